"""The seeded input generator follows its stated recipe: deterministic per
seed, codes uniform or Zipf(1.1) by code value, codebooks N(0, sigma),
scales U(0.5, 1.5), activations N(0, 1), every value binary16, and the
named workloads carry the Llama-2 layer shapes."""
import numpy as np
import pytest

from aq_inputs import WORKLOADS, LayerSpec, make_activations, make_layer, workload, workload_units


def test_same_seed_same_bytes_other_seed_other_bytes():
    spec = LayerSpec(64, 256, 2, 8)
    a, b = make_layer(spec, (1001, 0, 3)), make_layer(spec, (1001, 0, 3))
    c = make_layer(spec, (1001, 1, 3))  # another rank
    for f in ("codes", "codebooks", "scales"):
        assert getattr(a, f).tobytes() == getattr(b, f).tobytes()
        assert getattr(a, f).tobytes() != getattr(c, f).tobytes()
    assert np.array_equal(make_activations(256, 4, 7), make_activations(256, 4, 7))
    assert not np.array_equal(make_activations(256, 4, 7), make_activations(256, 4, 8))


@pytest.mark.parametrize("K,B", [(1, 16), (2, 8), (1, 8), (2, 16), (8, 8)])
def test_layout_and_types(K, B):
    layer = make_layer(LayerSpec(24, 64, K, B), 5)
    assert layer.codes.shape == (24, 8, K)
    assert layer.codes.dtype == (np.uint8 if B <= 8 else np.uint16)
    assert layer.codebooks.shape == (K, 1 << B, 8) and layer.codebooks.dtype == np.float16
    assert layer.scales.shape == (24,) and layer.scales.dtype == np.float16


def test_uniform_codes_cover_the_range():
    codes = make_layer(LayerSpec(512, 4096, 2, 8), 11).codes.astype(np.int64).ravel()
    counts = np.bincount(codes, minlength=256)
    assert counts.min() > 0 and codes.max() == 255
    expected = codes.size / 256
    chi2 = ((counts - expected) ** 2 / expected).sum()
    assert chi2 < 255 + 6 * np.sqrt(2 * 255)  # 255 degrees of freedom, six sigma


def test_zipf_codes_follow_the_power_law_by_code_value():
    codes = make_layer(LayerSpec(1024, 4096, 2, 8, code_dist="zipf"), 12).codes.astype(np.int64).ravel()
    counts = np.bincount(codes, minlength=256).astype(np.float64)
    # P(c) / P(0) = (c + 1)^-1.1
    for c in (1, 3, 15):
        ratio = counts[c] / counts[0]
        assert abs(ratio - (c + 1) ** -1.1) < 0.03 * (c + 1) ** -1.1 + 0.005
    assert counts[:8].sum() > counts[128:].sum()


def test_value_distributions():
    layer = make_layer(LayerSpec(4096, 512, 1, 16, codebook_sigma=0.02), 13)
    cb = layer.codebooks.astype(np.float64)
    assert abs(cb.mean()) < 1e-3 and abs(cb.std() - 0.02) < 2e-4
    s = layer.scales.astype(np.float64)
    assert s.min() >= 0.5 and s.max() <= 1.5 and abs(s.mean() - 1.0) < 0.02
    x = make_activations(4096, 16, 14).astype(np.float64)
    assert abs(x.mean()) < 0.02 and abs(x.std() - 1.0) < 0.02


def test_values_are_rounded_to_nearest_binary16():
    rng = np.random.Generator(np.random.PCG64(21))
    raw = rng.normal(0.0, 1.0, size=(64, 3))
    x = make_activations(64, 3, 21)
    # the nearer of the two binary16 neighbours (ties cannot occur for
    # continuous draws)
    err = np.abs(x.astype(np.float64) - raw)
    up = np.nextafter(x, np.float16(np.inf)).astype(np.float64)
    dn = np.nextafter(x, np.float16(-np.inf)).astype(np.float64)
    assert np.all(err <= np.abs(up - raw)) and np.all(err <= np.abs(dn - raw))


def test_rejects_width_not_multiple_of_group():
    with pytest.raises(ValueError):
        make_layer(LayerSpec(8, 12, 1, 16), 1)


def test_named_workloads_have_llama2_shapes():
    dims = {4096, 11008, 8192, 28672, 1024, 256, 512}
    for name in WORKLOADS:
        wl = workload(name)
        specs = [sp for _, sp, _, _ in workload_units(name)] + [
            sp for _, chain in wl.get("chains", []) for _, sp, _ in chain]
        assert specs, name
        for sp in specs:
            assert sp.out_features in dims and sp.in_features in dims, (name, sp)
            assert (sp.num_codebooks, sp.nbits) in {(1, 16), (2, 8), (1, 8), (2, 16), (8, 8)}
    assert workload("llama2-7b-1x16")["layers"][0][1] == LayerSpec(4096, 4096, 1, 16)
    assert workload("llama2-7b-1x16")["n"] == [1, 4, 16]
    # the decode workload is the 1x16 layer and the 2x8 MLP layers, each with its own batches
    units = workload_units("llama2-7b-decode")
    assert [(t, sp.scheme, n) for t, sp, n, _ in units] == [
        ("4096x4096", "1x16", (1, 4, 16)),
        ("11008x4096-uniform", "2x8", (1, 8)), ("4096x11008-uniform", "2x8", (1, 8)),
        ("11008x4096-zipf", "2x8", (1, 8)), ("4096x11008-zipf", "2x8", (1, 8))]
    with pytest.raises(KeyError):
        workload("no-such-workload")
