"""Parity of the CUDA path (through the C ABI) with the CPU oracle.

Codes, packed bytes and dequantised weights must match bit for bit; products
must satisfy |y_gpu - y_ref| <= 1e-2 * sum_i |s||W||x| + 1e-3 per element,
y_ref being the fp64 oracle.  Small layers are compared in full (several
tiles plus ragged tails); the full-size workloads are compared on sampled
rows, in the launch configuration the benchmark uses.
"""
import numpy as np
import pytest
import torch

import additive_quantized_matmul_b200 as aq
import oracle
from aq_inputs import LayerSpec, make_activations, make_layer, workload
from aqtest import (DevLayer, assert_close, dev, guarded, guards_intact, run_gemm, run_gemv,
                    to_f16, workspace)

pytestmark = pytest.mark.gpu

SCHEMES = [(1, 16), (2, 8), (1, 8), (2, 16), (8, 8)]
NEW_SCHEMES = [(1, 8), (2, 16), (8, 8)]
SMALL_SHAPES = [(8, 8), (37, 360), (256, 512), (1000, 1032), (64, 4096), (4100, 264)]


def _layer(out, inp, K, B, seed, **kw):
    return make_layer(LayerSpec(out, inp, K, B, codebook_sigma=kw.pop("sigma", 0.05), **kw), seed)


# ---------------------------------------------------------------------------
# pack / unpack / dequant: bit-exact
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("K,B", SCHEMES)
@pytest.mark.parametrize("out,inp", SMALL_SHAPES)
def test_pack_matches_oracle_bytes(K, B, out, inp):
    layer = _layer(out, inp, K, B, out * 7 + inp)
    dl = DevLayer(layer)
    want = oracle.pack(layer.codes, K, B)
    got = dl.packed.cpu().numpy()
    assert np.array_equal(got, want)
    back = torch.empty_like(dl.codes)
    aq.aq_unpack_codes(dl.desc, dl.packed, back)
    torch.cuda.synchronize()
    assert torch.equal(back, dl.codes)


@pytest.mark.parametrize("K,B", SCHEMES)
@pytest.mark.parametrize("out,inp", SMALL_SHAPES)
@pytest.mark.parametrize("scaled", [False, True])
def test_dequant_bit_exact(K, B, out, inp, scaled):
    layer = _layer(out, inp, K, B, out + inp + K)
    dl = DevLayer(layer)
    full, w = guarded(out * inp)
    aq.aq_dequant(dl.desc, dl.packed, dl.codebooks, dl.scales if scaled else None, w)
    torch.cuda.synchronize()
    assert guards_intact(full)
    want = oracle.decode(layer.codes, layer.codebooks, layer.scales if scaled else None)
    assert np.array_equal(w.cpu().numpy().view(np.uint16).reshape(out, inp), want.view(np.uint16))


def test_dequant_eight_codebooks_exact_sum_of_mixed_magnitudes():
    """8x8: the eight terms span many binades, so a sum rounded at every
    step (or in fp32) would differ from the exact sum rounded once."""
    rng = np.random.default_rng(5)
    K, B, out, inp = 8, 8, 64, 512
    mant = rng.integers(1024, 2048, size=(K, 256, 8))
    expo = rng.integers(-24, 6, size=(K, 256, 8))
    sign = rng.choice([-1.0, 1.0], size=(K, 256, 8))
    cb = (sign * mant * np.exp2(expo - 10.0)).astype(np.float16)
    layer = _layer(out, inp, K, B, 3)
    layer.codebooks[...] = cb
    dl = DevLayer(layer)
    full, w = guarded(out * inp)
    aq.aq_dequant(dl.desc, dl.packed, dl.codebooks, None, w)
    torch.cuda.synchronize()
    assert guards_intact(full)
    want = oracle.decode(layer.codes, layer.codebooks)
    assert np.array_equal(w.cpu().numpy().view(np.uint16).reshape(out, inp), want.view(np.uint16))


def test_dequant_signed_zero_and_extremes():
    layer = _layer(64, 256, 2, 8, 5)
    cb = layer.codebooks.copy()
    cb[0, :16] = -0.0
    cb[1, :16] = -0.0
    cb[0, 16:32] = 65504.0          # sums overflow to inf, as RN16 says
    cb[1, 16:32] = 32.0
    cb[0, 32:48] = np.float16(2.0 ** -24)  # subnormal sums
    cb[1, 32:48] = np.float16(2.0 ** -24)
    layer.codebooks = cb
    layer.codes[:, :, :] = np.random.default_rng(1).integers(0, 48, size=layer.codes.shape)
    dl = DevLayer(layer)
    w = torch.empty(64 * 256, dtype=torch.int16, device="cuda")
    aq.aq_dequant(dl.desc, dl.packed, dl.codebooks, None, w)
    torch.cuda.synchronize()
    want = oracle.decode(layer.codes, layer.codebooks)
    assert np.array_equal(w.cpu().numpy().view(np.uint16).reshape(64, 256), want.view(np.uint16))


# ---------------------------------------------------------------------------
# decode-time product (batch 1..16)
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("K,B", SCHEMES)
@pytest.mark.parametrize("out,inp", SMALL_SHAPES)
@pytest.mark.parametrize("batch", [1, 4, 16])
def test_gemv_matches_oracle(K, B, out, inp, batch):
    layer = _layer(out, inp, K, B, out * 3 + inp + batch)
    x = make_activations(inp, batch, 77 + batch)
    dl = DevLayer(layer)
    y = run_gemv(dl, x)
    ref, bound = oracle.matmul(layer.codes, layer.codebooks, layer.scales, x)
    assert_close(y, ref, bound, f"gemv {K}x{B} {out}x{inp} b{batch}")


@pytest.mark.parametrize("K,B", SCHEMES)
@pytest.mark.parametrize("batch", range(1, 17))
def test_gemv_every_batch(K, B, batch):
    layer = _layer(300, 1032, K, B, 1234)
    x = make_activations(1032, batch, batch)
    dl = DevLayer(layer)
    y = run_gemv(dl, x)
    ref, bound = oracle.matmul(layer.codes, layer.codebooks, layer.scales, x)
    assert_close(y, ref, bound, f"gemv {K}x{B} b{batch}")


@pytest.mark.parametrize("K,B", [(1, 16), (2, 16)])
@pytest.mark.parametrize("batch", [1, 5, 16])
def test_gemv_ragged_tall_layer_checked_in_full(K, B, batch):
    """20000 x 1032: 157 row tiles of only 17 64-feature stages, the last
    row tile ragged (32 rows) and the last stage one group.  1x16 runs on
    the CUDA cores at batch 1 (groups split five ways) and on the
    register-fragment kernel at 5 and 16 (one split); 2x16 runs on the
    tensor-core kernel, whose planner splits the sum of this shape (the
    workspace then holds partial sums).  Every output is checked against
    the oracle."""
    out, inp = 20000, 1032
    layer = _layer(out, inp, K, B, 4321)
    desc = aq.LayerDesc.make(out, inp, K, B)
    if (K, B) == (2, 16):
        assert aq.aq_gemv_workspace_bytes(desc, batch) > 16 + 4 * 1024  # a split of the sum is in use
    x = make_activations(inp, batch, 313 + batch)
    dl = DevLayer(layer)
    y = run_gemv(dl, x)
    ref, bound = oracle.matmul(layer.codes, layer.codebooks, layer.scales, x, threads=8)
    assert_close(y, ref, bound, f"tall {K}x{B} {out}x{inp} b{batch}")


def test_gemv_cuda_core_path_deterministic_and_reusable():
    """1x16 at batch 1 on the CUDA cores (4096 x 2048: 32 row ranges, 27
    group splits finished by the last CTA of each range): same bits twice,
    correct results with one workspace reused across activations."""
    layer = _layer(4096, 2048, 1, 16, 17)
    dl = DevLayer(layer)
    ws = workspace(aq.aq_gemv_workspace_bytes(dl.desc, 1))
    x = make_activations(2048, 1, 5)
    y1 = run_gemv(dl, x, ws)
    assert np.array_equal(y1, run_gemv(dl, x, ws))
    for rep in range(3):
        x2 = make_activations(2048, 1, (rep, 23))
        ref, bound = oracle.matmul(layer.codes, layer.codebooks, layer.scales, x2, threads=8)
        assert_close(run_gemv(dl, x2, ws), ref, bound, f"cuda-core 1x16 reuse {rep}")


@pytest.mark.parametrize("K,B", SCHEMES)
def test_gemv_deterministic_and_workspace_reusable(K, B):
    """Same inputs give the same bits; a workspace reused across calls with
    different activations gives correct results each time (the split-K
    arrival counters are back at zero after every call)."""
    layer = _layer(1024, 8192, K, B, 99)
    dl = DevLayer(layer)
    for batch in (1, 3, 16):
        ws = workspace(aq.aq_gemv_workspace_bytes(dl.desc, batch))
        x = make_activations(8192, batch, batch)
        y1 = run_gemv(dl, x, ws)
        assert np.array_equal(y1, run_gemv(dl, x, ws))
        ref, bound = oracle.matmul(layer.codes, layer.codebooks, layer.scales, x)
        assert_close(y1, ref, bound, f"gemv {K}x{B} b{batch}")
        for rep in range(3):
            x2 = make_activations(8192, batch, (batch, rep, 17))
            ref2, bound2 = oracle.matmul(layer.codes, layer.codebooks, layer.scales, x2)
            assert_close(run_gemv(dl, x2, ws), ref2, bound2, f"gemv {K}x{B} b{batch} reuse {rep}")


def test_gemv_without_scales_and_zipf_codes():
    layer = _layer(512, 2048, 2, 8, 3, code_dist="zipf")
    dl = DevLayer(layer)
    x = make_activations(2048, 1, 4)
    xd = dev(x.view(np.uint16))
    y = torch.empty(512, dtype=torch.int16, device="cuda")
    ws = workspace(aq.aq_gemv_workspace_bytes(dl.desc, 1))
    aq.aq_gemv(dl.desc, dl.packed, dl.codebooks, None, xd, 1, y, ws)
    torch.cuda.synchronize()
    ref, bound = oracle.matmul(layer.codes, layer.codebooks, None, x)
    assert_close(to_f16(y).astype(np.float64)[:, None], ref, bound, "gemv no scales")


def test_gemv_rejects_small_workspace_without_writing():
    layer = _layer(256, 512, 2, 8, 4)
    dl = DevLayer(layer)
    xd = dev(make_activations(512, 1, 1).view(np.uint16))
    full, y = guarded(256)
    ws = workspace(16)
    need = aq.aq_gemv_workspace_bytes(dl.desc, 1)
    with pytest.raises(aq.AQError) as e:
        aq.aq_gemv(dl.desc, dl.packed, dl.codebooks, dl.scales, xd, 1, y, ws, need - 1)
    assert e.value.name == "AQ_ERR_WORKSPACE"
    torch.cuda.synchronize()
    assert guards_intact(full) and bool((y == 0x7E5A).all())


# ---------------------------------------------------------------------------
# prefill product on the tensor cores
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("K,B", SCHEMES)
@pytest.mark.parametrize("out,inp", [(128, 64), (256, 512), (129, 136), (1000, 1032), (8, 8)])
@pytest.mark.parametrize("T", [1, 5, 8, 64, 136, 300, 520, 1032])
def test_gemm_matches_oracle(K, B, out, inp, T):
    layer = _layer(out, inp, K, B, out + inp * 5 + T)
    x = make_activations(inp, T, T)
    dl = DevLayer(layer)
    y = run_gemm(dl, x)
    ref, bound = oracle.matmul(layer.codes, layer.codebooks, layer.scales, x)
    assert_close(y, ref, bound, f"gemm {K}x{B} {out}x{inp} T{T}")


def test_gemm_deterministic():
    layer = _layer(512, 1024, 1, 16, 8)
    dl = DevLayer(layer)
    x = make_activations(1024, 256, 9)
    assert np.array_equal(run_gemm(dl, x), run_gemm(dl, x))


# ---------------------------------------------------------------------------
# bounded waits report instead of hanging
# ---------------------------------------------------------------------------

def test_bounded_wait_reports_timeout_and_context_survives():
    ws = workspace(16)
    aq.aq_selftest_bounded_wait(ws, 1000)
    assert aq.aq_workspace_status(ws) == 6  # AQ_ERR_TIMEOUT
    assert aq.aq_workspace_status(ws) == 0  # cleared by the read
    layer = _layer(64, 256, 1, 16, 2)
    dl = DevLayer(layer)
    x = make_activations(256, 2, 3)
    ref, bound = oracle.matmul(layer.codes, layer.codebooks, layer.scales, x)
    assert_close(run_gemv(dl, x), ref, bound, "after timeout")


# ---------------------------------------------------------------------------
# full-size workloads, sampled rows (same launch configuration as bench.py)
# ---------------------------------------------------------------------------

def _sample_rows(out, n=48, seed=0):
    rng = np.random.default_rng(seed)
    rows = set(rng.choice(out, size=min(n, out), replace=False).tolist())
    rows.update({0, out - 1, min(out - 1, 127), min(out - 1, 128)})
    return np.array(sorted(rows))


@pytest.mark.parametrize("name", ["tiny-2x8", "llama2-7b-1x16", "llama2-7b-mlp-2x8", "llama2-70b-1x16"])
def test_gemv_full_size_sampled(name):
    wl = workload(name)
    for i, (tag, spec) in enumerate(wl["layers"]):
        layer = make_layer(spec, (wl["seed"], i))
        dl = DevLayer(layer)
        for batch in wl["n"]:
            x = make_activations(spec.in_features, batch, (wl["seed"], i, batch))
            y = run_gemv(dl, x)
            rows = _sample_rows(spec.out_features, seed=i)
            ref, bound = oracle.matmul(layer.codes, layer.codebooks, layer.scales, x, rows=rows, threads=8)
            assert_close(y[rows], ref, bound, f"{name}/{tag} b{batch}")
        del dl
        torch.cuda.empty_cache()


def test_gemm_full_size_sampled():
    wl = workload("llama2-7b-prefill")
    for i, (tag, spec) in enumerate(wl["layers"]):
        layer = make_layer(spec, (wl["seed"], i))
        dl = DevLayer(layer)
        for T in wl["n"]:
            x = make_activations(spec.in_features, T, (wl["seed"], i, T))
            y = run_gemm(dl, x)
            rows = _sample_rows(spec.out_features, n=12, seed=i)
            ref, bound = oracle.matmul(layer.codes, layer.codebooks, layer.scales, x, rows=rows, threads=8)
            assert_close(y[rows], ref, bound, f"prefill/{tag} T{T}")
        del dl
        torch.cuda.empty_cache()


def test_dequant_full_size_sampled():
    spec = LayerSpec(28672, 8192, 1, 16)
    layer = make_layer(spec, 5)
    dl = DevLayer(layer)
    w = torch.empty(spec.out_features * spec.in_features, dtype=torch.int16, device="cuda")
    aq.aq_dequant(dl.desc, dl.packed, dl.codebooks, dl.scales, w)
    torch.cuda.synchronize()
    rows = _sample_rows(spec.out_features, n=64)
    got = w.view(spec.out_features, spec.in_features)[torch.from_numpy(rows).cuda()].cpu().numpy()
    want = oracle.decode(layer.codes[rows], layer.codebooks, layer.scales[rows])
    assert np.array_equal(got.view(np.uint16), want.view(np.uint16))


@pytest.mark.parametrize("K,B", NEW_SCHEMES)
def test_other_schemes_llama_shape_sampled(K, B):
    """1x8, 2x16 and 8x8 at a Llama-2-7B MLP shape: products at batch 1, 8
    and 16, a prefill product and the dequantised matrix, on sampled rows."""
    spec = LayerSpec(11008, 4096, K, B)
    layer = make_layer(spec, (K, B))
    dl = DevLayer(layer)
    rows = _sample_rows(spec.out_features, n=24, seed=K + B)
    for batch in (1, 8, 16):
        x = make_activations(spec.in_features, batch, (K, B, batch))
        y = run_gemv(dl, x)
        ref, bound = oracle.matmul(layer.codes, layer.codebooks, layer.scales, x, rows=rows, threads=8)
        assert_close(y[rows], ref, bound, f"{K}x{B} b{batch}")
    x = make_activations(spec.in_features, 512, (K, B, 512))
    y = run_gemm(dl, x)
    ref, bound = oracle.matmul(layer.codes, layer.codebooks, layer.scales, x, rows=rows[:8], threads=8)
    assert_close(y[rows[:8]], ref, bound, f"{K}x{B} T512")
    w = torch.empty(spec.out_features * spec.in_features, dtype=torch.int16, device="cuda")
    aq.aq_dequant(dl.desc, dl.packed, dl.codebooks, dl.scales, w)
    torch.cuda.synchronize()
    got = w.view(spec.out_features, spec.in_features)[torch.from_numpy(rows).cuda()].cpu().numpy()
    want = oracle.decode(layer.codes[rows], layer.codebooks, layer.scales[rows])
    assert np.array_equal(got.view(np.uint16), want.view(np.uint16))
    del dl
    torch.cuda.empty_cache()


@pytest.mark.parametrize("K,B", [(1, 16), (2, 8)])
@pytest.mark.parametrize("T", [256, 512, 2048])
def test_gemm_split_k_deterministic_and_reusable(K, B, T):
    """Layers small enough that the input features are split across CTAs:
    the split partial sums are added in split order, so repeated calls give
    identical bits, and the tile counters are back at zero after each call
    (the workspace is reused)."""
    layer = _layer(256, 4096, K, B, T + K)
    dl = DevLayer(layer)
    desc = dl.desc
    ws = workspace(aq.aq_gemm_workspace_bytes(desc, T))
    x = make_activations(4096, T, (T, 1))
    y1 = run_gemm(dl, x, ws)
    y2 = run_gemm(dl, x, ws)
    assert np.array_equal(y1, y2)
    rows = np.arange(0, 256, 17)
    ref, bound = oracle.matmul(layer.codes, layer.codebooks, layer.scales, x, rows=rows, threads=8)
    assert_close(y1[rows], ref, bound, f"split-K {K}x{B} T{T}")


@pytest.mark.parametrize("K,B", [(1, 16), (2, 8)])
@pytest.mark.parametrize("out,inp,T,ks", [(512, 2048, 392, 4), (256, 4096, 392, 8), (1000, 1032, 520, 2)])
def test_gemm_cluster_split_ragged_tokens_every_element(K, B, out, inp, T, ks):
    """Input-feature splits of 2, 4 and 8 that run as one thread-block
    cluster: each split owns BN / ks of a tile's 512 columns and adds every
    split's sums for them.  T leaves the last tile ragged (392 = 3 x 128 +
    8: at 4 splits one owner has 8 live columns, at 8 splits one has 8 and
    one none), and 1000 rows leave the last row tile ragged.  The workspace
    size pins the plan (ks splits, tiles of 128 x 512, fp32 sums); every
    element is checked against the oracle."""
    desc = aq.LayerDesc.make(out, inp, K, B)
    tiles = ((out + 127) // 128) * ((T + 511) // 512)
    assert aq.aq_gemm_workspace_bytes(desc, T) == 4112 + ks * tiles * 128 * 512 * 4
    layer = _layer(out, inp, K, B, out + inp + T + ks)
    dl = DevLayer(layer)
    x = make_activations(inp, T, (out, T, ks))
    y = run_gemm(dl, x)
    ref, bound = oracle.matmul(layer.codes, layer.codebooks, layer.scales, x, threads=8)
    assert_close(y, ref, bound, f"cluster split {ks} {K}x{B} {out}x{inp} T{T}")


@pytest.mark.parametrize("K,B", [(1, 16), (2, 8)])
@pytest.mark.parametrize("T", [2048, 2040])
def test_gemm_wave_tail_split(K, B, T):
    """A tile grid one wave and a bit: 38 row tiles x 4 token tiles = 152
    tiles on 148 SMs.  The last 4 tiles (rows 4352..4863, tokens 1536..)
    have their input features split 2 ways and are finished by the last of
    their splits; the workspace size pins that plan.  Every row of the tail
    tiles' row blocks and rows elsewhere are checked in full against the
    oracle (T = 2040 leaves the tail's token tile ragged)."""
    out, inp = 4864, 1024
    desc = aq.LayerDesc.make(out, inp, K, B)
    assert aq.aq_gemm_workspace_bytes(desc, T) == 4112 + 4 * 2 * 128 * 512 * 4
    layer = _layer(out, inp, K, B, T + K)
    dl = DevLayer(layer)
    x = make_activations(inp, T, (T, K, 5))
    y = run_gemm(dl, x)
    rows = np.concatenate([np.arange(4352, 4864), np.arange(0, 4352, 97)])
    ref, bound = oracle.matmul(layer.codes, layer.codebooks, layer.scales, x, rows=rows, threads=8)
    assert_close(y[rows], ref, bound, f"wave tail {K}x{B} T{T}")
    assert np.array_equal(run_gemm(dl, x)[rows], y[rows])  # deterministic


@pytest.mark.parametrize("K", [2, 1])
def test_gemv_tables_fall_back_to_exact_decode_beyond_binary16(K):
    """The batch-1 table path keeps its tables in binary16 and bounds their
    entries by 8 max|x| max|C| per CTA.  Here one codebook entry of 30 and
    activations of 300 in the first group make that bound 72000, beyond
    binary16, for the CTAs holding the first group: they decode each group
    exactly and multiply in fp32 instead, while the other group split keeps
    its tables.  Both must agree with the oracle."""
    layer = _layer(512, 1024, K, 8, 77)
    cb = layer.codebooks.copy()
    cb[0, 5, 0] = 30.0
    layer.codebooks = cb
    layer.codes[:64, 0, 0] = 5  # rows whose first group uses the large codeword
    x = make_activations(1024, 1, 78)
    x[:8, 0] = 300.0
    dl = DevLayer(layer)
    y = run_gemv(dl, x)
    ref, bound = oracle.matmul(layer.codes, layer.codebooks, layer.scales, x)
    assert np.abs(ref[:64]).max() > 1000  # the large terms are in the result
    assert_close(y, ref, bound, f"{K}x8 tables beyond binary16")
