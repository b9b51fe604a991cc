"""aq_gemv_noalloc: the decode-time product for callers that cannot allocate.

Some callers cannot call cudaMalloc (the host framework owns every device
allocation, or allocation is forbidden after start-up), so they cannot hand
aq_gemv a workspace.  aq_gemv_noalloc keeps its split-K scratch in a fixed
array inside the library instead.  These tests check, through the C ABI:

* two calls in a row, on layers whose usual workspace fits the array, give
  results within the tolerance of the oracle, as aq_gemv's do;
* layers whose usual workspace does not fit (a Llama-2-70B 1x16 layer at
  batch 16, which must split its sum more coarsely; a wide 2x8 layer at
  batch 1, whose table path's partial sums do not fit and which runs on the
  tensor cores instead) stay within the tolerance on sampled rows, and two
  calls on the same activations return the same bytes;
* a layer of 2^20 rows, whose plan needs no split (and so no scratch
  beyond the status word), runs through the same entry point.

This file is collected last, so that a run stopping at the first failure
has already run every other test; it also passes on its own in a fresh
process.
"""
import numpy as np
import pytest
import torch

import additive_quantized_matmul_b200 as aq
import oracle
from aq_inputs import LayerSpec, make_activations, make_layer
from aqtest import DevLayer, assert_close, dev, guarded, guards_intact, to_f16, workspace

pytestmark = pytest.mark.gpu

CASES = [
    ((4096, 4096, 1, 16), 1), ((4096, 4096, 1, 16), 16),
    ((1000, 1032, 2, 8), 1), ((1000, 1032, 2, 8), 5), ((256, 512, 2, 8), 4),
]
# usual workspace larger than the fixed array
OVER_CAP = [((28672, 8192, 1, 16), 16), ((32768, 16384, 2, 8), 1)]


def _noalloc(dl, x):
    batch = x.shape[1]
    full, y = guarded(dl.spec.out_features * batch)
    aq.aq_gemv_noalloc(dl.desc, dl.packed, dl.codebooks, dl.scales, dev(x.view(np.uint16)), batch, y)
    torch.cuda.synchronize()
    assert guards_intact(full), "aq_gemv_noalloc wrote outside its output"
    return to_f16(y).reshape(dl.spec.out_features, batch).astype(np.float64)


def _with_workspace(dl, x):
    batch = x.shape[1]
    y = torch.empty(dl.spec.out_features * batch, dtype=torch.int16, device="cuda")
    ws = workspace(aq.aq_gemv_workspace_bytes(dl.desc, batch))
    aq.aq_gemv(dl.desc, dl.packed, dl.codebooks, dl.scales, dev(x.view(np.uint16)), batch, y, ws)
    torch.cuda.synchronize()
    return to_f16(y).reshape(dl.spec.out_features, batch).astype(np.float64)


@pytest.mark.parametrize("shape,batch", CASES)
def test_noalloc_matches_oracle_like_workspace_entry_point(shape, batch):
    out, inp, K, B = shape
    spec = LayerSpec(out, inp, K, B, codebook_sigma=0.05)
    assert aq.aq_gemv_workspace_bytes(aq.LayerDesc.make(out, inp, K, B), batch) <= aq.GEMV_NOALLOC_SCRATCH_BYTES
    layer = make_layer(spec, out + inp + batch)
    dl = DevLayer(layer)
    for call in range(2):  # two calls in a row share the scratch array
        x = make_activations(inp, batch, (out, batch, call))
        ref, bound = oracle.matmul(layer.codes, layer.codebooks, layer.scales, x, threads=8)
        assert_close(_noalloc(dl, x), ref, bound, f"noalloc vs oracle, call {call}")
        assert_close(_with_workspace(dl, x), ref, bound, f"workspace entry point vs oracle, call {call}")


def _sample_rows(out, n=64, seed=0):
    rng = np.random.default_rng(seed)
    rows = set(rng.choice(out, size=n, replace=False).tolist())
    rows.update({0, 127, 128, out - 1})
    return np.array(sorted(rows))


@pytest.mark.parametrize("shape,batch", OVER_CAP)
def test_noalloc_coarser_split_when_the_usual_one_does_not_fit(shape, batch):
    out, inp, K, B = shape
    assert aq.aq_gemv_workspace_bytes(aq.LayerDesc.make(out, inp, K, B), batch) > aq.GEMV_NOALLOC_SCRATCH_BYTES
    layer = make_layer(LayerSpec(out, inp, K, B), (out, inp, batch))
    dl = DevLayer(layer)
    rows = _sample_rows(out, seed=out)
    x = make_activations(inp, batch, (out, batch))
    y1 = _noalloc(dl, x)
    y2 = _noalloc(dl, x)
    assert np.array_equal(y1.view(np.uint64), y2.view(np.uint64)), "two calls on the same x differ"
    ref, bound = oracle.matmul(layer.codes, layer.codebooks, layer.scales, x, rows=rows, threads=8)
    assert_close(y1[rows], ref, bound, f"noalloc {out}x{inp} {K}x{B} b{batch}")
    x2 = make_activations(inp, batch, (out, batch, 2))
    ref2, bound2 = oracle.matmul(layer.codes, layer.codebooks, layer.scales, x2, rows=rows, threads=8)
    assert_close(_noalloc(dl, x2)[rows], ref2, bound2, f"noalloc {out}x{inp} {K}x{B} b{batch}, second x")
    del dl
    torch.cuda.empty_cache()


def test_noalloc_layer_without_split():
    out, inp = 1 << 20, 64
    assert aq.aq_gemv_workspace_bytes(aq.LayerDesc.make(out, inp, 1, 16), 4) == 16
    layer = make_layer(LayerSpec(out, inp, 1, 16), 11)
    dl = DevLayer(layer)
    x = make_activations(inp, 4, 12)
    y = _noalloc(dl, x)
    rows = _sample_rows(out, seed=3)
    ref, bound = oracle.matmul(layer.codes, layer.codebooks, layer.scales, x, rows=rows, threads=8)
    assert_close(y[rows], ref, bound, "noalloc 2^20 x 64")
