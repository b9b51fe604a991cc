"""aq_gemv_noalloc: the decode-time product for callers that cannot allocate.

Some callers cannot call cudaMalloc (the host framework owns every device
allocation, or allocation is forbidden after start-up), so they cannot hand
aq_gemv a workspace.  aq_gemv_noalloc keeps its split-K scratch in a fixed
array inside the library instead.  These tests check, through the C ABI,
that two calls in a row give the same results as aq_gemv with a workspace
(within the tolerance the other tests use), and that a layer needing more
scratch than the array holds is refused without writing anything.

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
def test_noalloc_matches_workspace_entry_point(shape, batch):
    out, inp, K, B = shape
    spec = LayerSpec(out, inp, K, B, codebook_sigma=0.05)
    assert aq.aq_gemv_workspace_bytes(aq.LayerDesc.make(out, inp, K, B), batch) <= aq.GEMV_NOALLOC_SCRATCH_BYTES
    layer = make_layer(spec, out + inp + batch)
    dl = DevLayer(layer)
    for call in range(2):  # two calls in a row share the scratch array
        x = make_activations(inp, batch, (out, batch, call))
        y_na = _noalloc(dl, x)
        y_ws = _with_workspace(dl, x)
        _, bound = oracle.matmul(layer.codes, layer.codebooks, layer.scales, x)
        assert_close(y_na, y_ws, bound, f"noalloc vs workspace, call {call}")


def test_noalloc_refuses_layers_beyond_the_scratch():
    # 2x8 at batch 1 keeps one partial per row and 32-group block:
    # 32768 rows x 256 blocks x 4 bytes = 32 MiB > the fixed scratch
    desc = aq.LayerDesc.make(32768, 65536, 2, 8)
    assert aq.aq_gemv_workspace_bytes(desc, 1) > aq.GEMV_NOALLOC_SCRATCH_BYTES
    small = torch.zeros(64, dtype=torch.int16, device="cuda")  # never read: refused first
    full, y = guarded(64)
    with pytest.raises(aq.AQError) as e:
        aq.aq_gemv_noalloc(desc, small, small, small, small, 1, y)
    assert e.value.name == "AQ_ERR_WORKSPACE"
    torch.cuda.synchronize()
    assert guards_intact(full) and bool((y == 0x7E5A).all())
