"""Parameter gradient (aq_param_grad) against the oracle, through the C ABI.

dL/ds and dL/dC of L = sum(gy * y), y = diag(s) W x, for every scheme, at
sizes that span several 128 x 128 tiles with ragged rows, features and
tokens; each element within 1e-2 of the oracle's magnitude bound plus 1e-3.
"""
import numpy as np
import pytest
import torch

import additive_quantized_matmul_b200 as aq
import oracle
from aq_inputs import LayerSpec, make_activations, make_layer
from aqtest import DevLayer, dev, workspace
from conftest import ATOL, RTOL

pytestmark = pytest.mark.gpu

SCHEMES = [(1, 16), (2, 8), (1, 8), (2, 16), (8, 8)]


def _grads(dl, x, gy, want_s=True, want_c=True, scales=True):
    spec = dl.spec
    T = x.shape[1]
    gs = torch.full((spec.out_features,), float("nan"), dtype=torch.float32, device="cuda") if want_s else None
    gc = (torch.full(((spec.num_codebooks << spec.nbits) * 8,), float("nan"), dtype=torch.float32, device="cuda")
          if want_c else None)
    ws = workspace(aq.aq_param_grad_workspace_bytes(dl.desc, T))
    aq.aq_param_grad(dl.desc, dl.packed, dl.codebooks, dl.scales if scales else None,
                     dev(x.view(np.uint16)), dev(gy.view(np.uint16)), T, gs, gc, ws)
    torch.cuda.synchronize()
    assert aq.aq_workspace_status(ws) == 0
    return (None if gs is None else gs.cpu().numpy().astype(np.float64),
            None if gc is None else gc.cpu().numpy().astype(np.float64))


def _check(got, ref, bound, what):
    err = np.abs(got - ref)
    lim = RTOL * bound + ATOL
    bad = np.argwhere(~(err <= lim))
    assert bad.size == 0, f"{what}: {len(bad)} elements off, first {bad[:3].tolist()}, " \
                          f"err {err.ravel()[np.argmax(err - lim)]:.3g}"


@pytest.mark.parametrize("K,B", SCHEMES)
@pytest.mark.parametrize("out,inp,T", [(8, 8, 8), (128, 128, 64), (200, 264, 72), (300, 1032, 136)])
def test_param_grad_matches_oracle(K, B, out, inp, T):
    layer = make_layer(LayerSpec(out, inp, K, B, codebook_sigma=0.05), out + inp + T + K)
    dl = DevLayer(layer)
    x = make_activations(inp, T, (1, T))
    gy = make_activations(out, T, (2, T))
    gs, gc = _grads(dl, x, gy)
    rs, rsb, rc, rcb = oracle.backward(layer.codes, layer.codebooks, layer.scales, x, gy)
    _check(gs, rs, rsb, f"grad_s {K}x{B}")
    _check(gc, rc.ravel(), rcb.ravel(), f"grad_C {K}x{B}")


def test_param_grad_optional_outputs_and_unit_scales():
    layer = make_layer(LayerSpec(136, 520, 2, 8, code_dist="zipf", codebook_sigma=0.05), 4)
    dl = DevLayer(layer)
    x = make_activations(520, 40, 5)
    gy = make_activations(136, 40, 6)
    ones = np.ones(136, dtype=np.float16)
    rs, rsb, rc, rcb = oracle.backward(layer.codes, layer.codebooks, ones, x, gy)
    gs, gc = _grads(dl, x, gy, scales=False)
    _check(gs, rs, rsb, "grad_s, s = 1")
    _check(gc, rc.ravel(), rcb.ravel(), "grad_C, s = 1")
    gs2, none = _grads(dl, x, gy, want_c=False, scales=False)
    assert none is None
    _check(gs2, rs, rsb, "grad_s alone")
    none, gc2 = _grads(dl, x, gy, want_s=False, scales=False)
    assert none is None
    _check(gc2, rc.ravel(), rcb.ravel(), "grad_C alone")


@pytest.mark.parametrize("K,B", [(1, 16), (2, 8)])
def test_param_grad_llama_rows_long_tokens(K, B):
    """1024 x 4096 (32 feature tiles) and 1032 tokens (17 stages, ragged)."""
    layer = make_layer(LayerSpec(1024, 4096, K, B), (K, B, 9))
    dl = DevLayer(layer)
    x = make_activations(4096, 1032, (3, K))
    gy = make_activations(1024, 1032, (4, K))
    gs, gc = _grads(dl, x, gy)
    rs, rsb, rc, rcb = oracle.backward(layer.codes, layer.codebooks, layer.scales, x, gy)
    _check(gs, rs, rsb, f"grad_s {K}x{B}")
    _check(gc, rc.ravel(), rcb.ravel(), f"grad_C {K}x{B}")
