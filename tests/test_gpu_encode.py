"""Encoder (aq_encode) against the oracle, through the C ABI.

Integer-valued problems keep every score the kernel forms in fp32 an exact
integer, so both sides take the same decisions and the codes must match
bit for bit.  A real-valued problem (H = 2 X^T X of random activations) is
checked by objective: never worse than the start, and as good as the
oracle's within fp32 rounding.
"""
import numpy as np
import pytest
import torch

import additive_quantized_matmul_b200 as aq
import oracle
from aq_inputs import LayerSpec, make_layer
from aqtest import dev, workspace

pytestmark = pytest.mark.gpu


def _int_problem(out, inp, K, seed, rank=4):
    rng = np.random.default_rng(seed)
    w = rng.integers(-4, 5, size=(out, inp)).astype(np.float16)
    a = rng.integers(-1, 2, size=(rank, inp)).astype(np.float32)
    h = (a.T @ a + np.eye(inp, dtype=np.float32)).astype(np.float32)
    cb = rng.integers(-2, 3, size=(K, 256, 8)).astype(np.float16)
    c0 = rng.integers(0, 256, size=(out, inp // 8, K)).astype(np.uint8)
    return w, h, cb, c0


def _gpu_encode(w, h, cb, c0, beam):
    out, inp = w.shape
    K = cb.shape[0]
    desc = aq.LayerDesc.make(out, inp, K, 8)
    ci = torch.from_numpy(c0.copy()).cuda()
    co = torch.full_like(ci, 0xEE)
    ws = workspace(aq.aq_encode_workspace_bytes(desc))
    aq.aq_encode(desc, dev(w.view(np.uint16)), torch.from_numpy(h).cuda(), dev(cb.view(np.uint16)), ci, beam, co, ws)
    torch.cuda.synchronize()
    return co.cpu().numpy()


@pytest.mark.parametrize("K", [1, 2, 8])
@pytest.mark.parametrize("beam", [1, 4, 16])
def test_encode_matches_oracle_exactly_on_integer_problems(K, beam):
    out, inp = (5, 32) if K == 8 else (7, 64)
    w, h, cb, c0 = _int_problem(out, inp, K, K * 100 + beam)
    got = _gpu_encode(w, h, cb, c0, beam)
    want, _ = oracle.encode(w, h, cb, c0, beam)
    assert np.array_equal(got, want)


def test_encode_real_valued_objective():
    spec = LayerSpec(32, 64, 2, 8, codebook_sigma=0.05)
    layer = make_layer(spec, 11)
    rng = np.random.default_rng(12)
    w = rng.normal(0, 0.08, size=(32, 64)).astype(np.float16)
    x = rng.normal(0, 1, size=(256, 64)).astype(np.float32)
    h = (2.0 * x.T @ x / 256).astype(np.float32)
    c0 = layer.codes
    got = _gpu_encode(w, h, layer.codebooks, c0, 4)
    want, f_oracle = oracle.encode(w, h, layer.codebooks, c0, 4)
    f_gpu = oracle.objective(w, h, layer.codebooks, got)
    f_start = oracle.objective(w, h, layer.codebooks, c0)
    assert np.all(f_gpu <= f_start)
    assert np.all(f_gpu <= f_oracle * (1 + 1e-4) + 1e-6)
    assert (got == want).mean() > 0.95  # near-ties aside, the same codes
