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


# ---------------------------------------------------------------------------
# 16-bit codebooks (1x16, 2x16): every slot scores all 65536 codes
# ---------------------------------------------------------------------------

def _int_problem16(out, inp, K, seed, rank=3):
    rng = np.random.default_rng(seed)
    w = rng.integers(-4, 5, size=(out, inp)).astype(np.float16)
    a = rng.integers(-1, 2, size=(rank, inp)).astype(np.float32)
    h = (a.T @ a + np.eye(inp, dtype=np.float32)).astype(np.float32)
    cb = rng.integers(-2, 3, size=(K, 65536, 8)).astype(np.float16)
    c0 = rng.integers(0, 65536, size=(out, inp // 8, K)).astype(np.uint16)
    return w, h, cb, c0


def _gpu_encode16(w, h, cb, c0, beam):
    out, inp = w.shape
    K = cb.shape[0]
    desc = aq.LayerDesc.make(out, inp, K, 16)
    ci = torch.from_numpy(c0.view(np.int16).copy()).cuda()
    co = torch.full_like(ci, 0x7EEE)
    ws = workspace(aq.aq_encode_workspace_bytes(desc))
    aq.aq_encode(desc, dev(w.view(np.uint16)), torch.from_numpy(h).cuda(), dev(cb.view(np.uint16)), ci, beam, co, ws)
    torch.cuda.synchronize()
    return co.cpu().numpy().view(np.uint16)


@pytest.mark.parametrize("K,beam,out", [(1, 1, 19), (1, 4, 19), (2, 1, 5), (2, 4, 5), (2, 16, 3)])
def test_encode16_matches_oracle_exactly_on_integer_problems(K, beam, out):
    """Integer-valued problems: the fp32 scores are exact, so the kernel and
    the oracle rank every proposal alike (ties by parent beam, then code;
    the small integer codebooks hold many equal codewords) and the codes
    match bit for bit.  19 rows leave the second 16-row tile ragged."""
    w, h, cb, c0 = _int_problem16(out, 16, K, 1600 + 10 * K + beam)
    got = _gpu_encode16(w, h, cb, c0, beam)
    want, _ = oracle.encode(w, h, cb, c0, beam)
    assert got.shape == want.shape
    assert np.array_equal(got, want)


def test_encode16_real_valued_objective():
    """1x16 on a real-valued problem: never worse than the start, as good as
    the oracle within fp32 rounding, and nearly always the same codes."""
    rng = np.random.default_rng(21)
    out, inp = 8, 32
    cb = rng.normal(0, 0.05, size=(1, 65536, 8)).astype(np.float16)
    w = rng.normal(0, 0.08, size=(out, inp)).astype(np.float16)
    x = rng.normal(0, 1, size=(256, inp)).astype(np.float32)
    h = (2.0 * x.T @ x / 256).astype(np.float32)
    c0 = rng.integers(0, 65536, size=(out, inp // 8, 1)).astype(np.uint16)
    got = _gpu_encode16(w, h, cb, c0, 1)
    want, f_oracle = oracle.encode(w, h, cb, c0, 1)
    f_gpu = oracle.objective(w, h, cb, got)
    f_start = oracle.objective(w, h, cb, c0)
    assert np.all(f_gpu <= f_start)
    assert np.all(f_gpu <= f_oracle * (1 + 1e-4) + 1e-6)
    assert (got == want).mean() > 0.9
