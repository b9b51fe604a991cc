"""Degenerate layers whose products the CUDA path must reproduce exactly.

One-hot codebooks (every codeword is +e_p or -e_p) make each group of W the
sum of K signed unit vectors, so the product reduces to the textbook dense
matrix-vector product of that integer W.  With activations in {-1, 0, 1},
power-of-two row scales and K one-hot terms per group (at most
K * in / 8 <= 520 nonzero products per output), every partial sum any
kernel forms is an integer of magnitude below 2048,
exact in fp32 whatever the order; the final scale and binary16 rounding
are exact too.  So the decode-time product (table, CUDA-core and
tensor-core paths, any split) and the prefill product must equal the dense
product exactly, not just within the tolerance.  The same holds for a 1x16
layer whose codes all select one codeword (every gather hits one address).

The parameter gradient has the same property on these layers: with gy in
{-1, 0, 1} as well, M = gy x^T holds integers of magnitude at most T, and
dL/ds and dL/dC are sums of integers and half-integers far below 2^24, so
the order of the kernel's atomics and shared-memory scatter cannot change
them: they must equal the oracle's fp64 values exactly.
"""
import numpy as np
import pytest
import torch

import additive_quantized_matmul_b200 as aq
import oracle
from aq_inputs import Layer, LayerSpec
from aqtest import DevLayer, dev, run_gemm, run_gemv, workspace

pytestmark = pytest.mark.gpu

# (K, B, in_features), K * in / 8 <= 520.  1000 rows: 8 row tiles, the last
# ragged.  1x16 at 1032 takes the CUDA-core path at batch 1 and 2, at 4104
# the tensor cores; 8-bit schemes take the table path at batch 1.  Group
# counts 129, 513, 257, 65 leave a ragged last block of 32 groups.
CASES = [(1, 16, 1032), (1, 16, 4104), (2, 8, 520), (2, 8, 2056), (1, 8, 1032), (2, 16, 520), (8, 8, 520)]


def _one_hot_layer(out, inp, K, B, seed):
    rng = np.random.default_rng(seed)
    n = 1 << B
    cb = np.zeros((K, n, 8), dtype=np.float16)
    pos = rng.integers(0, 8, size=(K, n))
    sign = rng.choice(np.array([-1.0, 1.0]), size=(K, n))
    for k in range(K):
        cb[k, np.arange(n), pos[k]] = sign[k]
    codes = rng.integers(0, n, size=(out, inp // 8, K)).astype(np.uint8 if B <= 8 else np.uint16)
    scales = rng.choice(np.array([0.5, 1.0, 2.0]), size=out).astype(np.float16)
    return Layer(LayerSpec(out, inp, K, B), codes, cb, scales)


def _dense(layer):
    """W [out][in] in float64 from the construction (no decode routine)."""
    out, G, K = layer.codes.shape
    cb = layer.codebooks.astype(np.float64)
    W = np.zeros((out, G, 8))
    for k in range(K):
        W += cb[k][layer.codes[:, :, k].astype(np.int64)]
    return W.reshape(out, G * 8)


def _int_activations(inp, n, seed):
    return np.random.default_rng(seed).integers(-1, 2, size=(inp, n)).astype(np.float16)


def _expected(layer, x):
    y = layer.scales.astype(np.float64)[:, None] * (_dense(layer) @ x.astype(np.float64))
    assert np.abs(y).max() <= 2 * 520  # the bound of the module docstring
    assert np.array_equal(y.astype(np.float16).astype(np.float64), y)
    return y


@pytest.mark.parametrize("K,B,inp", CASES)
@pytest.mark.parametrize("batch", [1, 2, 4, 16])
def test_gemv_one_hot_codebooks_exact(K, B, inp, batch):
    layer = _one_hot_layer(1000, inp, K, B, 7 * K + B + batch)
    x = _int_activations(inp, batch, batch)
    want = _expected(layer, x)
    ref, _ = oracle.matmul(layer.codes, layer.codebooks, layer.scales, x)
    assert np.array_equal(ref, want)
    got = run_gemv(DevLayer(layer), x)
    bad = np.flatnonzero(got != want)
    assert bad.size == 0, f"{K}x{B} b{batch}: {bad.size} outputs differ, first {got.flat[bad[0]]} vs {want.flat[bad[0]]}"


@pytest.mark.parametrize("K,B,inp", CASES)
@pytest.mark.parametrize("T", [5, 64, 520])
def test_gemm_one_hot_codebooks_exact(K, B, inp, T):
    layer = _one_hot_layer(1000, inp, K, B, 11 * K + B + T)
    x = _int_activations(inp, T, T)
    want = _expected(layer, x)
    got = run_gemm(DevLayer(layer), x)
    bad = np.flatnonzero(got != want)
    assert bad.size == 0, f"{K}x{B} T{T}: {bad.size} outputs differ, first {got.flat[bad[0]]} vs {want.flat[bad[0]]}"


@pytest.mark.parametrize("code", [0, 65535])
@pytest.mark.parametrize("batch", [1, 4])
def test_gemv_every_code_the_same_codeword(code, batch):
    """1x16, 4096 x 1032: all 528 k codes select codeword `code`, so every
    gather of the launch reads one address."""
    layer = _one_hot_layer(4096, 1032, 1, 16, 3)
    layer = Layer(layer.spec, np.full_like(layer.codes, code), layer.codebooks, layer.scales)
    x = _int_activations(1032, batch, 40 + batch)
    want = _expected(layer, x)
    got = run_gemv(DevLayer(layer), x)
    assert np.array_equal(got, want)


@pytest.mark.parametrize("K,B,inp", CASES)
@pytest.mark.parametrize("T", [64, 136])
def test_param_grad_one_hot_codebooks_exact(K, B, inp, T):
    layer = _one_hot_layer(1000, inp, K, B, 13 * K + B + T)
    x = _int_activations(inp, T, T)
    gy = _int_activations(1000, T, T + 1)
    dl = DevLayer(layer)
    gs = torch.full((1000,), float("nan"), dtype=torch.float32, device="cuda")
    gc = torch.full(((K << B) * 8,), float("nan"), dtype=torch.float32, device="cuda")
    ws = workspace(aq.aq_param_grad_workspace_bytes(dl.desc, T))
    aq.aq_param_grad(dl.desc, dl.packed, dl.codebooks, dl.scales, dev(x.view(np.uint16)),
                     dev(gy.view(np.uint16)), T, gs, gc, ws)
    torch.cuda.synchronize()
    assert aq.aq_workspace_status(ws) == 0
    rs, _, rc, _ = oracle.backward(layer.codes, layer.codebooks, layer.scales, x, gy)
    assert np.abs(rc).max() < 2 ** 22 and np.abs(rs).max() < 2 ** 22
    got_s = gs.cpu().numpy().astype(np.float64)
    got_c = gc.cpu().numpy().astype(np.float64)
    bad_s = np.flatnonzero(got_s != rs)
    bad_c = np.flatnonzero(got_c != rc.ravel())
    assert bad_s.size == 0, f"{K}x{B} T{T} grad_s: {bad_s.size} differ"
    assert bad_c.size == 0, f"{K}x{B} T{T} grad_C: {bad_c.size} differ"
