"""Inputs fenced by NaN: no kernel reads an input past either end.

Every input array (codes, packed codes, codebooks, scales, activations,
output gradients) is copied into the middle of a larger allocation, between
two 4 KiB bands of binary16 NaN (0x7E00), starting 16-byte aligned and
ending exactly where the second band begins.  A kernel that read an input
element beyond its extent and used it would turn outputs into NaN; so every
product must still match the oracle within the tolerance and the dequantised
weights bit for bit, and afterwards the bands must be unchanged (no kernel
writes into its inputs).  Ragged shapes put every tail (rows, groups,
stages, batch, tokens) against a band.
"""
import numpy as np
import pytest
import torch

import additive_quantized_matmul_b200 as aq
import oracle
from aq_inputs import LayerSpec, make_activations, make_layer
from aqtest import assert_close, desc_of, guarded, guards_intact, to_f16, workspace

pytestmark = pytest.mark.gpu

BAND = 4096
NAN16 = np.array([0x00, 0x7E], dtype=np.uint8)  # binary16 0x7E00, little-endian


def fenced(a: np.ndarray, device="cuda"):
    """(buffer, view): the bytes of `a` at offset BAND of a buffer whose
    other bytes are binary16 NaN."""
    raw = np.ascontiguousarray(a).reshape(-1).view(np.uint8)
    n = raw.size
    host = np.resize(NAN16, 2 * BAND + n + (n & 1))
    host[BAND:BAND + n] = raw
    buf = torch.from_numpy(host).to(device)
    return buf, buf[BAND:BAND + n]


def bands_intact(buf, n) -> bool:
    host = buf.cpu().numpy()
    pattern = np.resize(NAN16, host.size)
    return bool(np.array_equal(host[:BAND], pattern[:BAND]) and
                np.array_equal(host[BAND + n:], pattern[BAND + n:]))


@pytest.mark.parametrize("K,B", [(1, 16), (2, 8), (1, 8), (2, 16), (8, 8)])
@pytest.mark.parametrize("out,inp", [(37, 360), (1000, 1032)])
def test_no_input_read_past_its_ends(K, B, out, inp):
    layer = make_layer(LayerSpec(out, inp, K, B, codebook_sigma=0.05), (out, inp, K, B))
    desc = desc_of(layer.spec)
    fences = []

    def put(a):
        buf, view = fenced(a)
        fences.append((buf, view.numel()))
        return view

    codes = put(layer.codes)
    packed_buf = torch.empty(aq.aq_packed_codes_bytes(desc), dtype=torch.uint8, device="cuda")
    aq.aq_pack_codes(desc, codes, packed_buf)
    torch.cuda.synchronize()
    packed = put(packed_buf.cpu().numpy())
    cb = put(layer.codebooks)
    sc = put(layer.scales)

    w_full, w = guarded(out * inp)
    aq.aq_dequant(desc, packed, cb, sc, w)
    torch.cuda.synchronize()
    want = oracle.decode(layer.codes, layer.codebooks, layer.scales).view(np.uint16).ravel()
    assert np.array_equal(w.cpu().numpy().view(np.uint16), want), "dequant"
    assert guards_intact(w_full)

    for batch in (1, 3, 16):
        x = make_activations(inp, batch, (inp, batch))
        xd = put(x)
        y_full, y = guarded(out * batch)
        ws = workspace(aq.aq_gemv_workspace_bytes(desc, batch))
        aq.aq_gemv(desc, packed, cb, sc, xd, batch, y, ws)
        torch.cuda.synchronize()
        assert guards_intact(y_full)
        ref, bound = oracle.matmul(layer.codes, layer.codebooks, layer.scales, x)
        assert_close(to_f16(y).astype(np.float64).reshape(out, batch), ref, bound, f"gemv b{batch}")

    for T in (5, 64):
        x = make_activations(inp, T, (inp, T, 1))
        xd = put(x)
        y_full, y = guarded(out * T)
        ws = workspace(aq.aq_gemm_workspace_bytes(desc, T))
        aq.aq_gemm(desc, packed, cb, sc, xd, T, y, ws)
        torch.cuda.synchronize()
        assert aq.aq_workspace_status(ws) == 0
        assert guards_intact(y_full)
        ref, bound = oracle.matmul(layer.codes, layer.codebooks, layer.scales, x)
        assert_close(to_f16(y).astype(np.float64).reshape(out, T), ref, bound, f"gemm T{T}")

    for buf, n in fences:
        assert bands_intact(buf, n), "a kernel wrote into an input"
