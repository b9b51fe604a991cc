"""Pins for the CPU oracle: checks that tie it to something other than itself.

Each test fixes the oracle against what the pages or the mathematics fix --
the pages' worked bit-rate examples and model sizes, closed forms,
invariants, exhaustive enumeration, library routines for special cases, and
exact brute force on tiny inputs -- chosen so that a dropped term, a wrong
index, a transposed operand or a wrong rounding fails at least one of them.

Pages: "Extreme Compression of Large Language Models via Additive
Quantization" -- AQLM wiki entry (brain.gartu.xyz), "Niveau intermédiaire";
devtrends.ru summary, "Как это работает технически?", "Схемы квантования",
"Почему это важно?".
"""
import json
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle
from aq_inputs import LayerSpec, make_activations, make_layer


# ---------------------------------------------------------------------------
# binary16 conversions (IEEE 754 definition) against numpy's float16
# ---------------------------------------------------------------------------

def test_half_to_double_all_patterns():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = bits.view(np.float16).astype(np.float64)
    got = np.array([oracle.half_to_double(int(b)) for b in bits])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])
    # signed zero keeps its sign
    assert np.signbit(got[0x8000]) and not np.signbit(got[0])


def test_double_to_half_roundtrip_all_finite():
    for b in range(65536):
        v = np.uint16(b).view(np.float16)
        if np.isnan(v):
            assert (oracle.double_to_half(float(v)) & 0x7C00) == 0x7C00
            continue
        assert oracle.double_to_half(float(v)) == b


def test_double_to_half_midpoints_round_to_even():
    pos = np.arange(0, 0x7C00, dtype=np.uint16).view(np.float16).astype(np.float64)
    mids = (pos[:-1] + pos[1:]) / 2.0  # exact in float64
    ref = mids.astype(np.float16).view(np.uint16)
    got = np.array([oracle.double_to_half(m) for m in mids], dtype=np.uint16)
    assert np.array_equal(got, ref)
    # ties go to the even significand: 1 + 2^-11 lies between 1 and 1 + 2^-10
    assert oracle.double_to_half(1.0 + 2.0 ** -11) == 0x3C00
    assert oracle.double_to_half(1.0 + 3 * 2.0 ** -11) == 0x3C02


def test_double_to_half_random_against_numpy():
    rng = np.random.default_rng(7)
    mag = 10.0 ** rng.uniform(-9, 5.5, size=100_000)
    v = mag * rng.choice([-1.0, 1.0], size=mag.size)
    with np.errstate(over="ignore"):
        ref = v.astype(np.float16).view(np.uint16)
    got = np.array([oracle.double_to_half(x) for x in v], dtype=np.uint16)
    assert np.array_equal(got, ref)


def test_double_to_half_edges():
    assert oracle.double_to_half(65504.0) == 0x7BFF
    assert oracle.double_to_half(65519.99) == 0x7BFF
    assert oracle.double_to_half(65520.0) == 0x7C00
    assert oracle.double_to_half(-1e9) == 0xFC00
    assert oracle.double_to_half(2.0 ** -25) == 0x0000  # tie to even (zero)
    assert oracle.double_to_half(2.0 ** -25 * 1.0000001) == 0x0001
    assert oracle.double_to_half(3 * 2.0 ** -25) == 0x0002  # tie 1.5 ulp -> 2
    assert oracle.double_to_half(-0.0) == 0x8000
    assert oracle.double_to_half(2.0 ** -14 - 2.0 ** -26) == 0x0400  # rounds up into normals


# ---------------------------------------------------------------------------
# Bit rate closed form and the storage it implies
# ---------------------------------------------------------------------------

def test_bitrate_page_examples(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "bitrate_examples.json")))
    for ex in g["examples"]:
        B = int(ex["codebook_size"]).bit_length() - 1
        assert (1 << B) == ex["codebook_size"]
        assert oracle.bits_per_weight(ex["K"], B, ex["group_size"]) == ex["bits_per_weight"]
    for case in g["schemes"]["cases"]:
        assert oracle.bits_per_weight(case["K"], case["B"], 8) == case["bits_per_weight"]


@pytest.mark.parametrize("K,B", [(1, 16), (2, 8), (1, 8), (2, 16), (8, 8)])
@pytest.mark.parametrize("out,inp", [(4096, 4096), (11008, 4096), (8, 256)])
def test_packed_size_matches_bitrate(K, B, out, inp):
    # aligned shapes carry no padding: bytes * 8 / weights == K * B / 8
    assert oracle.packed_bytes(out, inp, K, B) * 8 / (out * inp) == oracle.bits_per_weight(K, B)


def test_model_sizes_from_page(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "model_sizes.json")))
    for m in g["models"]:
        h, mlp, kv, L, V = m["hidden"], m["mlp"], m["kv"], m["layers"], m["vocab"]
        linears = [(h, h), (kv, h), (kv, h), (h, h), (mlp, h), (mlp, h), (h, mlp)]
        q = sum(oracle.layer_bytes(o, i, 1, 16) for o, i in linears) * L
        dense = 2 * V * h * 2 + (2 * L + 1) * h * 2  # embeddings, head, norms (binary16)
        size_gb = (q + dense) / 1e9
        assert abs(size_gb - m["printed_gb"]) < 0.05, (m["name"], size_gb)


def test_layer_bytes_terms():
    # codes, codebook and scales, each term checked on its own
    assert oracle.layer_bytes(1, 8, 1, 16) == 2 + 65536 * 16 + 2
    assert oracle.layer_bytes(3, 16, 2, 8) == 3 * 2 * 2 + 2 * 256 * 16 + 3 * 2


# ---------------------------------------------------------------------------
# Decode: W[o][8g+j] = RN16(sum_k C_k[codes[o][g][k]][j])
# ---------------------------------------------------------------------------

def _cb(K, B, sigma, seed):
    rng = np.random.default_rng(seed)
    return rng.normal(0, sigma, size=(K, 1 << B, 8)).astype(np.float16)


def test_decode_exhaustive_2x8_group():
    cb = _cb(2, 8, 0.05, 1)
    i0, i1 = np.meshgrid(np.arange(256), np.arange(256), indexing="ij")
    codes = np.stack([i0.ravel(), i1.ravel()], axis=-1).astype(np.uint8)[:, None, :]
    w = oracle.decode(codes, cb)  # [65536][8]
    ref = (cb[0][i0.ravel()].astype(np.float64) + cb[1][i1.ravel()].astype(np.float64)).astype(np.float16)
    assert np.array_equal(w.view(np.uint16), ref.view(np.uint16))


def test_decode_1x16_is_verbatim():
    cb = _cb(1, 16, 0.02, 2)
    codes = np.arange(65536, dtype=np.uint16).reshape(4096, 16, 1)
    w = oracle.decode(codes, cb)  # row o holds codewords 16o .. 16o+15
    assert np.array_equal(w.reshape(65536, 8).view(np.uint16), cb[0].view(np.uint16))


def test_decode_one_hot_codebook_reconstructs_exactly():
    # K=1, B=8: codeword c = v_c * e_(c mod 8); any W whose groups are
    # codewords is reconstructed exactly, in the right row and column.
    v = (np.arange(256) - 128.0) / 4.0  # distinct, exactly representable
    cb = np.zeros((1, 256, 8), dtype=np.float16)
    cb[0, np.arange(256), np.arange(256) % 8] = v
    rng = np.random.default_rng(3)
    out, G = 5, 7
    codes = rng.integers(0, 256, size=(out, G, 1)).astype(np.uint8)
    W = np.zeros((out, G * 8))
    for o in range(out):
        for g in range(G):
            c = codes[o, g, 0]
            W[o, 8 * g + c % 8] = v[c]
    assert np.array_equal(oracle.decode(codes, cb).astype(np.float64), W)


def test_decode_additivity():
    cb = _cb(2, 8, 0.05, 4)
    rng = np.random.default_rng(5)
    codes = rng.integers(0, 256, size=(9, 6, 2)).astype(np.uint8)
    w2 = oracle.decode(codes, cb)
    w0 = oracle.decode(codes[:, :, 0:1], cb[0:1])  # single codebooks decode exactly
    w1 = oracle.decode(codes[:, :, 1:2], cb[1:2])
    ref = (w0.astype(np.float64) + w1.astype(np.float64)).astype(np.float16)
    assert np.array_equal(w2.view(np.uint16), ref.view(np.uint16))


def test_decode_integer_codebooks_exact():
    rng = np.random.default_rng(6)
    cb = rng.integers(-8, 9, size=(2, 256, 8)).astype(np.float16)
    codes = rng.integers(0, 256, size=(4, 3, 2)).astype(np.uint8)
    w = oracle.decode(codes, cb).astype(np.float64)
    for o in range(4):
        for g in range(3):
            for j in range(8):
                want = int(cb[0, codes[o, g, 0], j]) + int(cb[1, codes[o, g, 1], j])
                assert w[o, 8 * g + j] == want


def test_decode_permutation_invariance():
    cb = _cb(2, 8, 0.05, 8)
    rng = np.random.default_rng(9)
    codes = rng.integers(0, 256, size=(6, 4, 2)).astype(np.uint8)
    perm = [rng.permutation(256) for _ in range(2)]
    cbp = np.stack([cb[k][perm[k]] for k in range(2)])  # cbp[k][c] = cb[k][perm[k][c]]
    inv = [np.argsort(p) for p in perm]
    codesp = np.stack([inv[k][codes[:, :, k]] for k in range(2)], axis=-1).astype(np.uint8)
    assert np.array_equal(oracle.decode(codes, cb).view(np.uint16),
                          oracle.decode(codesp, cbp).view(np.uint16))


def test_decode_scaled_is_one_rounding():
    layer = make_layer(LayerSpec(16, 64, 2, 8, codebook_sigma=0.05), 10)
    w = oracle.decode(layer.codes, layer.codebooks)
    ws = oracle.decode(layer.codes, layer.codebooks, layer.scales)
    ref = (layer.scales.astype(np.float64)[:, None] * w.astype(np.float64)).astype(np.float16)
    assert np.array_equal(ws.view(np.uint16), ref.view(np.uint16))


def test_decode_rounds_the_sum_not_the_terms():
    # 1 + 2^-11 ties to 1.0 (even); 1 + 2^-11 + 2^-11 would be 1 + 2^-10
    cb = np.zeros((2, 256, 8), dtype=np.float16)
    cb[0, 1, :] = 1.0
    cb[1, 2, :] = 2.0 ** -11
    codes = np.array([[[1, 2]]], dtype=np.uint8)
    assert np.all(oracle.decode(codes, cb).view(np.uint16) == 0x3C00)
    cb[1, 2, :] = 3 * 2.0 ** -11  # 1 + 3*2^-11 ties to 1 + 2^-9 (even)
    assert np.all(oracle.decode(codes, cb).view(np.uint16) == 0x3C02)


def test_decode_signed_zero_follows_ieee_sum():
    # the sum starts from the first codeword: -0 alone stays -0,
    # (-0) + (-0) = -0 and (+0) + (-0) = +0 under round-to-nearest
    cb = np.zeros((2, 256, 8), dtype=np.float16)
    cb[:, 1, :] = -0.0
    neg = np.array([[[1, 1]]], dtype=np.uint8)
    mixed = np.array([[[0, 1]]], dtype=np.uint8)
    assert np.all(oracle.decode(neg, cb).view(np.uint16) == 0x8000)
    assert np.all(oracle.decode(mixed, cb).view(np.uint16) == 0x0000)
    assert np.all(oracle.decode(neg[:, :, :1], cb[:1]).view(np.uint16) == 0x8000)


# ---------------------------------------------------------------------------
# Product y = diag(s) W x
# ---------------------------------------------------------------------------

def _dyadic_layer(out, inp, K, B, seed):
    rng = np.random.default_rng(seed)
    cb = (rng.integers(-32, 33, size=(K, 1 << B, 8)) / 8.0).astype(np.float16)
    codes = rng.integers(0, 1 << B, size=(out, inp // 8, K)).astype(np.uint8 if B <= 8 else np.uint16)
    s = rng.choice([0.5, 0.75, 1.0, 1.25, 1.5], size=out).astype(np.float16)
    return codes, cb, s


@pytest.mark.parametrize("out,inp,K,B,n", [(1, 8, 1, 2, 1), (3, 16, 2, 2, 2), (4, 16, 2, 8, 3),
                                           (2, 8, 1, 8, 1), (4, 8, 2, 2, 4), (2, 16, 8, 8, 2),
                                           (3, 8, 2, 16, 1), (2, 16, 4, 3, 2)])
def test_matmul_brute_force_exact(out, inp, K, B, n):
    """Triple loop over (g, j, k) in exact rationals, without forming W."""
    codes, cb, s = _dyadic_layer(out, inp, K, B, out * 100 + inp + K + B)
    rng = np.random.default_rng(n)
    x = (rng.integers(-16, 17, size=(inp, n)) / 4.0).astype(np.float16)
    y, _ = oracle.matmul(codes, cb, s, x)
    for o in range(out):
        for b in range(n):
            acc = Fraction(0)
            for g in range(inp // 8):
                for j in range(8):
                    for k in range(K):
                        acc += Fraction(float(cb[k, codes[o, g, k], j])) * Fraction(float(x[8 * g + j, b]))
            assert y[o, b] == float(Fraction(float(s[o])) * acc)


def test_decode_eight_codebooks_one_rounding_of_exact_sum():
    """K = 8: each weight is the exact sum of eight binary16 terms of widely
    different magnitudes, rounded once (checked against numpy's binary16
    conversion of the exact rational sum, which is exact in a double)."""
    rng = np.random.default_rng(21)
    K, B = 8, 8
    mant = rng.integers(1024, 2048, size=(K, 1 << B, 8))
    expo = rng.integers(-24, 6, size=(K, 1 << B, 8))
    sign = rng.choice([-1.0, 1.0], size=(K, 1 << B, 8))
    cb = (sign * mant * np.exp2(expo - 10.0)).astype(np.float16)
    assert np.all(np.isfinite(cb))
    out, G = 6, 5
    codes = rng.integers(0, 1 << B, size=(out, G, K)).astype(np.uint8)
    w = oracle.decode(codes, cb)
    for o in range(out):
        for g in range(G):
            for j in range(8):
                exact = sum(Fraction(float(cb[k, codes[o, g, k], j])) for k in range(K))
                assert w[o, 8 * g + j].view(np.uint16) == np.float16(float(exact)).view(np.uint16)


def test_decode_eight_codebooks_rounds_the_sum_not_the_terms():
    # 1 + 7 * 2^-12 = 1 + 1.75 ulp: one rounding gives 1 + 2 ulp, while
    # rounding after every addition would stay at 1
    cb = np.zeros((8, 256, 8), dtype=np.float16)
    cb[0, 1, 0] = 1.0
    cb[1:, 1, 0] = 2.0 ** -12
    codes = np.ones((1, 1, 8), dtype=np.uint8)
    w = oracle.decode(codes, cb)
    assert float(w[0, 0]) == 1.0 + 2.0 ** -9


def test_matmul_uses_rounded_weights():
    cb = np.zeros((2, 256, 8), dtype=np.float16)
    cb[0, 1, 0] = 1.0
    cb[1, 2, 0] = 2.0 ** -11  # W[0][0] = RN16(1 + 2^-11) = 1
    codes = np.array([[[1, 2]]], dtype=np.uint8)
    x = np.zeros((8, 1), dtype=np.float16)
    x[0, 0] = 1.0
    y, _ = oracle.matmul(codes, cb, np.ones(1, np.float16), x)
    assert y[0, 0] == 1.0


def test_matmul_one_hot_reduces_to_dense_product():
    v = (np.arange(256) - 128.0) / 4.0
    cb = np.zeros((1, 256, 8), dtype=np.float16)
    cb[0, np.arange(256), np.arange(256) % 8] = v
    rng = np.random.default_rng(11)
    out, G, n = 13, 9, 5
    codes = rng.integers(0, 256, size=(out, G, 1)).astype(np.uint8)
    W = np.zeros((out, G * 8))
    for o in range(out):
        for g in range(G):
            W[o, 8 * g + codes[o, g, 0] % 8] = v[codes[o, g, 0]]
    x = make_activations(G * 8, n, 12)
    y, _ = oracle.matmul(codes, cb, np.ones(out, np.float16), x)
    ref = W @ x.astype(np.float64)
    np.testing.assert_allclose(y, ref, rtol=1e-13, atol=1e-13)


def test_matmul_matches_numpy_on_random_layer():
    layer = make_layer(LayerSpec(40, 96, 2, 8, codebook_sigma=0.05), 13)
    x = make_activations(96, 3, 14)
    y, bound = oracle.matmul(layer.codes, layer.codebooks, layer.scales, x)
    W = oracle.decode(layer.codes, layer.codebooks).astype(np.float64)
    ref = layer.scales.astype(np.float64)[:, None] * (W @ x.astype(np.float64))
    np.testing.assert_allclose(y, ref, rtol=0, atol=1e-12 * bound.max())
    refb = np.abs(layer.scales.astype(np.float64))[:, None] * (np.abs(W) @ np.abs(x.astype(np.float64)))
    np.testing.assert_allclose(bound, refb, rtol=1e-12)
    assert np.all(bound >= np.abs(y) * (1 - 1e-12))


def test_matmul_linearity_and_rows():
    layer = make_layer(LayerSpec(24, 64, 1, 16), 15)
    x = make_activations(64, 2, 16)
    y, _ = oracle.matmul(layer.codes, layer.codebooks, layer.scales, x)
    y2, _ = oracle.matmul(layer.codes, layer.codebooks, layer.scales, (x.astype(np.float64) * 2).astype(np.float16))
    assert np.array_equal(y2, 2 * y)
    s4 = (layer.scales.astype(np.float64) * 4).astype(np.float16)
    y4, _ = oracle.matmul(layer.codes, layer.codebooks, s4, x)
    assert np.array_equal(y4, 4 * y)
    rows = np.array([23, 0, 7, 7])
    yr, _ = oracle.matmul(layer.codes, layer.codebooks, layer.scales, x, rows=rows)
    assert np.array_equal(yr, y[rows])
    yt, _ = oracle.matmul(layer.codes, layer.codebooks, layer.scales, x, threads=4)
    assert np.array_equal(yt, y)


# ---------------------------------------------------------------------------
# Packed layout
# ---------------------------------------------------------------------------

def test_pack_hand_worked_offsets(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "pack_offsets.json")))
    L = g["layer"]
    assert oracle.packed_bytes(L["out"], L["in"], 1, 16) == L["packed_bytes"]
    assert oracle.packed_bytes(L["out"], L["in"], 2, 8) == L["packed_bytes"]
    G = L["in"] // 8
    # 1x16: every code distinct, so its position identifies it
    codes = (np.arange(L["out"] * G, dtype=np.uint32) + 1).astype(np.uint16).reshape(L["out"], G, 1)
    packed = oracle.pack(codes, 1, 16)
    for e in g["offsets"]:
        word = int(packed[e["byte"]]) | (int(packed[e["byte"] + 1]) << 8)
        assert word == codes[e["o"], e["g"], 0]
    # 2x8: byte 0 of the word is codebook 0, byte 1 codebook 1
    c2 = np.zeros((L["out"], G, 2), dtype=np.uint8)
    c2[13, 40] = (0xAB, 0xCD)
    p2 = oracle.pack(c2, 2, 8)
    assert p2[2186] == 0xAB and p2[2187] == 0xCD
    assert int(p2.astype(np.int64).sum()) == 0xAB + 0xCD


def test_pack_hand_worked_offsets_wide_words(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "pack_offsets_wide.json")))
    L = g["layer"]
    G = L["in"] // 8
    for sch in g["schemes"]:
        K, B, W = sch["K"], sch["B"], sch["W"]
        assert oracle.packed_bytes(L["out"], L["in"], K, B) == sch["packed_bytes"]
        dt = np.uint8 if B <= 8 else np.uint16
        # one nonzero code at a time: its bytes must sit at the worked offset
        for key, byte in g["offsets_bytes"][str(W)].items():
            o, gg = map(int, key.split(","))
            codes = np.zeros((L["out"], G, K), dtype=dt)
            codes[o, gg, 0] = 0x5A
            p = oracle.pack(codes, K, B)
            assert p[byte] == 0x5A and int(p.astype(np.int64).sum()) == 0x5A, (K, B, key)
        for e in g["offsets_in_words"]:
            codes = np.zeros((L["out"], G, K), dtype=dt)
            codes[e["o"], e["g"], 0] = 0x33
            p = oracle.pack(codes, K, B)
            assert p[e["word"] * W] == 0x33, (K, B, e)
    # byte order inside a word
    c = np.zeros((L["out"], G, 2), dtype=np.uint16)
    c[0, 0] = (0x1234, 0xABCD)
    assert list(oracle.pack(c, 2, 16)[:4]) == [0x34, 0x12, 0xCD, 0xAB]
    c8 = np.zeros((L["out"], G, 8), dtype=np.uint8)
    c8[0, 0] = np.arange(1, 9)
    assert list(oracle.pack(c8, 8, 8)[:8]) == list(range(1, 9))


@pytest.mark.parametrize("out,inp,K,B", [(1, 8, 1, 16), (20, 520, 1, 16), (20, 520, 2, 8),
                                         (37, 8 * 45, 2, 8), (256, 512, 2, 8), (20, 520, 1, 8),
                                         (37, 8 * 45, 2, 16), (20, 520, 8, 8), (1, 8, 8, 8)])
def test_pack_roundtrip_and_padding(out, inp, K, B):
    spec = LayerSpec(out, inp, K, B)
    layer = make_layer(spec, out + inp)
    packed = oracle.pack(layer.codes, K, B)
    assert np.array_equal(oracle.unpack(packed, out, inp, K, B), layer.codes)
    rows = -(-out // 8) * 8
    gp = -(-(inp // 8) // 32) * 32
    assert packed.size == rows * gp * K * B // 8
    # zero padding: the byte sum equals the code-byte sum
    assert int(packed.astype(np.int64).sum()) == int(layer.codes.view(np.uint8).astype(np.int64).sum())


# ---------------------------------------------------------------------------
# Gradient with respect to scales and codebooks
# ---------------------------------------------------------------------------

def _loss(codes, cb, s, x, gy):
    """L = sum(gy * y) from the forward product, in exact rationals."""
    y, _ = oracle.matmul(codes, cb, s, x)
    return sum(Fraction(float(gy[o, b])) * Fraction(float(y[o, b]))
               for o in range(y.shape[0]) for b in range(y.shape[1]))


@pytest.mark.parametrize("out,inp,K,B,n", [(3, 16, 2, 3, 2), (2, 24, 1, 4, 3), (4, 8, 8, 2, 1),
                                           (2, 16, 2, 8, 2), (3, 8, 1, 16, 2)])
def test_backward_matches_finite_differences_exactly(out, inp, K, B, n):
    """Dyadic inputs keep every decode exact, so L is linear in each codebook
    entry and each scale and a unit finite difference of the forward product
    is the exact partial derivative."""
    codes, cb, s = _dyadic_layer(out, inp, K, B, out + inp + K + B + n)
    rng = np.random.default_rng(out * 31 + n)
    x = (rng.integers(-8, 9, size=(inp, n)) / 4.0).astype(np.float16)
    gy = (rng.integers(-8, 9, size=(out, n)) / 4.0).astype(np.float16)
    gs, _, gc, _ = oracle.backward(codes, cb, s, x, gy)
    base = _loss(codes, cb, s, x, gy)
    # every scale
    for o in range(out):
        s2 = s.copy()
        s2[o] = s2[o] + np.float16(0.25)
        assert (_loss(codes, cb, s2, x, gy) - base) * 4 == Fraction(float(gs[o])), o
    # codebook entries that are used, and one that is not (gradient 0)
    used = {(k, int(codes[o, g, k])) for o in range(out) for g in range(inp // 8) for k in range(K)}
    probe = sorted(used)[:6] + [(k, c) for k in range(K) for c in range(1 << B) if (k, c) not in used][:1]
    for k, c in probe:
        for j in (0, 3, 7):
            cb2 = cb.copy()
            cb2[k, c, j] = cb2[k, c, j] + np.float16(0.125)
            assert (_loss(codes, cb2, s, x, gy) - base) * 8 == Fraction(float(gc[k, c, j])), (k, c, j)


def test_backward_euler_identity():
    """L is linear in the codebooks (exact decode) and in s, so
    sum(C * dL/dC) = L = sum_o s_o dL/ds_o."""
    codes, cb, s = _dyadic_layer(5, 64, 2, 4, 9)
    rng = np.random.default_rng(3)
    x = (rng.integers(-8, 9, size=(64, 4)) / 4.0).astype(np.float16)
    gy = (rng.integers(-8, 9, size=(5, 4)) / 4.0).astype(np.float16)
    gs, _, gc, _ = oracle.backward(codes, cb, s, x, gy)
    L = _loss(codes, cb, s, x, gy)
    assert sum(Fraction(float(a)) * Fraction(float(b)) for a, b in zip(cb.ravel(), gc.ravel())) == L
    assert sum(Fraction(float(a)) * Fraction(float(b)) for a, b in zip(s, gs)) == L


def test_backward_bounds_dominate():
    layer = make_layer(LayerSpec(40, 264, 2, 8, codebook_sigma=0.05), 8)
    x = make_activations(264, 6, 1)
    gy = make_activations(40, 6, 2)
    gs, gsb, gc, gcb = oracle.backward(layer.codes, layer.codebooks, layer.scales, x, gy)
    assert np.all(np.abs(gs) <= gsb) and np.all(np.abs(gc) <= gcb)
    assert np.all(gcb >= 0) and gsb.min() > 0


# ---------------------------------------------------------------------------
# Encoder: beam search of the codes for fixed codebooks
# ---------------------------------------------------------------------------

def _int_problem(out, inp, K, B, seed):
    """Small-integer weights, codebooks and a positive definite H: every
    objective is an exact integer in fp32 and fp64."""
    rng = np.random.default_rng(seed)
    w = rng.integers(-4, 5, size=(out, inp)).astype(np.float16)
    a = rng.integers(-1, 2, size=(inp, inp)).astype(np.float32)
    h = (a.T @ a + np.eye(inp, dtype=np.float32)).astype(np.float32)
    cb = rng.integers(-2, 3, size=(K, 1 << B, 8)).astype(np.float16)
    c0 = rng.integers(0, 1 << B, size=(out, inp // 8, K)).astype(np.uint8 if B <= 8 else np.uint16)
    return w, h, cb, c0


def _np_objective(w, h, cb, codes):
    out, inp = w.shape
    K = cb.shape[0]
    res = []
    for o in range(out):
        what = np.concatenate([sum(cb[k, codes[o, g, k]].astype(np.float64) for k in range(K))
                               for g in range(inp // 8)])
        e = w[o].astype(np.float64) - what
        res.append(float(e @ h.astype(np.float64) @ e))
    return np.array(res)


def test_encode_one_group_full_beam_is_exhaustive():
    """One group, beam = 2^B: the first slot keeps every code, the second
    tries every pair, so the result is the brute-force optimum (any H)."""
    w, h, cb, c0 = _int_problem(5, 8, 2, 3, 1)
    codes, obj = oracle.encode(w, h, cb, c0, beam=8)
    for o in range(5):
        best = min(_np_objective(w[o:o + 1], h, cb, np.array([[[a, b]]], dtype=np.uint8))[0]
                   for a in range(8) for b in range(8))
        assert obj[o] == best


def test_encode_identity_h_single_codebook_is_nearest_codeword():
    w, _, cb, c0 = _int_problem(4, 32, 1, 4, 2)
    h = np.eye(32, dtype=np.float32)
    codes, _ = oracle.encode(w, h, cb, c0, beam=1)
    for o in range(4):
        for g in range(4):
            d = ((cb[0].astype(np.float64) - w[o, 8 * g:8 * g + 8].astype(np.float64)) ** 2).sum(axis=1)
            assert d[codes[o, g, 0]] == d.min()
            assert codes[o, g, 0] == int(np.flatnonzero(d == d.min())[0])  # ties: smallest code


def test_encode_beam_one_is_greedy_coordinate_pass():
    w, h, cb, c0 = _int_problem(3, 24, 2, 2, 3)
    codes, obj = oracle.encode(w, h, cb, c0, beam=1)
    for o in range(3):
        cur = c0[o:o + 1].copy()
        for g in range(3):
            for k in range(2):
                scores = []
                for c in range(4):
                    t = cur.copy()
                    t[0, g, k] = c
                    scores.append(_np_objective(w[o:o + 1], h, cb, t)[0])
                cur[0, g, k] = int(np.argmin(scores))  # first minimum: smallest code
        assert np.array_equal(codes[o], cur[0])
        assert obj[o] == _np_objective(w[o:o + 1], h, cb, cur)[0]


@pytest.mark.parametrize("K,B,beam", [(1, 4, 1), (2, 3, 4), (2, 4, 8), (8, 2, 3)])
def test_encode_never_worse_than_start_and_objective_consistent(K, B, beam):
    w, h, cb, c0 = _int_problem(6, 32, K, B, K * 10 + B + beam)
    codes, obj = oracle.encode(w, h, cb, c0, beam=beam)
    start = _np_objective(w, h, cb, c0)
    assert np.all(obj <= start)
    assert np.array_equal(obj, _np_objective(w, h, cb, codes))
    assert np.array_equal(oracle.objective(w, h, cb, codes), obj)


def test_encode_ties_resolved_by_parent_beam_then_code():
    """Hand-worked tie (one group, K = 3, B = 2, beam 2, H = I, lane 0 only).
    Target 3; codebook 0 holds 2 (code 1) and 0 (code 2), codebook 1 holds 0
    (code 0) and -2 (code 1), codebook 2 holds 0 (code 0) and 3 (code 1);
    every other codeword is 100.  Codebook 0 keeps beams [code 1 (error 1),
    code 2 (error 9)].  Codebook 1: the best is (beam 0, code 0) with error
    1, then (beam 0, code 1) and (beam 1, code 0) tie at 9 -- the lower
    parent beam goes first, so the second beam is (1, 1).  Codebook 2: that
    beam plus code 1 reaches the target exactly, giving codes (1, 1, 1);
    ordering ties by code alone would give (2, 0, 1) at the same objective."""
    cb = np.full((3, 4, 8), 0.0, dtype=np.float16)
    cb[:, :, 0] = 100.0
    cb[0, 1, 0], cb[0, 2, 0] = 2.0, 0.0
    cb[1, 0, 0], cb[1, 1, 0] = 0.0, -2.0
    cb[2, 0, 0], cb[2, 1, 0] = 0.0, 3.0
    w = np.zeros((1, 8), dtype=np.float16)
    w[0, 0] = 3.0
    c0 = np.zeros((1, 1, 3), dtype=np.uint8)
    codes, obj = oracle.encode(w, np.eye(8, dtype=np.float32), cb, c0, beam=2)
    assert codes[0, 0].tolist() == [1, 1, 1]
    assert obj[0] == 0.0


def test_encode_full_beam_is_sequential_exhaustive_per_group():
    """beam = 2^B: each group's code pair is the brute-force optimum given
    the groups before it (already chosen) and after it (still initial)."""
    w, h, cb, c0 = _int_problem(3, 24, 2, 2, 7)
    codes, obj = oracle.encode(w, h, cb, c0, beam=4)
    for o in range(3):
        cur = c0[o:o + 1].copy()
        for g in range(3):
            best = None
            for a in range(4):
                for b in range(4):
                    t = cur.copy()
                    t[0, g] = (a, b)
                    f = _np_objective(w[o:o + 1], h, cb, t)[0]
                    if best is None or f < best[0]:
                        best = (f, a, b)
            cur[0, g] = best[1:]
        assert np.array_equal(codes[o], cur[0]), o
        assert obj[o] == _np_objective(w[o:o + 1], h, cb, cur)[0]
