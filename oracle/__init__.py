"""CPU oracle for additive-quantised matrix products (numpy-facing wrapper).

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference arm of ``bench.py`` may import this package.  The
CUDA library never imports, links or calls it, and it imports nothing from
the CUDA library.

The arithmetic lives in ``aq_oracle.c`` (plain C, fp64, no blocking); this
module compiles it with gcc on first use and marshals numpy arrays.  What it
computes, after "Extreme Compression of Large Language Models via Additive
Quantization" (AQLM wiki entry, "Niveau intermédiaire"; devtrends.ru summary,
"Как это работает технически?"):

* ``decode``:  W[o][8g+j] = RN16(sum_k C_k[codes[o][g][k]][j]) (optionally
  RN16(s[o] * W[o][i]));
* ``matmul``:  y[o][b] = s[o] * sum_i W[o][i] * x[i][b] in fp64, plus the
  per-element magnitude sum_i |s||W||x| used to scale the tolerance;
* ``backward``: gradients of sum(gy * y) with respect to the row scales and
  the codebook entries (the decode's rounding taken as the identity), with
  magnitude bounds;
* ``encode`` / ``objective``: beam search of each group's codes for fixed
  codebooks under e^T H e (the quantisation objective of the wiki entry),
  group after group, and that objective for given codes;
* ``pack`` / ``unpack``: the library's documented packed code layout;
* ``bits_per_weight`` and ``layer_bytes``: the bit-rate closed form and the
  storage it implies.

Binary16 values cross this interface as ``np.uint16`` bit patterns or
``np.float16`` arrays (viewed as uint16).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "aq_oracle.c")
_BUILD = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD, "libaqoracle.so")
_lock = threading.Lock()
_lib = None

_c_i64 = ctypes.c_int64
_c_int = ctypes.c_int
_vp = ctypes.c_void_p


def build(force: bool = False) -> str:
    """Compile ``aq_oracle.c`` into ``_build/libaqoracle.so`` (gcc, fp64,
    no fast-math, no FMA contraction)."""
    os.makedirs(_BUILD, exist_ok=True)
    stale = (not os.path.exists(_LIB_PATH)
             or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC))
    if force or stale:
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fopenmp",
               "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            lib.aqo_half_to_double.argtypes = [ctypes.c_uint16]
            lib.aqo_half_to_double.restype = ctypes.c_double
            lib.aqo_double_to_half.argtypes = [ctypes.c_double]
            lib.aqo_double_to_half.restype = ctypes.c_uint16
            lib.aqo_bits_per_weight.argtypes = [_c_int, _c_int, _c_int]
            lib.aqo_bits_per_weight.restype = ctypes.c_double
            lib.aqo_layer_bytes.argtypes = [_c_i64, _c_i64, _c_int, _c_int]
            lib.aqo_layer_bytes.restype = ctypes.c_double
            lib.aqo_decode.argtypes = [_c_i64, _c_i64, _c_int, _c_int, _vp, _vp, _vp, _vp]
            lib.aqo_decode.restype = _c_int
            lib.aqo_matmul.argtypes = [_c_i64, _c_i64, _c_int, _c_int, _vp, _vp, _vp,
                                       _vp, _c_i64, _vp, _c_i64, _vp, _vp, _c_int]
            lib.aqo_matmul.restype = _c_int
            lib.aqo_backward.argtypes = [_c_i64, _c_i64, _c_int, _c_int, _vp, _vp, _vp, _vp, _vp,
                                         _c_i64, _vp, _vp, _vp, _vp]
            lib.aqo_backward.restype = _c_int
            lib.aqo_encode.argtypes = [_c_i64, _c_i64, _c_int, _c_int, _vp, _vp, _vp, _vp, _c_int, _vp, _vp]
            lib.aqo_encode.restype = _c_int
            lib.aqo_objective.argtypes = [_c_i64, _c_i64, _c_int, _c_int, _vp, _vp, _vp, _vp, _vp]
            lib.aqo_objective.restype = _c_int
            lib.aqo_packed_bytes.argtypes = [_c_i64, _c_i64, _c_int, _c_int]
            lib.aqo_packed_bytes.restype = _c_i64
            lib.aqo_pack.argtypes = [_c_i64, _c_i64, _c_int, _c_int, _vp, _vp]
            lib.aqo_pack.restype = _c_int
            lib.aqo_unpack.argtypes = [_c_i64, _c_i64, _c_int, _c_int, _vp, _vp]
            lib.aqo_unpack.restype = _c_int
            lib.aqo_max_threads.argtypes = []
            lib.aqo_max_threads.restype = _c_int
            _lib = lib
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data


def _bits(a) -> np.ndarray:
    """binary16 array (float16 or uint16) -> contiguous uint16 bit patterns."""
    a = np.ascontiguousarray(a)
    if a.dtype == np.float16:
        return a.view(np.uint16)
    if a.dtype != np.uint16:
        raise TypeError(f"expected float16/uint16, got {a.dtype}")
    return a


def _codes(codes, K, B) -> np.ndarray:
    want = np.uint8 if B <= 8 else np.uint16
    codes = np.ascontiguousarray(codes)
    if codes.dtype != want:
        raise TypeError(f"codes must be {np.dtype(want).name} for B={B}")
    if codes.ndim != 3 or codes.shape[2] != K:
        raise ValueError("codes must be [out][in/8][K]")
    return codes


# -- scalar helpers ---------------------------------------------------------

def half_to_double(h: int) -> float:
    return _load().aqo_half_to_double(int(h) & 0xFFFF)


def double_to_half(v: float) -> int:
    return int(_load().aqo_double_to_half(float(v)))


def bits_per_weight(K: int, B: int, g: int = 8) -> float:
    return _load().aqo_bits_per_weight(K, B, g)


def layer_bytes(out: int, inp: int, K: int, B: int) -> float:
    return _load().aqo_layer_bytes(out, inp, K, B)


def max_threads() -> int:
    return _load().aqo_max_threads()


# -- array functions --------------------------------------------------------

def decode(codes, codebooks, scales=None) -> np.ndarray:
    """Dequantised W ``[out][in]`` as float16 (exact sum, one RN-even)."""
    cb = _bits(codebooks)
    K, ncw, g = cb.shape
    B = int(ncw).bit_length() - 1
    if g != 8 or (1 << B) != ncw:
        raise ValueError("codebooks must be [K][2**B][8]")
    codes = _codes(codes, K, B)
    out, G, _ = codes.shape
    s = None if scales is None else _bits(scales)
    w = np.empty((out, G * 8), dtype=np.uint16)
    rc = _load().aqo_decode(out, G * 8, K, B, _ptr(codes), _ptr(cb), _ptr(s), _ptr(w))
    if rc:
        raise RuntimeError(f"aqo_decode failed ({rc})")
    return w.view(np.float16)


def matmul(codes, codebooks, scales, x, rows=None, threads: int = 1):
    """``(y, bound)`` in float64; y = diag(s) W x for all rows or ``rows``."""
    cb = _bits(codebooks)
    K, ncw, _ = cb.shape
    B = int(ncw).bit_length() - 1
    codes = _codes(codes, K, B)
    out, G, _ = codes.shape
    xb = _bits(x)
    if xb.ndim != 2 or xb.shape[0] != G * 8:
        raise ValueError("x must be [in][n]")
    n = xb.shape[1]
    s = None if scales is None else _bits(scales)
    r = None if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
    nrows = out if r is None else len(r)
    y = np.empty((nrows, n), dtype=np.float64)
    bound = np.empty((nrows, n), dtype=np.float64)
    rc = _load().aqo_matmul(out, G * 8, K, B, _ptr(codes), _ptr(cb), _ptr(s), _ptr(xb),
                            n, _ptr(r), nrows, _ptr(y), _ptr(bound), int(threads))
    if rc:
        raise RuntimeError(f"aqo_matmul failed ({rc})")
    return y, bound


def backward(codes, codebooks, scales, x, gy):
    """Gradients of sum(gy * y), y = diag(s) W x, with respect to the row
    scales and the codebooks (rounding of the decode taken as the identity).

    Returns ``(grad_s [out], grad_s_bound, grad_cb [K][2^B][8], grad_cb_bound)``
    in float64; the bounds are the same sums of absolute terms."""
    cb = _bits(codebooks)
    K, ncw, _ = cb.shape
    B = int(ncw).bit_length() - 1
    codes = _codes(codes, K, B)
    out, G, _ = codes.shape
    xb, gyb = _bits(x), _bits(gy)
    if xb.ndim != 2 or xb.shape[0] != G * 8 or gyb.shape != (out, xb.shape[1]):
        raise ValueError("x must be [in][n] and gy [out][n]")
    n = xb.shape[1]
    s = None if scales is None else _bits(scales)
    gs = np.empty(out, dtype=np.float64)
    gsb = np.empty(out, dtype=np.float64)
    gc = np.empty((K, ncw, 8), dtype=np.float64)
    gcb = np.empty((K, ncw, 8), dtype=np.float64)
    rc = _load().aqo_backward(out, G * 8, K, B, _ptr(codes), _ptr(cb), _ptr(s), _ptr(xb), _ptr(gyb), n,
                              _ptr(gs), _ptr(gsb), _ptr(gc), _ptr(gcb))
    if rc:
        raise RuntimeError(f"aqo_backward failed ({rc})")
    return gs, gsb, gc, gcb


def _enc_args(w, h, codebooks):
    wb = _bits(w)
    out, inp = wb.shape
    hf = np.ascontiguousarray(h, dtype=np.float32)
    if hf.shape != (inp, inp):
        raise ValueError("h must be [in][in]")
    cb = _bits(codebooks)
    K, ncw, _ = cb.shape
    B = int(ncw).bit_length() - 1
    return wb, hf, cb, out, inp, K, B


def encode(w, h, codebooks, codes_init, beam: int):
    """Beam search of the codes of every row of ``w`` ([out][in] binary16)
    for fixed codebooks under the objective e^T H e, e = w - sum_k C_k[i_k]
    (``h`` [in][in] float32): group by group from ``codes_init``, a beam over
    the group's K codes (codebook by codebook), the best beam kept before the
    next group.  Returns ``(codes [out][in/8][K], objective [out])``."""
    wb, hf, cb, out, inp, K, B = _enc_args(w, h, codebooks)
    ci = np.ascontiguousarray(np.asarray(codes_init).reshape(out, inp // 8, K), dtype=np.uint32)
    co = np.empty_like(ci)
    obj = np.empty(out, dtype=np.float64)
    rc = _load().aqo_encode(out, inp, K, B, _ptr(wb), _ptr(hf), _ptr(cb), _ptr(ci), int(beam), _ptr(co), _ptr(obj))
    if rc:
        raise RuntimeError(f"aqo_encode failed ({rc})")
    return co.astype(np.uint8 if B <= 8 else np.uint16), obj


def objective(w, h, codebooks, codes):
    """e^T H e per row for the given codes (exact codeword sums, double)."""
    wb, hf, cb, out, inp, K, B = _enc_args(w, h, codebooks)
    ci = np.ascontiguousarray(np.asarray(codes).reshape(out, inp // 8, K), dtype=np.uint32)
    obj = np.empty(out, dtype=np.float64)
    rc = _load().aqo_objective(out, inp, K, B, _ptr(wb), _ptr(hf), _ptr(cb), _ptr(ci), _ptr(obj))
    if rc:
        raise RuntimeError(f"aqo_objective failed ({rc})")
    return obj


def packed_bytes(out: int, inp: int, K: int, B: int) -> int:
    n = _load().aqo_packed_bytes(out, inp, K, B)
    if n < 0:
        raise ValueError("unsupported layer for the packed layout")
    return int(n)


def pack(codes, K: int, B: int) -> np.ndarray:
    codes = _codes(codes, K, B)
    out, G, _ = codes.shape
    buf = np.empty(packed_bytes(out, G * 8, K, B), dtype=np.uint8)
    if _load().aqo_pack(out, G * 8, K, B, _ptr(codes), _ptr(buf)):
        raise RuntimeError("aqo_pack failed")
    return buf


def unpack(packed, out: int, inp: int, K: int, B: int) -> np.ndarray:
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    if packed.size != packed_bytes(out, inp, K, B):
        raise ValueError("packed buffer has the wrong size")
    codes = np.empty((out, inp // 8, K), dtype=np.uint8 if B <= 8 else np.uint16)
    if _load().aqo_unpack(out, inp, K, B, _ptr(packed), _ptr(codes)):
        raise RuntimeError("aqo_unpack failed")
    return codes
