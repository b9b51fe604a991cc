"""Python binding of libaq_b200.so, the sm_100a additive-quantised product library.

Thin marshalling over the C ABI declared in ``include/aq.h``: every function
here has the name of the C entry point it calls, takes torch tensors (device
memory) and the current CUDA stream, checks nothing beyond what is needed to
build the call, and raises :class:`AQError` on a non-zero status.  All
computation happens in the library's CUDA kernels; there is no CPU path.

Layer storage (see ``include/aq.h``): codes ``[out][in/8][K]`` (uint8 for
2x8, 16-bit for 1x16), packed with :func:`aq_pack_codes`; codebooks
``[K][2**B][8]`` float16; scales ``[out]`` float16; activations ``[in][n]``
float16; outputs ``[out][n]`` float16.
"""
from __future__ import annotations

import ctypes
import os

__all__ = [
    "AQError", "LayerDesc", "lib", "library_path", "aq_version", "aq_status_string",
    "aq_packed_codes_bytes", "aq_gemv_workspace_bytes", "aq_gemm_workspace_bytes",
    "aq_workspace_status", "aq_selftest_bounded_wait", "aq_pack_codes", "aq_unpack_codes",
    "aq_dequant", "aq_gemv", "aq_gemv_ordered", "aq_gemv_noalloc", "aq_gemm", "aq_gemm_ordered",
    "aq_param_grad_workspace_bytes",
    "aq_param_grad", "aq_encode_workspace_bytes", "aq_encode", "aq_gather_probe_sink_bytes",
    "aq_gather_probe", "EXPORTED_SYMBOLS",
    "GEMV_NOALLOC_SCRATCH_BYTES",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
library_path = os.path.join(_HERE, "libaq_b200.so")

AQ_OK = 0
STATUS_NAMES = {0: "AQ_OK", 1: "AQ_ERR_INVALID_ARG", 2: "AQ_ERR_UNSUPPORTED",
                3: "AQ_ERR_MISALIGNED", 4: "AQ_ERR_WORKSPACE", 5: "AQ_ERR_CUDA",
                6: "AQ_ERR_TIMEOUT"}

# Every symbol include/aq.h declares.
EXPORTED_SYMBOLS = (
    "aq_status_string", "aq_version", "aq_packed_codes_bytes", "aq_gemv_workspace_bytes",
    "aq_gemm_workspace_bytes", "aq_workspace_status", "aq_selftest_bounded_wait",
    "aq_pack_codes", "aq_unpack_codes", "aq_dequant", "aq_gemv", "aq_gemv_ordered", "aq_gemv_noalloc", "aq_gemm",
    "aq_gemm_ordered",
    "aq_param_grad_workspace_bytes", "aq_param_grad", "aq_encode_workspace_bytes", "aq_encode",
    "aq_gather_probe_sink_bytes", "aq_gather_probe",
)

# AQ_GEMV_NOALLOC_SCRATCH_BYTES of include/aq.h: the fixed scratch behind
# aq_gemv_noalloc.
GEMV_NOALLOC_SCRATCH_BYTES = 4 << 20


class AQError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        self.name = STATUS_NAMES.get(status, str(status))
        super().__init__(f"{fn} failed: {self.name} ({aq_status_string(status)})")


class LayerDesc(ctypes.Structure):
    """``aq_layer_desc``: out_features, in_features, group_size, num_codebooks, nbits."""

    _fields_ = [("out_features", ctypes.c_int32), ("in_features", ctypes.c_int32),
                ("group_size", ctypes.c_int32), ("num_codebooks", ctypes.c_int32),
                ("nbits", ctypes.c_int32)]

    @classmethod
    def make(cls, out_features: int, in_features: int, num_codebooks: int, nbits: int,
             group_size: int = 8) -> "LayerDesc":
        return cls(out_features, in_features, group_size, num_codebooks, nbits)


def _load() -> ctypes.CDLL:
    if not os.path.exists(library_path):
        raise ImportError(
            f"{library_path} is missing: build it with "
            "`python additive_quantized_matmul_b200/build.py` (nvcc, sm_100a)")
    L = ctypes.CDLL(library_path)
    vp, sz, i32 = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int
    dp = ctypes.POINTER(LayerDesc)
    sig = {
        "aq_status_string": ([i32], ctypes.c_char_p),
        "aq_version": ([], i32),
        "aq_packed_codes_bytes": ([dp], sz),
        "aq_gemv_workspace_bytes": ([dp, i32], sz),
        "aq_gemm_workspace_bytes": ([dp, i32], sz),
        "aq_workspace_status": ([vp, vp], i32),
        "aq_selftest_bounded_wait": ([vp, i32, vp], i32),
        "aq_pack_codes": ([dp, vp, vp, vp], i32),
        "aq_unpack_codes": ([dp, vp, vp, vp], i32),
        "aq_dequant": ([dp, vp, vp, vp, vp, vp], i32),
        "aq_gemv": ([dp, vp, vp, vp, vp, i32, vp, vp, sz, vp], i32),
        "aq_gemv_ordered": ([dp, vp, vp, vp, vp, i32, vp, vp, sz, vp], i32),
        "aq_gemm": ([dp, vp, vp, vp, vp, i32, vp, vp, sz, vp], i32),
        "aq_gemm_ordered": ([dp, vp, vp, vp, vp, i32, vp, vp, sz, vp], i32),
        "aq_gemv_noalloc": ([dp, vp, vp, vp, vp, i32, vp, vp], i32),
        "aq_param_grad_workspace_bytes": ([dp, i32], sz),
        "aq_param_grad": ([dp, vp, vp, vp, vp, vp, i32, vp, vp, vp, sz, vp], i32),
        "aq_encode_workspace_bytes": ([dp], sz),
        "aq_encode": ([dp, vp, vp, vp, vp, i32, vp, vp, sz, vp], i32),
        "aq_gather_probe_sink_bytes": ([i32], sz),
        "aq_gather_probe": ([vp, vp, sz, i32, vp, vp], i32),
    }
    for name, (args, res) in sig.items():
        fn = getattr(L, name)
        fn.argtypes = args
        fn.restype = res
    return L


lib = _load()


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(fn: str, status: int):
    if status != AQ_OK:
        raise AQError(fn, status)


def aq_status_string(status: int) -> str:
    return lib.aq_status_string(status).decode()


def aq_version() -> int:
    return lib.aq_version()


def aq_packed_codes_bytes(desc: LayerDesc) -> int:
    return lib.aq_packed_codes_bytes(ctypes.byref(desc))


def aq_gemv_workspace_bytes(desc: LayerDesc, batch: int) -> int:
    return lib.aq_gemv_workspace_bytes(ctypes.byref(desc), batch)


def aq_gemm_workspace_bytes(desc: LayerDesc, T: int) -> int:
    return lib.aq_gemm_workspace_bytes(ctypes.byref(desc), T)


def aq_workspace_status(workspace, stream=None) -> int:
    """Status word of a workspace (read and cleared; synchronises ``stream``)."""
    return lib.aq_workspace_status(_ptr(workspace), _stream(stream))


def aq_selftest_bounded_wait(workspace, spin_limit: int, stream=None) -> None:
    _check("aq_selftest_bounded_wait",
           lib.aq_selftest_bounded_wait(_ptr(workspace), spin_limit, _stream(stream)))


def aq_pack_codes(desc: LayerDesc, codes, packed, stream=None) -> None:
    _check("aq_pack_codes", lib.aq_pack_codes(ctypes.byref(desc), _ptr(codes), _ptr(packed),
                                              _stream(stream)))


def aq_unpack_codes(desc: LayerDesc, packed, codes, stream=None) -> None:
    _check("aq_unpack_codes", lib.aq_unpack_codes(ctypes.byref(desc), _ptr(packed), _ptr(codes),
                                                  _stream(stream)))


def aq_dequant(desc: LayerDesc, packed, codebooks, scales, w, stream=None) -> None:
    _check("aq_dequant", lib.aq_dequant(ctypes.byref(desc), _ptr(packed), _ptr(codebooks),
                                        _ptr(scales), _ptr(w), _stream(stream)))


def aq_gemv(desc: LayerDesc, packed, codebooks, scales, x, batch: int, y, workspace,
            workspace_bytes: int | None = None, stream=None) -> None:
    if workspace_bytes is None:
        workspace_bytes = workspace.numel() * workspace.element_size()
    _check("aq_gemv", lib.aq_gemv(ctypes.byref(desc), _ptr(packed), _ptr(codebooks), _ptr(scales),
                                  _ptr(x), batch, _ptr(y), _ptr(workspace), workspace_bytes,
                                  _stream(stream)))


def aq_gemv_ordered(desc: LayerDesc, packed, codebooks, scales, x, batch: int, y, workspace,
                    workspace_bytes: int | None = None, stream=None) -> None:
    """aq_gemv launched without programmatic dependent launch: no weight is
    read before the previous work on the stream has completed."""
    if workspace_bytes is None:
        workspace_bytes = workspace.numel() * workspace.element_size()
    _check("aq_gemv_ordered", lib.aq_gemv_ordered(ctypes.byref(desc), _ptr(packed), _ptr(codebooks), _ptr(scales),
                                                  _ptr(x), batch, _ptr(y), _ptr(workspace), workspace_bytes,
                                                  _stream(stream)))


def aq_gemv_noalloc(desc: LayerDesc, packed, codebooks, scales, x, batch: int, y, stream=None) -> None:
    """aq_gemv for callers that cannot allocate device memory: the split-K
    scratch is a fixed array inside the library (see include/aq.h); calls
    that overlap on the GPU must not be issued."""
    _check("aq_gemv_noalloc", lib.aq_gemv_noalloc(ctypes.byref(desc), _ptr(packed), _ptr(codebooks),
                                                  _ptr(scales), _ptr(x), batch, _ptr(y), _stream(stream)))


def aq_gemm(desc: LayerDesc, packed, codebooks, scales, x, T: int, y, workspace,
            workspace_bytes: int | None = None, stream=None) -> None:
    if workspace_bytes is None:
        workspace_bytes = workspace.numel() * workspace.element_size()
    _check("aq_gemm", lib.aq_gemm(ctypes.byref(desc), _ptr(packed), _ptr(codebooks), _ptr(scales),
                                  _ptr(x), T, _ptr(y), _ptr(workspace), workspace_bytes,
                                  _stream(stream)))


def aq_gemm_ordered(desc: LayerDesc, packed, codebooks, scales, x, T: int, y, workspace,
                    workspace_bytes: int | None = None, stream=None) -> None:
    """aq_gemm launched without programmatic dependent launch: no weight is
    read before the previous work on the stream has completed."""
    if workspace_bytes is None:
        workspace_bytes = workspace.numel() * workspace.element_size()
    _check("aq_gemm_ordered", lib.aq_gemm_ordered(ctypes.byref(desc), _ptr(packed), _ptr(codebooks), _ptr(scales),
                                                  _ptr(x), T, _ptr(y), _ptr(workspace), workspace_bytes,
                                                  _stream(stream)))


def aq_param_grad_workspace_bytes(desc: LayerDesc, T: int) -> int:
    return lib.aq_param_grad_workspace_bytes(ctypes.byref(desc), T)


def aq_param_grad(desc: LayerDesc, packed, codebooks, scales, x, gy, T: int, grad_scales, grad_codebooks,
                  workspace, workspace_bytes: int | None = None, stream=None) -> None:
    """dL/ds [out] and dL/dC [K][2^B][8] (fp32, overwritten; either may be
    None) for L = sum(gy * y), y = diag(s) W x; x [in][T], gy [out][T]."""
    if workspace_bytes is None:
        workspace_bytes = workspace.numel() * workspace.element_size()
    _check("aq_param_grad", lib.aq_param_grad(ctypes.byref(desc), _ptr(packed), _ptr(codebooks), _ptr(scales),
                                              _ptr(x), _ptr(gy), T, _ptr(grad_scales), _ptr(grad_codebooks),
                                              _ptr(workspace), workspace_bytes, _stream(stream)))


def aq_encode_workspace_bytes(desc: LayerDesc) -> int:
    return lib.aq_encode_workspace_bytes(ctypes.byref(desc))


def aq_encode(desc: LayerDesc, w, h, codebooks, codes_in, beam: int, codes_out, workspace,
              workspace_bytes: int | None = None, stream=None) -> None:
    """Beam search of the codes minimising e^T H e per row; w [out][in]
    binary16, h [in][in] fp32, codes [out][in/8][K] uint8 (8-bit codebooks)
    or uint16 (16-bit)."""
    if workspace_bytes is None:
        workspace_bytes = workspace.numel() * workspace.element_size()
    _check("aq_encode", lib.aq_encode(ctypes.byref(desc), _ptr(w), _ptr(h), _ptr(codebooks), _ptr(codes_in), beam,
                                      _ptr(codes_out), _ptr(workspace), workspace_bytes, _stream(stream)))


def aq_gather_probe_sink_bytes(mode: int) -> int:
    return lib.aq_gather_probe_sink_bytes(mode)


def aq_gather_probe(codebook, codes, n: int, mode: int, sink, stream=None) -> None:
    """Measurement aid: read codebook[codes[i]] for each of the n 16-bit codes
    (mode 0: from L2 into shared memory with cp.async, as the tensor-core
    GEMV's decoders do; mode 1: from the codebook split over 8-CTA
    clusters' shared memory; mode 2: through L1 into registers, as the
    batch-1 CUDA-core GEMV does; mode 3: no codeword, ``codes`` itself read
    once as a stream, the read-only HBM bandwidth; ``codebook`` may then be
    None; mode 4: the codebook sliced over 8-CTA clusters' shared memory,
    each code handled by the CTA holding its slice); per-thread XOR
    checksums go to ``sink``."""
    _check("aq_gather_probe", lib.aq_gather_probe(_ptr(codebook), _ptr(codes), n, mode, _ptr(sink), _stream(stream)))
