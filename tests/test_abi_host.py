"""Host-side checks of the C ABI (no GPU needed, no kernel launched).

The library must load, export every function include/aq.h declares, size
buffers like the documented layout (checked against the oracle's
independent implementation), and reject bad arguments before any launch.
Every call below either touches no device memory or carries an argument
the host validation rejects, so nothing here can reach a kernel.
"""
import ctypes
import os
import re
import subprocess

import pytest

import additive_quantized_matmul_b200 as aq
import oracle
from conftest import ROOT

HEADER = os.path.join(ROOT, "include", "aq.h")
FAKE = 0x10000  # 16-byte aligned, never dereferenced: every call using it is rejected first


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(aq_[a-z_]+)\s*\(", text)))


def test_header_and_binding_agree():
    assert declared_functions() == sorted(aq.EXPORTED_SYMBOLS)


def test_library_exports_every_declared_symbol():
    out = subprocess.run(["nm", "-D", "--defined-only", aq.library_path],
                         capture_output=True, text=True, check=True).stdout
    exported = set(re.findall(r"\bT (aq_\w+)", out))
    missing = set(declared_functions()) - exported
    assert not missing, missing
    for name in declared_functions():
        assert hasattr(aq.lib, name)


def test_library_has_no_oracle_or_torch_dependency():
    out = subprocess.run(["nm", "-D", aq.library_path], capture_output=True, text=True).stdout
    assert "aqo_" not in out
    ldd = subprocess.run(["ldd", aq.library_path], capture_output=True, text=True).stdout
    assert "torch" not in ldd and "aqoracle" not in ldd


def test_version_and_status_strings():
    assert aq.aq_version() == 10000
    for s in range(7):
        assert aq.aq_status_string(s)
    assert aq.aq_status_string(99) == "unknown status"


SCHEMES = ((1, 16), (2, 8), (1, 8), (2, 16), (8, 8))


@pytest.mark.parametrize("out,inp,K,B", [(1, 8, 1, 16), (20, 520, 1, 16), (20, 520, 2, 8),
                                         (4096, 4096, 1, 16), (11008, 4096, 2, 8),
                                         (4096, 11008, 2, 8), (28672, 8192, 1, 16), (37, 360, 2, 8),
                                         (20, 520, 1, 8), (37, 360, 2, 16), (20, 520, 8, 8),
                                         (4096, 4096, 8, 8), (11008, 4096, 2, 16)])
def test_packed_bytes_matches_oracle(out, inp, K, B):
    d = aq.LayerDesc.make(out, inp, K, B)
    assert aq.aq_packed_codes_bytes(d) == oracle.packed_bytes(out, inp, K, B)


@pytest.mark.parametrize("desc,why", [
    ((0, 64, 8, 1, 16), "no rows"), ((16, 0, 8, 1, 16), "no columns"), ((16, 12, 8, 1, 16), "in % 8"),
    ((16, 64, 4, 1, 16), "group size"), ((16, 64, 8, 4, 8), "4x8"), ((16, 64, 8, 2, 4), "2x4"),
    ((16, 64, 8, 1, 12), "1x12"), ((16, 64, 8, 3, 8), "3x8"), ((16, 64, 8, 8, 16), "8x16"),
    ((-1, 64, 8, 1, 16), "negative"),
    ((8, 1 << 24, 8, 2, 8), "in = 2^24 (65536 blocks of 32 groups: one grid row too many)"),
    ((8, 65535 * 256 + 8, 8, 1, 16), "in above 65535 * 256"),
    ((1 << 20, 1 << 21, 8, 2, 8), "out * in above 2^40"),
    ((1 << 28 + 1, 8, 8, 2, 8), "out above 2^28"),
])
def test_invalid_descriptors(desc, why):
    d = aq.LayerDesc(*desc)
    assert aq.aq_packed_codes_bytes(d) == 0, why
    assert aq.aq_gemv_workspace_bytes(d, 1) == 0, why
    want = 2 if desc[2] != 8 or (desc[3], desc[4]) not in SCHEMES else 1
    if desc[0] < 1 or desc[1] < 8 or desc[1] % 8:
        want = 1
    st = aq.lib.aq_gemv(ctypes.byref(d), FAKE, FAKE, FAKE, FAKE, 1, FAKE, FAKE, 1 << 20, None)
    assert st == want, why
    st = aq.lib.aq_dequant(ctypes.byref(d), FAKE, FAKE, None, FAKE, None)
    assert st == want, why


def test_largest_input_width_is_accepted():
    """in = 65535 * 256 is the widest layer: its 65535 blocks of 32 groups
    are the most split-K grid rows a launch can have."""
    for K, B in SCHEMES:
        d = aq.LayerDesc.make(8, 65535 * 256, K, B)
        assert aq.aq_packed_codes_bytes(d) == oracle.packed_bytes(8, 65535 * 256, K, B)
        for b in (1, 2, 16):
            assert aq.aq_gemv_workspace_bytes(d, b) >= 16


def test_workspace_sizes_host_only():
    d = aq.LayerDesc.make(4096, 4096, 1, 16)
    for b in range(1, 17):
        assert aq.aq_gemv_workspace_bytes(d, b) >= 16
    assert aq.aq_gemv_workspace_bytes(d, 0) == 0
    assert aq.aq_gemv_workspace_bytes(d, 17) == 0
    assert aq.aq_gemm_workspace_bytes(d, 2048) >= 16
    assert aq.aq_gemm_workspace_bytes(d, 0) == 0


def _gemv(d, packed=FAKE, cb=FAKE, s=FAKE, x=FAKE, batch=1, y=FAKE, ws=FAKE, wsb=1 << 30, fn="aq_gemv"):
    return getattr(aq.lib, fn)(ctypes.byref(d), packed, cb, s, x, batch, y, ws, wsb, None)


def _gemm(d, packed=FAKE, cb=FAKE, s=FAKE, x=FAKE, T=64, y=FAKE, ws=FAKE, wsb=1 << 30, fn="aq_gemm"):
    return getattr(aq.lib, fn)(ctypes.byref(d), packed, cb, s, x, T, y, ws, wsb, None)


@pytest.mark.parametrize("fn", ["aq_gemv", "aq_gemv_ordered"])
def test_gemv_argument_errors(fn):
    d = aq.LayerDesc.make(64, 256, 2, 8)
    assert _gemv(d, batch=0, fn=fn) == 1
    assert _gemv(d, batch=17, fn=fn) == 1
    assert _gemv(d, packed=None, fn=fn) == 1
    assert _gemv(d, cb=None, fn=fn) == 1
    assert _gemv(d, x=None, fn=fn) == 1
    assert _gemv(d, y=None, fn=fn) == 1
    assert _gemv(d, packed=FAKE + 8, fn=fn) == 3
    assert _gemv(d, x=FAKE + 2, fn=fn) == 3
    assert _gemv(d, y=FAKE + 4, fn=fn) == 3
    assert _gemv(d, cb=FAKE + 1, fn=fn) == 3
    assert _gemv(d, s=FAKE + 1, fn=fn) == 3
    assert _gemv(d, ws=None, fn=fn) == 4
    assert _gemv(d, wsb=8, fn=fn) == 4
    assert _gemv(d, ws=FAKE + 8, fn=fn) == 3
    assert getattr(aq.lib, fn)(None, FAKE, FAKE, FAKE, FAKE, 1, FAKE, FAKE, 1 << 20, None) == 1


@pytest.mark.parametrize("fn", ["aq_gemm", "aq_gemm_ordered"])
def test_gemm_argument_errors(fn):
    d = aq.LayerDesc.make(64, 256, 1, 16)
    assert _gemm(d, T=0, fn=fn) == 1
    assert _gemm(d, T=-5, fn=fn) == 1
    assert _gemm(d, x=None, fn=fn) == 1
    assert _gemm(d, y=FAKE + 2, fn=fn) == 3
    assert _gemm(d, ws=None, fn=fn) == 4
    assert _gemm(d, wsb=0, fn=fn) == 4


def test_pack_and_misc_argument_errors():
    d = aq.LayerDesc.make(64, 256, 1, 16)
    assert aq.lib.aq_pack_codes(ctypes.byref(d), None, FAKE, None) == 1
    assert aq.lib.aq_pack_codes(ctypes.byref(d), FAKE, FAKE + 4, None) == 3
    assert aq.lib.aq_pack_codes(ctypes.byref(d), FAKE + 1, FAKE, None) == 3  # u16 codes odd address
    assert aq.lib.aq_unpack_codes(ctypes.byref(d), FAKE + 8, FAKE, None) == 3
    assert aq.lib.aq_dequant(ctypes.byref(d), FAKE, FAKE, FAKE + 1, FAKE, None) == 3
    assert aq.lib.aq_workspace_status(None, None) == 1
    assert aq.lib.aq_workspace_status(FAKE + 4, None) == 3
    assert aq.lib.aq_selftest_bounded_wait(FAKE, 0, None) == 1
    assert aq.lib.aq_selftest_bounded_wait(FAKE, (1 << 20) + 1, None) == 1
    assert aq.lib.aq_selftest_bounded_wait(None, 10, None) == 1


def test_binding_raises_on_error():
    d = aq.LayerDesc.make(64, 256, 1, 16)
    with pytest.raises(aq.AQError) as e:
        aq.aq_gemv(d, FAKE, FAKE, FAKE, FAKE, 0, FAKE, FAKE, 1 << 20, stream=0)
    assert e.value.name == "AQ_ERR_INVALID_ARG"


def test_gemv_noalloc_argument_errors():
    d = aq.LayerDesc.make(64, 256, 1, 16)
    f = aq.lib.aq_gemv_noalloc
    assert f(ctypes.byref(d), FAKE, FAKE, FAKE, FAKE, 0, FAKE, None) == 1
    assert f(ctypes.byref(d), FAKE, FAKE, FAKE, FAKE, 17, FAKE, None) == 1
    assert f(ctypes.byref(d), None, FAKE, FAKE, FAKE, 1, FAKE, None) == 1
    assert f(ctypes.byref(d), FAKE, FAKE, FAKE, FAKE + 8, 1, FAKE, None) == 3
    assert f(None, FAKE, FAKE, FAKE, FAKE, 1, FAKE, None) == 1



def test_workspace_layout_is_shared_by_every_call():
    """Counters live in a fixed area after the 16-byte status word, and
    partial sums or tables only after it: a plan that splits needs the
    4112-byte prefix, one that does not needs the status word alone."""
    prefix = 16 + 4 * 1024
    for (o, i, K, B), b in [((4096, 4096, 1, 16), 1), ((4096, 4096, 1, 16), 16), ((11008, 4096, 2, 8), 1),
                            ((4096, 11008, 2, 8), 8)]:
        d = aq.LayerDesc.make(o, i, K, B)
        assert aq.aq_gemv_workspace_bytes(d, b) > prefix  # these split
        assert (aq.aq_gemv_workspace_bytes(d, b) - prefix) % (4 * ((o + 7) // 8 * 8) * b) == 0
    # 64 groups: one CTA's tables cover every group, no split
    assert aq.aq_gemv_workspace_bytes(aq.LayerDesc.make(256, 512, 2, 8), 1) == 16
    # 2^20 rows: 8192 row tiles fill the GPU without a split, and would need
    # more counters than the fixed area holds
    huge = aq.LayerDesc.make(1 << 20, 64, 1, 16)
    assert aq.aq_gemv_workspace_bytes(huge, 4) == 16
    assert aq.aq_gemm_workspace_bytes(huge, 64) == 16
    # a prefill split over the input features (here 8 splits, one cluster)
    # keeps its fp32 partial sums after the counters area
    assert aq.aq_gemm_workspace_bytes(aq.LayerDesc.make(256, 4096, 2, 8), 512) == prefix + 8 * 256 * 512 * 4
    assert aq.aq_encode_workspace_bytes(aq.LayerDesc.make(64, 256, 2, 8)) == prefix + 32 * 2 * 256 * 4
    # the coarsest split of the no-allocation entry point always fits its array
    assert aq.aq_gemv_workspace_bytes(aq.LayerDesc.make(1 << 28, 8, 1, 16), 1) <= aq.GEMV_NOALLOC_SCRATCH_BYTES


def test_noalloc_scratch_size_matches_header():
    text = open(HEADER).read()
    m = re.search(r"#define AQ_GEMV_NOALLOC_SCRATCH_BYTES \((\d+)u << (\d+)\)", text)
    assert m and int(m.group(1)) << int(m.group(2)) == aq.GEMV_NOALLOC_SCRATCH_BYTES


def test_param_grad_argument_errors():
    d = aq.LayerDesc.make(64, 256, 2, 8)
    f = aq.lib.aq_param_grad

    def call(T=64, x=FAKE, gy=FAKE, gs=FAKE, gc=FAKE, ws=FAKE, wsb=1 << 20, packed=FAKE, s=FAKE):
        return f(ctypes.byref(d), packed, FAKE, s, x, gy, T, gs, gc, ws, wsb, None)

    assert aq.aq_param_grad_workspace_bytes(d, 64) >= 16
    assert aq.aq_param_grad_workspace_bytes(d, 12) == 0  # T % 8
    assert call(T=0) == 1 and call(T=12) == 1 and call(T=4) == 1
    assert call(x=None) == 1 and call(gy=None) == 1 and call(packed=None) == 1
    assert call(x=FAKE + 8) == 3 and call(gy=FAKE + 2) == 3
    assert call(gs=FAKE + 4) == 3 and call(gc=FAKE + 8) == 3 and call(s=FAKE + 1) == 3
    assert call(ws=None) == 4 and call(wsb=4) == 4
    bad = aq.LayerDesc.make(64, 256, 4, 8)
    assert f(ctypes.byref(bad), FAKE, FAKE, FAKE, FAKE, FAKE, 64, FAKE, FAKE, FAKE, 1 << 20, None) == 2


def test_encode_argument_errors():
    d = aq.LayerDesc.make(64, 256, 2, 8)
    f = aq.lib.aq_encode

    def call(desc=d, w=FAKE, h=FAKE, cb=FAKE, ci=FAKE, beam=4, co=FAKE + 64, ws=FAKE, wsb=1 << 20):
        return f(ctypes.byref(desc), w, h, cb, ci, beam, co, ws, wsb, None)

    assert aq.aq_encode_workspace_bytes(d) >= 16 + 32 * 2 * 256 * 4
    assert call(beam=0) == 1 and call(beam=17) == 1
    assert call(w=None) == 1 and call(h=None) == 1 and call(ci=None) == 1 and call(co=None) == 1
    assert call(co=FAKE) == 1  # codes_out aliases codes_in
    assert call(w=FAKE + 2) == 3 and call(h=FAKE + 4) == 3 and call(cb=FAKE + 8) == 3
    assert call(ws=None) == 4 and call(wsb=16) == 4
    # 16-bit codes: the q table [G][K][65536] and the residual [out][in], fp32
    assert aq.aq_encode_workspace_bytes(aq.LayerDesc.make(64, 256, 1, 16)) == 4112 + 32 * 65536 * 4 + 64 * 256 * 4
    assert aq.aq_encode_workspace_bytes(aq.LayerDesc.make(64, 256, 2, 16)) == 4112 + 32 * 2 * 65536 * 4 + 64 * 256 * 4
    assert call(desc=aq.LayerDesc.make(64, 256, 1, 16), wsb=16) == 4
    assert call(desc=aq.LayerDesc.make(64, 16392, 2, 8)) == 1   # in > 16384


def test_gather_probe_argument_errors():
    f = aq.lib.aq_gather_probe
    assert all(aq.aq_gather_probe_sink_bytes(m) > 0 for m in (0, 1, 2, 3, 4))
    assert aq.aq_gather_probe_sink_bytes(5) == 0 and aq.aq_gather_probe_sink_bytes(-1) == 0
    assert f(FAKE, FAKE, 64, 5, FAKE, None) == 1       # unknown mode
    assert f(None, FAKE, 64, 4, FAKE, None) == 1       # the slice mode reads the codebook
    assert f(None, None, 64, 3, FAKE, None) == 1       # the stream mode still needs codes
    assert f(None, FAKE, 64, 3, None, None) == 1       # and a sink
    assert f(None, FAKE + 8, 64, 3, FAKE, None) == 3   # misaligned codes (no codebook needed)
    assert f(FAKE, FAKE, 0, 0, FAKE, None) == 1        # no codes
    assert f(FAKE, FAKE, 12, 0, FAKE, None) == 1       # n not a multiple of 8
    assert f(None, FAKE, 64, 0, FAKE, None) == 1
    assert f(FAKE, None, 64, 1, FAKE, None) == 1
    assert f(FAKE, FAKE, 64, 0, None, None) == 1
    assert f(FAKE + 8, FAKE, 64, 0, FAKE, None) == 3   # misaligned codebook
    assert f(FAKE, FAKE + 2, 64, 1, FAKE, None) == 3   # misaligned codes


def test_binding_fails_loudly_without_the_library(tmp_path):
    """A copy of the package without libaq_b200.so must refuse to import
    (there is no CPU path to fall back to)."""
    import shutil
    import subprocess
    import sys
    pkg = tmp_path / "additive_quantized_matmul_b200"
    pkg.mkdir()
    shutil.copy(os.path.join(ROOT, "additive_quantized_matmul_b200", "__init__.py"), pkg / "__init__.py")
    code = ("import sys; sys.path.insert(0, sys.argv[1])\n"
            "try:\n    import additive_quantized_matmul_b200\n"
            "except ImportError as e:\n    print('ImportError:', e); sys.exit(3)\n"
            "sys.exit(0)\n")
    r = subprocess.run([sys.executable, "-c", code, str(tmp_path)], capture_output=True, text=True, timeout=120,
                       cwd=str(tmp_path))
    assert r.returncode == 3, r.stdout + r.stderr
    assert "libaq_b200.so is missing" in r.stdout and "build.py" in r.stdout


def test_prefill_plans_pinned_by_workspace_size():
    """The prefill planner's choices for Llama-2-7B shapes, read back from
    the workspace each needs (status word and counters, then fp32 sums):
    a 4096-row layer at 512 tokens splits its input features 4 ways in one
    cluster (32 tiles x 4 slices of 128 x 512); the 11008-row MLP layers at
    2048 tokens split the 48 tiles of their third wave 3 ways; layers that
    fill the SMs with whole tiles need no sums."""
    prefix = 4112
    slice_bytes = 128 * 512 * 4
    for K, B in ((1, 16), (2, 8)):
        assert aq.aq_gemm_workspace_bytes(aq.LayerDesc.make(4096, 4096, K, B), 512) == prefix + 32 * 4 * slice_bytes
        assert aq.aq_gemm_workspace_bytes(aq.LayerDesc.make(4096, 11008, K, B), 512) == prefix + 32 * 4 * slice_bytes
        assert aq.aq_gemm_workspace_bytes(aq.LayerDesc.make(11008, 4096, K, B), 2048) == prefix + 48 * 3 * slice_bytes
        assert aq.aq_gemm_workspace_bytes(aq.LayerDesc.make(11008, 4096, K, B), 512) == 16
        assert aq.aq_gemm_workspace_bytes(aq.LayerDesc.make(4096, 11008, K, B), 2048) == 16
