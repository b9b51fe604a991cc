"""Helpers for the GPU tests: move seeded layers to the device, guard-banded
output buffers, and tolerance checks against the oracle."""
from __future__ import annotations

import numpy as np
import torch

import additive_quantized_matmul_b200 as aq
from aq_inputs import Layer, LayerSpec, make_activations, make_layer
from conftest import within_tolerance

GUARD = 4096  # elements of canary before and after every output
CANARY = 0x7E5A


def desc_of(spec: LayerSpec) -> aq.LayerDesc:
    return aq.LayerDesc.make(spec.out_features, spec.in_features, spec.num_codebooks, spec.nbits)


def dev(a: np.ndarray) -> torch.Tensor:
    if a.dtype == np.uint16:
        a = a.view(np.int16)
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


class DevLayer:
    """A layer on the device: packed codes, codebooks, scales."""

    def __init__(self, layer: Layer):
        self.layer = layer
        self.spec = layer.spec
        self.desc = desc_of(layer.spec)
        self.codes = dev(layer.codes)
        self.packed = torch.empty(aq.aq_packed_codes_bytes(self.desc), dtype=torch.uint8, device="cuda")
        aq.aq_pack_codes(self.desc, self.codes, self.packed)
        self.codebooks = dev(layer.codebooks.view(np.uint16))
        self.scales = dev(layer.scales.view(np.uint16))


def guarded(n: int, dtype=torch.int16):
    """Buffer of n elements with canary bands; returns (full, inner view)."""
    full = torch.full((n + 2 * GUARD,), CANARY, dtype=dtype, device="cuda")
    return full, full[GUARD:GUARD + n]


def guards_intact(full: torch.Tensor) -> bool:
    g = torch.cat([full[:GUARD], full[-GUARD:]])
    return bool((g == CANARY).all().item())


def workspace(nbytes: int) -> torch.Tensor:
    return torch.zeros(max(nbytes, 16) // 16 * 16 + 16, dtype=torch.uint8, device="cuda")


def to_f16(t: torch.Tensor) -> np.ndarray:
    return t.cpu().numpy().view(np.float16)


def run_gemv(dl: DevLayer, x: np.ndarray, ws=None):
    batch = x.shape[1]
    xd = dev(x.view(np.uint16))
    full, y = guarded(dl.spec.out_features * batch)
    if ws is None:
        ws = workspace(aq.aq_gemv_workspace_bytes(dl.desc, batch))
    aq.aq_gemv(dl.desc, dl.packed, dl.codebooks, dl.scales, xd, batch, y, ws)
    torch.cuda.synchronize()
    assert guards_intact(full), "gemv wrote outside its output"
    return to_f16(y).reshape(dl.spec.out_features, batch).astype(np.float64)


def run_gemm(dl: DevLayer, x: np.ndarray, ws=None):
    T = x.shape[1]
    xd = dev(x.view(np.uint16))
    full, y = guarded(dl.spec.out_features * T)
    if ws is None:
        ws = workspace(aq.aq_gemm_workspace_bytes(dl.desc, T))
    aq.aq_gemm(dl.desc, dl.packed, dl.codebooks, dl.scales, xd, T, y, ws)
    torch.cuda.synchronize()
    assert aq.aq_workspace_status(ws) == 0, "a bounded wait gave up"
    assert guards_intact(full), "gemm wrote outside its output"
    return to_f16(y).reshape(dl.spec.out_features, T).astype(np.float64)


def assert_close(y_gpu, y_ref, bound, what=""):
    ok, err, lim = within_tolerance(y_gpu, y_ref, bound)
    if not ok.all():
        idx = np.argwhere(~ok)[:5]
        raise AssertionError(f"{what}: {int((~ok).sum())} elements out of tolerance, first "
                             f"{[(tuple(i), float(y_gpu[tuple(i)]), float(y_ref[tuple(i)]), float(lim[tuple(i)])) for i in idx]}")
    assert np.isfinite(y_gpu).all()


__all__ = ["DevLayer", "LayerSpec", "make_layer", "make_activations", "run_gemv", "run_gemm",
           "assert_close", "guarded", "guards_intact", "workspace", "dev", "to_f16", "desc_of"]
