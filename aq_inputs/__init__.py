"""Seeded synthetic inputs for additive-quantised layers.

This module only draws random numbers.  It holds none of the method's
arithmetic (no decoding, no multiplication, no layout).  Both the CPU oracle
(tests, benchmark baseline) and the CUDA path (tests, benchmark, smoke) take
their inputs from here, so that both sides see identical bytes.

A layer in the additive-quantisation scheme of "Extreme Compression of Large
Language Models via Additive Quantization" (Egiazarian et al., ICML 2024) is
stored as

* ``codes``      ``[out][in/8][K]``  uint8 when B <= 8, else uint16;
* ``codebooks``  ``[K][2**B][8]``    IEEE binary16;
* ``scales``     ``[out]``           IEEE binary16 (one per output row);

and the activations are ``x`` ``[in][n]`` IEEE binary16 (``n`` = batch for
decode, tokens for prefill).

Value distributions follow the workloads this library is measured on:
codebooks N(0, sigma) with sigma 0.05 (small layer) or 0.02 (Llama-2-shaped
layers), row scales U(0.5, 1.5), activations N(0, 1), codes uniform over
[0, 2**B) or Zipf-skewed with P(c) proportional to (c + 1) ** -1.1 (rank =
code value, no permutation).  Every float is drawn in float64 and rounded to
binary16 by numpy's round-to-nearest-even conversion.
"""
from __future__ import annotations

import dataclasses
from typing import Iterable

import numpy as np

GROUP = 8  # in_group_size: consecutive input weights per code group


@dataclasses.dataclass(frozen=True)
class LayerSpec:
    """Shape and value recipe of one quantised linear layer."""

    out_features: int
    in_features: int
    num_codebooks: int  # K
    nbits: int  # B
    codebook_sigma: float = 0.02
    code_dist: str = "uniform"  # "uniform" | "zipf"
    zipf_s: float = 1.1
    scale_lo: float = 0.5
    scale_hi: float = 1.5

    @property
    def groups(self) -> int:
        return self.in_features // GROUP

    @property
    def scheme(self) -> str:
        return f"{self.num_codebooks}x{self.nbits}"

    def code_dtype(self):
        return np.uint8 if self.nbits <= 8 else np.uint16


@dataclasses.dataclass
class Layer:
    spec: LayerSpec
    codes: np.ndarray  # [out][G][K]
    codebooks: np.ndarray  # [K][2**B][8] float16
    scales: np.ndarray  # [out] float16


def _rng(seed) -> np.random.Generator:
    if isinstance(seed, Iterable) and not isinstance(seed, (str, bytes)):
        seed = [int(v) for v in seed]
    return np.random.Generator(np.random.PCG64(seed))


def _zipf_probs(n: int, s: float) -> np.ndarray:
    p = (np.arange(n, dtype=np.float64) + 1.0) ** (-s)
    return p / p.sum()


def make_codes(spec: LayerSpec, rng: np.random.Generator) -> np.ndarray:
    n = 1 << spec.nbits
    shape = (spec.out_features, spec.groups, spec.num_codebooks)
    if spec.code_dist == "uniform":
        codes = rng.integers(0, n, size=shape, dtype=np.int64)
    elif spec.code_dist == "zipf":
        codes = rng.choice(n, size=shape, p=_zipf_probs(n, spec.zipf_s))
    else:
        raise ValueError(f"unknown code distribution {spec.code_dist!r}")
    return codes.astype(spec.code_dtype())


def make_layer(spec: LayerSpec, seed) -> Layer:
    """Draw codes, codebooks and row scales for ``spec`` from ``seed``."""
    if spec.in_features % GROUP:
        raise ValueError("in_features must be a multiple of 8")
    rng = _rng(seed)
    codes = make_codes(spec, rng)
    cb = rng.normal(0.0, spec.codebook_sigma,
                    size=(spec.num_codebooks, 1 << spec.nbits, GROUP))
    scales = rng.uniform(spec.scale_lo, spec.scale_hi, size=spec.out_features)
    return Layer(spec, codes, cb.astype(np.float16), scales.astype(np.float16))


def make_activations(in_features: int, n: int, seed, sigma: float = 1.0) -> np.ndarray:
    """x ``[in][n]`` float16, N(0, sigma)."""
    rng = _rng(seed)
    return rng.normal(0.0, sigma, size=(in_features, n)).astype(np.float16)


# ---------------------------------------------------------------------------
# Named workloads (sizes of Llama-2-7B / 70B linear layers).
# ---------------------------------------------------------------------------

LLAMA2_7B_BLOCK = {
    "q": (4096, 4096), "k": (4096, 4096), "v": (4096, 4096), "o": (4096, 4096),
    "gate": (11008, 4096), "up": (11008, 4096), "down": (4096, 11008),
}


def workload(name: str) -> dict:
    """Return ``{"layers": [(tag, LayerSpec), ...], "n": [...], "seed": int}``."""
    if name == "tiny-2x8":
        sp = LayerSpec(256, 512, 2, 8, codebook_sigma=0.05)
        return {"layers": [("tiny", sp)], "n": [1, 4], "seed": 1000}
    if name == "llama2-7b-1x16":
        sp = LayerSpec(4096, 4096, 1, 16)
        return {"layers": [("4096x4096", sp)], "n": [1, 4, 16], "seed": 1001}
    if name == "llama2-7b-decode":
        # the decode-time products the headline metric covers: the 1x16
        # 4096 x 4096 layer at batch 1, 4, 16 and the 2x8 MLP layers
        # (uniform and Zipf codes) at batch 1 and 8, each part keeping its
        # own batches and seed
        return {"parts": ["llama2-7b-1x16", "llama2-7b-mlp-2x8"]}
    if name == "llama2-7b-mlp-2x8":
        layers = []
        for dist in ("uniform", "zipf"):
            layers.append((f"11008x4096-{dist}", LayerSpec(11008, 4096, 2, 8, code_dist=dist)))
            layers.append((f"4096x11008-{dist}", LayerSpec(4096, 11008, 2, 8, code_dist=dist)))
        return {"layers": layers, "n": [1, 8], "seed": 1002}
    if name == "llama2-70b-1x16":
        shapes = [(8192, 8192), (28672, 8192), (8192, 28672), (1024, 8192)]
        layers = [(f"{o}x{i}", LayerSpec(o, i, 1, 16)) for o, i in shapes]
        return {"layers": layers, "n": [1, 16], "seed": 1003}
    if name == "llama2-7b-prefill":
        layers = []
        for K, B in ((1, 16), (2, 8)):
            for tag, (o, i) in LLAMA2_7B_BLOCK.items():
                layers.append((f"{tag}-{K}x{B}", LayerSpec(o, i, K, B)))
        return {"layers": layers, "n": [512, 2048], "seed": 1004}
    if name == "llama2-7b-grad":
        # parameter gradient (codebooks, scales) of block shapes over 2048 tokens
        layers = [(f"{tag}-{K}x{B}", LayerSpec(o, i, K, B)) for K, B in ((1, 16), (2, 8))
                  for tag, (o, i) in (("q", LLAMA2_7B_BLOCK["q"]), ("gate", LLAMA2_7B_BLOCK["gate"]))]
        return {"layers": layers, "n": [2048], "seed": 1007}
    if name == "llama2-7b-encode":
        # code assignment (beam 8) for a 2x8 q projection and MLP up shape,
        # and a 1x16 q projection (65536 codes scored per group)
        layers = [("q-2x8", LayerSpec(4096, 4096, 2, 8)), ("gate-2x8", LayerSpec(11008, 4096, 2, 8)),
                  ("q-1x16", LayerSpec(4096, 4096, 1, 16))]
        return {"layers": layers, "n": [8], "seed": 1008}
    if name == "llama2-7b-schemes":
        # the other schemes the pages name, at the Llama-2-7B MLP up shape
        layers = [(f"11008x4096-{K}x{B}", LayerSpec(11008, 4096, K, B)) for K, B in ((1, 8), (2, 16), (8, 8))]
        return {"layers": layers, "n": [1, 16], "seed": 1006}
    if name == "llama2-7b-block":
        # the seven linears of one decoder block per scheme, run as a chain:
        # each entry is (tag, spec, input) with input None for the block's
        # input vector, else the tag of the layer whose output it consumes
        # (q, k, v read the block input; o reads v; gate and up read o;
        # down reads up)
        src = {"q": None, "k": None, "v": None, "o": "v", "gate": "o", "up": "o", "down": "up"}
        chains = []
        for K, B in ((1, 16), (2, 8)):
            chains.append((f"block-{K}x{B}",
                           [(tag, LayerSpec(o, i, K, B), src[tag]) for tag, (o, i) in LLAMA2_7B_BLOCK.items()]))
        return {"layers": [], "chains": chains, "n": [1], "seed": 1005}
    raise KeyError(name)


def workload_units(name: str) -> list:
    """Flatten a workload into ``[(tag, spec, batches, seed), ...]`` (a
    composite workload lists the parts it is made of)."""
    wl = workload(name)
    if "parts" in wl:
        return [u for part in wl["parts"] for u in workload_units(part)]
    return [(tag, spec, tuple(wl["n"]), wl["seed"]) for tag, spec in wl["layers"]]


WORKLOADS = ("tiny-2x8", "llama2-7b-decode", "llama2-7b-1x16", "llama2-7b-mlp-2x8",
             "llama2-70b-1x16", "llama2-7b-prefill", "llama2-7b-block", "llama2-7b-schemes", "llama2-7b-grad",
             "llama2-7b-encode")
