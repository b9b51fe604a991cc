"""Planted mistakes in the oracle must fail its pins.

Each mutant below is a copy of ``oracle/aq_oracle.c`` with one plausible
slip (a dropped term, a wrong index, a transposed operand, a lost scale or
sign, a wrong rounding rule).  The copy is compiled with the oracle's own
flags into a temporary directory and ``tests/test_oracle_pins.py`` runs
against it in a child process; the pins must fail for every mutant.  A
mutant that survives is a part of the oracle no pin checks.  Everything
happens on the CPU; the committed oracle is not touched.
"""
import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

from conftest import ROOT

SRC = os.path.join(ROOT, "oracle", "aq_oracle.c")

# (name, text in aq_oracle.c (must occur exactly once), replacement)
MUTANTS = [
    # binary16 conversions
    ("half: subnormal scale", "v = ldexp((double)f, -24);", "v = ldexp((double)f, -25);"),
    ("half: normal exponent bias", "v = ldexp((double)(1024 + f), e - 25);", "v = ldexp((double)(1024 + f), e - 24);"),
    ("half: ties away from zero", "if (d > 0.5) return fl + 1.0;", "if (d >= 0.5) return fl + 1.0;"),
    # (">" for ">=" here is no mistake: the exponent carry below sends 65520
    # to infinity too; taking the largest finite value as the limit is one)
    ("half: overflow threshold", "if (a >= 65520.0) return", "if (a >= 65504.0) return"),
    ("half: carry into exponent lost", "        m = 1024.0;\n        e += 1;", "        m = 1024.0;"),
    # bit rate and storage
    ("bitrate: K dropped", "return (double)K * (double)B / (double)g;", "return (double)B / (double)g;"),
    ("storage: codebook count dropped",
     "double codebook_bytes = (double)K * ldexp(1.0, B) * AQO_GROUP * 2.0;",
     "double codebook_bytes = ldexp(1.0, B) * AQO_GROUP * 2.0;"),
    ("storage: scales dropped", "return code_bits / 8.0 + codebook_bytes + 2.0 * (double)out;",
     "return code_bits / 8.0 + codebook_bytes;"),
    # decode
    ("decode: only the first codebook", "sum = (k == 0) ? term : sum + term;", "sum = (k == 0) ? term : sum;"),
    ("decode: sum starts from +0", "sum = (k == 0) ? term : sum + term;", "sum = sum + term;"),
    ("decode: sum not rounded", "row[g * AQO_GROUP + j] = aqo_half_to_double(aqo_double_to_half(sum));",
     "row[g * AQO_GROUP + j] = sum;"),
    ("decode: codebook 0 for every k",
     "aqo_half_to_double(codebooks[((int64_t)k * ncw + c) * AQO_GROUP + j]);",
     "aqo_half_to_double(codebooks[((int64_t)0 * ncw + c) * AQO_GROUP + j]);"),
    ("decode: lanes reversed",
     "aqo_half_to_double(codebooks[((int64_t)k * ncw + c) * AQO_GROUP + j]);",
     "aqo_half_to_double(codebooks[((int64_t)k * ncw + c) * AQO_GROUP + (AQO_GROUP - 1 - j)]);"),
    ("decode: codes of a group in reverse order",
     "uint32_t c = code_at(codes, B, (o * G + g) * K + k);\n                double term",
     "uint32_t c = code_at(codes, B, (o * G + g) * K + (K - 1 - k));\n                double term"),
    ("decode: scale ignored", "w[o * in + i] = scales ? aqo_double_to_half(s * row[i])",
     "w[o * in + i] = scales ? aqo_double_to_half(row[i])"),
    # product
    ("matmul: scale dropped", "y[r * n + b] = s * acc;", "y[r * n + b] = acc;"),
    ("matmul: sign flipped", "y[r * n + b] = s * acc;", "y[r * n + b] = -s * acc;"),
    ("matmul: x transposed", "acc += row[i] * xd[i * n + b];", "acc += row[i] * xd[b * in + i];"),
    ("matmul: bound without abs", "mag += fabs(row[i] * xd[i * n + b]);", "mag += row[i] * xd[i * n + b];"),
    ("matmul: bound without scale", "if (bound) bound[r * n + b] = fabs(s) * mag;",
     "if (bound) bound[r * n + b] = mag;"),
    ("matmul: listed rows ignored", "int64_t o = rows ? rows[r] : r;", "int64_t o = r;"),
    # gradient
    ("backward: codebook grad without scale", "if (grad_cb) grad_cb[base + j] += s * m[g * AQO_GROUP + j];",
     "if (grad_cb) grad_cb[base + j] += m[g * AQO_GROUP + j];"),
    ("backward: codebook grad lane shifted", "if (grad_cb) grad_cb[base + j] += s * m[g * AQO_GROUP + j];",
     "if (grad_cb) grad_cb[base + j] += s * m[g * AQO_GROUP + (j + 1) % AQO_GROUP];"),
    ("backward: scale grad sign flipped", "gs += row[i] * m[i];", "gs -= row[i] * m[i];"),
    ("backward: gy transposed", "double t = aqo_half_to_double(gy[o * n + b]) * xd[i * n + b];",
     "double t = aqo_half_to_double(gy[b * out + o]) * xd[i * n + b];"),
    ("backward: codebook bound without scale",
     "if (grad_cb_bound) grad_cb_bound[base + j] += fabs(s) * mabs[g * AQO_GROUP + j];",
     "if (grad_cb_bound) grad_cb_bound[base + j] += mabs[g * AQO_GROUP + j];"),
    # encoder
    ("encode: worst proposals kept", "if (prop_less(&props[q], &props[best])) best = q;",
     "if (prop_less(&props[best], &props[q])) best = q;"),
    ("encode: beams carried across groups", "if (sl % K == 0) nb = 1;", "if (sl == 0) nb = 1;"),
    ("encode: proposal not applied", "nxt[r * S + sl] = props[r].code;", ""),
    ("encode: objective drops one codebook",
     "for (int k = 0; k < K; ++k)\n                sum += aqo_half_to_double",
     "for (int k = 1; k < K; ++k)\n                sum += aqo_half_to_double"),
    ("encode: ties by code first", "if (a->parent != b->parent) return a->parent < b->parent;", ""),
    # packed layout
    ("pack: tile transposed", "(g % 32) * 8 * W + (o % 8) * W;", "(g % 32) * W + (o % 8) * 32 * W;"),
    ("pack: big-endian words", "packed[at + b] = (uint8_t)(word >> (8 * b));",
     "packed[at + b] = (uint8_t)(word >> (8 * (W - 1 - b)));"),
    ("pack: codes of a word swapped",
     "word |= (uint64_t)code_at(codes, B, (o * G + g) * K + k) << (k * B);",
     "word |= (uint64_t)code_at(codes, B, (o * G + g) * K + k) << ((K - 1 - k) * B);"),
    ("pack: groups not padded", "int64_t gp = (in / AQO_GROUP + 31) / 32 * 32;", "int64_t gp = in / AQO_GROUP;"),
    ("pack: rows not padded", "int64_t rows = (out + 7) / 8 * 8;", "int64_t rows = out;"),
    # (a 16-bit mask for 8-bit codes is no mistake: the uint8_t store masks)
    ("unpack: codes shifted by bytes", "uint64_t c = (word >> (k * B)) & mask;", "uint64_t c = (word >> (k * 8)) & mask;"),
    # more of the gradient and the encoder
    ("backward: scale bound without abs", "gsb += fabs(row[i]) * mabs[i];", "gsb += row[i] * mabs[i];"),
    ("encode: beam width ignored", "int keep = np < beam ? np : beam;", "int keep = 1;"),
    ("encode: every survivor from beam 0", "nxt[r * S + t] = cur[props[r].parent * S + t];", "nxt[r * S + t] = cur[t];"),
    ("encode: H taken as its diagonal", "for (int64_t b = 0; b < in; ++b) t += h[a * in + b] * e[b];",
     "t += h[a * in + a] * e[a];"),
    ("objective: first row's codes for every row", "row_error(in, K, B, codes + o * S, wd, codebooks, e);",
     "row_error(in, K, B, codes, wd, codebooks, e);"),
    ("storage: weights counted as groups", "double code_bits = (double)out * (double)(in / AQO_GROUP) * K * B;",
     "double code_bits = (double)out * (double)in * K * B;"),
]

# Runs the pins against the oracle built from the mutated source.
_CHILD = r"""
import os, sys
sys.path.insert(0, {root!r})
sys.path.insert(0, os.path.join({root!r}, "tests"))
import oracle
oracle._SRC = {src!r}
oracle._BUILD = {build!r}
oracle._LIB_PATH = os.path.join({build!r}, "libaqoracle.so")
oracle._lib = None
import pytest
sys.exit(pytest.main([os.path.join({root!r}, "tests", "test_oracle_pins.py"), "-x", "-q",
                      "-p", "no:cacheprovider", "-m", "not gpu"]))
"""


def _run_mutant(tmp_root, idx, old, new):
    d = os.path.join(tmp_root, f"m{idx}")
    os.makedirs(d)
    src = open(SRC).read().replace(old, new)
    path = os.path.join(d, "aq_oracle.c")
    with open(path, "w") as f:
        f.write(src)
    code = _CHILD.format(root=ROOT, src=path, build=os.path.join(d, "_build"))
    p = subprocess.run([sys.executable, "-c", code], cwd=d, capture_output=True, text=True, timeout=600)
    return p.returncode, p.stdout[-2000:] + p.stderr[-2000:]


def test_mutation_targets_exist_once():
    text = open(SRC).read()
    for name, old, _ in MUTANTS:
        assert text.count(old) == 1, f"{name}: the mutated text must occur exactly once"


def test_pins_fail_for_every_planted_mistake(tmp_path):
    jobs = min(8, os.cpu_count() or 1)
    with ThreadPoolExecutor(max_workers=jobs) as pool:
        futs = [pool.submit(_run_mutant, str(tmp_path), i, old, new) for i, (_, old, new) in enumerate(MUTANTS)]
        results = [f.result() for f in futs]
    survivors, broken = [], []
    for (name, _, _), (rc, out) in zip(MUTANTS, results):
        if rc == 0:
            survivors.append(name)
        elif rc != 1:  # 1: tests failed; anything else is a harness problem
            broken.append((name, rc, out))
    assert not broken, broken
    assert not survivors, f"mutants no pin catches: {survivors}"
