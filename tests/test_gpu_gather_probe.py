"""aq_gather_probe: the codeword-read ceiling of the 1x16 product (modes 0-2, 4)
and the read-only HBM stream (mode 3).

Modes 0-2 and 4 read codebook[codes[i]] for every code and XOR each 32-bit word
they read into a per-thread checksum.  These tests check, through the C ABI,
that each mode reads exactly the codewords the codes select: the XOR of all
checksums must equal the XOR of those codewords, computed here with numpy
from the same inputs (a property of the data, not of the method).  Mode 3
reads the code array itself once: its checksums XOR to the XOR of the
array's 32-bit words.
"""
import numpy as np
import pytest
import torch

import additive_quantized_matmul_b200 as aq

pytestmark = pytest.mark.gpu


def _expected_xor(cb_words: np.ndarray, codes: np.ndarray) -> np.ndarray:
    # XOR over i of the four 32-bit words of codeword codes[i]
    return np.bitwise_xor.reduce(cb_words[codes.astype(np.int64)], axis=0)


@pytest.mark.parametrize("mode", [0, 1, 2, 4])
@pytest.mark.parametrize("n", [8, 4096 * 512, 4096 * 512 + 8 * 37])
def test_probe_reads_the_selected_codewords(mode, n):
    rng = np.random.default_rng(n + mode)
    cb_words = rng.integers(0, 2**32, size=(65536, 4), dtype=np.uint64).astype(np.uint32)
    codes = rng.integers(0, 65536, size=n, dtype=np.int64).astype(np.uint16)
    cb = torch.from_numpy(cb_words.view(np.int32)).cuda()
    cd = torch.from_numpy(codes.view(np.int16)).cuda()
    sink_bytes = aq.aq_gather_probe_sink_bytes(mode)
    sink = torch.zeros(sink_bytes // 4, dtype=torch.int32, device="cuda")
    aq.aq_gather_probe(cb, cd, n, mode, sink)
    torch.cuda.synchronize()
    got = np.bitwise_xor.reduce(sink.cpu().numpy().view(np.uint32).reshape(-1, 4), axis=0)
    assert np.array_equal(got, _expected_xor(cb_words, codes))


def test_probe_back_to_back_calls_keep_the_checksum():
    # calls overlap through programmatic dependent launch; each waits for
    # the previous one before writing the sink
    rng = np.random.default_rng(5)
    cb_words = rng.integers(0, 2**32, size=(65536, 4), dtype=np.uint64).astype(np.uint32)
    codes = rng.integers(0, 65536, size=1 << 20, dtype=np.int64).astype(np.uint16)
    cb = torch.from_numpy(cb_words.view(np.int32)).cuda()
    cd = torch.from_numpy(codes.view(np.int16)).cuda()
    sink = torch.zeros(aq.aq_gather_probe_sink_bytes(0) // 4, dtype=torch.int32, device="cuda")
    for _ in range(5):
        aq.aq_gather_probe(cb, cd, codes.size, 0, sink)
    torch.cuda.synchronize()
    got = np.bitwise_xor.reduce(sink.cpu().numpy().view(np.uint32).reshape(-1, 4), axis=0)
    assert np.array_equal(got, _expected_xor(cb_words, codes))


@pytest.mark.parametrize("n", [8, 8 * 592 * 256 * 8, 8 * 592 * 256 * 8 * 3 + 8 * 4099, (1 << 26) + 8 * 5])
def test_stream_probe_reads_every_word_once(n):
    rng = np.random.default_rng(n)
    codes = rng.integers(0, 65536, size=n, dtype=np.int64).astype(np.uint16)
    cd = torch.from_numpy(codes.view(np.int16)).cuda()
    sink = torch.zeros(aq.aq_gather_probe_sink_bytes(3) // 4, dtype=torch.int32, device="cuda")
    aq.aq_gather_probe(None, cd, n, 3, sink)
    aq.aq_gather_probe(None, cd, n, 3, sink)  # a second call rewrites the same checksums
    torch.cuda.synchronize()
    got = np.bitwise_xor.reduce(sink.cpu().numpy().view(np.uint32).reshape(-1, 4), axis=0)
    want = np.bitwise_xor.reduce(codes.view(np.uint32).reshape(-1, 4), axis=0)
    assert np.array_equal(got, want)
