"""Parity of chained decode-time products, launched back to back.

In a decoder each product's activations are the previous product's output,
and aq_gemv launches with programmatic dependent launch: a kernel may start
reading its weights while the kernel before it on the stream is still
running, and must read x and write y and the workspace only after that
kernel has finished.  These tests run the products the way a decoder (and
the benchmark) does -- every launch on one stream, no host synchronisation
between them, one workspace shared by all -- and check each product
element by element against the oracle applied to the GPU output it
consumed, so every step is held to the tolerance on its own.

* the seven linears of a Llama-2-7B decoder block (q, k, v read the block
  input; o reads v; gate and up read o; down reads up), 1x16 and 2x8, at
  batch 1 and at a tensor-core batch (4);
* four such blocks in one CUDA graph, each block reading the previous
  block's down-projection output (16 dependent products deep);
* the benchmark's rotation: 76 copies of a 4096 x 4096 1x16 layer at
  distinct addresses, batch 1, 4 and 16, in one CUDA graph, all copies of a
  batch sharing one workspace;
* the block's seven prefill products (aq_gemm, also launched with
  programmatic dependent launch) at 512 and 136 tokens.

Weights of the multi-block chain are drawn with codebook spreads that keep
the activations' magnitude about constant from layer to layer (gain ~1), so
a deep chain stays far from binary16 overflow.
"""
import numpy as np
import pytest
import torch

import additive_quantized_matmul_b200 as aq
import oracle
from aq_inputs import LLAMA2_7B_BLOCK, LayerSpec, make_activations, make_layer
from aqtest import DevLayer, assert_close, dev, to_f16, workspace

pytestmark = pytest.mark.gpu

# block order and the layer each one reads (None: the block input)
BLOCK = ["q", "k", "v", "o", "gate", "up", "down"]
SOURCE = {"q": None, "k": None, "v": None, "o": "v", "gate": "o", "up": "o", "down": "up"}


def _block_layers(K, B, seed, unit_gain=False):
    layers = {}
    for li, tag in enumerate(BLOCK):
        out, inp = LLAMA2_7B_BLOCK[tag]
        # gain ~1: the decoded weight's spread (K codebook terms) times
        # sqrt(in) times the RMS row scale (~1.04) is about one
        sigma = 1.0 / (np.sqrt(K * inp) * 1.04) if unit_gain else 0.02
        base = seed if isinstance(seed, tuple) else (seed,)
        layers[tag] = make_layer(LayerSpec(out, inp, K, B, codebook_sigma=sigma), (*base, li))
    return layers


def _launch_block(dls, x_in, ys, batch, ws, stream):
    """The seven products of one block on `stream`, no synchronisation."""
    for tag in BLOCK:
        dl = dls[tag]
        src = SOURCE[tag]
        inp = x_in if src is None else ys[src]
        aq.aq_gemv(dl.desc, dl.packed, dl.codebooks, dl.scales, inp, batch, ys[tag], ws, stream=stream)


def _check_block(layers, x_in_host, ys, batch, what):
    """Each product against the oracle on the input the GPU actually used."""
    got = {tag: to_f16(ys[tag]).reshape(-1, batch) for tag in BLOCK}
    for tag in BLOCK:
        L = layers[tag]
        src = SOURCE[tag]
        x = x_in_host if src is None else got[src]
        assert np.isfinite(x.astype(np.float64)).all()
        ref, bound = oracle.matmul(L.codes, L.codebooks, L.scales, x, threads=8)
        assert_close(got[tag].astype(np.float64), ref, bound, f"{what} {tag}")
    return got


def _block_buffers(batch):
    return {tag: torch.empty(LLAMA2_7B_BLOCK[tag][0] * batch, dtype=torch.int16, device="cuda") for tag in BLOCK}


def _block_workspace(dls, batch):
    return workspace(max(aq.aq_gemv_workspace_bytes(dl.desc, batch) for dl in dls.values()))


@pytest.mark.parametrize("K,B", [(1, 16), (2, 8)])
@pytest.mark.parametrize("batch", [1, 4])
def test_decoder_block_chain_matches_oracle(K, B, batch):
    layers = _block_layers(K, B, 7100 + 10 * K + batch)
    dls = {tag: DevLayer(L) for tag, L in layers.items()}
    x = make_activations(4096, batch, (7101, K, batch))
    xd = dev(x.view(np.uint16))
    ws = _block_workspace(dls, batch)
    stream = torch.cuda.Stream()
    for rep in range(2):  # the second pass reuses the workspace left by the first
        ys = _block_buffers(batch)
        torch.cuda.synchronize()
        _launch_block(dls, xd, ys, batch, ws, stream)
        torch.cuda.synchronize()
        assert aq.aq_workspace_status(ws, stream=stream) == 0, "a bounded wait gave up"
        _check_block(layers, x, ys, batch, f"{K}x{B} b{batch} pass {rep}")


@pytest.mark.parametrize("K,B", [(1, 16), (2, 8)])
def test_chained_blocks_in_one_cuda_graph(K, B):
    """Four blocks, each reading the previous block's down output, captured
    as one CUDA graph of 28 launches and replayed twice."""
    nblocks, batch = 4, 1
    blocks = [_block_layers(K, B, (7200, K, b), unit_gain=True) for b in range(nblocks)]
    dls = [{tag: DevLayer(L) for tag, L in layers.items()} for layers in blocks]
    x = make_activations(4096, batch, (7201, K))
    xd = dev(x.view(np.uint16))
    ws = workspace(max(aq.aq_gemv_workspace_bytes(dl.desc, batch) for d in dls for dl in d.values()))
    ys = [_block_buffers(batch) for _ in range(nblocks)]
    stream = torch.cuda.Stream()

    def chain():
        inp = xd
        for b in range(nblocks):
            _launch_block(dls[b], inp, ys[b], batch, ws, stream)
            inp = ys[b]["down"]

    with torch.cuda.stream(stream):
        chain()  # eager once before capture
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        chain()
    for rep in range(2):
        for b in range(nblocks):
            for t in ys[b].values():
                t.fill_(0x7E00)  # binary16 NaN: a product that did not run shows
        torch.cuda.synchronize()
        with torch.cuda.stream(stream):
            graph.replay()
        torch.cuda.synchronize()
        assert aq.aq_workspace_status(ws, stream=stream) == 0, "a bounded wait gave up"
        x_host = x
        for b in range(nblocks):
            got = _check_block(blocks[b], x_host, ys[b], batch, f"{K}x{B} graph replay {rep} block {b}")
            x_host = got["down"]
    del graph


@pytest.mark.parametrize("batch", [1, 4, 16])
def test_rotated_copies_in_one_cuda_graph(batch):
    """76 copies of one 4096 x 4096 1x16 layer at distinct addresses,
    launched back to back in a graph with one shared workspace, as the
    benchmark does: every output equals the oracle within the tolerance and
    all copies agree bit for bit (same weights, same x)."""
    ncopies = 76
    layer = make_layer(LayerSpec(4096, 4096, 1, 16), 7300)
    dl = DevLayer(layer)
    copies = [(dl.packed.clone(), dl.codebooks.clone(), dl.scales.clone()) for _ in range(ncopies)]
    x = make_activations(4096, batch, (7301, batch))
    xd = dev(x.view(np.uint16))
    ys = [torch.empty(4096 * batch, dtype=torch.int16, device="cuda") for _ in range(ncopies)]
    ws = workspace(aq.aq_gemv_workspace_bytes(dl.desc, batch))
    stream = torch.cuda.Stream()

    def step():
        for (p, c, s), y in zip(copies, ys):
            aq.aq_gemv(dl.desc, p, c, s, xd, batch, y, ws, stream=stream)

    with torch.cuda.stream(stream):
        step()
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        step()
    for y in ys:
        y.fill_(0x7E00)
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        graph.replay()
        graph.replay()
    torch.cuda.synchronize()
    assert aq.aq_workspace_status(ws, stream=stream) == 0, "a bounded wait gave up"
    ref, bound = oracle.matmul(layer.codes, layer.codebooks, layer.scales, x, threads=8)
    first = ys[0].cpu().numpy()
    assert_close(to_f16(ys[0]).reshape(4096, batch).astype(np.float64), ref, bound, f"copy 0 b{batch}")
    for i, y in enumerate(ys[1:], 1):
        assert np.array_equal(y.cpu().numpy(), first), f"copy {i} differs from copy 0 (b{batch})"
    del graph


@pytest.mark.parametrize("K,B", [(1, 16), (2, 8)])
@pytest.mark.parametrize("batch", [1, 4, 16])
def test_ordered_entry_point_same_bits_as_gemv(K, B, batch):
    """aq_gemv_ordered (ordinary launches, no weight read before the
    previous kernel completes) runs the same plan as aq_gemv: the block
    chain gives the same bits either way, and both match the oracle."""
    layers = _block_layers(K, B, 7400 + 10 * K + batch)
    dls = {tag: DevLayer(L) for tag, L in layers.items()}
    x = make_activations(4096, batch, (7401, K, batch))
    xd = dev(x.view(np.uint16))
    ws = _block_workspace(dls, batch)
    stream = torch.cuda.Stream()
    ys_pdl, ys_ord = _block_buffers(batch), _block_buffers(batch)
    torch.cuda.synchronize()
    _launch_block(dls, xd, ys_pdl, batch, ws, stream)
    for tag in BLOCK:
        dl = dls[tag]
        src = SOURCE[tag]
        inp = xd if src is None else ys_ord[src]
        aq.aq_gemv_ordered(dl.desc, dl.packed, dl.codebooks, dl.scales, inp, batch, ys_ord[tag], ws, stream=stream)
    torch.cuda.synchronize()
    assert aq.aq_workspace_status(ws, stream=stream) == 0, "a bounded wait gave up"
    for tag in BLOCK:
        assert torch.equal(ys_pdl[tag], ys_ord[tag]), f"{K}x{B} b{batch} {tag}: ordered launch differs"
    _check_block(layers, x, ys_ord, batch, f"ordered {K}x{B} b{batch}")


@pytest.mark.parametrize("K,B", [(1, 16), (2, 8)])
@pytest.mark.parametrize("T", [512, 136])
def test_prefill_block_chain_under_programmatic_launch(K, B, T):
    """The seven prefill products of a Llama-2-7B block on one stream, no
    host synchronisation, one workspace: aq_gemm launches with programmatic
    dependent launch (a kernel reads its weights while the previous product
    may still run; x, y and the workspace only after it).  512 tokens: the
    4096-row products split their input features 4 ways in clusters; 136
    tokens: ragged 256-token tiles.  Each product is checked on sampled rows
    against the oracle applied to the GPU input it consumed, and the same
    chain through aq_gemm_ordered gives the same bits."""
    layers = _block_layers(K, B, (T, K, 3), unit_gain=True)
    dls = {tag: DevLayer(layers[tag]) for tag in BLOCK}
    x_host = make_activations(LLAMA2_7B_BLOCK["q"][1], T, (T, K, 4))
    x = dev(x_host.view(np.uint16))
    ws = workspace(max(aq.aq_gemm_workspace_bytes(dls[tag].desc, T) for tag in BLOCK))
    stream = torch.cuda.Stream()

    def chain(fn):
        ys = {tag: torch.empty(LLAMA2_7B_BLOCK[tag][0] * T, dtype=torch.int16, device="cuda") for tag in BLOCK}
        for tag in BLOCK:
            dl = dls[tag]
            src = SOURCE[tag]
            fn(dl.desc, dl.packed, dl.codebooks, dl.scales, x if src is None else ys[src], T, ys[tag], ws,
               stream=stream)
        torch.cuda.synchronize()
        return ys

    ys = chain(aq.aq_gemm)
    assert aq.aq_workspace_status(ws, stream=stream) == 0, "a bounded wait gave up"
    got = {tag: to_f16(ys[tag]).reshape(-1, T) for tag in BLOCK}
    rng = np.random.default_rng(T + K)
    for tag in BLOCK:
        L = layers[tag]
        src = SOURCE[tag]
        xin = x_host if src is None else got[src]
        assert np.isfinite(xin.astype(np.float64)).all()
        out = LLAMA2_7B_BLOCK[tag][0]
        rows = np.unique(np.concatenate([rng.choice(out, size=20, replace=False), [0, 127, 128, out - 1]]))
        ref, bound = oracle.matmul(L.codes, L.codebooks, L.scales, xin, rows=rows, threads=8)
        assert_close(got[tag][rows].astype(np.float64), ref, bound, f"prefill chain {K}x{B} T{T} {tag}")
    ys2 = chain(aq.aq_gemm_ordered)
    for tag in BLOCK:
        assert torch.equal(ys[tag], ys2[tag]), f"ordered launch differs at {tag}"
