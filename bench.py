"""Benchmark of the additive-quantised decode-time product on B200.

Default workload (``llama2-7b-decode``): the decode-time products the metric
names, 1x16 and 2x8 at Llama-2-7B shapes --
* 4096 x 4096 layers in 1x16 (K = 1, B = 16, g = 8; 2 bits per weight) at
  batch 1, 4 and 16;
* the MLP layers 11008 x 4096 and 4096 x 11008 in 2x8 (K = 2, B = 8), with
  uniform and with Zipf(1.1)-skewed codes, at batch 1 and 8.
One step = the product at each batch for every layer of a rotation set of
distinct copies per shape (about 4 GB of layer bytes per shape, 30x the L2
cache, so codes and codebooks come from HBM, not L2), ordered batch-major
so that a layer is re-read only after every other layer.  The timed region
replays a CUDA graph of one step K times, bracketed by a barrier and device
synchronisation; time comes from CUDA events on the launching stream, max
over ranks.  Per-kernel times are the median over further replays of the
same graph.

Metric: achieved throughput of algorithmic bytes (codes + codebooks +
scales + x + y per product; the dense matrix is never counted) in GB/s,
plus microseconds per layer for each shape and batch.  The roofline object
reports the dominant kernel against the measured HBM copy bandwidth, with
the read-only HBM stream and the 1x16 codeword-read ceiling beside it.

``--impl reference`` times the CPU oracle (the plain fp64 C implementation
the tests compare against) on a bounded sample of the same workload.

Launch: ``python bench.py [--gpus N --steps K --warmup W]``; for N > 1 under
``torch.distributed.run`` (one rank per GPU, independent layers per rank,
no collective on the data path: weak scaling).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from aq_inputs import LayerSpec, make_activations, make_layer, workload_units  # noqa: E402

METRIC = "AQ-GEMV µs/layer & achieved HBM GB/s vs roofline (1x16, 2x8; batch 1–16)"
WORKLOAD = "llama2-7b-decode"
L2_BYTES = 126 * 1024 * 1024
ROTATION_BYTES = 4e9  # layer bytes per shape in the rotation set of a decode step


def alg_bytes(spec: LayerSpec, n: int) -> int:
    """Algorithmic bytes of one product: codes, codebooks, scales, x, y."""
    codes = spec.out_features * spec.groups * spec.num_codebooks * spec.nbits // 8
    cbs = spec.num_codebooks * (1 << spec.nbits) * 8 * 2
    return codes + cbs + 2 * spec.out_features + 2 * spec.in_features * n + 2 * spec.out_features * n


def bits_per_weight(spec: LayerSpec) -> dict:
    """Stored bits per weight of one layer: the closed form K*B/8 (codes
    only) and with the codebooks and row scales counted."""
    return {"codes": spec.num_codebooks * spec.nbits / 8,
            "stored": round(8 * alg_bytes(spec, 0) / (spec.out_features * spec.in_features), 3)}


def measured_peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


# ---------------------------------------------------------------------------
# distributed plumbing
# ---------------------------------------------------------------------------

def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def init_dist(world: int, backend: str):
    if world <= 1:
        return None
    import datetime

    import torch.distributed as dist
    os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
    dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))
    return dist


def max_over_ranks(value: float, dist, device=None) -> float:
    if dist is None:
        return value
    import torch
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ---------------------------------------------------------------------------
# clocks sampled during the timed region
# ---------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int, path: str | None = None):
        self.gpu = gpu_index
        self.proc = None
        self.path = path

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.25)
        return self

    def __exit__(self, *exc):
        time.sleep(0.15)
        self.lines = []
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [l for l in out.splitlines() if l.strip()]
        if self.path:
            with open(self.path, "w") as f:
                f.write("\n".join(self.lines) + "\n")

    def summary(self) -> dict:
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for l in self.lines:
            f = [v.strip() for v in l.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        # samples under load: the top half of the observed clock range
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------------------
# CPU oracle (baseline and reference arm)
# ---------------------------------------------------------------------------

_SAMPLE_INPUTS = {}


def _sample_layer(tag, spec, seed):
    key = (tag, seed)
    if key not in _SAMPLE_INPUTS:
        _SAMPLE_INPUTS[key] = make_layer(spec, (seed, 0))
    return _SAMPLE_INPUTS[key]


def oracle_sample(units, frac: float, threads: int):
    """Time the oracle on the first ``frac`` of the rows (at least 8) of one
    layer of each unit, at each of the unit's batches.

    Returns (seconds, algorithmic bytes the sample stands for)."""
    import oracle
    dt = nbytes = 0.0
    for tag, spec, batches, seed in units:
        layer = _sample_layer(tag, spec, seed)
        rows = int(min(spec.out_features, max(8, round(frac * spec.out_features))))
        sel = np.arange(rows, dtype=np.int64)
        for b in batches:
            x = make_activations(spec.in_features, b, (seed, 0, b))
            t0 = time.perf_counter()
            oracle.matmul(layer.codes, layer.codebooks, layer.scales, x, rows=sel, threads=threads)
            dt += time.perf_counter() - t0
            nbytes += alg_bytes(spec, b) * rows / spec.out_features
    return dt, nbytes


def _sized_sample(units, threads: int, budget_s: float):
    """Row fraction whose oracle sample takes about ``budget_s`` seconds."""
    f = 1.0 / 512
    for _ in range(3):  # small samples carry a fixed cost: re-measure nearer the target
        dt, _ = oracle_sample(units, f, threads)
        target = min(1.0, f * budget_s / max(dt, 1e-4))
        if target <= 4 * f:
            return float(target)
        f = target / 4
    return float(target)


def _describe(units, frac: float) -> str:
    parts = [f"{tag} {spec.scheme} b{'/'.join(map(str, n))}" for tag, spec, n, _ in units]
    return (f"first {frac:.2%} of the rows (at least 8) of one layer of each shape: " + "; ".join(parts)
            + " (fp64 C oracle, OpenMP over rows), scaled to the layers' algorithmic bytes")


def cpu_model() -> str:
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def cpu_baseline(units, budget_s: float = 10.0, single_budget_s: float = 3.0) -> dict:
    import oracle
    threads = os.cpu_count() or 1
    frac = _sized_sample(units, threads, budget_s)
    dt, nbytes = oracle_sample(units, frac, threads)
    frac1 = _sized_sample(units, 1, single_budget_s)
    dt1, nbytes1 = oracle_sample(units, frac1, 1)
    return {"value": nbytes / dt / 1e9, "unit": "GB/s", "cores": min(threads, oracle.max_threads()),
            "kind": "oracle", "sample": _describe(units, frac),
            "single_thread": {"value": nbytes1 / dt1 / 1e9, "row_fraction": round(frac1, 5)},
            "nproc": threads, "cpu_model": cpu_model()}


def run_reference(args) -> None:
    world, rank, _ = dist_env()
    if rank != 0:
        return
    import oracle
    threads = os.cpu_count() or 1
    units = workload_units(args.workload)
    frac = _sized_sample(units, threads, 2.0)  # ~2 s of oracle work per step
    for _ in range(args.warmup):
        oracle_sample(units, frac, threads)
    total_t, total_b = 0.0, 0.0
    for _ in range(args.steps):
        dt, nb = oracle_sample(units, frac, threads)
        total_t += dt
        total_b += nb
    value = total_b / total_t / 1e9
    cores = min(threads, oracle.max_threads())
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * total_t / max(args.steps, 1), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": args.workload,
                   "layers": [f"{tag} {spec.scheme} g8" for tag, spec, _, _ in units],
                   "batches": {tag: list(n) for tag, _, n, _ in units},
                   "row_fraction_per_step": round(frac, 5)},
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": cores, "kind": "oracle",
                         "sample": _describe(units, frac) + ", per step"},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------

def count_graph_kernels(graph) -> int:
    """Kernel nodes in a captured graph (needs ``keep_graph=True``)."""
    from cuda.bindings import runtime as rt
    raw = graph.raw_cuda_graph()
    g = raw if isinstance(raw, rt.cudaGraph_t) else rt.cudaGraph_t(init_value=int(raw))
    err, _, n = rt.cudaGraphGetNodes(g, 0)
    if int(err) != 0:
        raise RuntimeError(f"cudaGraphGetNodes: {err}")
    err, nodes, n = rt.cudaGraphGetNodes(g, n)
    if int(err) != 0:
        raise RuntimeError(f"cudaGraphGetNodes: {err}")
    kernel = rt.cudaGraphNodeType.cudaGraphNodeTypeKernel
    count = 0
    for nd in nodes[:n]:
        err, t = rt.cudaGraphNodeGetType(nd)
        if int(err) == 0 and t == kernel:
            count += 1
    return count


def recorded_traffic(layer: str, batch: int):
    """DRAM bytes per launch of the product on ``layer`` at ``batch`` from
    the committed ncu record, or None when there is none or the kernel
    sources changed since the counters were taken."""
    import hashlib
    p = os.path.join(ROOT, "profiles", "traffic_gemv_llama2-7b-1x16.json")
    if not os.path.exists(p):
        return None
    rec = json.load(open(p))
    if layer != rec.get("layer"):
        return None
    h = hashlib.sha256()
    for f in rec["sources"]:
        h.update(open(os.path.join(ROOT, f), "rb").read())
    if h.hexdigest() != rec["sources_sha256"]:
        return None
    return rec["per_launch_bytes"].get(str(batch))


def encode_flops(spec: LayerSpec, beam: int) -> int:
    """Arithmetic of one aq_encode call: (H e)_g for every row and group
    (2 out in^2) plus scoring every code of every slot for each live beam
    (one at a group's first slot, `beam` after it; about 18 flops per
    score)."""
    G = spec.in_features // 8
    beams_per_group = 1 + (spec.num_codebooks - 1) * beam
    return (2 * spec.out_features * spec.in_features ** 2
            + spec.out_features * G * beams_per_group * (1 << spec.nbits) * 18)


def encode_inputs(spec: LayerSpec, beam: int, seed) -> dict:
    """Synthetic encoder inputs on the device: weights, H = 2 X^T X / n from
    random activations, starting codes; the codes buffer it writes."""
    import torch
    rng = np.random.default_rng(seed)
    w = rng.normal(0, 0.02, size=(spec.out_features, spec.in_features)).astype(np.float16)
    x = torch.from_numpy(rng.normal(0, 1, size=(512, spec.in_features)).astype(np.float32)).cuda()
    h = (2.0 / 512) * (x.T @ x)
    c0 = rng.integers(0, 1 << spec.nbits, size=(spec.out_features, spec.in_features // 8, spec.num_codebooks))
    codes = torch.from_numpy(c0.astype(np.uint8) if spec.nbits == 8 else c0.astype(np.uint16).view(np.int16)).cuda()
    return {"w": torch.from_numpy(w.view(np.int16)).cuda(), "h": h.contiguous(), "codes_in": codes,
            "codes_out": torch.empty_like(codes)}


def flops(spec: LayerSpec, n: int) -> int:
    return 2 * spec.out_features * spec.in_features * n


def gather_ceiling(aq, units, kernels, stream, reps: int = 5):
    """Codeword-read ceiling of each 1x16 shape: aq_gather_probe (the same
    random 16-byte codeword reads as the GEMV, one per code, nothing else)
    over the same rotated layer copies, captured in a CUDA graph and timed
    with CUDA events like the GEMV; mode 0 reads from L2 into shared memory
    as the tensor-core GEMV's decoders do, mode 1 from the codebook split
    over 8-CTA clusters' shared memory, mode 2 through L1 into registers as
    the batch-1 CUDA-core GEMV does, mode 4 from the codebook sliced over
    8-CTA clusters with each code handled by the CTA holding its slice."""
    import torch
    rows, seen = [], set()
    for u in units:
        spec = u.get("spec")
        if spec is None or (spec.num_codebooks, spec.nbits) != (1, 16) or u["tag"] in seen:
            continue
        seen.add(u["tag"])
        n = spec.out_features * spec.in_features // 64 * 8  # the layer's codes, a multiple of 8
        row = {"layer": u["tag"], "codes": n}
        for mode, key in ((0, "l2_cp_async"), (1, "dsmem_cluster8"), (2, "l1_ldg"), (4, "slice_cluster8")):
            sink = torch.zeros(aq.aq_gather_probe_sink_bytes(mode) // 4, dtype=torch.int32, device=stream.device)

            def once():
                for packed, cb, _ in u["copies"]:
                    aq.aq_gather_probe(cb, packed, n, mode, sink, stream=stream)

            with torch.cuda.stream(stream):
                once()
            torch.cuda.synchronize()
            graph = torch.cuda.CUDAGraph(keep_graph=True)
            with torch.cuda.graph(graph, stream=stream):
                once()
            graph.instantiate()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            with torch.cuda.stream(stream):
                graph.replay()
                e0.record(stream)
                for _ in range(reps):
                    graph.replay()
                e1.record(stream)
            torch.cuda.synchronize()
            us = 1e3 * e0.elapsed_time(e1) / (reps * len(u["copies"]))
            row[f"{key}_us_per_layer"] = round(us, 3)
            row[f"{key}_gathers_per_s"] = round(n / (us * 1e-6), -6)
            del graph
        # the ceiling is the fastest route the products take: through L1
        # into registers (CUDA-core and register-fragment kernels) or from L2
        # into shared memory; the codebook-slice route (mode 4) is reported
        # beside it as the route a kernel could take instead
        row["ceiling_us_per_layer"] = min(row["l2_cp_async_us_per_layer"], row["l1_ldg_us_per_layer"])
        row["slice_vs_l1"] = round(row["l1_ldg_us_per_layer"] / row["slice_cluster8_us_per_layer"], 3)
        for k in kernels:
            if k["layer"] == u["tag"] and "us_per_layer" in k:
                row[f"gemv_n{k['n']}_us"] = k["us_per_layer"]
                row[f"gemv_n{k['n']}_frac_of_ceiling"] = round(row["ceiling_us_per_layer"] / k["us_per_layer"], 3)
        rows.append(row)
    return rows or None


def hbm_read_probe(aq, dev, stream, copy_gbs: float, nbytes: int = 4 << 30, reps: int = 7) -> dict:
    """Read-only HBM bandwidth: aq_gather_probe mode 3 streams one array of
    ``nbytes`` (32x the L2 cache) once per call; median of ``reps`` calls
    timed with CUDA events on the launching stream."""
    import torch
    buf = torch.empty(nbytes, dtype=torch.uint8, device=dev)  # contents do not matter
    sink = torch.zeros(aq.aq_gather_probe_sink_bytes(3) // 4, dtype=torch.int32, device=dev)
    n = nbytes // 2
    times = []
    with torch.cuda.stream(stream):
        aq.aq_gather_probe(None, buf, n, 3, sink, stream=stream)
        for _ in range(reps):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            aq.aq_gather_probe(None, buf, n, 3, sink, stream=stream)
            e1.record(stream)
            e1.synchronize()
            times.append(e0.elapsed_time(e1) * 1e-3)
    del buf
    gbs = nbytes / statistics.median(times) / 1e9
    return {"gbs": round(gbs, 1), "bytes": nbytes, "reps": reps, "vs_copy_peak": round(gbs / copy_gbs, 4),
            "how": "aq_gather_probe mode 3: one 4 GiB array read once per call with 16-byte loads, "
                   "median of CUDA-event times"}


def run_gpu(args) -> None:
    import torch

    import additive_quantized_matmul_b200 as aq
    from aq_inputs import workload

    world, rank, local = dist_env()
    torch.cuda.set_device(local)
    dist = init_dist(world, "nccl")
    dev = torch.device("cuda", local)
    wl = workload(args.workload)
    layer_units = workload_units(args.workload)
    op = {"llama2-7b-prefill": "gemm", "llama2-7b-grad": "grad", "llama2-7b-encode": "encode"}.get(args.workload, "gemv")
    tensor_op = op in ("gemm", "grad")  # reported in TFLOP/s against the tensor peak
    alu_op = op == "encode"             # fp32 CUDA-core work, reported against the derived fp32 FMA peak
    peaks = measured_peaks()

    # ---- units: one (layer shape, batch) product kind each, over a rotation
    #      set of copies at distinct addresses (> 3x L2 per shape) -----------
    def device_layer(spec, seed):
        desc = aq.LayerDesc.make(spec.out_features, spec.in_features, spec.num_codebooks, spec.nbits)
        L = make_layer(spec, seed)
        codes = torch.from_numpy(L.codes.view(np.int16) if spec.nbits > 8 else L.codes).to(dev)
        packed = torch.empty(aq.aq_packed_codes_bytes(desc), dtype=torch.uint8, device=dev)
        aq.aq_pack_codes(desc, codes, packed)
        cb = torch.from_numpy(L.codebooks.view(np.int16)).to(dev)
        sc = torch.from_numpy(L.scales.view(np.int16)).to(dev)
        return desc, packed, cb, sc

    units = []
    rotation = max(3 * L2_BYTES, args.rotation_gb * 1e9)
    for si, (tag, spec, batches, seed) in enumerate(layer_units):
        desc, packed0, cb0, sc0 = device_layer(spec, (seed, rank, si))  # seeded per rank and shape
        lb = alg_bytes(spec, 0)
        ncopies = args.layers or (1 if alu_op else 3 if tensor_op else max(4, int(rotation / lb) + 1))
        copies = [(packed0.clone(), cb0.clone(), sc0.clone()) for _ in range(ncopies)]
        del packed0, cb0, sc0
        for n in batches:
            x = torch.from_numpy(make_activations(spec.in_features, n, (seed, rank, si, n)).view(np.int16)).to(dev)
            nbytes = {"gemm": aq.aq_gemm_workspace_bytes, "grad": aq.aq_param_grad_workspace_bytes,
                      "gemv": aq.aq_gemv_workspace_bytes,
                      "encode": lambda d, n: aq.aq_encode_workspace_bytes(d)}[op](desc, n)
            units.append({
                "tag": tag, "spec": spec, "n": n, "desc": desc, "copies": copies, "x": x,
                "bytes": alg_bytes(spec, n), "flops": encode_flops(spec, n) if op == "encode" else flops(spec, n),
                **(encode_inputs(spec, n, (seed, rank, si)) if op == "encode" else {}),
                **({"gy": torch.from_numpy(make_activations(spec.out_features, n, (seed, rank, si, n, 1))
                                           .view(np.int16)).to(dev),
                    "grad_s": torch.empty(spec.out_features, dtype=torch.float32, device=dev),
                    "grad_cb": torch.empty((spec.num_codebooks << spec.nbits) * 8, dtype=torch.float32, device=dev)}
                   if op == "grad" else {}),
                "ys": [torch.empty(spec.out_features * n, dtype=torch.int16, device=dev) for _ in range(ncopies)],
                "ws": torch.zeros(max(nbytes, 16), dtype=torch.uint8, device=dev),
                # two events per group of same-shape launches (event nodes between
                # every launch would add their own cost to each measurement)
                "evs": [torch.cuda.Event(enable_timing=True, external=True) for _ in range(2)],
            })
    # chained decoder blocks: one unit per scheme, each copy a whole block of
    # layers whose inputs are the block input or an earlier layer's output
    for ci, (tag, chain) in enumerate(wl.get("chains", [])):
        layers = [device_layer(spec, (wl["seed"], rank, ci, li)) for li, (_, spec, _) in enumerate(chain)]
        block_bytes = sum(alg_bytes(spec, 1) for _, spec, _ in chain)
        ncopies = args.layers or max(4, int(3 * L2_BYTES / block_bytes) + 1)
        copies = [[(p.clone(), c.clone(), q.clone()) for _, p, c, q in layers] for _ in range(ncopies)]
        tags = [t for t, _, _ in chain]
        wsb = max(aq.aq_gemv_workspace_bytes(d, 1) for d, _, _, _ in layers)
        units.append({
            "tag": tag, "n": 1, "copies": copies,
            "chain": [(d, spec, None if s_ is None else tags.index(s_)) for (d, _, _, _), (_, spec, s_) in zip(layers, chain)],
            "x": torch.from_numpy(make_activations(chain[0][1].in_features, 1, (wl["seed"], rank, ci)).view(np.int16)).to(dev),
            "ys": [[torch.empty(spec.out_features, dtype=torch.int16, device=dev) for _, spec, _ in chain]
                   for _ in range(ncopies)],
            "bytes": block_bytes, "flops": sum(flops(spec, 1) for _, spec, _ in chain),
            "ws": torch.zeros(max(wsb, 16), dtype=torch.uint8, device=dev),
            "evs": [torch.cuda.Event(enable_timing=True, external=True) for _ in range(2)],
        })
        del layers
    torch.cuda.synchronize()
    stream = torch.cuda.Stream(device=dev)

    def run(u, i, x_in, y_out, s):
        """Copy i of unit u on stream s: one product, or a whole chained block
        (whose last layer writes y_out, the others their own buffers)."""
        if "chain" in u:
            ys = u["ys"][i]
            for li, (desc, spec, src) in enumerate(u["chain"]):
                packed, cb, sc = u["copies"][i][li]
                inp = x_in if src is None else ys[src]
                out = y_out if li == len(u["chain"]) - 1 else ys[li]
                aq.aq_gemv(desc, packed, cb, sc, inp, 1, out, u["ws"], stream=s)
            return
        packed, cb, sc = u["copies"][i]
        if op == "encode":
            aq.aq_encode(u["desc"], u["w"], u["h"], cb, u["codes_in"], u["n"], u["codes_out"], u["ws"], stream=s)
            return
        if op == "grad":
            aq.aq_param_grad(u["desc"], packed, cb, sc, x_in, u["gy"], u["n"], u["grad_s"], u["grad_cb"], u["ws"],
                             stream=s)
        elif op == "gemm":
            aq.aq_gemm(u["desc"], packed, cb, sc, x_in, u["n"], y_out, u["ws"], stream=s)
        else:
            aq.aq_gemv(u["desc"], packed, cb, sc, x_in, u["n"], y_out, u["ws"], stream=s)

    def out_buf(u, i):
        return u["ys"][i][-1] if "chain" in u else u["ys"][i]

    def call(u, i, s):
        run(u, i, u["x"], out_buf(u, i), s)

    def one_step(record: bool):
        s = torch.cuda.current_stream()
        for u in units:
            if record:
                u["evs"][0].record(s)
            for i in range(len(u["copies"])):
                call(u, i, s)
            if record:
                u["evs"][1].record(s)

    with torch.cuda.stream(stream):
        one_step(False)  # eager warm-up (the library is compiled ahead of time)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph(keep_graph=True)
    with torch.cuda.graph(graph, stream=stream):
        one_step(True)
    launches_per_step = count_graph_kernels(graph)
    graph.instantiate()
    torch.cuda.synchronize()
    for _ in range(max(args.warmup, 0)):
        graph.replay()
    torch.cuda.synchronize()

    t_start = torch.cuda.Event(enable_timing=True)
    t_stop = torch.cuda.Event(enable_timing=True)
    cvd = os.environ.get("CUDA_VISIBLE_DEVICES", "")
    gpu_index = int(cvd.split(",")[local]) if cvd.replace(",", "").isdigit() else local
    # the raw clock samples go to the CSV named by AQ_CLOCK_LOG ({rank} is
    # replaced by the rank), if set; the JSON line carries their summary
    log = os.environ.get("AQ_CLOCK_LOG")
    if log:
        log = log.replace("{rank}", str(rank))
        os.makedirs(os.path.dirname(os.path.abspath(log)), exist_ok=True)
    sampler = ClockSampler(gpu_index, log)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    with sampler:
        with torch.cuda.stream(stream):
            t_start.record(stream)
            for _ in range(args.steps):
                graph.replay()
            t_stop.record(stream)
        torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    elapsed_ms = max_over_ranks(t_start.elapsed_time(t_stop), dist, dev)

    # per-kernel times: average duration per launch of each group of
    # same-shape launches (events on the launching stream), median over
    # further replays of the same graph
    per_unit = [[] for _ in units]
    with torch.cuda.stream(stream):
        for _ in range(max(1, args.median_replays)):
            graph.replay()
            torch.cuda.synchronize()
            for ui, u in enumerate(units):
                per_unit[ui].append(1e3 * u["evs"][0].elapsed_time(u["evs"][1]) / len(u["copies"]))
    status_ok = all(aq.aq_workspace_status(u["ws"]) == 0 for u in units)

    kernels = []
    step_bytes = step_flops = 0
    for u, times in zip(units, per_unit):
        us = statistics.median(times)
        nb, nf = u["bytes"], u["flops"]
        step_bytes += nb * len(u["copies"])
        step_flops += nf * len(u["copies"])
        k = {"layer": u["tag"], "n": u["n"], "us_per_layer": round(us, 3),
             "gbs": round(nb / (us * 1e-6) / 1e9, 1), "tflops": round(nf / (us * 1e-6) / 1e12, 2),
             "bytes_per_call": nb, "copies": len(u["copies"]), "total_us": us * len(u["copies"]),
             "us_range": [round(min(times), 3), round(max(times), 3)]}
        if "chain" in u:  # one call is a whole block of layers
            k["layers_per_call"] = len(u["chain"])
            k["us_per_block"] = k.pop("us_per_layer")
        if op == "gemv" and "spec" in u:
            k["bits_per_weight"] = bits_per_weight(u["spec"])
        k["frac_hbm"] = round(k["gbs"] / peaks["hbm_gbs"], 4)
        k["frac_tensor"] = round(k["tflops"] / peaks["bf16_tflops_sustained"], 4)
        kernels.append(k)
    dom = max(kernels, key=lambda k: k["total_us"])
    if alu_op:
        value = world * step_flops * args.steps / (elapsed_ms * 1e-3) / 1e12
        unit = "TFLOP/s"
        fp32_peak = 148 * 128 * 2 * 1.965e9 / 1e12  # SMs x fp32 FMA lanes x 2 flops x max SM clock
        roofline = {"bound": "alu", "achieved": dom["tflops"], "peak": round(fp32_peak, 1), "unit": "TFLOP/s",
                    "frac": round(dom["tflops"] / fp32_peak, 4), "traffic": None,
                    "kernel": f"aq_encode {dom['layer']} beam={dom['n']}",
                    "peak_source": "derived: 148 SMs x 128 fp32 FMA/clk x 2 x 1965 MHz"}
    elif tensor_op:
        value = world * step_flops * args.steps / (elapsed_ms * 1e-3) / 1e12
        unit = "TFLOP/s"
        roofline = {"bound": "tensor", "achieved": dom["tflops"], "peak": peaks["bf16_tflops_sustained"],
                    "unit": "TFLOP/s", "frac": dom["frac_tensor"], "traffic": None,
                    "kernel": f"aq_{'param_grad' if op == 'grad' else 'gemm'} {dom['layer']} T={dom['n']}",
                    "peak_source": f"{peaks['source']} bf16_tflops_sustained (cuBLAS bf16; fp16 tcgen05 has the same rate)"}
    else:
        value = world * step_bytes * args.steps / (elapsed_ms * 1e-3) / 1e9
        unit = "GB/s"
        roofline = {"bound": "hbm", "achieved": dom["gbs"], "peak": peaks["hbm_gbs"], "unit": "GB/s",
                    "frac": dom["frac_hbm"], "traffic": recorded_traffic(dom["layer"], dom["n"]),
                    "kernel": f"aq_gemv {dom['layer']} batch {dom['n']}",
                    "peak_source": f"{peaks['source']} hbm_gbs (STREAM-style copy)"}
    for k in kernels:
        del k["total_us"]

    # ---- read-only HBM stream beside the copy figure of the peak -------------
    if op == "gemv" and not args.skip_hbm_probe:
        roofline["hbm_read_probe"] = hbm_read_probe(aq, dev, stream, peaks["hbm_gbs"])

    # ---- codeword-read ceiling of the 1x16 shapes (secondary bound) ----------
    if op == "gemv" and not args.skip_ceiling:
        ceiling = gather_ceiling(aq, units, kernels, stream)
        if ceiling:
            roofline["gather_ceiling"] = ceiling

    # ---- end-to-end through the public API with host buffers ----------------
    e2e = None
    if not args.skip_e2e and op not in ("grad", "encode"):  # the gradient's outputs are parameters, not a per-step result
        hx = [torch.empty((len(u["copies"]), u["x"].numel()), dtype=torch.int16).pin_memory() for u in units]
        hy = [torch.empty((len(u["copies"]), out_buf(u, 0).numel()), dtype=torch.int16).pin_memory() for u in units]
        dx = [torch.empty(h.shape, dtype=torch.int16, device=dev) for h in hx]
        dy = [torch.empty(h.shape, dtype=torch.int16, device=dev) for h in hy]
        for h, u in zip(hx, units):
            h.copy_(u["x"].cpu().reshape(1, -1).expand(h.shape[0], -1))
        h2d = sum(h.numel() * 2 for h in hx)
        d2h = sum(h.numel() * 2 for h in hy)
        e_steps = max(1, min(args.steps, args.e2e_steps))

        # Transfers overlap the products: a unit's copies go in chunks; a
        # chunk's inputs come in on one stream while earlier chunks compute,
        # its results go out on another; per-chunk events keep the buffers
        # safe across steps (a chunk's next inputs wait until its products
        # ran, its next products until its results left).  Every step still
        # moves all its inputs in and all its results out, and ends when the
        # results are on the host.
        cin, cout = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
        chunks = [[(c0, min(len(u["copies"]), c0 + max(1, -(-len(u["copies"]) // 4))))
                   for c0 in range(0, len(u["copies"]), max(1, -(-len(u["copies"]) // 4)))] for u in units]
        ev_used, ev_out = {}, {}

        def e2e_step():
            s = torch.cuda.current_stream()
            for ui, u in enumerate(units):
                for c0, c1 in chunks[ui]:
                    key = (ui, c0)
                    if key in ev_used:
                        cin.wait_event(ev_used[key])
                    with torch.cuda.stream(cin):
                        dx[ui][c0:c1].copy_(hx[ui][c0:c1], non_blocking=True)
                    e_in = torch.cuda.Event()
                    e_in.record(cin)
                    s.wait_event(e_in)
                    if key in ev_out:
                        s.wait_event(ev_out[key])
                    for i in range(c0, c1):
                        run(u, i, dx[ui][i], dy[ui][i], s)
                    e_c = torch.cuda.Event()
                    e_c.record(s)
                    ev_used[key] = e_c
                    cout.wait_event(e_c)
                    with torch.cuda.stream(cout):
                        hy[ui][c0:c1].copy_(dy[ui][c0:c1], non_blocking=True)
                    e_o = torch.cuda.Event()
                    e_o.record(cout)
                    ev_out[key] = e_o
            s.wait_stream(cout)

        e2e_step()
        torch.cuda.synchronize()
        if dist is not None:
            dist.barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(e_steps):
            e2e_step()
        e1.record()
        torch.cuda.synchronize()
        e_ms = max_over_ranks(e0.elapsed_time(e1), dist, dev)
        tot = (step_flops / 1e12) if tensor_op else (step_bytes / 1e9)
        e2e = {"value": round(world * tot * e_steps / (e_ms * 1e-3), 2), "unit": unit,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": e_steps,
               "api": "additive_quantized_matmul_b200 (C ABI via ctypes), eager, pinned host buffers, "
                      "transfers on their own streams overlapping the products (4 chunks per shape and batch)"}

    cpu = None
    if rank == 0 and world == 1 and not args.skip_cpu and op == "gemv" and layer_units:
        cpu = cpu_baseline(layer_units)

    if rank == 0:
        shapes = [f"{t} {sp.scheme} g8" for t, sp, _, _ in layer_units]
        shapes += [f"{t}: " + ", ".join(f"{lt} {sp.out_features}x{sp.in_features} {sp.scheme}" for lt, sp, _ in ch)
                   for t, ch in wl.get("chains", [])]
        line = {
            "metric": METRIC, "value": round(value, 2), "unit": unit, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(elapsed_ms / args.steps, 4), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f16", "accumulate": "f32",
            "data": "synthetic",
            "config": {"workload": args.workload,
                       "layers": shapes,
                       "n": {t: list(n) for t, _, n, _ in layer_units} if layer_units else [1],
                       "copies_per_shape": {u["tag"]: len(u["copies"]) for u in units},
                       **({"chain": "per block: q, k, v read the block input; o reads v; gate and up "
                                    "read o; down reads up (one stream, each launch waits on the previous)"}
                          if wl.get("chains") else {}),
                       "l2": "inputs larger than L2: per shape, copies at distinct addresses whose "
                             "bytes exceed 3x the 126 MB L2 (about 4 GB per decode-time shape), visited in "
                             "turn before any is re-read",
                       "kernel_times": f"median over {max(1, args.median_replays)} replays of the step's graph",
                       "parallelism": f"replicas x{world} (independent layers per rank)"},
            "kernels": kernels, "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
            "clocks": sampler.summary(), "status_ok": status_ok,
            "gpu_launches": launches_per_step * args.steps,
        }
        if op == "gemv" and layer_units:
            line["us_per_layer"] = {f"{k['layer']} b{k['n']}": k["us_per_layer"] for k in kernels}
        print(json.dumps(line), flush=True)
    del graph
    if dist is not None:
        dist.destroy_process_group()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--skip-ceiling", action="store_true",
                    help="do not time the 1x16 codeword-read ceiling (aq_gather_probe)")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=WORKLOAD,
                    help="llama2-7b-decode (default), llama2-7b-1x16, llama2-7b-mlp-2x8, llama2-70b-1x16, "
                         "llama2-7b-prefill, llama2-7b-block, llama2-7b-schemes, llama2-7b-grad, "
                         "llama2-7b-encode, tiny-2x8")
    ap.add_argument("--layers", type=int, default=0, help="copies per shape (0: --rotation-gb of layer bytes)")
    ap.add_argument("--rotation-gb", type=float, default=ROTATION_BYTES / 1e9,
                    help="layer bytes per shape in the rotation set of a decode step (at least 3x L2)")
    ap.add_argument("--median-replays", type=int, default=10,
                    help="replays of the step's graph after the timed region for per-kernel medians")
    ap.add_argument("--skip-hbm-probe", action="store_true", help="do not time the read-only HBM stream")
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--skip-e2e", action="store_true")
    ap.add_argument("--skip-cpu", action="store_true")
    args = ap.parse_args()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
