"""Benchmark of the additive-quantised decode-time product on B200.

Workload: Llama-2-7B-shaped 1x16 layers (out = in = 4096, g = 8, K = 1,
B = 16; 2 bits per weight), decode-time products at batch 1, 4 and 16.
One step = the product at each batch for every layer of a rotation set of
distinct layers whose bytes exceed three times the L2 cache (codes and
codebooks come from HBM, not L2), ordered batch-major so that a layer is
re-read only after every other layer.  The timed region replays a CUDA graph
of one step K times, bracketed by a barrier and device synchronisation;
time comes from CUDA events on the launching stream, max over ranks.

Metric: achieved throughput of algorithmic bytes (codes + codebooks +
scales + x + y per product; the dense matrix is never counted) in GB/s,
plus microseconds per layer for each batch.  The roofline object reports
the dominant kernel against the measured HBM copy bandwidth.

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

from aq_inputs import LayerSpec, make_activations, make_layer  # noqa: E402

METRIC = "AQ-GEMV µs/layer & achieved HBM GB/s vs roofline (1x16, 2x8; batch 1–16)"
WORKLOAD = "llama2-7b-1x16"
SPEC = LayerSpec(4096, 4096, 1, 16)
BATCHES = (1, 4, 16)
SEED = 1001
L2_BYTES = 126 * 1024 * 1024


def alg_bytes(spec: LayerSpec, n: int) -> int:
    """Algorithmic bytes of one product: codes, codebooks, scales, x, y."""
    codes = spec.out_features * spec.groups * spec.num_codebooks * spec.nbits // 8
    cbs = spec.num_codebooks * (1 << spec.nbits) * 8 * 2
    return codes + cbs + 2 * spec.out_features + 2 * spec.in_features * n + 2 * spec.out_features * n


def measured_peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"], "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "source": "fallback"}


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
                 "--format=csv,noheader,nounits", "-lms", "100"],
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


def oracle_sample(rows: int, threads: int, repeats: int = 1):
    """Time the oracle on ``rows`` rows of one layer at every batch.

    Returns (seconds, algorithmic bytes the sample stands for)."""
    import oracle
    if not _SAMPLE_INPUTS:
        _SAMPLE_INPUTS["layer"] = make_layer(SPEC, (SEED, 0, 0))
        _SAMPLE_INPUTS["xs"] = {b: make_activations(SPEC.in_features, b, (SEED, 0, b)) for b in BATCHES}
    layer, xs = _SAMPLE_INPUTS["layer"], _SAMPLE_INPUTS["xs"]
    sel = np.arange(rows, dtype=np.int64)
    frac = rows / SPEC.out_features
    t0 = time.perf_counter()
    for _ in range(repeats):
        for b in BATCHES:
            oracle.matmul(layer.codes, layer.codebooks, layer.scales, xs[b], rows=sel, threads=threads)
    dt = time.perf_counter() - t0
    nbytes = repeats * sum(alg_bytes(SPEC, b) for b in BATCHES) * frac
    return dt, nbytes


def cpu_baseline(budget_s: float = 10.0) -> dict:
    import oracle
    threads = os.cpu_count() or 1
    # calibrate on a small sample, then size the measured sample to the budget
    dt, _ = oracle_sample(64, threads)
    rows = int(min(SPEC.out_features, max(64, 64 * budget_s / max(dt, 1e-3))))
    dt, nbytes = oracle_sample(rows, threads)
    return {"value": nbytes / dt / 1e9, "unit": "GB/s", "cores": min(threads, oracle.max_threads()),
            "kind": "oracle",
            "sample": f"{rows} of {SPEC.out_features} rows of one 4096x4096 1x16 layer at batch "
                      f"1, 4, 16 (fp64 C oracle, OpenMP over rows), scaled to the layer's bytes"}


def run_reference(args) -> None:
    world, rank, _ = dist_env()
    if rank != 0:
        return
    import oracle
    threads = os.cpu_count() or 1
    dt, _ = oracle_sample(32, threads)
    rows = int(min(SPEC.out_features, max(16, 32 * 2.0 / max(dt, 1e-3))))  # ~2 s per step
    for _ in range(args.warmup):
        oracle_sample(rows, threads)
    total_t, total_b = 0.0, 0.0
    for _ in range(args.steps):
        dt, nb = oracle_sample(rows, threads)
        total_t += dt
        total_b += nb
    value = total_b / total_t / 1e9
    cores = min(threads, oracle.max_threads())
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * total_t / max(args.steps, 1), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD, "layer": "4096x4096 1x16 g8", "batches": list(BATCHES),
                   "sample_rows_per_step": rows},
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": cores, "kind": "oracle",
                         "sample": f"{rows} rows of one 4096x4096 1x16 layer at batch 1, 4, 16 per step"},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------

def count_graph_kernels(graph) -> int | None:
    try:
        from cuda.bindings import runtime as rt
        g = graph.raw_cuda_graph()
        err, _, n = rt.cudaGraphGetNodes(g, 0)
        if int(err) != 0:
            return None
        err, nodes, n = rt.cudaGraphGetNodes(g, n)
        kinds = [rt.cudaGraphNodeGetType(nd)[1] for nd in nodes]
        return sum(1 for k in kinds if k == rt.cudaGraphNodeType.cudaGraphNodeTypeKernel)
    except Exception:
        return None


def run_gpu(args) -> None:
    import torch

    import additive_quantized_matmul_b200 as aq

    world, rank, local = dist_env()
    torch.cuda.set_device(local)
    dist = init_dist(world, "nccl")
    dev = torch.device("cuda", local)
    desc = aq.LayerDesc.make(SPEC.out_features, SPEC.in_features, SPEC.num_codebooks, SPEC.nbits)

    layer_bytes = alg_bytes(SPEC, 0)
    nlayers = args.layers or max(8, int(3 * L2_BYTES / layer_bytes) + 1)
    # ---- build the rotation set of distinct layers (seeded per rank) --------
    layers = []
    for i in range(nlayers):
        L = make_layer(SPEC, (SEED, rank, i))  # seeded per rank and layer
        codes = torch.from_numpy(L.codes.view(np.int16)).to(dev)
        packed = torch.empty(aq.aq_packed_codes_bytes(desc), dtype=torch.uint8, device=dev)
        aq.aq_pack_codes(desc, codes, packed)
        cb = torch.from_numpy(L.codebooks.view(np.int16)).to(dev)
        sc = torch.from_numpy(L.scales.view(np.int16)).to(dev)
        layers.append((packed, cb, sc))
        del codes, L
    xs = {b: torch.from_numpy(make_activations(SPEC.in_features, b, (SEED, rank, b)).view(np.int16)).to(dev)
          for b in BATCHES}
    ys = {b: [torch.empty(SPEC.out_features * b, dtype=torch.int16, device=dev) for _ in range(nlayers)]
          for b in BATCHES}
    ws = {b: torch.zeros(aq.aq_gemv_workspace_bytes(desc, b), dtype=torch.uint8, device=dev)
          for b in BATCHES}
    torch.cuda.synchronize()

    stream = torch.cuda.Stream(device=dev)
    # events around every product inside the graph (external record nodes)
    evs = {b: [torch.cuda.Event(enable_timing=True, external=True) for _ in range(nlayers + 1)]
           for b in BATCHES}

    def one_step(record: bool):
        s = torch.cuda.current_stream()
        for b in BATCHES:
            if record:
                evs[b][0].record(s)
            for i, (packed, cb, sc) in enumerate(layers):
                aq.aq_gemv(desc, packed, cb, sc, xs[b], b, ys[b][i], ws[b], stream=s)
                if record:
                    evs[b][i + 1].record(s)

    # eager warm-up (also JIT-free: the library is AOT compiled)
    with torch.cuda.stream(stream):
        one_step(False)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        one_step(True)
    launches_per_step = count_graph_kernels(graph)
    torch.cuda.synchronize()

    for _ in range(max(args.warmup, 0)):
        graph.replay()
    torch.cuda.synchronize()

    t_start = torch.cuda.Event(enable_timing=True)
    t_stop = torch.cuda.Event(enable_timing=True)
    gpu_index = int(os.environ.get("CUDA_VISIBLE_DEVICES", str(local)).split(",")[local]) \
        if os.environ.get("CUDA_VISIBLE_DEVICES", "").replace(",", "").isdigit() else local
    os.makedirs(os.path.join(ROOT, "gpurun_out"), exist_ok=True)
    sampler = ClockSampler(gpu_index, os.path.join(ROOT, "gpurun_out", f"clocks_rank{rank}.csv"))
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
    elapsed_ms = t_start.elapsed_time(t_stop)
    elapsed_ms = max_over_ranks(elapsed_ms, dist, dev)

    # per-product durations from the last replay inside the timed region
    per_b = {}
    for b in BATCHES:
        t = [evs[b][i].elapsed_time(evs[b][i + 1]) for i in range(nlayers)]
        per_b[b] = {"us_per_call": 1e3 * float(np.mean(t)), "us_median": 1e3 * float(np.median(t))}
    step_bytes = nlayers * sum(alg_bytes(SPEC, b) for b in BATCHES)
    value = world * step_bytes * args.steps / (elapsed_ms * 1e-3) / 1e9
    peaks = measured_peaks()
    kernels = []
    for b in BATCHES:
        us = per_b[b]["us_per_call"]
        gbs = alg_bytes(SPEC, b) / (us * 1e-6) / 1e9
        kernels.append({"batch": b, "us_per_layer": round(us, 3), "gbs": round(gbs, 1),
                        "frac_hbm": round(gbs / peaks["hbm_gbs"], 4),
                        "bytes_per_call": alg_bytes(SPEC, b)})
    dom = max(kernels, key=lambda k: k["us_per_layer"])
    roofline = {"bound": "hbm", "achieved": dom["gbs"], "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": round(dom["gbs"] / peaks["hbm_gbs"], 4), "traffic": None,
                "kernel": f"aq_gemv batch {dom['batch']} (4096x4096 1x16)",
                "peak_source": f"{peaks['source']} hbm_gbs (MEASURED_PEAKS.json copy bandwidth)"}

    # ---- end-to-end through the public API with host buffers ----------------
    e2e = None
    if not args.skip_e2e:
        hx = {b: torch.empty((nlayers, SPEC.in_features * b), dtype=torch.int16).pin_memory() for b in BATCHES}
        hy = {b: torch.empty((nlayers, SPEC.out_features * b), dtype=torch.int16).pin_memory() for b in BATCHES}
        for b in BATCHES:
            hx[b].copy_(xs[b].cpu().reshape(1, -1).expand(nlayers, -1))
        dx = {b: torch.empty((nlayers, SPEC.in_features * b), dtype=torch.int16, device=dev) for b in BATCHES}
        dy = {b: torch.empty((nlayers, SPEC.out_features * b), dtype=torch.int16, device=dev) for b in BATCHES}
        h2d = sum(hx[b].numel() * 2 for b in BATCHES)
        d2h = sum(hy[b].numel() * 2 for b in BATCHES)
        e_steps = max(1, min(args.steps, args.e2e_steps))

        def e2e_step():
            for b in BATCHES:
                dx[b].copy_(hx[b], non_blocking=True)
            for b in BATCHES:
                for i, (packed, cb, sc) in enumerate(layers):
                    aq.aq_gemv(desc, packed, cb, sc, dx[b][i], b, dy[b][i], ws[b])
            for b in BATCHES:
                hy[b].copy_(dy[b], non_blocking=True)

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
        e2e = {"value": round(world * step_bytes * e_steps / (e_ms * 1e-3) / 1e9, 2), "unit": "GB/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": e_steps,
               "api": "additive_quantized_matmul_b200.aq_gemv (C ABI via ctypes), eager"}

    cpu = None
    if rank == 0 and world == 1 and not args.skip_cpu:
        cpu = cpu_baseline()

    if rank == 0:
        line = {
            "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(elapsed_ms / args.steps, 4), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f16", "accumulate": "f32",
            "data": "synthetic",
            "config": {"workload": WORKLOAD, "layer": "4096x4096 1x16 g8 (2 bits/weight)",
                       "batches": list(BATCHES), "layers_per_step": nlayers,
                       "l2": f"inputs larger than L2: {nlayers} distinct layers, "
                             f"{nlayers * layer_bytes / 1e6:.0f} MB of codes+codebooks per pass, "
                             f"batch-major order (> 3x the 126 MB L2)",
                       "parallelism": f"replicas x{world} (independent layers per rank)"},
            "us_per_layer": {str(k["batch"]): k["us_per_layer"] for k in kernels},
            "kernels": kernels, "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
            "clocks": sampler.summary(),
            "gpu_launches": None if launches_per_step is None else launches_per_step * args.steps,
        }
        print(json.dumps(line), flush=True)
    del graph
    if dist is not None:
        dist.destroy_process_group()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--layers", type=int, default=0, help="rotation set size (0: > 3x L2)")
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
