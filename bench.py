"""Benchmark of the edge-aware attention layer (forward + backward) on B200.

Workload (one step): one forward and one backward of the layer over one
batch of the SBM-shaped training preset (B=32 graphs, n=192 padded nodes,
n_real ~ U[44,187], dx=256, de=64, dy=64, H=8, dh=32, bf16 storage, fp32
accumulation), synthetic seeded inputs (edge_aware_graph_b200/inputs.py).
`--workload large-train` runs the Large-shaped training step (B=4, n=1024)
instead; `planar-sample` / `tree-sample` the sampling-time forward.
Metric: edge pairs (B*n^2, padded) per second, and the fraction of the HBM
roofline of the dominant kernel.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Under torchrun (N > 1) every rank runs its own batch of the same shape
(weak scaling) and the step adds the data-parallel all-reduce of the weight
gradients over NCCL; rank 0 prints one JSON line.  `--impl reference` times
the fp64 CPU oracle (the reference arm) on a bounded sample of the workload.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np

# --workload: the SBM-shaped training step (default), the Large-shaped
# training step (B=4, n=1024), or the sampling-time forward on Planar- /
# Tree-shaped batches (forward only, many calls per model)
WORKLOADS = {"sbm-train": "sbm", "large-train": "large", "planar-sample": "planar", "tree-sample": "tree",
             "block-sbm-train": "sbm", "block-large-train": "large"}
BLOCK = ("block-sbm-train", "block-large-train")
TRAINING = ("sbm-train", "large-train")
DESCRIBE = {
    "sbm": "sbm-shaped training step (fwd+bwd): B=32, n=192 padded, n_real~U[44,187], 2-5 blocks, "
           "dx=256 de=64 dy=64 H=8 dh=32, bf16 storage / fp32 accumulation",
    "large": "large-shaped training step (fwd+bwd): B=4, n=1024 padded, n_real~U[768,1024], 8 blocks, "
             "dx=256 de=64 dy=64 H=8 dh=32, bf16 storage / fp32 accumulation",
}
SAMPLE_ROTATION = 6     # batches cycled by the sampling workload: 6 x ~77 MB > L2
METRIC = "edge-pairs/sec (B·n²) fwd and fwd+bwd on 1 B200; % of HBM roofline"
UNIT = "edge-pairs/s"
FALLBACK_HBM_GBS = 6650.0

# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) of one launch of
# the dominant kernels on each workload, from one ncu capture of the kernels as
# they are (the summaries under profiles/ give the commands).  A kernel that
# changes reports null until it is captured again.  Planar: one batch's
# E' (32 MiB) fits in L2, so within the captured launch its writes stay in L2
# and reach DRAM later, under the next batch's launch.
NCU_TRAFFIC = {
    ("sbm", "k_fwd_stream"): 162472448 + 97329664,
    ("sbm", "k_bwd_stream"): 257099520 + 109985792,
    ("large", "k_fwd_stream"): 734333184 + 481042944,
    ("large", "k_bwd_stream"): 1771164416 + 507204608,
    ("planar", "k_fwd_stream"): 39935744 + 764672,
    ("sbm", "k_eblk_fwd"): 63142912 + 99683840,
    ("sbm", "k_eblk_bwd"): 182036992 + 124005632,
    ("large", "k_eblk_fwd"): 487750000 + 485110000,
    ("large", "k_eblk_bwd"): 1040000000 + 510180000,
}


def env_rank():
    return (int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)),
            int(os.environ.get("LOCAL_RANK", 0)))


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            pk = json.load(f)
        return float(pk["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


# ------------------------------------------------------------------ clocks


class ClockSampler:
    """Samples SM clock and throttle reasons through NVML in a thread."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
               0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}

    def __init__(self, device_index: int, period_s: float = 0.002):
        self.samples, self.reasons = [], set()
        self.period = period_s
        self.max_mhz = None
        self._stop = threading.Event()
        self._thr = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self.nv = None

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                r = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for bit, name in self.REASONS.items():
                    if r & bit and name != "gpu_idle":
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def start(self):
        if self.nv:
            self._thr = threading.Thread(target=self._run, daemon=True)
            self._thr.start()

    def stop(self):
        if self._thr:
            self._stop.set()
            self._thr.join()
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons), "samples": len(self.samples)}


# ------------------------------------------------------------------ bytes


def compulsory_bytes(p, training=True):
    """Algorithmic bytes of the layer (no recomputation, each tensor once)."""
    s = 2 if p.dtype == "bf16" else 4
    pairs, nodes = p.B * p.n * p.n, p.B * p.n
    fwd = pairs * p.de * s * 2 + nodes * p.dx * s * 2
    bwd = pairs * p.de * s * 3 + nodes * p.dx * s * 3
    return fwd + (bwd if training else 0)


def pair_kernel_bytes(p, which):
    """Algorithmic bytes of one launch of the pair kernels: the E-sized
    streams only (forward: E read, E' write; backward: E and dE' read, dE
    write).  Node-sized terms (Q, K, V, O, LSE, ...) are left out."""
    s = 2 if p.dtype == "bf16" else 4
    per_pair = p.de * s * (2 if which == "fwd" else 3)
    return p.B * p.n * p.n * per_pair


# ------------------------------------------------------------------ our arm


def memory_report(buf, step, torch):
    """Device memory of the step: what the buffers hold (inputs, outputs,
    saved state, the two workspaces) and the allocation peak over one step
    above what was allocated before it (the library allocates nothing)."""
    torch.cuda.synchronize()
    before = torch.cuda.memory_allocated()
    torch.cuda.reset_peak_memory_stats()
    step()
    torch.cuda.synchronize()
    peak_delta = torch.cuda.max_memory_allocated() - before
    mib = lambda b: b / 2**20
    E = buf.E.numel() * buf.E.element_size()
    return {"peak_mib_delta_per_step": mib(peak_delta), "held_mib": mib(before),
            "workspace_fwd_mib": mib(buf.ws_fwd.numel()), "workspace_bwd_mib": mib(buf.ws_bwd.numel()),
            "saved_mib": mib(buf.saved.numel()), "edge_tensor_mib": mib(E),
            "workspace_bwd_per_pair_bytes": buf.ws_bwd.numel() / (buf.E.shape[0] * buf.E.shape[1] ** 2)}


def run_ours(args):
    if args.workload in BLOCK:
        return run_block(args)
    if args.workload not in TRAINING:
        return run_sample(args, WORKLOADS[args.workload])
    WORKLOAD = WORKLOADS[args.workload]
    import torch
    import torch.distributed as dist

    from edge_aware_graph_b200 import dp, eaga
    from edge_aware_graph_b200 import inputs as I
    from edge_aware_graph_b200.buffers import LayerBuffers

    rank, world, local = env_rank()
    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    p = I.preset(WORKLOAD, seed=dp.rank_seed(I.preset(WORKLOAD).seed, rank))
    d = I.draw_inputs(p, with_grads=True)
    W = I.draw_weights(I.preset(WORKLOAD))          # one model: the same weights on every rank
    buf = LayerBuffers(p.B, p.n, p.dx, p.de, p.dy, p.H, p.dh, dtype=p.dtype, backward=True)
    buf.load_inputs(d, W)
    stream = torch.cuda.current_stream()
    flat_dw = buf.dW_flat

    def layer(s):
        buf.forward(s, variant=args.variant)
        buf.backward(s, variant=args.variant)

    def step():
        layer(torch.cuda.current_stream())
        dp.allreduce_weight_grads(flat_dw)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()

    # ---- per-kernel times: eager steps with CUDA events around the pair kernels
    nk = min(args.steps, 20)
    ev_f = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(nk)]
    ev_b = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(nk)]
    ev_r = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(nk)]
    for a, b in ev_f + ev_b + ev_r:   # torch creates the CUDA event on first record
        a.record(stream)
        b.record(stream)
    torch.cuda.synchronize()
    for k in range(nk):
        eaga.set_profile_events(0, *ev_f[k])
        eaga.set_profile_events(1, *ev_b[k])
        eaga.set_profile_events(2, *ev_r[k])
        step()
    torch.cuda.synchronize()
    eaga.set_profile_events(0)
    eaga.set_profile_events(1)
    eaga.set_profile_events(2)
    fwd_ms = statistics.mean(a.elapsed_time(b) for a, b in ev_f)
    bwd_ms = statistics.mean(a.elapsed_time(b) for a, b in ev_b)
    rows_ms = statistics.mean(a.elapsed_time(b) for a, b in ev_r)

    # ---- the step's kernels as one CUDA graph (launch gaps removed); the
    # weight-gradient all-reduce (N > 1) stays outside the graph
    graph = None
    if not args.no_graph:
        graph = torch.cuda.CUDAGraph()
        cap = torch.cuda.Stream()
        cap.wait_stream(stream)
        with torch.cuda.stream(cap):
            layer(cap)                     # warm the capture stream
        torch.cuda.synchronize()
        with torch.cuda.graph(graph, stream=cap):
            layer(cap)
        torch.cuda.synchronize()

    def timed_step():
        if graph is not None:
            graph.replay()
            dp.allreduce_weight_grads(flat_dw)
        else:
            step()

    for _ in range(3):
        timed_step()
    # ---- timed region: K steps
    K = args.steps
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.start()
    t0.record(stream)
    for k in range(K):
        timed_step()
    t1.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clk = clocks.stop()
    ms_total = t0.elapsed_time(t1)
    ms_total = dp.max_over_ranks(ms_total, "cuda")
    if graph is not None:
        torch.cuda.synchronize()
        del graph

    # ---- end to end through the public API with host buffers
    e2e = run_e2e(args, buf, d, stream, step)
    e2e["ms"] = dp.max_over_ranks(e2e["ms"], "cuda")

    launches = (eaga.kernel_launches(buf.dims, False) + eaga.kernel_launches(buf.dims, True)) * K
    mem = memory_report(buf, step, torch)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return None

    pairs_step = p.B * p.n * p.n
    ms_step = ms_total / K
    value = world * pairs_step * K / (ms_total / 1e3)
    peak, peak_kind = measured_peaks()
    kb = pair_kernel_bytes(p, "bwd")
    achieved = kb / (rows_ms / 1e3) / 1e9
    kf = pair_kernel_bytes(p, "fwd")
    step_bytes = compulsory_bytes(p)
    out = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K, "warmup": args.warmup,
        "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded SBM-shaped graphs; edge_aware_graph_b200/inputs.py)",
        "config": {"workload": DESCRIBE[WORKLOAD] + ("" if args.variant == "layer" else
                                                     f"; ablation variant: {args.variant}"),
                   "global_batch": p.B * world, "seq_len": p.n, "parallelism": f"dp{world}",
                   "l2": f"inputs larger than L2 (E, dE' {p.B * p.n * p.n * p.de * 2 / 2**20:.0f} MiB each; "
                         "E', dE written each step)",
                   "launch": "CUDA graph of the step's kernels" if not args.no_graph else "eager"},
        "roofline": {"bound": "hbm", "kernel": "k_bwd_stream (backward row pair kernel)", "achieved": achieved,
                     "peak": peak, "peak_kind": peak_kind, "unit": "GB/s", "frac": achieved / peak,
                     "traffic": NCU_TRAFFIC.get((WORKLOAD, "k_bwd_stream")),
                     "algorithmic_bytes": kb, "ms_per_launch": rows_ms,
                     "backward_pair_kernels_ms": bwd_ms},
        "roofline_fwd": {"bound": "hbm", "kernel": "k_fwd_stream (forward pair kernel)",
                         "achieved": kf / (fwd_ms / 1e3) / 1e9, "peak": peak, "unit": "GB/s",
                         "frac": kf / (fwd_ms / 1e3) / 1e9 / peak,
                         "traffic": NCU_TRAFFIC.get((WORKLOAD, "k_fwd_stream")),
                         "algorithmic_bytes": kf, "ms_per_launch": fwd_ms},
        "step_roofline": {"compulsory_bytes": step_bytes, "achieved_gbs": step_bytes / (ms_step / 1e3) / 1e9,
                          "frac_of_measured": step_bytes / (ms_step / 1e3) / 1e9 / peak,
                          "frac_of_8tbs": step_bytes / (ms_step / 1e3) / 1e9 / 8000.0},
        "clocks": clk,
        "e2e": {"value": world * pairs_step / (e2e["ms"] / 1e3), "unit": UNIT,
                "h2d_bytes_per_step": e2e["h2d"], "d2h_bytes_per_step": e2e["d2h"], "steps": e2e["steps"]},
        "gpu_launches": launches,
        "memory": mem,
    }
    if world == 1 and not args.no_cpu_baseline:
        graphs = min(args.cpu_graphs, p.B) if WORKLOAD == "sbm" else 1
        reps = args.cpu_reps if WORKLOAD == "sbm" else 1
        out["cpu_baseline"] = cpu_baseline(p, d, W, graphs, reps, variant=args.variant)
        out["cpu_baseline_1thread"] = cpu_baseline(p, d, W, 1, 1, threads=1, variant=args.variant)
    return out


def run_rows(args):
    """Row-sharded training step (edge_aware_graph_b200/rowshard.py): every rank
    holds the same graphs and owns a slab of each graph's rows; a step is the
    slab's forward and backward plus one all-reduce of the gradient parts.
    Under torchrun the N ranks split the rows N ways (total work fixed: strong
    scaling).  With one GPU, --row-slabs K runs rank 0's slab of a K-way split
    alone (no exchange), the share one GPU of K would take."""
    WORKLOAD = WORKLOADS[args.workload]
    import torch
    import torch.distributed as dist

    from edge_aware_graph_b200 import dp, eaga, rowshard
    from edge_aware_graph_b200 import inputs as I
    from edge_aware_graph_b200.buffers import LayerBuffers

    rank, world, local = env_rank()
    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=torch.device("cuda", local))
    ways = world if world > 1 else max(1, args.row_slabs)
    p = I.preset(WORKLOAD)
    d = I.draw_inputs(p, with_grads=True)
    W = I.draw_weights(p)
    buf = LayerBuffers(p.B, p.n, p.dx, p.de, p.dy, p.H, p.dh, dtype=p.dtype, backward=True)
    buf.load_inputs(d, W)
    row0, rows = rowshard.row_slabs(p.n, ways)[rank if world > 1 else 0]
    E_r = buf.E[:, row0:row0 + rows].contiguous()
    dEo_r = buf.dEout[:, row0:row0 + rows].contiguous()
    Eo_r, dE_r = torch.empty_like(E_r), torch.empty_like(E_r)
    del buf.E, buf.Eout, buf.dEout, buf.dE             # the rank holds slabs only
    dX32 = torch.zeros(p.B, p.n, p.dx, dtype=torch.float32, device="cuda")
    dy32 = torch.zeros(p.B, p.dy, dtype=torch.float32, device="cuda")
    stream = torch.cuda.current_stream()

    def step():
        rowshard.forward_rows(buf.dims, row0, rows, buf.X, E_r, buf.y, buf.M, buf.W, buf.Xout, Eo_r, buf.saved,
                              buf.ws_fwd, stream)
        rowshard.backward_rows(buf.dims, row0, rows, buf.X, E_r, buf.y, buf.M, buf.W, buf.saved, buf.dXout, dEo_r,
                               buf.dX, dE_r, buf.dy, buf.dW, buf.ws_bwd, stream)
        if world > 1:
            dX32.copy_(buf.dX)
            dy32.copy_(buf.dy)
            rowshard.allreduce_parts([dX32, dy32, buf.dW_flat])

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    nk = min(args.steps, 20)
    ev_r = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(nk)]
    for a, b in ev_r:
        a.record(stream)
        b.record(stream)
    torch.cuda.synchronize()
    for k in range(nk):
        eaga.set_profile_events(2, *ev_r[k])
        step()
    torch.cuda.synchronize()
    eaga.set_profile_events(2)
    rows_ms = statistics.mean(a.elapsed_time(b) for a, b in ev_r)

    K = args.steps
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.start()
    t0.record(stream)
    for _ in range(K):
        step()
    t1.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clk = clocks.stop()
    ms_total = dp.max_over_ranks(t0.elapsed_time(t1), "cuda")
    launches = (eaga.kernel_launches(buf.dims, False) + eaga.kernel_launches(buf.dims, True)) * K
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return None
    ms_step = ms_total / K
    pairs_step = p.B * p.n * p.n if world > 1 else p.B * rows * p.n
    peak, peak_kind = measured_peaks()
    kb = 3 * p.B * rows * p.n * p.de * 2          # the slab's E, dE' read and dE written
    return {
        "metric": METRIC, "value": pairs_step / (ms_step / 1e3), "unit": UNIT, "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "strong" if world > 1 else "one rank's share", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded graphs; edge_aware_graph_b200/inputs.py)",
        "config": {"workload": DESCRIBE[WORKLOAD] + f"; rows split {ways} ways (rank 0's slab: rows {row0}.."
                   f"{row0 + rows - 1} of every graph" + ("" if world > 1 else ", run alone") + ")",
                   "global_batch": p.B, "seq_len": p.n, "parallelism": f"rows{ways}",
                   "l2": "inputs larger than L2" if E_r.numel() * 2 > (126 << 20) else "slab smaller than L2",
                   "launch": "eager"},
        "roofline": {"bound": "hbm", "kernel": "k_bwd_stream (backward row pair kernel, the slab)",
                     "achieved": kb / (rows_ms / 1e3) / 1e9, "peak": peak, "peak_kind": peak_kind, "unit": "GB/s",
                     "frac": kb / (rows_ms / 1e3) / 1e9 / peak, "traffic": None, "algorithmic_bytes": kb,
                     "ms_per_launch": rows_ms},
        "clocks": clk, "e2e": None, "gpu_launches": launches,
    }


def run_sample(args, name):
    """Sampling-time forward: the forward alone, called once per step on one of
    SAMPLE_ROTATION resident batches in turn (inputs larger than L2), the
    rotation's calls replayed as one CUDA graph."""
    import torch
    import torch.distributed as dist

    from edge_aware_graph_b200 import dp, eaga
    from edge_aware_graph_b200 import inputs as I
    from edge_aware_graph_b200.buffers import LayerBuffers, host_to_storage_tensor

    rank, world, local = env_rank()
    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    p0 = I.preset(name)
    R = SAMPLE_ROTATION
    W = I.draw_weights(p0)                          # one model on every rank
    bufs, ds = [], []
    for r in range(R):
        p = I.preset(name, seed=dp.rank_seed(p0.seed, rank * R + r))
        d = I.draw_inputs(p, with_grads=False)
        buf = LayerBuffers(p.B, p.n, p.dx, p.de, p.dy, p.H, p.dh, dtype=p.dtype, backward=False)
        buf.load_inputs(d, W)
        bufs.append(buf)
        ds.append(d)
    stream = torch.cuda.current_stream()

    def call(r, s):
        bufs[r].forward(s)

    for k in range(max(args.warmup, R)):
        call(k % R, stream)
    torch.cuda.synchronize()

    # ---- forward pair kernel times: eager calls with CUDA events around it
    nk = min(args.steps, 24)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(nk)]
    for a, b in ev:
        a.record(stream)
        b.record(stream)
    torch.cuda.synchronize()
    for k in range(nk):
        eaga.set_profile_events(0, *ev[k])
        call(k % R, stream)
    torch.cuda.synchronize()
    eaga.set_profile_events(0)
    fwd_ms = statistics.mean(a.elapsed_time(b) for a, b in ev)

    graph = None
    if not args.no_graph:
        graph = torch.cuda.CUDAGraph()
        cap = torch.cuda.Stream()
        cap.wait_stream(stream)
        with torch.cuda.stream(cap):
            for r in range(R):
                call(r, cap)
        torch.cuda.synchronize()
        with torch.cuda.graph(graph, stream=cap):
            for r in range(R):
                call(r, cap)
        torch.cuda.synchronize()

    def rotation():
        if graph is not None:
            graph.replay()
        else:
            for r in range(R):
                call(r, stream)

    rotation()
    reps = max(1, (args.steps + R - 1) // R)
    K = reps * R
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.start()
    t0.record(stream)
    for _ in range(reps):
        rotation()
    t1.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clk = clocks.stop()
    ms_total = dp.max_over_ranks(t0.elapsed_time(t1), "cuda")
    if graph is not None:
        del graph

    # ---- end to end through the public API: inputs from pinned host memory,
    # X' and E' read back, every call
    host_in = [{k: host_to_storage_tensor(d[k], bufs[0].dtype).pin_memory() for k in ("X", "E", "y")}
               for d in ds]
    host_M = [torch.from_numpy(np.ascontiguousarray(d["M"])).pin_memory() for d in ds]
    host_out = [(torch.empty(b.Xout.shape, dtype=b.Xout.dtype).pin_memory(),
                 torch.empty(b.Eout.shape, dtype=b.Eout.dtype).pin_memory()) for b in bufs]
    h2d = sum(t.numel() * t.element_size() for t in host_in[0].values()) + host_M[0].numel()
    d2h = sum(t.numel() * t.element_size() for t in host_out[0])

    def e2e_call(r):
        b = bufs[r]
        for k in ("X", "E", "y"):
            getattr(b, k).copy_(host_in[r][k], non_blocking=True)
        b.M.copy_(host_M[r], non_blocking=True)
        call(r, stream)
        host_out[r][0].copy_(b.Xout, non_blocking=True)
        host_out[r][1].copy_(b.Eout, non_blocking=True)

    for r in range(R):
        e2e_call(r)
    torch.cuda.synchronize()
    ne = max(args.e2e_steps, R)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for k in range(ne):
        e2e_call(k % R)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = dp.max_over_ranks(e0.elapsed_time(e1) / ne, "cuda")

    launches = eaga.kernel_launches(bufs[0].dims, False) * K
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return None

    pairs_call = p0.B * p0.n * p0.n
    value = world * pairs_call * K / (ms_total / 1e3)
    peak, peak_kind = measured_peaks()
    kf = pair_kernel_bytes(p0, "fwd")
    achieved = kf / (fwd_ms / 1e3) / 1e9
    call_bytes = compulsory_bytes(p0, training=False)
    ms_call = ms_total / K
    out = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K, "warmup": args.warmup,
        "ms_per_step": ms_call, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16", "data": f"synthetic (seeded {name.capitalize()}-shaped graphs; edge_aware_graph_b200/inputs.py)",
        "config": {"workload": f"{name}-shaped sampling-time forward: B={p0.B}, n={p0.n} (all nodes real), "
                               f"dx={p0.dx} de={p0.de} dy={p0.dy} H={p0.H} dh={p0.dh}, bf16 storage / fp32 "
                               "accumulation, saved state written",
                   "global_batch": p0.B * world, "seq_len": p0.n, "parallelism": f"dp{world}",
                   "l2": f"inputs larger than L2: {R} resident batches called in turn "
                         f"(E {p0.B * p0.n * p0.n * p0.de * 2 / 2**20:.0f} MiB each)",
                   "launch": (f"CUDA graph of {R} forward calls" if not args.no_graph else "eager")},
        "roofline": {"bound": "hbm", "kernel": "k_fwd_stream (forward pair kernel)", "achieved": achieved,
                     "peak": peak, "peak_kind": peak_kind, "unit": "GB/s", "frac": achieved / peak,
                     "traffic": NCU_TRAFFIC.get((name, "k_fwd_stream")),
                     "algorithmic_bytes": kf, "ms_per_launch": fwd_ms},
        "step_roofline": {"compulsory_bytes": call_bytes, "achieved_gbs": call_bytes / (ms_call / 1e3) / 1e9,
                          "frac_of_measured": call_bytes / (ms_call / 1e3) / 1e9 / peak,
                          "frac_of_8tbs": call_bytes / (ms_call / 1e3) / 1e9 / 8000.0},
        "clocks": clk,
        "e2e": {"value": world * pairs_call / (e2e_ms / 1e3), "unit": UNIT,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": ne},
        "gpu_launches": launches,
    }
    if world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline_forward(p0, ds[0], W, args.cpu_seconds)
    return out


def run_e2e(args, buf, d, stream, step):
    """Steps whose timed region includes the pinned-host -> device copy of the
    step's inputs and the device -> host read of its results."""
    import torch

    from edge_aware_graph_b200.buffers import host_to_storage_tensor
    names_in = ["X", "E", "y", "dXout", "dEout"]
    host_in = {k: host_to_storage_tensor(d[k], buf.dtype).pin_memory() for k in names_in}
    host_M = torch.from_numpy(np.ascontiguousarray(d["M"])).pin_memory()
    outs = [buf.Xout, buf.Eout, buf.dX, buf.dE, buf.dy, buf.dW_flat]
    host_out = [torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in outs]
    dev_in = {"X": buf.X, "E": buf.E, "y": buf.y, "dXout": buf.dXout, "dEout": buf.dEout}
    h2d = sum(t.numel() * t.element_size() for t in host_in.values()) + host_M.numel()
    d2h = sum(t.numel() * t.element_size() for t in outs)

    def e2e_step():
        for k in names_in:
            dev_in[k].copy_(host_in[k], non_blocking=True)
        buf.M.copy_(host_M, non_blocking=True)
        step()
        for h, t in zip(host_out, outs):
            h.copy_(t, non_blocking=True)

    for _ in range(2):
        e2e_step()
    torch.cuda.synchronize()
    n = args.e2e_steps
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(n):
        e2e_step()
    t1.record(stream)
    torch.cuda.synchronize()
    return {"ms": t0.elapsed_time(t1) / n, "h2d": h2d, "d2h": d2h, "steps": n}


# ------------------------------------------------------------------ the block around the layer


def block_step_bytes(p):
    """Algorithmic bytes of one block training step: the layer's (compulsory_bytes)
    plus the block's edge streams (forward: E' read, Eout write; backward: E',
    dEout read, dE' write) and node streams (forward: X' read, Xout write;
    backward: X', dXout read, dX' write)."""
    s = 2 if p.dtype == "bf16" else 4
    pairs, nodes = p.B * p.n * p.n, p.B * p.n
    return compulsory_bytes(p) + pairs * p.de * s * 5 + nodes * p.dx * s * 5


def cpu_baseline_block(p, d, W, Wb, dyo, graphs):
    """The block oracle (fp64: the layer's C oracle and the block's numpy
    restatement), as it stands, forward + backward of the first `graphs`
    graphs of the batch."""
    import oracle
    from oracle import block as OB
    oracle.build()
    sl = {k: d[k][:graphs] for k in ("X", "E", "y", "M", "dXout", "dEout")}
    dims = dict(H=p.H, dh=p.dh)
    t = time.perf_counter()
    OB.block_forward(dims, sl["X"], sl["E"], sl["y"], sl["M"], W, Wb)
    OB.block_backward(dims, sl["X"], sl["E"], sl["y"], sl["M"], W, Wb, sl["dXout"], sl["dEout"], dyo[:graphs])
    dt = time.perf_counter() - t
    return {"value": graphs * p.n * p.n / dt, "unit": UNIT, "cores": oracle.threads_used(), "kind": "oracle",
            "sample": f"{graphs} of {p.B} graphs of the workload (n={p.n}), block forward + backward, fp64",
            "seconds": dt}


def run_block(args):
    """Training step of the graph-transformer block around the layer (layer,
    LayerNorms, FFNs, global update; forward + backward) on the SBM- or
    Large-shaped batch."""
    name = WORKLOADS[args.workload]
    import torch
    import torch.distributed as dist

    from edge_aware_graph_b200 import dp, eaga
    from edge_aware_graph_b200 import inputs as I
    from edge_aware_graph_b200.buffers import BlockBuffers, host_to_storage_tensor

    rank, world, local = env_rank()
    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=torch.device("cuda", local))
    base = I.preset(name)
    p = I.preset(name, seed=dp.rank_seed(base.seed, rank))
    d = I.draw_inputs(p, with_grads=True)
    W, Wb = I.draw_weights(base), I.draw_block_weights(base)     # one model on every rank
    dyo = I.draw_block_upstream(p)
    buf = BlockBuffers(p.B, p.n, p.dx, p.de, p.dy, p.H, p.dh, dtype=p.dtype, backward=True)
    buf.load_inputs(d, W)
    buf.load_block(Wb, dyo)
    stream = torch.cuda.current_stream()

    def block(s):
        buf.block_forward(s)
        buf.block_backward(s)

    def step():
        block(torch.cuda.current_stream())
        dp.allreduce_weight_grads(buf.dW_flat)
        dp.allreduce_weight_grads(buf.dWb_flat)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    nk = min(args.steps, 20)
    points = (0, 2, 3, 4)
    evs = {q: [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(nk)]
           for q in points}
    for q in points:
        for a, b in evs[q]:
            a.record(stream)
            b.record(stream)
    torch.cuda.synchronize()
    for k in range(nk):
        for q in points:
            eaga.set_profile_events(q, *evs[q][k])
        step()
    torch.cuda.synchronize()
    for q in points:
        eaga.set_profile_events(q)
    kms = {q: statistics.mean(a.elapsed_time(b) for a, b in evs[q]) for q in points}

    graph = None
    if not args.no_graph:
        graph = torch.cuda.CUDAGraph()
        cap = torch.cuda.Stream()
        cap.wait_stream(stream)
        with torch.cuda.stream(cap):
            block(cap)
        torch.cuda.synchronize()
        with torch.cuda.graph(graph, stream=cap):
            block(cap)
        torch.cuda.synchronize()

    def timed_step():
        if graph is not None:
            graph.replay()
            dp.allreduce_weight_grads(buf.dW_flat)
            dp.allreduce_weight_grads(buf.dWb_flat)
        else:
            step()

    for _ in range(3):
        timed_step()
    K = args.steps
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.start()
    t0.record(stream)
    for _ in range(K):
        timed_step()
    t1.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clk = clocks.stop()
    ms_total = dp.max_over_ranks(t0.elapsed_time(t1), "cuda")
    if graph is not None:
        torch.cuda.synchronize()
        del graph

    # end to end through the public API: inputs from pinned host memory, every
    # output and gradient read back, inside the timed region
    names_in = ["X", "E", "y", "dXout", "dEout", "dyout"]
    src = dict(d)
    src["dyout"] = dyo
    host_in = {k: host_to_storage_tensor(src[k], buf.dtype).pin_memory() for k in names_in}
    host_M = torch.from_numpy(np.ascontiguousarray(d["M"])).pin_memory()
    outs = [buf.Xout, buf.Eout, buf.yout, buf.dX, buf.dE, buf.dy, buf.dW_flat, buf.dWb_flat]
    host_out = [torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in outs]
    h2d = sum(t.numel() * t.element_size() for t in host_in.values()) + host_M.numel()
    d2h = sum(t.numel() * t.element_size() for t in outs)

    def e2e_step():
        for k in names_in:
            getattr(buf, k).copy_(host_in[k], non_blocking=True)
        buf.M.copy_(host_M, non_blocking=True)
        step()
        for h, t in zip(host_out, outs):
            h.copy_(t, non_blocking=True)

    for _ in range(2):
        e2e_step()
    torch.cuda.synchronize()
    a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a0.record(stream)
    for _ in range(args.e2e_steps):
        e2e_step()
    a1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = dp.max_over_ranks(a0.elapsed_time(a1) / args.e2e_steps, "cuda")

    launches = (eaga.block_kernel_launches(buf.dims, False) + eaga.block_kernel_launches(buf.dims, True)) * K
    torch.cuda.synchronize()
    before = torch.cuda.memory_allocated()
    torch.cuda.reset_peak_memory_stats()
    step()
    torch.cuda.synchronize()
    mem = {"peak_mib_delta_per_step": (torch.cuda.max_memory_allocated() - before) / 2**20,
           "held_mib": before / 2**20, "block_workspace_bwd_mib": buf.bws_bwd.numel() / 2**20,
           "block_saved_mib": buf.bsaved.numel() / 2**20,
           "block_workspace_bwd_per_pair_bytes": buf.bws_bwd.numel() / (p.B * p.n * p.n)}
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return None

    pairs = p.B * p.n * p.n
    ms_step = ms_total / K
    value = world * pairs * K / (ms_total / 1e3)
    peak, peak_kind = measured_peaks()
    kern = {
        "k_eblk_bwd (edge sub-block backward)": (pairs * p.de * 2 * 3, kms[4], None),
        "k_eblk_fwd (edge sub-block forward)": (pairs * p.de * 2 * 2, kms[3], None),
        "k_bwd_stream (layer backward row pair kernel)": (pair_kernel_bytes(p, "bwd"), kms[2],
                                                          NCU_TRAFFIC.get((name, "k_bwd_stream"))),
        "k_fwd_stream (layer forward pair kernel)": (pair_kernel_bytes(p, "fwd"), kms[0],
                                                     NCU_TRAFFIC.get((name, "k_fwd_stream"))),
    }
    kern["k_eblk_bwd (edge sub-block backward)"] = kern["k_eblk_bwd (edge sub-block backward)"][:2] + (
        NCU_TRAFFIC.get((name, "k_eblk_bwd")),)
    kern["k_eblk_fwd (edge sub-block forward)"] = kern["k_eblk_fwd (edge sub-block forward)"][:2] + (
        NCU_TRAFFIC.get((name, "k_eblk_fwd")),)
    rl = lambda k: {"bound": "hbm", "kernel": k, "achieved": kern[k][0] / (kern[k][1] / 1e3) / 1e9, "peak": peak,
                    "peak_kind": peak_kind, "unit": "GB/s",
                    "frac": kern[k][0] / (kern[k][1] / 1e3) / 1e9 / peak, "traffic": kern[k][2],
                    "algorithmic_bytes": kern[k][0], "ms_per_launch": kern[k][1]}
    dominant = max(kern, key=lambda k: kern[k][1])
    sb = block_step_bytes(p)
    out = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K, "warmup": args.warmup,
        "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": f"synthetic (seeded {name.upper()}-shaped graphs; edge_aware_graph_b200/inputs.py)",
        "config": {"workload": "graph-transformer block training step (the layer, LayerNorms, node / edge / "
                               "global FFNs and the global update; fwd+bwd) on the " + DESCRIBE[name],
                   "global_batch": p.B * world, "seq_len": p.n, "parallelism": f"dp{world}",
                   "l2": f"inputs larger than L2 (E, E', dE', dEout {pairs * p.de * 2 / 2**20:.0f} MiB each)",
                   "launch": "CUDA graph of the step's kernels" if not args.no_graph else "eager"},
        "roofline": rl(dominant),
        "roofline_kernels": {k: rl(k) for k in kern},
        "step_roofline": {"compulsory_bytes": sb, "achieved_gbs": sb / (ms_step / 1e3) / 1e9,
                          "frac_of_measured": sb / (ms_step / 1e3) / 1e9 / peak},
        "clocks": clk,
        "e2e": {"value": world * pairs / (e2e_ms / 1e3), "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "steps": args.e2e_steps},
        "gpu_launches": launches,
        "memory": mem,
    }
    if world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline_block(p, d, W, Wb, dyo, 2 if name == "sbm" else 1)
    return out


def run_reference_block(args, world):
    """The oracle arm of the block workloads: the block oracle's forward +
    backward on --ref-graphs graphs (one at n = 1024) per step."""
    from edge_aware_graph_b200 import inputs as I
    name = WORKLOADS[args.workload]
    p = I.preset(name)
    d = I.draw_inputs(p, with_grads=True)
    W, Wb, dyo = I.draw_weights(p), I.draw_block_weights(p), I.draw_block_upstream(p)
    g = 1 if name == "large" else max(1, min(args.ref_graphs, p.B))
    for _ in range(args.warmup):
        cpu_baseline_block(p, d, W, Wb, dyo, 1)
    res = [cpu_baseline_block(p, d, W, Wb, dyo, g) for _ in range(args.steps)]
    secs = sum(r["seconds"] for r in res)
    value = args.steps * g * p.n * p.n / secs
    cb = dict(res[0])
    cb["value"] = value
    cb.pop("seconds", None)
    return {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": secs / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": f"synthetic (seeded {name.upper()}-shaped graphs)",
            "config": {"workload": "graph-transformer block training step on the " + DESCRIBE[name]
                                   + f"; bounded sample of {g} graph(s) per step",
                       "global_batch": g, "seq_len": p.n, "parallelism": "cpu"},
            "cpu_baseline": cb,
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


# ------------------------------------------------------------------ oracle arm


def cpu_baseline(p, d, W, graphs, reps=1, threads=None, variant="layer"):
    """The fp64 oracle, as it stands, on a bounded sample: the first `graphs`
    graphs of the batch, forward + backward, `reps` times, on all usable host
    cores (or on `threads` threads)."""
    import oracle
    oracle.build()
    oracle.set_threads(threads)
    sl = {k: d[k][:graphs] for k in ("X", "E", "y", "M", "dXout", "dEout")}
    dims = dict(H=p.H, dh=p.dh)
    t = time.perf_counter()
    for _ in range(reps):
        oracle.forward(dims, sl["X"], sl["E"], sl["y"], sl["M"], W, variant=variant)
        oracle.backward(dims, sl["X"], sl["E"], sl["y"], sl["M"], W, sl["dXout"], sl["dEout"], variant=variant)
    dt = time.perf_counter() - t
    cores = oracle.threads_used()
    oracle.set_threads(None)
    pairs = reps * graphs * p.n * p.n
    return {"value": pairs / dt, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"{graphs} of {p.B} graphs of the workload (n={p.n}), forward + backward, fp64, "
                      f"{reps} time(s)",
            "seconds": dt}


def cpu_baseline_forward(p, d, W, min_seconds):
    """The fp64 oracle, as it stands, on the forward of the whole batch,
    repeated until `min_seconds` have passed (a bounded sample)."""
    import oracle
    oracle.build()
    dims = dict(H=p.H, dh=p.dh)
    reps, t = 0, time.perf_counter()
    while True:
        oracle.forward(dims, d["X"], d["E"], d["y"], d["M"], W)
        reps += 1
        dt = time.perf_counter() - t
        if dt >= min_seconds or reps >= 1000:
            break
    pairs = reps * p.B * p.n * p.n
    return {"value": pairs / dt, "unit": UNIT, "cores": oracle.threads_used(), "kind": "oracle",
            "sample": f"the forward of all {p.B} graphs of the batch (n={p.n}), fp64, {reps} time(s)",
            "seconds": dt}


def run_reference(args):
    rank, world, _ = env_rank()
    if rank != 0:
        return None
    from edge_aware_graph_b200 import inputs as I
    if args.workload in BLOCK:
        return run_reference_block(args, world)
    if args.workload not in TRAINING:
        return run_reference_sample(args, WORKLOADS[args.workload], world)
    WORKLOAD = WORKLOADS[args.workload]
    p = I.preset(WORKLOAD)
    if WORKLOAD == "large":
        args.ref_graphs = 1
    d = I.draw_inputs(p, with_grads=True)
    W = I.draw_weights(p)
    for _ in range(args.warmup):
        cpu_baseline(p, d, W, 1)
    res = [cpu_baseline(p, d, W, args.ref_graphs) for _ in range(args.steps)]
    secs = sum(r["seconds"] for r in res)
    pairs = args.steps * args.ref_graphs * p.n * p.n
    value = pairs / secs
    cb = dict(res[0])
    cb["value"] = value
    cb.pop("seconds", None)
    return {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": secs / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded SBM-shaped graphs)",
            "config": {"workload": DESCRIBE[WORKLOAD] + f"; bounded sample of {args.ref_graphs} graph(s) per step",
                       "global_batch": args.ref_graphs,
                       "seq_len": p.n, "parallelism": "cpu"},
            "cpu_baseline": cb,
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def run_reference_sample(args, name, world):
    """The oracle arm of the sampling workload: the oracle's forward on
    --ref-graphs graphs of the batch per step."""
    from edge_aware_graph_b200 import inputs as I
    p = I.preset(name)
    d = I.draw_inputs(p, with_grads=False)
    W = I.draw_weights(p)
    import oracle
    oracle.build()
    g = max(1, min(args.ref_graphs, p.B))
    sl = {k: d[k][:g] for k in ("X", "E", "y", "M")}
    dims = dict(H=p.H, dh=p.dh)
    for _ in range(args.warmup):
        oracle.forward(dims, sl["X"], sl["E"], sl["y"], sl["M"], W)
    t = time.perf_counter()
    for _ in range(args.steps):
        oracle.forward(dims, sl["X"], sl["E"], sl["y"], sl["M"], W)
    secs = time.perf_counter() - t
    value = args.steps * g * p.n * p.n / secs
    return {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": secs / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": f"synthetic (seeded {name.capitalize()}-shaped graphs)",
            "config": {"workload": f"{name}-shaped sampling-time forward, bounded sample of {g} graph(s) "
                                   "per step", "global_batch": g, "seq_len": p.n, "parallelism": "cpu"},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": oracle.threads_used(), "kind": "oracle",
                             "sample": f"the forward of {g} of {p.B} graphs (n={p.n}), fp64, per step"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--parallel", default="batch", choices=["batch", "rows"],
                    help="split graphs over the ranks (batch) or each graph's rows (rows: eaga_*_rows)")
    ap.add_argument("--row-slabs", type=int, default=2,
                    help="with --parallel rows on one GPU: rank 0's slab of this many")
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--cpu-graphs", type=int, default=32)
    ap.add_argument("--cpu-reps", type=int, default=3)
    ap.add_argument("--ref-graphs", type=int, default=2)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-graph", action="store_true", help="launch the step's kernels one by one")
    ap.add_argument("--workload", default="sbm-train", choices=list(WORKLOADS),
                    help="sbm-train: the training step (default); planar-sample / tree-sample: the "
                         "sampling-time forward on Planar- / Tree-shaped batches")
    ap.add_argument("--variant", default="layer", choices=["layer", "light_edge", "unnormalised"],
                    help="training workloads: the layer (default) or one of its ablation variants")
    ap.add_argument("--cpu-seconds", type=float, default=10.0,
                    help="sampling workloads: seconds of oracle forward calls in cpu_baseline")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        out = run_reference(args)
    elif args.parallel == "rows" and args.workload in TRAINING:
        out = run_rows(args)
    else:
        out = run_ours(args)
    if out is not None:
        print(json.dumps(out), flush=True)


if __name__ == "__main__":
    main()
