"""Benchmark of the truly-sparse layer's hot path on B200.

Workload: the single FC layer W 4096 x 4096 at 95% sparsity (838,861 nnz, uniform positions),
bf16 values and activations with fp32 accumulation, batch N in {1, 8, 32}.  One step = the
forward SpMM, the transposed SpMM (input gradient) and the SDDMM (weight gradient) at each of
the three batch sizes: 9 launches.  The format build and one restructure pass are timed
separately and reported under "preprocess" (their cost is reported, not hidden).

Metric: achieved HBM GB/s under the algorithmic byte model (values + indices + row/col
pointers + the dense operands read once + outputs written once) and useful GFLOP/s
(2 nnz N per op).  L2 is kept cold by rotating over R independent copies of every operand
(layout, values, activations, outputs) whose total exceeds 3x the L2 size; each step runs on
the next copy.  Timing: CUDA events on the launching stream around K replays of CUDA graphs
(one graph per copy, one step each), synchronised on both sides; max over ranks.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

--impl reference times the CPU oracle (plain fp64 loops, one thread) on the same workload,
each step a bounded sample of rows.  Under torchrun only rank 0 runs it.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "SpMM HBM GB/s (frac. of peak) & useful GFLOP/s=2·nnz·N at 90–99% sparsity"
WORKLOAD = "fc-4096x4096-s95-bf16"
BATCHES = (1, 8, 32)
OPS = ("forward", "backward_input", "backward_weight")
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0


# ----------------------------------------------------------------------------- byte / flop model

def op_bytes(op: str, M: int, K: int, nnz: int, N: int, s: int, ib: int = 4) -> int:
    """Algorithmic bytes of one op: compulsory traffic, dense operands once; ib = bytes of a
    column / row index (4 as the format specifies, 2 with 16-bit indices; perm stays 4)."""
    if op == "forward":
        return nnz * (s + ib) + 4 * (M + 1) + K * N * s + M * N * s
    if op == "backward_input":
        return nnz * (s + ib + 4) + 4 * (K + 1) + M * N * s + K * N * s
    if op == "backward_weight":
        return nnz * (ib + s) + 4 * (M + 1) + K * N * s + M * N * s
    raise ValueError(op)


def op_flops(nnz: int, N: int) -> int:
    return 2 * nnz * N


def peaks() -> dict:
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "source": "measured", "sm_max_mhz": p.get("sm_max_mhz")}
    return {"hbm_gbs": FALLBACK_HBM_GBS, "source": "fallback", "sm_max_mhz": 1965.0}


# ----------------------------------------------------------------------------- distributed plumbing

def dist_setup(n_gpus: int):
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return rank, world, local


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    """The maximum of x over all ranks (the job's time is its slowest rank's)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank: float, world: int, ms_per_step_max: float) -> float:
    """Whole-job rate: every rank processes units_per_rank per step (weak scaling, replicas),
    and the step time is the maximum over ranks."""
    return units_per_rank * world / (ms_per_step_max * 1e-3)


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons while the timed region runs."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.dev), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, FileNotFoundError):
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        self.out = ""
        if self.proc is not None:
            time.sleep(0.15)
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                self.out, _ = self.proc.communicate()

    def summary(self) -> dict:
        rows = []
        for line in (self.out or "").strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 7:
                continue
            try:
                rows.append((float(parts[0]), float(parts[1]), parts[3:7]))
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        reasons = sorted({names[i] for _, _, r in rows for i, v in enumerate(r) if v.lower() == "active"})
        return {"sm_mhz": float(np.median([r[0] for r in rows])), "sm_max_mhz": max(r[1] for r in rows),
                "reasons": reasons, "samples": len(rows)}


# ----------------------------------------------------------------------------- our implementation

def run_ours(args, rank: int, world: int, local: int) -> dict:
    import torch

    from sparse_spmm_b200 import build as build_mod
    from sparse_spmm_b200 import snk
    from sparse_spmm_b200 import workloads as wl

    build_mod.build()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    props = torch.cuda.get_device_properties(dev)
    l2 = int(getattr(props, "L2_cache_size", 126 * 2**20))

    layer = wl.uniform_layer(4096, 4096, 0.95, "bf16", seed=args.seed, name="W")
    M, K, nnz = layer.M, layer.K, layer.nnz
    s = 2
    batches = [int(b) for b in args.batches.split(",")]

    def dev_bf16(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(dev)

    row_h, col_h, val_h = layer.row, layer.col, layer.values
    xs = {N: wl.activations(K, N, "bf16", args.seed, stream=2) for N in batches}
    dys = {N: wl.activations(M, N, "bf16", args.seed, stream=3) for N in batches}

    # hot bytes of one copy: format arrays read by the products + values + activations + outputs
    hot = nnz * (4 + 4 + 4 + s + s) + 8 * (M + K) + sum((K + M) * N * s * 2 for N in batches)
    R = max(2, int(np.ceil(3.0 * l2 / hot)))
    if args.rotate:
        R = args.rotate

    stream = torch.cuda.Stream(device=dev)
    torch.cuda.synchronize()

    # build R copies (timing the build of the first)
    copies = []
    t_build = None
    ws_bytes = snk.snk_workspace_bytes(M, K, nnz, args.parts)
    for i in range(R):
        row, col, val = torch.from_numpy(row_h).to(dev), torch.from_numpy(col_h).to(dev), dev_bf16(val_h)
        ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
        torch.cuda.synchronize()
        with torch.cuda.stream(stream):
            t0 = time.perf_counter()  # the build call alone (it ends with its own stream sync)
            L = snk.Layout(M, K, row, col, val, num_parts=args.parts, workspace=ws)
            t1 = time.perf_counter()
        if i == 0:
            t_build = t1 - t0
        c = {"L": L}
        for N in batches:
            c[("X", N)] = dev_bf16(xs[N])
            c[("dY", N)] = dev_bf16(dys[N])
            c[("Y", N)] = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
            c[("dX", N)] = torch.empty((K, N), dtype=torch.bfloat16, device=dev)
            c[("dW", N)] = torch.empty(nnz, dtype=torch.bfloat16, device=dev)
        copies.append(c)
    P = copies[0]["L"].num_parts
    torch.cuda.synchronize()

    def launch(c, op, N, st):
        L = c["L"]
        if op == "forward":
            L.forward(c[("X", N)], Y=c[("Y", N)], stream=st)
        elif op == "backward_input":
            L.backward_input(c[("dY", N)], dX=c[("dX", N)], stream=st)
        else:
            L.backward_weight(c[("dY", N)], c[("X", N)], dW=c[("dW", N)], stream=st)

    def step(c, st):
        for N in batches:
            for op in OPS:
                launch(c, op, N, st)

    launches_per_step = len(batches) * len(OPS)  # every N <= 64: one kernel per op

    # warm-up (also JIT-free: the library is precompiled) then capture one graph per copy
    with torch.cuda.stream(stream):
        for i in range(max(1, args.warmup)):
            step(copies[i % R], stream)
    torch.cuda.synchronize()
    graphs = []
    for c in copies:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            step(c, stream)
        graphs.append(g)
    torch.cuda.synchronize()

    # per-op graphs: R launches of one (op, N), to time each kernel alone (L2-cold)
    reps = 20

    def time_ops(ib: int) -> dict:
        res = {}
        for N in batches:
            for op in OPS:
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g, stream=stream):
                    for c in copies:
                        launch(c, op, N, stream)
                with torch.cuda.stream(stream):
                    g.replay()
                stream.synchronize()
                e0 = torch.cuda.Event(enable_timing=True)
                e1 = torch.cuda.Event(enable_timing=True)
                with torch.cuda.stream(stream):
                    e0.record(stream)
                    for _ in range(reps):
                        g.replay()
                    e1.record(stream)
                e1.synchronize()
                us = e0.elapsed_time(e1) * 1e3 / (reps * R)
                b = op_bytes(op, M, K, nnz, N, s, ib)
                res[f"{op}@N={N}"] = {"us": round(us, 3), "bytes": b, "gbs": round(b / us / 1e3, 1),
                                      "gflops": round(op_flops(nnz, N) / us / 1e3, 1)}
                del g
        return res

    torch.cuda.nvtx.range_push("per-op graphs, int32 indices")
    per_op = time_ops(4)
    torch.cuda.nvtx.range_pop()
    # the same ops reading 16-bit column / row indices (bit-identical results), with their
    # own byte model; the step above and the headline use the int32 format
    for c in copies:
        c["L"].set_index_bits(16)
    torch.cuda.nvtx.range_push("per-op graphs, 16-bit indices")
    per_op16 = time_ops(2)
    torch.cuda.nvtx.range_pop()
    for c in copies:
        c["L"].set_index_bits(32)
    us32 = sum(v["us"] for v in per_op.values())
    us16 = sum(v["us"] for v in per_op16.values())
    index16 = {"ops_us_sum": round(us16, 3), "int32_ops_us_sum": round(us32, 3),
               "time_ratio_vs_int32": round(us16 / us32, 4),
               "gbs_own_model": round(sum(v["bytes"] for v in per_op16.values()) / us16 / 1e3, 1),
               "byte_model": "col / csc_row 2 B per nonzero, perm 4 B", "per_op_us": {k: v["us"] for k, v in per_op16.items()}}

    # warm-up of the step graphs, then the timed region
    with torch.cuda.stream(stream):
        for i in range(args.warmup):
            graphs[i % R].replay()
    torch.cuda.synchronize()
    barrier(world)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        torch.cuda.synchronize()
        torch.cuda.nvtx.range_push("timed steps")
        with torch.cuda.stream(stream):
            e0.record(stream)
            for i in range(args.steps):
                graphs[i % R].replay()
            e1.record(stream)
        e1.synchronize()
        torch.cuda.nvtx.range_pop()
        torch.cuda.synchronize()
    barrier(world)
    ms = max_over_ranks(e0.elapsed_time(e1), world)
    ms_per_step = ms / args.steps

    step_bytes = sum(op_bytes(op, M, K, nnz, N, s) for N in batches for op in OPS)
    step_flops = sum(op_flops(nnz, N) for N in batches for op in OPS)
    value = job_throughput(step_bytes, world, ms_per_step) / 1e9
    gflops = job_throughput(step_flops, world, ms_per_step) / 1e9

    # end to end through the public API: pinned host inputs in, results out, every step
    pinned = {}
    for N in batches:
        pinned[("X", N)] = torch.from_numpy(xs[N].view(np.int16)).view(torch.bfloat16).pin_memory()
        pinned[("dY", N)] = torch.from_numpy(dys[N].view(np.int16)).view(torch.bfloat16).pin_memory()
        pinned[("Y", N)] = torch.empty((M, N), dtype=torch.bfloat16).pin_memory()
        pinned[("dX", N)] = torch.empty((K, N), dtype=torch.bfloat16).pin_memory()
        pinned[("dW", N)] = torch.empty(nnz, dtype=torch.bfloat16).pin_memory()
    h2d = sum(pinned[("X", N)].numel() * s + pinned[("dY", N)].numel() * s for N in batches)
    d2h = sum((pinned[("Y", N)].numel() + pinned[("dX", N)].numel() + pinned[("dW", N)].numel()) * s
              for N in batches)

    # Three streams, as a user would pipeline a stream of steps: step i's uploads (h2d) run
    # while step i-1 computes, and its downloads (d2h) while step i+1 computes; events order
    # upload -> compute -> download of each step, which runs on its own rotated copy.
    h2d_s = torch.cuda.Stream(device=dev)
    d2h_s = torch.cuda.Stream(device=dev)

    def e2e_step(c):
        up = torch.cuda.Event()
        with torch.cuda.stream(h2d_s):
            if "done" in c:  # this copy's previous results have been read back
                h2d_s.wait_event(c["done"])
            for N in batches:
                c[("X", N)].copy_(pinned[("X", N)], non_blocking=True)
                c[("dY", N)].copy_(pinned[("dY", N)], non_blocking=True)
            up.record(h2d_s)
        stream.wait_event(up)
        for N in batches:
            for op in OPS:
                launch(c, op, N, stream)
        computed = torch.cuda.Event()
        computed.record(stream)
        with torch.cuda.stream(d2h_s):
            d2h_s.wait_event(computed)
            for N in batches:
                pinned[("Y", N)].copy_(c[("Y", N)], non_blocking=True)
                pinned[("dX", N)].copy_(c[("dX", N)], non_blocking=True)
                pinned[("dW", N)].copy_(c[("dW", N)], non_blocking=True)
            c["done"] = torch.cuda.Event()
            c["done"].record(d2h_s)

    e2e_steps = max(20, min(args.steps, 2000))
    for i in range(3):
        e2e_step(copies[i % R])
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.nvtx.range_push("e2e steps")
    e0.record(h2d_s)
    for i in range(e2e_steps):
        e2e_step(copies[i % R])
    e1.record(d2h_s)
    torch.cuda.nvtx.range_pop()
    e1.synchronize()
    barrier(world)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world) / e2e_steps
    e2e_value = job_throughput(step_bytes, world, e2e_ms) / 1e9

    # preprocessing: build (timed above, host wall clock incl. its one sync) and one restructure
    L0 = copies[0]["L"]
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    with torch.cuda.stream(stream):
        L0.restructure(nnz // 10, seed=args.seed)
    t_rs = time.perf_counter() - t0

    pk = peaks()
    dom_key = max(per_op, key=lambda k: per_op[k]["us"])
    dom_op = dom_key.split("@")[0]
    dom_launches = [k for k in per_op if k.startswith(dom_op + "@")]
    dom_bytes = sum(per_op[k]["bytes"] for k in dom_launches)
    dom_us = sum(per_op[k]["us"] for k in dom_launches)
    achieved = dom_bytes / dom_us / 1e3
    traffic = traffic_for(dom_op)
    roofline = {"bound": "hbm", "achieved": round(achieved, 1), "peak": pk["hbm_gbs"], "unit": "GB/s",
                "frac": round(achieved / pk["hbm_gbs"], 4), "traffic": traffic,
                "kernel": KERNEL_NAMES[dom_op], "launches_averaged": dom_launches,
                "peak_source": pk["source"] + " (hbm_gbs, copy burst)"}

    out = {
        "metric": METRIC, "value": round(value, 1), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_per_step, 6), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": WORKLOAD, "M": M, "K": K, "nnz": nnz, "batches": batches, "ops": list(OPS),
                   "num_parts": P, "l2": f"cold: {R} rotated copies x {hot / 1e6:.1f} MB >= 3x L2 ({l2 / 2**20:.0f} MiB)",
                   "parallelism": f"replicas x{world}"},
        "frac_of_peak": round(value / world / pk["hbm_gbs"], 4),
        "frac_of_nominal_8tbs": round(value / world / 8000.0, 4),
        "gflops": round(gflops, 1),
        "roofline": roofline,
        "e2e": {"value": round(e2e_value, 2), "unit": "GB/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": round(e2e_ms, 4), "steps": e2e_steps,
                "pipelining": "uploads, products and downloads on three streams, ordered per step by events"},
        "clocks": clk.summary(),
        "gpu_launches": launches_per_step * args.steps,
        "per_op": per_op,
        "index16": index16,
        "preprocess": {"build_ms": round(t_build * 1e3, 3), "restructure_ms": round(t_rs * 1e3, 3),
                       "restructure_drop": nnz // 10, "note": "host wall clock incl. the one status sync"},
    }
    if rank == 0 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(layer, xs, dys, batches, budget_s=args.cpu_seconds)
    for g in graphs:
        del g
    return out


KERNEL_NAMES = {"forward": "k_spmm_small<bf16,*,*,false,int32_t>", "backward_input": "k_spmm_small<bf16,*,*,true,int32_t>",
                "backward_weight": "k_sddmm_small<bf16,*,*,int32_t,false>"}


def traffic_for(op: str):
    """DRAM bytes per launch from the committed ncu summary, if it matches the current source."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        t = json.load(f)
    src = os.path.join(ROOT, "sparse_spmm_b200", "csrc", "spmm.cu")
    h = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
    if t.get("spmm_cu_sha256_16") != h:
        return None
    ent = t.get("ops", {}).get(op)
    return ent.get("dram_bytes_per_launch_avg") if ent else None


# ----------------------------------------------------------------------------- CPU oracle legs

def _oracle_inputs(layer, xs, dys, batches):
    import oracle
    ref = oracle.build(layer.M, layer.K, layer.row, layer.col, layer.values, 1)
    v64 = oracle.widen(ref["values"])
    X64 = {N: oracle.widen(xs[N].reshape(-1)).reshape(xs[N].shape) for N in batches}
    dY64 = {N: oracle.widen(dys[N].reshape(-1)).reshape(dys[N].shape) for N in batches}
    return ref, v64, X64, dY64


def _oracle_step(layer, ref, v64, X64, dY64, batches, rows_sel):
    """One oracle step restricted to the entries of rows_sel (all three ops, every N)."""
    import oracle
    m = np.isin(ref["row"], rows_sel)
    r, c, v = ref["row"][m], ref["col"][m], v64[m]
    for N in batches:
        oracle.forward(layer.M, layer.K, r, c, v, X64[N])
        oracle.backward_input(layer.M, layer.K, r, c, v, dY64[N])
        oracle.backward_weight(r, c, dY64[N], X64[N])
    return int(m.sum())


def cpu_baseline(layer, xs, dys, batches, budget_s: float = 15.0) -> dict:
    """The oracle as it stands (plain fp64 loops, 1 thread) timed on a bounded sample."""
    ref, v64, X64, dY64 = _oracle_inputs(layer, xs, dys, batches)
    s = 2
    done_bytes, t_total, steps = 0, 0.0, 0
    rng = np.random.default_rng(0)
    frac_rows = 256
    while t_total < budget_s and steps < 1000:
        rows_sel = np.sort(rng.choice(layer.M, size=frac_rows, replace=False))
        t0 = time.perf_counter()
        n_sel = _oracle_step(layer, ref, v64, X64, dY64, batches, rows_sel)
        t_total += time.perf_counter() - t0
        f = frac_rows / layer.M
        done_bytes += sum(op_bytes(op, layer.M, layer.K, layer.nnz, N, s) for N in batches for op in OPS) * \
            (n_sel / layer.nnz) if n_sel else 0
        steps += 1
    return {"value": round(done_bytes / t_total / 1e9, 4), "unit": "GB/s", "cores": 1, "kind": "oracle",
            "host_cores": len(os.sched_getaffinity(0)),
            "sample": f"{steps} samples of {frac_rows} random rows (fwd, dX, dW at N={list(batches)}), "
                      f"{t_total:.1f} s of oracle time; bytes scaled by the sampled share of nnz"}


def run_reference(args, rank: int, world: int) -> dict:
    from sparse_spmm_b200 import workloads as wl
    layer = wl.uniform_layer(4096, 4096, 0.95, "bf16", seed=args.seed, name="W")
    batches = [int(b) for b in args.batches.split(",")]
    xs = {N: wl.activations(layer.K, N, "bf16", args.seed, stream=2) for N in batches}
    dys = {N: wl.activations(layer.M, N, "bf16", args.seed, stream=3) for N in batches}
    ref, v64, X64, dY64 = _oracle_inputs(layer, xs, dys, batches)
    s = 2
    full_bytes = sum(op_bytes(op, layer.M, layer.K, layer.nnz, N, s) for N in batches for op in OPS)
    # size each step so that warm-up + steps fit in about two minutes
    probe_rows = np.arange(0, layer.M, 64)
    t0 = time.perf_counter()
    n_probe = _oracle_step(layer, ref, v64, X64, dY64, batches, probe_rows)
    t_probe = time.perf_counter() - t0
    per_nnz = t_probe / max(n_probe, 1)
    budget = 120.0 / max(1, args.steps + args.warmup)
    rows_per_step = int(np.clip(budget / per_nnz / (layer.nnz / layer.M), 1, layer.M))
    rng = np.random.default_rng(1)
    for _ in range(args.warmup):
        _oracle_step(layer, ref, v64, X64, dY64, batches, rng.choice(layer.M, rows_per_step, replace=False))
    t_total, done = 0.0, 0.0
    for _ in range(args.steps):
        sel = np.sort(rng.choice(layer.M, rows_per_step, replace=False))
        t0 = time.perf_counter()
        n_sel = _oracle_step(layer, ref, v64, X64, dY64, batches, sel)
        t_total += time.perf_counter() - t0
        done += full_bytes * n_sel / layer.nnz
    value = done / t_total / 1e9
    sample = f"each step: fwd, dX, dW at N={batches} over the entries of {rows_per_step} random rows of 4096"
    return {"impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(t_total / args.steps * 1e3, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {"workload": WORKLOAD, "batches": batches, "ops": list(OPS),
                                            "parallelism": "rank 0 only (CPU oracle)"},
            "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": 1, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def run_profile(args) -> None:
    """Two passes of the step's launches (forward, transposed, SDDMM per batch) on one layout,
    no timing: pass 0 warms up, pass 1 is what an ncu capture selects.  For profiling only."""
    import torch

    from sparse_spmm_b200 import build as build_mod
    from sparse_spmm_b200 import snk
    from sparse_spmm_b200 import workloads as wl

    build_mod.build()
    torch.cuda.set_device(0)
    relu = False
    if args.profile_workload == "gpt2-w1":  # GPT-2 c_fc, 3072 x 768 at 90% (magnitude-pruned), fp32, N = 1024
        layer = wl.magnitude_pruned_layer(3072, 768, 0.90, args.seed, "W1")
        batches = [1024]
    elif args.profile_workload == "gpt2-w2":  # GPT-2 c_proj, 768 x 3072 at 90%, fp32, N = 1024
        layer = wl.magnitude_pruned_layer(768, 3072, 0.90, args.seed + 1, "W2")
        batches = [1024]
    elif args.profile_workload == "conv-512x2048-s80":  # 1x1 conv, fp32, N = 6272, X = ReLU(N(0,1))
        layer = wl.uniform_layer(512, 2048, 0.80, "f32", args.seed, "W")
        batches = [6272]
        relu = True
    elif args.profile_workload == "tiny-fc":  # 512 x 512 at 90%, fp32, N = 8
        layer = wl.uniform_layer(512, 512, 0.90, "f32", args.seed, "W")
        batches = [8]
    elif args.profile_workload == "llama-up":  # 11008 x 4096 at 99%, Zipf(1.2) rows, bf16, N = 1, 4, 16
        layer = wl.zipf_layer(11008, 4096, 0.99, "bf16", 1.2, args.seed, "W_up")
        batches = [1, 4, 16]
    elif args.profile_workload == "llama-down":  # 4096 x 11008 at 99%, Zipf(1.2) rows, bf16, N = 1, 4, 16
        layer = wl.zipf_layer(4096, 11008, 0.99, "bf16", 1.2, args.seed + 1, "W_down")
        batches = [1, 4, 16]
    else:  # the bench workload
        layer = wl.uniform_layer(4096, 4096, 0.95, "bf16", seed=args.seed, name="W")
        batches = [int(b) for b in args.batches.split(",")]

    def dev_t(a):
        if a.dtype == np.uint16:
            return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()
        return torch.from_numpy(a).cuda()

    L = snk.Layout(layer.M, layer.K, dev_t(layer.row), dev_t(layer.col), dev_t(layer.values), num_parts=args.parts)
    data = {N: (dev_t(wl.activations(layer.K, N, layer.dtype, args.seed, stream=2, relu=relu)),
                dev_t(wl.activations(layer.M, N, layer.dtype, args.seed, stream=3))) for N in batches}
    torch.cuda.synchronize()
    for _ in range(2):
        for N in batches:
            X, dY = data[N]
            L.forward(X)
            L.backward_input(dY)
            L.backward_weight(dY, X)
    torch.cuda.synchronize()
    print(json.dumps({"profile_passes": 2, "launches_per_pass": 3 * len(batches), "batches": batches,
                      "workload": args.profile_workload}))


# ----------------------------------------------------------------------------- sweep over every config

def _graph_time_us(fns, reps: int = 3, rounds: int = 3) -> float:
    """Per-call µs of the calls in `fns` (one per rotated copy), captured into one CUDA graph
    and replayed `reps` times; best of `rounds`."""
    import torch
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):  # eager warm-up: library handles (cuBLAS) exist before capture
        for f in fns:
            f()
    s.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        for f in fns:
            f()
    with torch.cuda.stream(s):
        g.replay()
    s.synchronize()
    best = float("inf")
    for _ in range(rounds):
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(s):
            e0.record(s)
            for _ in range(reps):
                g.replay()
            e1.record(s)
        e1.synchronize()
        best = min(best, e0.elapsed_time(e1) * 1e3 / (reps * len(fns)))
    del g
    return best


def fp32_fma_peak(sm_count: int) -> dict:
    """Measured fp32 FMA rate (TFLOP/s) from the library's probe, best of 3 ~10 ms launches."""
    import torch
    from sparse_spmm_b200 import snk
    blocks = 4 * sm_count
    sink = torch.zeros(blocks, device="cuda")
    iters = 60000
    snk.snk_probe_fp32_fma(blocks, 1000, sink)
    best = float("inf")
    flops = 0
    for _ in range(3):
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record()
        flops = snk.snk_probe_fp32_fma(blocks, iters, sink)
        e1.record()
        e1.synchronize()
        best = min(best, e0.elapsed_time(e1) * 1e-3)
    return {"tflops": round(flops / best / 1e12, 2), "blocks": blocks, "iters": iters}


def run_sweep(args) -> None:
    """Every config, op and batch of the workload list: L2-cold per-op CUDA graphs, achieved
    GB/s and GFLOP/s under the byte model, fractions of the measured HBM and fp32 FMA peaks,
    a single launch after an L2 flush, and (forward) the dense and dense+mask products of the
    same W on the same GPU (torch.matmul, i.e. cuBLAS), as the pages' ratio style.  One JSON
    line per measurement."""
    import torch

    from sparse_spmm_b200 import build as build_mod
    from sparse_spmm_b200 import snk
    from sparse_spmm_b200 import workloads as wl

    build_mod.build()
    torch.cuda.set_device(0)
    sm_count = torch.cuda.get_device_properties(0).multi_processor_count
    pk = peaks()
    l2 = 126 * 2 ** 20

    def dev_t(a):
        if a.dtype == np.uint16:
            return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()
        return torch.from_numpy(np.ascontiguousarray(a)).cuda()

    with ClockSampler(0) as clk:
        f32 = fp32_fma_peak(sm_count)
    f32["clocks"] = clk.summary()
    print(json.dumps({"sweep": "fp32_fma_peak", **f32}), flush=True)

    flush = torch.empty(3 * l2 // 4, dtype=torch.float32, device="cuda")
    works = [wl.tiny_fc(), wl.fc_4096(), wl.gpt2_mlp(), wl.llama_mlp()]
    works += [wl.conv1x1(M, K, sp) for (M, K) in wl.CONV_SHAPES for sp in wl.CONV_SPARSITIES]
    opname = {"forward": "forward", "backward_input": "backward_input", "backward_weight": "backward_weight"}
    for work in works:
        s = 2 if work.dtype == "bf16" else 4
        tdt = torch.bfloat16 if work.dtype == "bf16" else torch.float32
        for make in work.layers:
            layer = make()
            M, K, nnz = layer.M, layer.K, layer.nnz
            hot = nnz * (s + 12) + 8 * (M + K) + max(work.batches) * (M + K) * s * 2
            R = int(min(40, max(2, np.ceil(3 * l2 / hot))))
            copies = [snk.Layout(M, K, dev_t(layer.row), dev_t(layer.col), dev_t(layer.values)) for _ in range(R)]
            for N in work.batches:
                X = [dev_t(wl.activations(K, N, work.dtype, args.seed, 2, work.relu_x)) for _ in range(R)]
                dY = [dev_t(wl.activations(M, N, work.dtype, args.seed, 3)) for _ in range(R)]
                Y = [torch.empty(M, N, dtype=tdt, device="cuda") for _ in range(R)]
                dX = [torch.empty(K, N, dtype=tdt, device="cuda") for _ in range(R)]
                dW = [torch.empty(nnz, dtype=tdt, device="cuda") for _ in range(R)]
                torch.cuda.synchronize()
                for op in work.ops:
                    if op == "restructure":
                        continue
                    if op == "forward":
                        fns = [lambda i=i: copies[i].forward(X[i], Y=Y[i]) for i in range(R)]
                    elif op == "backward_input":
                        fns = [lambda i=i: copies[i].backward_input(dY[i], dX=dX[i]) for i in range(R)]
                    else:
                        fns = [lambda i=i: copies[i].backward_weight(dY[i], X[i], dW=dW[i]) for i in range(R)]
                    us = _graph_time_us(fns, reps=3 if N >= 1024 else 10)
                    # one launch right after an L2 flush (a 3 x L2 buffer written), best of 3
                    single = float("inf")
                    for _ in range(3):
                        flush.fill_(1.0)
                        e0 = torch.cuda.Event(enable_timing=True)
                        e1 = torch.cuda.Event(enable_timing=True)
                        e0.record()
                        fns[0]()
                        e1.record()
                        e1.synchronize()
                        single = min(single, e0.elapsed_time(e1) * 1e3)
                    b = op_bytes(opname[op], M, K, nnz, N, s)
                    fl = op_flops(nnz, N)
                    rec = {"sweep": work.name, "layer": layer.name, "M": M, "K": K, "nnz": nnz, "op": op, "N": N,
                           "us": round(us, 2), "single_launch_us": round(single, 2), "gbs": round(b / us / 1e3, 1),
                           "frac_hbm": round(b / us / 1e3 / pk["hbm_gbs"], 4),
                           "gflops": round(fl / us / 1e3, 1), "frac_fp32": round(fl / us / 1e6 / f32["tflops"], 4),
                           "bound": "alu" if fl / (f32["tflops"] * 1e12) > b / (pk["hbm_gbs"] * 1e9) else "hbm"}
                    if op == "forward":
                        # dense and dense+mask products of the same W (cuBLAS via torch), L2-cold too
                        Wd = torch.zeros(M, K, dtype=tdt, device="cuda")
                        Wd[dev_t(layer.row).long(), dev_t(layer.col).long()] = dev_t(layer.values)
                        Md = (Wd != 0).to(tdt)
                        Rd = int(min(R, max(2, np.ceil(3 * l2 / (M * K * s * 2 + (M + K) * N * s)))))
                        Wds = [Wd.clone() for _ in range(Rd)]
                        Mds = [Md.clone() for _ in range(Rd)]
                        Tmp = [torch.empty_like(Wd) for _ in range(Rd)]
                        dense = [lambda i=i: torch.matmul(Wds[i], X[i], out=Y[i]) for i in range(Rd)]
                        masked = [lambda i=i: (torch.mul(Wds[i], Mds[i], out=Tmp[i]),
                                               torch.matmul(Tmp[i], X[i], out=Y[i])) for i in range(Rd)]
                        rec["dense_us"] = round(_graph_time_us(dense), 2)
                        rec["dense_mask_us"] = round(_graph_time_us(masked), 2)
                        rec["speedup_vs_dense"] = round(rec["dense_us"] / us, 2)
                        rec["speedup_vs_dense_mask"] = round(rec["dense_mask_us"] / us, 2)
                        del Wd, Md, Wds, Mds, Tmp
                    print(json.dumps(rec), flush=True)
                del X, dY, Y, dX, dW
            if "restructure" in work.ops:
                k = int(round(0.1 * nnz))
                L = copies[0]
                L.restructure(k, seed=args.seed)  # warm-up
                torch.cuda.synchronize()
                e0 = torch.cuda.Event(enable_timing=True)
                e1 = torch.cuda.Event(enable_timing=True)
                e0.record()
                L.restructure(k, seed=args.seed + 1)
                e1.record()
                e1.synchronize()
                print(json.dumps({"sweep": work.name, "layer": layer.name, "op": "restructure", "drop": k,
                                  "ms": round(e0.elapsed_time(e1), 3)}), flush=True)
            del copies
            torch.cuda.empty_cache()

    # sparse 3x3 convolutions at ResNet-50 layer shapes (channel-major input, batch 32):
    # patch matrix + forward SpMM, against cuDNN's dense fp32 convolution (TF32 off)
    torch.backends.cudnn.allow_tf32 = False
    for (Cc, HW, sp) in ((256, 14, 0.90), (256, 14, 0.95), (512, 7, 0.90), (512, 7, 0.95)):
        Nb, H, W = 32, HW, HW
        P = Nb * H * W
        layer = wl.uniform_layer(Cc, 9 * Cc, sp, "f32", args.seed, "W3x3")
        xin = np.maximum(np.random.default_rng(args.seed).normal(size=(Cc, P)), 0).astype(np.float32)
        hot = layer.nnz * 8 + Cc * P * 4 * 11  # W, input, patch matrix (9x), output
        R = int(min(20, max(2, np.ceil(3 * l2 / hot))))
        Ls = [snk.Layout(Cc, 9 * Cc, dev_t(layer.row), dev_t(layer.col), dev_t(layer.values)) for _ in range(R)]
        xs = [dev_t(xin) for _ in range(R)]
        patches = [torch.empty((9 * Cc, P), device="cuda") for _ in range(R)]
        ys = [torch.empty((Cc, P), device="cuda") for _ in range(R)]
        fns = [lambda i=i: snk.sparse_conv3x3(Ls[i], xs[i], Nb, H, W, patch=patches[i], Y=ys[i]) for i in range(R)]
        us = _graph_time_us(fns, reps=5)
        im2 = [lambda i=i: snk.snk_im2col3x3(xs[i], Cc, Nb, H, W, out=patches[i]) for i in range(R)]
        us_patch = _graph_time_us(im2, reps=5)
        Wd = torch.zeros(Cc, 9 * Cc, device="cuda")
        Wd[dev_t(layer.row).long(), dev_t(layer.col).long()] = dev_t(layer.values)
        Wd4 = Wd.view(Cc, Cc, 3, 3)
        xn = [x.view(Cc, Nb, H, W).permute(1, 0, 2, 3).contiguous() for x in xs]  # NCHW for cuDNN
        dense = [lambda i=i: torch.nn.functional.conv2d(xn[i], Wd4, padding=1) for i in range(R)]
        us_dense = _graph_time_us(dense, reps=5)
        fl = op_flops(layer.nnz, P)
        b = layer.nnz * 8 + 4 * (Cc + 1) + Cc * P * 4 * 2  # W once, input once, output once
        print(json.dumps({"sweep": f"conv3x3-{Cc}x{Cc}-{H}x{W}-b32-s{int(round(sp * 100))}-f32", "layer": "W3x3",
                          "M": Cc, "K": 9 * Cc, "nnz": layer.nnz, "op": "conv3x3", "N": P, "us": round(us, 2),
                          "patch_us": round(us_patch, 2), "gbs_implicit_model": round(b / us / 1e3, 1),
                          "gflops": round(fl / us / 1e3, 1), "frac_fp32": round(fl / us / 1e6 / f32["tflops"], 4),
                          "dense_cudnn_fp32_us": round(us_dense, 2), "speedup_vs_dense": round(us_dense / us, 2)}),
              flush=True)
        del Ls, xs, patches, ys, xn, Wd, Wd4
        torch.cuda.empty_cache()


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20000)
    ap.add_argument("--warmup", type=int, default=200)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--batches", default="1,8,32")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--parts", type=int, default=0, help="nnz-balanced parts (0 = library default)")
    ap.add_argument("--rotate", type=int, default=0, help="number of rotated copies (0 = enough for 3x L2)")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--profile", action="store_true",
                    help="run two untimed passes of the step (for ncu captures) and exit")
    ap.add_argument("--profile-workload", default="fc",
                    choices=("fc", "gpt2-w1", "gpt2-w2", "conv-512x2048-s80", "tiny-fc", "llama-up", "llama-down"),
                    help="workload of --profile: the bench's FC layer or another config's layer")
    ap.add_argument("--sweep", action="store_true",
                    help="time every config, op and batch (plus dense baselines); JSON lines; exit")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    if args.profile:
        run_profile(args)
        return 0
    if args.sweep:
        run_sweep(args)
        return 0
    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        world = int(os.environ.get("WORLD_SIZE", "1"))
        if rank != 0:
            return 0
        print(json.dumps(run_reference(args, rank, world)), flush=True)
        return 0

    rank, world, local = dist_setup(args.gpus)
    out = run_ours(args, rank, world, local)
    if rank == 0:
        print(json.dumps(out), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
