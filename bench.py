#!/usr/bin/env python
"""Benchmark: converged GRU states per second by parallel Newton on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--T T]

A step is one whole solve of the untrained dense GRU workload (Din = D = 64,
B = 16 sequences per GPU, T = 65536, fp32, weights N(0, 1/D), inputs N(0, 1),
quasi-DEER to tol 1e-5): the input projection, then every Newton iteration
(fused cell + diagonal Jacobian + single-pass scan + convergence reduction)
until the on-device test stops it.  value = B*T*D states x steps x ranks /
(max over ranks of the device time of the K timed steps).

Sequences are independent, so N GPUs run N replicas of the per-GPU batch
(weak scaling, no data-path collective); the launcher is torchrun, one rank
per GPU, NCCL only for the barrier and the max-over-ranks timing.

``--impl reference`` times the fp64 CPU oracle instead (the reference arm of
this benchmark; rank 0 only), on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "converged states/sec (B*T*D per s, Newton to tol)"
UNIT = "states/s"
WORKLOAD = "untrained dense GRU Din=D=64, B=16/GPU, T={T}, fp32, quasi-DEER tol 1e-5"
# bytes each state moves per Newton iteration in a fused single pass:
# P (3 fp32 pre-activations) + previous guess + new guess
BYTES_PER_STATE_ITER = 20
# ncu DRAM traffic of the solver kernel (read + write bytes of one launch,
# captured at T = 16384: 4.812 GB over 14 iterations x 16.78 M states) and the
# hash of the kernel source it was measured on.  Traffic grows with states x
# iterations, so the full launch's is scaled from it; reported only while the
# source is unchanged.
NCU_TRAFFIC = {"bytes_per_state_iter": 4.812e9 / (14 * 16 * 16384 * 64),
               "source_sha1": "6cb957761e3f"}


def log(*a):
    print(*a, file=sys.stderr, flush=True)


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def kernel_sha():
    src = os.path.join(ROOT, "newton_solve_nonlinear_b200", "csrc", "newton_dense_tc.cu")
    return hashlib.sha1(open(src, "rb").read()).hexdigest()[:12]


class Clocks:
    """Sample SM clocks and throttle reasons with nvidia-smi during a region."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = os.path.join("/tmp", f"bench_clocks_{os.getpid()}.csv")

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            self.proc.wait(timeout=10)

    def summary(self):
        if self.proc is None or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        rows = []
        for line in open(self.path):
            f = [x.strip() for x in line.split(",")]
            if len(f) >= 9:
                rows.append(f)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        smax = max(float(r[2]) for r in rows if r[2].replace(".", "").isdigit())
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i] == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "reasons": reasons, "samples": len(rows)}


def cpu_baseline_oracle(T_sample: int = 1024, B_sample: int = 16):
    """Time the fp64 oracle (as it stands) on a bounded sample of the workload."""
    import numpy as np
    import oracle
    from oracle.cells import GRU
    from newton_solve_nonlinear_b200.inputs import make_workload
    try:
        from threadpoolctl import threadpool_info
        cores = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:  # pragma: no cover
        cores = 1
    w = make_workload("untrained", B=B_sample, T=T_sample)
    c = GRU.from_workload(w)
    x, h0 = w.x.double().numpy(), w.h0.double().numpy()
    t0 = time.perf_counter()
    r = oracle.newton_solve(c, x, h0, "QUASI", w.tol)
    secs = time.perf_counter() - t0
    states = w.B * w.T * w.d
    return {"value": states / secs, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"fp64 numpy oracle quasi-DEER to tol 1e-5 on B={w.B}, T={w.T}, D=64 "
                      f"({r['iters']} iterations, {secs:.1f} s); same distributions"}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    steps = []
    base = None
    for i in range(args.warmup + args.steps):
        cb = cpu_baseline_oracle(T_sample=256, B_sample=4)
        if i >= args.warmup:
            steps.append(cb["value"])
        base = cb
    v = statistics.median(steps)
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": None,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": {"workload": WORKLOAD.format(T=args.T), "sample": base["sample"]},
            "cpu_baseline": {"value": v, "unit": UNIT, "cores": base["cores"], "kind": "oracle",
                             "sample": base["sample"]},
            "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def run_ours(args):
    import torch
    import torch.distributed as dist
    from newton_solve_nonlinear_b200 import binding
    from newton_solve_nonlinear_b200.inputs import make_workload

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=300), device_id=dev)

    def barrier():
        if world > 1:
            dist.barrier()

    w = make_workload("untrained", T=args.T, seed=rank)
    B, T, D, din = w.B, w.T, w.d, w.din
    states = B * T * D
    g = lambda t: t.to(dev).contiguous()
    w_ih, b_ih, w_hh, b_hh, x, h0 = map(g, (w.w_ih, w.b_ih, w.w_hh, w.b_hh, w.x, w.h0))
    cell = binding.make_cell("dense", din, D, torch.float32)
    ws = binding.alloc_workspace(binding.workspace_size("dense", din, D, B, T, "QUASI"), dev)
    P = torch.empty(B, T, 3 * D, dtype=torch.float32, device=dev)
    out = torch.empty(B, T, D, dtype=torch.float32, device=dev)
    info = torch.zeros(4, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step(ev_mid=None):
        binding.input_projection(x, w_ih, b_ih, d=D, out=P)
        if ev_mid is not None:
            ev_mid.record(stream)
        binding.newton_iterate(P, w_hh, b_hh, h0, kind="dense", din=din, mode="QUASI",
                               tol=w.tol, info_dev=info, out=out, workspace=ws)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    iters, status = int(info[0]), int(info[1])
    if status != 0:
        log(f"warning: solve status {binding.STATUS.get(status)} after {iters} iterations")

    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
            torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    with Clocks(local) as clk:
        barrier()
        torch.cuda.synchronize()
        for e0, e1, e2 in evs:
            e0.record(stream)
            step(e1)
            e2.record(stream)
        torch.cuda.synchronize()
        barrier()
    total_ms = sum(e0.elapsed_time(e2) for e0, _, e2 in evs)
    solver_ms = [e1.elapsed_time(e2) for _, e1, e2 in evs]
    proj_ms = [e0.elapsed_time(e1) for e0, e1, _ in evs]
    t = torch.tensor([total_ms], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    max_ms = float(t.item())
    value = world * args.steps * states / (max_ms / 1e3)

    # end to end through the public call: pinned host x in, host h out, each step
    x_host = w.x.pin_memory()
    h_host = torch.empty(B, T, D, dtype=torch.float32).pin_memory()
    x_dev = torch.empty_like(x)
    e2e_steps = max(1, min(args.steps, 5))
    barrier()
    torch.cuda.synchronize()
    ea, eb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ea.record(stream)
    for _ in range(e2e_steps):
        x_dev.copy_(x_host, non_blocking=True)
        r = binding.newton_solve(w_ih, b_ih, w_hh, b_hh, x_dev, h0, kind="dense", mode="QUASI",
                                 tol=w.tol, out=out, workspace=ws)
        h_host.copy_(out, non_blocking=True)
    eb.record(stream)
    torch.cuda.synchronize()
    te = torch.tensor([ea.elapsed_time(eb)], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(te, op=dist.ReduceOp.MAX)
    e2e_value = world * e2e_steps * states / (float(te.item()) / 1e3)

    cpu = None
    if rank == 0 and world == 1:
        cpu = cpu_baseline_oracle()

    peak, peak_kind = peaks()
    solver_avg_s = statistics.mean(solver_ms) / 1e3
    algo_bytes = iters * states * BYTES_PER_STATE_ITER
    achieved = algo_bytes / solver_avg_s / 1e9
    traffic = (NCU_TRAFFIC["bytes_per_state_iter"] * iters * states
               if NCU_TRAFFIC["source_sha1"] == kernel_sha() else None)
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": max_ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": WORKLOAD.format(T=T), "B": B, "T": T, "D": D, "din": din,
                   "mode": "QUASI", "tol": w.tol, "iters": iters,
                   "status": binding.STATUS.get(status),
                   "l2": (f"inputs larger than L2 (126 MB): x {x.numel() * 4 / 1e6:.0f} MB, "
                          f"P {P.numel() * 4 / 1e6:.0f} MB, h {out.numel() * 4 / 1e6:.0f} MB per solve"),
                   "parallelism": f"replicas over sequences x{world}",
                   "projection_ms": statistics.mean(proj_ms),
                   "solver_ms": statistics.mean(solver_ms)},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "traffic": traffic,
                     "kernel": "quasi_tc_kernel<64> (persistent, all iterations)",
                     "algorithmic_bytes": f"{BYTES_PER_STATE_ITER} B/state/iteration x {iters} "
                                          f"iterations x {states} states",
                     "peak_kind": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs)"},
        "e2e": {"value": e2e_value, "unit": UNIT,
                "h2d_bytes_per_step": x_host.numel() * 4,
                "d2h_bytes_per_step": h_host.numel() * 4 + 16},
        "gpu_launches": 2 * args.steps,
        "clocks": clk.summary(),
    }
    if cpu is not None:
        line["cpu_baseline"] = cpu
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--T", type=int, default=65536)
    args = ap.parse_args()
    if args.warmup < 3:
        log("warmup raised to 3 (timing rule)")
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
