#!/usr/bin/env python
"""Benchmark: converged GRU states per second by parallel Newton on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--T T]

A step is one whole solve: the input projection, then every Newton iteration
until the on-device test stops it.  The default workload is the untrained
dense GRU (Din = D = 64, B = 16 sequences per GPU, T = 65536, fp32, weights
N(0, 1/D), inputs N(0, 1), quasi-DEER to tol 1e-5: fused cell + diagonal
Jacobian + single-pass scan + convergence reduction per iteration).
``--workload`` selects another solver family with the same line format:
diag (diagonal-recurrence GRU, exact Newton), dense_deer (full-Jacobian DEER
on tensor cores), quasi_elk and elk (damped steps on the near-unstable GRU).
value = B*T*D states x steps x ranks / (max over ranks of the device time of
the K timed steps).

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
# Parts (ramped sizes) whose copies the host-buffer calls overlap with the solves.
# Every part costs a solve's fixed overhead (a launch, and per iteration a grid
# barrier and a pipeline refill), while the first part's copy in and the last
# part's copy out overlap nothing: large copies against a short solve want
# more parts, a short sequence with many iterations fewer.  Measured on the
# streamed call (one B200): untrained GRU best at 7 (9.26 ms; 5: 9.54, 9: 9.53);
# quasi-ELK (28 iterations, 5.1 M states) at 2 (4.52 ms; 7: 6.38); dense DEER
# at 2 (3.20 ms; 7: 4.71).
E2E_PARTS = 7
# The benchmarked solves, one per row family of the hot path.  "untrained"
# (the default) is the headline; the others measure the other solver kernels
# with the same JSON line.  Roofline units per state and Newton iteration:
#   hbm    algorithmic bytes a fused single pass moves: P (3 fp32
#          pre-activations) + previous guess + new guess = 20 B; quasi-ELK
#          forward (P + guess, writes m, P, a, b) + backward (reads 16, guess 4,
#          writes 4) = 56 B;
#   tensor D x D Jacobian products, 2 D^3 flop per step = 2 D^2 per state;
#   alu    dense ELK cyclic reduction, about 14 D^3 flop per step (J^T J 2 D^3,
#          each step eliminated once: inverse + two products 6 D^3, folded once:
#          three products 6 D^3) = 14 D^2 per state.
BENCHES = {
    "untrained": dict(
        workload="untrained", mode="QUASI", lam=0.0, bound="hbm", per_state=20,
        kernel="quasi_tc2_kernel<64, quasi> (persistent, all iterations)",
        desc="untrained dense GRU Din=D=64, B={B}/GPU, T={T}, fp32, quasi-DEER tol 1e-5",
        cpu_sample=dict(B=16, T=12288), ref_sample=dict(B=16, T=4096), roll_sample=dict()),
    "diag": dict(
        workload="diag", mode="QUASI", lam=0.0, bound="hbm", per_state=20,
        kernel="diag2_kernel (persistent, all iterations)",
        desc="diagonal-recurrence GRU Din=D=2048, B={B}/GPU, T={T}, bf16 x and W_ih, fp32 state, "
             "quasi-DEER (exact Newton) tol 1e-4",
        cpu_sample=dict(B=1, T=16384), ref_sample=dict(B=1, T=2048), roll_sample=dict(T=256)),
    "dense_deer": dict(
        workload="dense_deer", mode="DEER", lam=0.0, bound="tensor", per_state=None,
        kernel="deer_mma_kernel (persistent, all iterations)",
        desc="dense GRU Din=16, D=32, B={B}/GPU, T={T}, fp32 cell, TF32 Jacobian products, DEER tol 1e-5",
        cpu_sample=dict(B=4, T=32768), ref_sample=dict(B=4, T=4096), roll_sample=dict(), e2e_parts=2),
    "quasi_elk": dict(
        workload="near_unstable", mode="QUASI_ELK", lam=0.1, bound="hbm", per_state=56,
        kernel="quasi_tc2_kernel<64, quasi-ELK> (persistent, all iterations)",
        desc="near-unstable dense GRU Din=D=64 (spectral radius 1.5), B={B}/GPU, T={T}, fp32, "
             "quasi-ELK lambda 0.1, tol 1e-4",
        cpu_sample=dict(B=8, T=8000), ref_sample=dict(B=2, T=2000), roll_sample=dict(), e2e_parts=2),
    "elk": dict(
        workload="near_unstable", mode="ELK", lam=0.01, bound="alu", per_state=None,
        kernel="dense_elk_kernel<64> (persistent, all iterations)",
        desc="near-unstable dense GRU Din=D=64 (spectral radius 1.5), B={B}/GPU, T={T}, fp32, "
             "ELK lambda 0.01, tol 1e-4",
        cpu_sample=dict(B=1, T=5000), ref_sample=dict(B=1, T=1000), roll_sample=dict(), e2e_parts=2),
    # the backward pass through the evaluated diagonal-cell sequence (not a solve):
    # reads P 12 + h 4 + dL/dh 4, writes dL/dP 12 = 32 B per state
    "adjoint": dict(
        workload="diag", mode="ADJOINT", lam=0.0, bound="hbm", per_state=32,
        kernel="adjoint_diag_kernel (one reverse pass)",
        desc="backward pass of the diagonal-recurrence GRU Din=D=2048, B={B}/GPU, T={T}: "
             "dL/dP, dL/dh0, dL/du, dL/db_hh from the converged states and dL/dh",
        cpu_sample=dict(B=1, T=1024), ref_sample=dict(B=1, T=512)),
}
# the dense cell's backward pass with the Jacobian's diagonal: the step is four
# kernels; algorithmic bytes per state over all of them: h_{t-1} copy 8, GEMM
# U h_{t-1} (reads h 4, writes 12), reverse scan (reads P 12, U h 12, h 4,
# dL/dh 4; writes dL/dP 12, grow 12), dW_hh GEMM (reads grow 12, h 4) = 96 B
BENCHES["adjoint_dense"] = dict(
    workload="untrained", mode="ADJOINT", lam=0.0, bound="hbm", per_state=96,
    kernel="the backward step: h_{t-1} copy, proj_gemm_kernel (U h), adjoint_diag_kernel<dense>, "
           "outer_sum_partial_kernel + outer_sum_reduce_kernel",
    desc="backward pass of the dense GRU Din=D=64, B={B}/GPU, T={T}, with the Jacobian's diagonal: "
         "dL/dP, dL/dh0, dL/dW_hh [3D, D], dL/db_hh from the converged states and dL/dh",
    cpu_sample=dict(B=16, T=32768), ref_sample=dict(B=4, T=16384))
ADJ_METRIC = "backward states/sec (B*T*D per s, gradients through the evaluated sequence)"
SCAN_METRIC = "affine-scan elements/sec (B*T*D per s, h_t = a_t h_(t-1) + b_t)"
# the diagonal-recurrence LSTM (state (c, h) per lane; exact Newton over 2x2 lane
# blocks): reads P 16 + the guess (c, h) 8, writes (c, h) 8 = 32 B per lane-step
BENCHES["lstm"] = dict(
    workload="lstm", mode="LSTM", lam=0.0, bound="hbm", per_state=32,
    kernel="lstm_diag_kernel (persistent, all iterations)",
    desc="diagonal-recurrence LSTM Din=D=2048, B={B}/GPU, T={T}, bf16 x and W_ih, fp32 state (c, h), "
         "exact Newton (2x2 lane Jacobians) tol 1e-4",
    cpu_sample=dict(B=1, T=8192), ref_sample=dict(B=1, T=1024), roll_sample=dict(T=256))
# fp32 FMA peak for the ALU-bound row: 148 SMs x 128 fp32 lanes x 2 flop x
# 1965 MHz (the part's maximum SM clock), in TFLOP/s.
ALU_PEAK_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12
# ncu DRAM traffic of the solver kernel per state and iteration (read + write
# bytes of one launch captured at T = 16384, / (iterations x states)) and the
# hash of the kernel source it was measured on.  Traffic grows with states x
# iterations, so the full launch's is scaled from it; reported only while the
# source is unchanged.
NCU_TRAFFIC = {"bytes_per_state_iter": (4.100330e9 + 0.991507e9) / (14 * 16 * 16384 * 64),
               "source_sha1": "8db10b5d6c9f"}


def log(*a):
    print(*a, file=sys.stderr, flush=True)


def max_over_ranks(ms: float, device) -> float:
    """The slowest rank's time: device timings are combined with a MAX
    all-reduce (a no-op without a process group)."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_value(states_per_rank: int, steps: int, world: int, max_ms: float) -> float:
    """Whole-job throughput: the states every rank solved over the slowest
    rank's time (weak scaling: each rank owns its own batch)."""
    return world * steps * states_per_rank / (max_ms / 1e3)


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def tf32_peak():
    """Dense TF32 TFLOP/s: the measured bf16 burst peak x 1/2 (nominal ratio)."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        return float(json.load(open(p))["bf16_tflops"]) / 2
    return 1590.0 / 2


def kernel_sha():
    """Hash of the headline solver kernel's sources (the .cu and the headers it uses)."""
    csrc = os.path.join(ROOT, "newton_solve_nonlinear_b200", "csrc")
    h = hashlib.sha1()
    for f in ("newton_dense_tc2.cu", "common.cuh", "lookback.cuh", "solver.cuh", "tc_utils.cuh"):
        h.update(open(os.path.join(csrc, f), "rb").read())
    return h.hexdigest()[:12]


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


def cpu_baseline_oracle(spec: dict, sample: dict, jac_every: int = 1):
    """Time the fp64 oracle (as it stands) on a bounded sample of the workload:
    the same generator and distributions, fewer sequences and steps."""
    import oracle
    from oracle.cells import GRU
    from newton_solve_nonlinear_b200.inputs import make_workload
    try:
        from threadpoolctl import threadpool_info
        cores = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:  # pragma: no cover
        cores = 1
    mode = spec["mode"]
    if mode == "LSTM":
        from oracle.lstm import LSTM, lstm_newton_solve
        from newton_solve_nonlinear_b200.inputs import make_lstm_workload
        lw = make_lstm_workload(**sample)
        lc = LSTM(w_ih=lw.w_ih.double().numpy(), b_ih=lw.b_ih.double().numpy(), u=lw.u.double().numpy(),
                  b_hh=lw.b_hh.double().numpy())
        t0 = time.perf_counter()
        r = lstm_newton_solve(lc, lw.x.double().numpy(), lw.c0.double().numpy(), lw.h0.double().numpy(), lw.tol)
        secs = time.perf_counter() - t0
        return {"value": lw.states / secs, "unit": UNIT, "cores": cores, "kind": "oracle",
                "sample": f"fp64 numpy oracle, exact Newton to tol {lw.tol:g} on B={lw.B}, T={lw.T}, D={lw.d} "
                          f"({r['iters']} iterations, {secs:.1f} s); same distributions"}
    w = make_workload(spec["workload"], **sample)
    c = GRU.from_workload(w)
    x, h0 = w.x.double().numpy(), w.h0.double().numpy()
    if mode == "ADJOINT":
        import numpy as np
        from oracle.adjoint import adjoint
        from oracle.cells import rollout
        h = rollout(c, x, h0)
        g = np.random.default_rng(0).normal(size=h.shape)
        t0 = time.perf_counter()
        adjoint(c, x, h0, h, g, jacobian="diag")
        secs = time.perf_counter() - t0
        states = w.B * w.T * w.d
        return {"value": states / secs, "unit": UNIT, "cores": cores, "kind": "oracle",
                "sample": f"fp64 numpy oracle backward pass (reverse recurrence, dP, parameter and input "
                          f"gradients) on B={w.B}, T={w.T}, D={w.d} ({secs:.1f} s); same distributions"}
    t0 = time.perf_counter()
    if mode in ("ELK", "QUASI_ELK"):
        r = oracle.elk_solve(c, x, h0, mode, spec["lam"], w.tol)
    else:
        r = oracle.newton_solve(c, x, h0, mode, w.tol, jac_every=jac_every)
    secs = time.perf_counter() - t0
    states = w.B * w.T * w.d
    return {"value": states / secs, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"fp64 numpy oracle, {mode} to tol {w.tol:g} on B={w.B}, T={w.T}, "
                      f"D={w.d} ({r['iters']} iterations, {secs:.1f} s"
                      + (f", Jacobian every {jac_every} iterations" if jac_every != 1 else "")
                      + "); same distributions"}


def cpu_rollout_baseline(spec: dict) -> dict | None:
    """The plain sequential evaluation on the host (oracle/rollout.c: fp64 and
    fp32, one thread and OpenMP over the batch's sequences), on the sample
    `roll_sample` of the workload (the whole workload where it fits in seconds).
    Reported beside the GPU solve: what a CPU does without the parallel method."""
    import numpy as np
    from oracle import crollout
    from oracle.cells import GRU
    from newton_solve_nonlinear_b200.inputs import make_workload
    sample = spec.get("roll_sample")
    if sample is None:
        return None
    if spec["mode"] == "LSTM":  # the diagonal LSTM: (c, h) per lane
        from oracle.lstm import LSTM
        from newton_solve_nonlinear_b200.inputs import make_lstm_workload
        w = make_lstm_workload(**sample)
        c = LSTM(w_ih=w.w_ih.double().numpy(), b_ih=w.b_ih.double().numpy(), u=w.u.double().numpy(),
                 b_hh=w.b_hh.double().numpy())
        x, c0, h0 = w.x.double().numpy(), w.c0.double().numpy(), w.h0.double().numpy()
        roll = lambda xx, cc, hh, dt, thr: crollout.lstm_rollout(c, xx, cc, hh, dt, threads=thr)
    else:
        w = make_workload(spec["workload"], **sample)
        c = GRU.from_workload(w)
        x, h0 = w.x.double().numpy(), w.h0.double().numpy()
        c0 = h0
        roll = lambda xx, cc, hh, dt, thr: crollout.rollout(c, xx, hh, dt, threads=thr)
    states = w.B * w.T * w.d
    nthr = min(crollout.max_threads(), w.B)
    out = {"unit": UNIT, "cores": os.cpu_count(), "threads": nthr, "cpu": cpu_model(),
           "sample": f"B={w.B}, T={w.T}, D={w.d}, Din={w.din} on {nthr} threads, the first sequence alone "
                     f"on one thread (sequential rollout, gcc -O3 -fopenmp)"}
    for name, dt in (("fp64", np.float64), ("fp32", np.float32)):
        t0 = time.perf_counter()
        roll(x, c0, h0, dt, nthr)
        out[name] = states / (time.perf_counter() - t0)
        t0 = time.perf_counter()
        roll(x[:1], c0[:1], h0[:1], dt, 1)
        out[name + "_1thread"] = states / w.B / (time.perf_counter() - t0)
    return out


def cpu_model() -> str:
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    if args.workload == "scan":
        return run_reference_scan(args)
    spec = BENCHES[args.workload]
    steps = []
    base = None
    for i in range(args.warmup + args.steps):
        cb = cpu_baseline_oracle(spec, spec["ref_sample"], args.jac_every)
        if i >= args.warmup:
            steps.append(cb["value"])
        base = cb
    v = statistics.median(steps)
    from newton_solve_nonlinear_b200.inputs import WORKLOADS
    metric = ADJ_METRIC if spec["mode"] == "ADJOINT" else METRIC
    full = WORKLOADS[spec["workload"]] if spec["workload"] in WORKLOADS else dict(B=8, T=4096)
    T = args.T or full["T"]
    line = {"impl": "reference", "metric": metric, "value": v, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": None,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": {"workload": spec["desc"].format(B=full["B"], T=T), "sample": base["sample"]},
            "cpu_baseline": {"value": v, "unit": UNIT, "cores": base["cores"], "kind": "oracle",
                             "sample": base["sample"]},
            "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def run_reference_scan(args):
    """The oracle's serial fp64 scan on a bounded sample of the scan workload."""
    import numpy as np
    from oracle.scan import affine_scan
    from newton_solve_nonlinear_b200.inputs import make_scan_input
    B, T, D = 2, (args.T or 65536), 64
    s = make_scan_input(B, T, D, seed=0)
    A, b, h0 = s.A.double().numpy(), s.b.double().numpy(), s.h0.double().numpy()
    vals = []
    for i in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        affine_scan(A, b, h0)
        if i >= args.warmup:
            vals.append(B * T * D / (time.perf_counter() - t0))
    v = statistics.median(vals)
    sample = f"fp64 numpy serial recurrence on B={B}, T={T}, D={D} (same distributions, one thread over t)"
    line = {"impl": "reference", "metric": SCAN_METRIC, "value": v, "unit": "elements/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": None, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": f"affine scan alone h_t = a_t h_(t-1) + b_t, [B=16, T={T}, D=64], "
                                   f"a ~ U(0.5, 1), b ~ N(0, 1), h0 = 0", "sample": sample},
            "cpu_baseline": {"value": v, "unit": "elements/s", "cores": 1, "kind": "oracle", "sample": sample},
            "e2e": {"value": v, "unit": "elements/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def run_adjoint(args):
    """The backward pass through the converged solve (diagonal or dense cell), timed alone."""
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

    spec = BENCHES[args.workload]
    over = {"T": args.T} if args.T else {}
    w = make_workload(spec["workload"], seed=rank, **over)
    B, T, D = w.B, w.T, w.d
    states = B * T * D
    g = lambda t: t.to(dev).contiguous()
    # the forward solve gives the states; the upstream gradient is synthetic
    sol = binding.solve_workload(w, "QUASI", device=dev)
    P = binding.input_projection(g(w.x), g(w.w_ih), g(w.b_ih), d=D, kind=w.kind)
    h, h0, u, bh = sol.h, g(w.h0), g(w.w_hh), g(w.b_hh)
    dh = torch.randn(B, T, D, generator=torch.Generator().manual_seed(rank)).to(dev)
    ws = binding.alloc_workspace(binding.adjoint_workspace_size(D, B, T, kind=w.kind), dev)
    out = dict(dP=torch.empty_like(P), dh0=torch.empty_like(h0), dw_hh=torch.empty_like(u),
               db_hh=torch.empty_like(bh))
    stream = torch.cuda.current_stream(dev)
    step = lambda: binding.adjoint(u, bh, P, h0, h, dh, workspace=ws, out=out)
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    with Clocks(local) as clk:
        barrier()
        torch.cuda.synchronize()
        for e0, e1 in evs:
            e0.record(stream)
            step()
            e1.record(stream)
        torch.cuda.synchronize()
        barrier()
    ms = [e0.elapsed_time(e1) for e0, e1 in evs]
    max_ms = max_over_ranks(sum(ms), dev)
    value = job_value(states, args.steps, world, max_ms)
    st = binding.lib().pararnn_adjoint_status(ws.data_ptr(), stream.cuda_stream)
    # end to end through the public host-buffer call: P, h0, h and dL/dh from
    # page-locked host memory; dL/dP, dL/dh0 and the parameter gradients back;
    # the library overlaps the copies with the parts' passes
    hP, hh, hdh, hh0 = (t.cpu().pin_memory() for t in (P, h, dh, h0))
    parts = max(1, min(E2E_PARTS, B))
    hout = dict(dP=torch.empty(P.shape).pin_memory(), dh0=torch.empty(h0.shape).pin_memory(),
                dw_hh=torch.empty(u.shape).pin_memory(), db_hh=torch.empty(bh.shape).pin_memory())
    ws_host = binding.alloc_workspace(int(binding.lib().pararnn_adjoint_host_workspace_size(
        binding.make_cell(w.kind if w.kind == "dense" else "diag", 1, D, torch.float32), B, T, parts)), dev)
    e2e_step = lambda: binding.adjoint_host(u, bh, hP, hh0, hh, hdh, parts=parts, out=hout, workspace=ws_host,
                                            stream=stream)
    e2e_step()
    e2e_steps = max(1, min(args.steps, 3))
    barrier()
    torch.cuda.synchronize()
    ea, eb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ea.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    eb.record(stream)
    torch.cuda.synchronize()
    e2e_value = job_value(states, e2e_steps, world, max_over_ranks(ea.elapsed_time(eb), dev))
    cpu = cpu_baseline_oracle(spec, spec["cpu_sample"]) if rank == 0 and world == 1 else None
    hbm_peak, peak_kind = peaks()
    avg_s = statistics.mean(ms) / 1e3
    achieved = states * spec["per_state"] / avg_s / 1e9
    line = {
        "metric": ADJ_METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": max_ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": spec["desc"].format(B=B, T=T), "name": args.workload, "B": B, "T": T, "D": D,
                   "cell": w.kind, "status": binding.STATUS.get(st),
                   "l2": f"inputs larger than L2 (126 MB): P {P.numel() * 4 / 1e6:.0f} MB, "
                         f"h and dL/dh {h.numel() * 8 / 1e6:.0f} MB, dL/dP {P.numel() * 4 / 1e6:.0f} MB",
                   "parallelism": f"replicas over sequences x{world}"},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
                     "frac": achieved / hbm_peak, "traffic": None, "kernel": spec["kernel"],
                     "algorithmic": f"{spec['per_state']} B/state x {states} states",
                     "peak_kind": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs)"},
        "e2e": {"value": e2e_value, "unit": UNIT,
                "h2d_bytes_per_step": (P.numel() + h.numel() + dh.numel() + h0.numel()) * 4,
                "d2h_bytes_per_step": (P.numel() + h0.numel() + u.numel() + bh.numel()) * 4, "parts": parts},
        "gpu_launches": (4 if w.kind == "dense" else 1) * args.steps,
        "clocks": clk.summary(),
    }
    if cpu is not None:
        line["cpu_baseline"] = cpu
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


def run_lstm(args):
    """The diagonal-recurrence LSTM solve (projection + every Newton iteration)."""
    import torch
    import torch.distributed as dist
    from newton_solve_nonlinear_b200 import binding
    from newton_solve_nonlinear_b200.inputs import make_lstm_workload

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

    spec = BENCHES[args.workload]
    over = {"T": args.T} if args.T else {}
    w = make_lstm_workload(seed=rank, **over)
    B, T, D = w.B, w.T, w.d
    states = B * T * D
    g = lambda t: t.to(dev).contiguous()
    w_ih, b_ih, u, b_hh, x, c0, h0 = map(g, (w.w_ih, w.b_ih, w.u, w.b_hh, w.x, w.c0, w.h0))
    ws = binding.alloc_workspace(binding.lstm_workspace_size(w.din, D, B, T, w.x_dtype), dev)
    out = (torch.empty(B, T, D, device=dev), torch.empty(B, T, D, device=dev))
    stream = torch.cuda.current_stream(dev)
    step = lambda: binding.lstm_solve(w_ih, b_ih, u, b_hh, x, c0, h0, tol=w.tol, out=out, workspace=ws)
    res = None
    for _ in range(args.warmup):
        res = step()[2]
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    with Clocks(local) as clk:
        barrier()
        torch.cuda.synchronize()
        for e0, e1 in evs:
            e0.record(stream)
            res = step()[2]
            e1.record(stream)
        torch.cuda.synchronize()
        barrier()
    ms = [e0.elapsed_time(e1) for e0, e1 in evs]
    max_ms = max_over_ranks(sum(ms), dev)
    value = job_value(states, args.steps, world, max_ms)
    # end to end through the public host-buffer call: x, c0, h0 from page-locked
    # host memory, (c, h) back; the library streams the sequence through the
    # device in time parts and overlaps the copies with the parts' solves
    hx, hc0, hh0 = w.x.pin_memory(), w.c0.float().pin_memory(), w.h0.float().pin_memory()
    hc, hh = torch.empty(B, T, D).pin_memory(), torch.empty(B, T, D).pin_memory()
    parts = max(1, min(E2E_PARTS, (T + 127) // 128))
    ws_host = binding.alloc_workspace(binding.lstm_host_streamed_workspace_size(w.din, D, B, T, parts, w.x.dtype),
                                      dev)
    # the weights stay resident on the device, as in the device-timed steps
    e2e_step = lambda: binding.lstm_solve_host_streamed(w_ih, b_ih, u, b_hh, hx, hc0, hh0,
                                                        tol=w.tol, parts=parts, out=(hc, hh), workspace=ws_host,
                                                        stream=stream)
    e2e_step()
    e2e_steps = max(1, min(args.steps, 3))
    barrier()
    torch.cuda.synchronize()
    ea, eb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ea.record(stream)
    e2e_iters = []
    for _ in range(e2e_steps):
        _, _, r_e2e = e2e_step()
        if r_e2e.status != "OK":
            raise SystemExit(f"lstm: end-to-end solve status {r_e2e.status}")
        e2e_iters.append(r_e2e.iters)
    eb.record(stream)
    torch.cuda.synchronize()
    e2e_value = job_value(states, e2e_steps, world, max_over_ranks(ea.elapsed_time(eb), dev))
    cpu = cpu_baseline_oracle(spec, spec["cpu_sample"]) if rank == 0 and world == 1 else None
    roll = cpu_rollout_baseline(spec) if rank == 0 and world == 1 else None
    hbm_peak, peak_kind = peaks()
    avg_s = statistics.mean(ms) / 1e3
    achieved = res.iters * states * spec["per_state"] / avg_s / 1e9
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": max_ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": spec["desc"].format(B=B, T=T), "name": args.workload, "B": B, "T": T, "D": D,
                   "din": w.din, "cell": "lstm_diag", "mode": "DEER (exact, 2x2 lane blocks)", "tol": w.tol,
                   "iters": res.iters, "status": res.status,
                   "l2": f"inputs larger than L2 (126 MB): x {w.x.numel() * 2 / 1e6:.0f} MB, "
                         f"P {states * 16 / 1e6:.0f} MB, (c, h) {states * 8 / 1e6:.0f} MB",
                   "parallelism": f"replicas over sequences x{world}"},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
                     "frac": achieved / hbm_peak, "traffic": None, "kernel": spec["kernel"],
                     "algorithmic": f"{spec['per_state']} B/lane-step/iteration x {res.iters} iterations x "
                                    f"{states} lane-steps (the solve's time includes the projection)",
                     "peak_kind": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs)"},
        "e2e": {"value": e2e_value, "unit": UNIT,
                "h2d_bytes_per_step": w.x.numel() * w.x.element_size() + 2 * B * D * 4,
                "d2h_bytes_per_step": 2 * states * 4 + 16 * parts, "parts": parts, "split": "time",
                "iters_summed_over_parts": e2e_iters, "copy_gbs": copy_bandwidth(dev)},
        "gpu_launches": 2 * args.steps,
        "clocks": clk.summary(),
    }
    if cpu is not None:
        line["cpu_baseline"] = cpu
    if roll is not None:
        line["cpu_rollout"] = roll
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


def _dist_setup():
    """(world, rank, local rank, device, barrier) of this process; NCCL only when
    launched as several ranks."""
    import torch
    import torch.distributed as dist
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1 and not dist.is_initialized():
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=300), device_id=dev)

    def barrier():
        if world > 1:
            dist.barrier()
    return world, rank, local, dev, barrier


def copy_bandwidth(dev, nbytes: int = 256 << 20) -> dict:
    """Pinned host <-> device copy bandwidth of this machine, GB/s (the ceiling of
    every end-to-end number that moves its inputs and results over the host
    link): one copy each way, then both at once, timed with CUDA events."""
    import torch
    n = nbytes // 4
    hsrc, hdst = torch.empty(n).pin_memory(), torch.empty(n).pin_memory()
    d1, d2 = torch.empty(n, device=dev), torch.empty(n, device=dev)
    s1, s2 = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    out = {}
    for name in ("h2d", "d2h", "both"):
        for rep in range(2):  # the first pass warms the link
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            if name in ("h2d", "both"):
                with torch.cuda.stream(s1):
                    d1.copy_(hsrc, non_blocking=True)
            if name in ("d2h", "both"):
                with torch.cuda.stream(s2):
                    hdst.copy_(d2, non_blocking=True)
            cur = torch.cuda.current_stream(dev)
            cur.wait_stream(s1)
            cur.wait_stream(s2)
            e1.record()
            torch.cuda.synchronize()
        moved = nbytes * (2 if name == "both" else 1)
        out[name] = moved / (e0.elapsed_time(e1) / 1e3) / 1e9
    return out


def bench_solve(args, name: str, *, full: bool = True, steps: int | None = None):
    """Time one solver family (projection + the whole Newton loop per step) and
    return its JSON line.  ``full`` adds the end-to-end (host buffers) number,
    the CPU baselines and the clock record; the per-family entries of the
    default run's ``workloads`` key leave those out."""
    import torch
    from newton_solve_nonlinear_b200 import binding
    from newton_solve_nonlinear_b200.inputs import make_workload

    world, rank, local, dev, barrier = _dist_setup()
    steps = args.steps if steps is None else steps
    spec = BENCHES[name]
    mode, lam = spec["mode"], spec["lam"]
    over = {"T": args.T} if (args.T and name == args.workload) else {}
    w = make_workload(spec["workload"], seed=rank, **over)
    B, T, D, din, kind = w.B, w.T, w.d, w.din, w.kind
    states = B * T * D
    g = lambda t: t.to(dev).contiguous()
    w_ih, b_ih, w_hh, b_hh, x, h0 = map(g, (w.w_ih, w.b_ih, w.w_hh, w.b_hh, w.x, w.h0))
    ws = binding.alloc_workspace(
        binding.workspace_size(kind, din, D, B, T, mode, w.x_dtype), dev)
    P = torch.empty(B, T, 3 * D, dtype=torch.float32, device=dev)
    out = torch.empty(B, T, D, dtype=torch.float32, device=dev)
    # one report per timed step, read after the timed region
    infos = torch.zeros(max(steps, 1) + 1, 4, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream(dev)

    k = args.jac_every if name == args.workload else 1
    if k != 1:
        if mode != "DEER":
            raise SystemExit("--jac-every needs a DEER workload")
        ws = binding.alloc_workspace(binding.lib().pararnn_reuse_workspace_size(
            binding.make_cell(kind, din, D, w.x_dtype), B, T), dev)

    def step(info, ev_mid=None):
        if k != 1:  # one synchronous call: projection and the solve with the Jacobian reused
            if ev_mid is not None:
                ev_mid.record(stream)
            r = binding.newton_solve(w_ih, b_ih, w_hh, b_hh, x, h0, kind=kind, mode=mode, tol=w.tol,
                                     jac_every=k, out=out, workspace=ws, stream=stream)
            info[0], info[1] = r.iters, {v: c for c, v in binding.STATUS.items()}[r.status]
            return
        binding.input_projection(x, w_ih, b_ih, d=D, kind=kind, out=P)
        if ev_mid is not None:
            ev_mid.record(stream)
        binding.newton_iterate(P, w_hh, b_hh, h0, kind=kind, din=din, mode=mode, lam=lam,
                               tol=w.tol, info_dev=info, out=out, workspace=ws, dtype=w.x_dtype)

    for _ in range(args.warmup):
        step(infos[-1])
    torch.cuda.synchronize()

    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
            torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    clk = Clocks(local) if full else None
    if clk is not None:
        clk.__enter__()
    barrier()
    torch.cuda.synchronize()
    for i, (e0, e1, e2) in enumerate(evs):
        e0.record(stream)
        step(infos[i], e1)
        e2.record(stream)
    torch.cuda.synchronize()
    barrier()
    if clk is not None:
        clk.__exit__(None, None, None)
    total_ms = sum(e0.elapsed_time(e2) for e0, _, e2 in evs)
    solver_ms = [e1.elapsed_time(e2) for _, e1, e2 in evs]
    proj_ms = [e0.elapsed_time(e1) for e0, e1, _ in evs]
    max_ms = max_over_ranks(total_ms, dev)
    value = job_value(states, steps, world, max_ms)
    # the timed solves' own reports: every one must have converged, and the
    # iteration count the roofline uses is theirs
    rep = infos[:steps].cpu()
    step_iters = [int(v) for v in rep[:, 0]]
    step_status = [binding.STATUS.get(int(v), str(int(v))) for v in rep[:, 1]]
    if any(st != "OK" for st in step_status):
        raise SystemExit(f"{name}: a timed solve did not converge: iterations {step_iters}, "
                         f"statuses {step_status}")
    iters = max(step_iters)

    e2e = None
    parts = max(1, min(spec.get("e2e_parts", E2E_PARTS), (T + 127) // 128)) if k == 1 else 1
    if full:
        # end to end through the public host-buffer call: page-locked x and h0 in,
        # h out; the library streams the sequence through the device in time
        # parts (the whole batch in each) and overlaps the copies with the solves
        x_host = w.x.contiguous().pin_memory()
        h0_host = w.h0.float().contiguous().pin_memory()
        h_host = torch.empty(B, T, D, dtype=torch.float32).pin_memory()
        ws_host = binding.alloc_workspace(
            binding.host_streamed_workspace_size(kind, din, D, B, T, mode, parts, w.x_dtype), dev)
        e2e_steps = max(1, min(steps, 5))

        def e2e_step():
            if k != 1:  # copies around the reuse solve (no host-buffer variant of it)
                x.copy_(x_host, non_blocking=True)
                h0.copy_(h0_host, non_blocking=True)
                binding.newton_solve(w_ih, b_ih, w_hh, b_hh, x, h0, kind=kind, mode=mode, tol=w.tol,
                                     jac_every=k, out=out, workspace=ws, stream=stream)
                h_host.copy_(out, non_blocking=True)
                return None
            return binding.newton_solve_host_streamed(w_ih, b_ih, w_hh, b_hh, x_host, h0_host, kind=kind,
                                                      mode=mode, lam=lam, tol=w.tol, parts=parts, out=h_host,
                                                      workspace=ws_host, stream=stream)

        e2e_step()
        barrier()
        torch.cuda.synchronize()
        ea, eb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ea.record(stream)
        e2e_iters = []
        for _ in range(e2e_steps):
            r = e2e_step()
            if r is not None and r.status != "OK":
                raise SystemExit(f"{name}: end-to-end solve status {r.status}")
            if r is not None:
                e2e_iters.append(r.iters)
        eb.record(stream)
        torch.cuda.synchronize()
        e2e = {"value": job_value(states, e2e_steps, world, max_over_ranks(ea.elapsed_time(eb), dev)),
               "unit": UNIT,
               "h2d_bytes_per_step": x_host.numel() * x_host.element_size() + h0_host.numel() * 4,
               "d2h_bytes_per_step": h_host.numel() * 4 + 16 * parts, "parts": parts,
               "split": "time" if k == 1 else "none",
               "iters_summed_over_parts": e2e_iters,
               "copy_gbs": copy_bandwidth(dev)}
        del ws_host

    cpu = roll = None
    if full and rank == 0 and world == 1:
        cpu = cpu_baseline_oracle(spec, spec["cpu_sample"], k)
        roll = cpu_rollout_baseline(spec)

    hbm_peak, peak_kind = peaks()
    solver_avg_s = statistics.mean(solver_ms) / 1e3
    traffic = None
    if spec["bound"] == "hbm":
        per_state = spec["per_state"]
        achieved = iters * states * per_state / solver_avg_s / 1e9
        peak, unit = hbm_peak, "GB/s"
        algo = f"{per_state} B/state/iteration x {iters} iterations x {states} states"
        pk = f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs)"
        if name == "untrained" and NCU_TRAFFIC["source_sha1"] == kernel_sha():
            traffic = NCU_TRAFFIC["bytes_per_state_iter"] * iters * states
    elif spec["bound"] == "tensor":
        per_state = 2 * D * D
        fresh = (iters + k - 1) // k  # iterations that form new Jacobian products
        achieved = fresh * states * per_state / solver_avg_s / 1e12
        peak, unit = tf32_peak(), "TFLOP/s"
        algo = f"2 D^3 flop/step = {per_state} flop/state/iteration x {fresh} x {states} states"
        if k != 1:
            algo += f" (Jacobian every {k} iterations: {fresh} of {iters} form products; time includes the projection)"
        pk = "TF32 dense = MEASURED_PEAKS.json bf16_tflops x 1/2 (nominal TF32:bf16 ratio)"
    else:
        per_state = 14 * D * D
        achieved = iters * states * per_state / solver_avg_s / 1e12
        peak, unit = ALU_PEAK_TFLOPS, "TFLOP/s"
        algo = f"14 D^3 flop/step = {per_state} flop/state/iteration x {iters} x {states} states"
        pk = "fp32 FMA: 148 SMs x 128 lanes x 2 flop x 1965 MHz"
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": steps,
        "warmup": args.warmup, "ms_per_step": max_ms / steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": spec["desc"].format(B=B, T=T), "name": name,
                   "B": B, "T": T, "D": D, "din": din, "cell": kind, "mode": mode,
                   "lambda": lam if mode in ("ELK", "QUASI_ELK") else None,
                   "jac_every": k,
                   "tol": w.tol, "iters": iters, "status": "OK", "iters_per_step": step_iters,
                   "l2": (f"inputs larger than L2 (126 MB) summed per solve: "
                          f"x {x.numel() * x.element_size() / 1e6:.0f} MB, "
                          f"P {P.numel() * 4 / 1e6:.0f} MB, h {out.numel() * 4 / 1e6:.0f} MB"),
                   "parallelism": f"replicas over sequences x{world}",
                   "projection_ms": statistics.mean(proj_ms),
                   "solver_ms": statistics.mean(solver_ms)},
        "roofline": {"bound": spec["bound"], "achieved": achieved, "peak": peak, "unit": unit,
                     "frac": achieved / peak, "traffic": traffic, "kernel": spec["kernel"],
                     "algorithmic": algo, "peak_kind": pk},
        "gpu_launches": 2 * steps,
    }
    if e2e is not None:
        line["e2e"] = e2e
    if clk is not None:
        line["clocks"] = clk.summary()
    if cpu is not None:
        line["cpu_baseline"] = cpu
    if roll is not None:
        line["cpu_rollout"] = roll
    del ws, P, out
    torch.cuda.empty_cache()
    return line


def bench_scan(args, *, steps: int | None = None, full: bool = False):
    """The affine scan alone (pararnn_affine_scan, diagonal): [16, 65536, 64],
    a ~ U(0.5, 1), b ~ N(0, 1), h0 = 0; 12 B per element (a, b in, h out)."""
    import torch
    from newton_solve_nonlinear_b200 import binding
    from newton_solve_nonlinear_b200.inputs import make_scan_input

    world, rank, local, dev, barrier = _dist_setup()
    steps = args.steps if steps is None else steps
    B, T, D = 16, (args.T if (args.T and args.workload == "scan") else 65536), 64
    s = make_scan_input(B, T, D, seed=rank)
    A, b, h0 = s.A.to(dev), s.b.to(dev), s.h0.to(dev)
    ws = binding.alloc_workspace(int(binding.lib().pararnn_affine_scan_workspace_size(B, T, D, 0)), dev)
    h = torch.empty_like(b)
    stream = torch.cuda.current_stream(dev)
    run = lambda: binding.affine_scan(A, b, h0, out=h, workspace=ws, stream=stream)
    for _ in range(args.warmup):
        run()
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    clk = Clocks(local) if full else None
    if clk is not None:
        clk.__enter__()
    barrier()
    torch.cuda.synchronize()
    for e0, e1 in evs:
        e0.record(stream)
        run()
        e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    if clk is not None:
        clk.__exit__(None, None, None)
    st = binding.lib().pararnn_affine_scan_status(ws.data_ptr(), stream.cuda_stream)
    if st != 0:
        raise SystemExit(f"scan: status {binding.STATUS.get(st, st)}")
    ms = [e0.elapsed_time(e1) for e0, e1 in evs]
    max_ms = max_over_ranks(sum(ms), dev)
    n = B * T * D
    value = job_value(n, steps, world, max_ms)
    hbm_peak, peak_kind = peaks()
    achieved = n * 12 / (statistics.mean(ms) / 1e3) / 1e9
    line = {
        "metric": SCAN_METRIC, "value": value, "unit": "elements/s", "n_gpus": world, "steps": steps,
        "warmup": args.warmup, "ms_per_step": max_ms / steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": f"affine scan alone h_t = a_t h_(t-1) + b_t, [B={B}, T={T}, D={D}], "
                               f"a ~ U(0.5, 1), b ~ N(0, 1), h0 = 0", "name": "scan", "B": B, "T": T, "D": D,
                   "l2": f"inputs larger than L2 (126 MB): a, b {2 * n * 4 / 1e6:.0f} MB, h {n * 4 / 1e6:.0f} MB",
                   "parallelism": f"replicas over sequences x{world}"},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
                     "frac": achieved / hbm_peak, "traffic": None, "kernel": "scan_diag_kernel (one pass)",
                     "algorithmic": f"12 B/element x {n} elements",
                     "peak_kind": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs)"},
        "gpu_launches": steps,
    }
    if full:
        # end to end through the public host-buffer call: a, b, h0 from page-locked
        # host memory, h back; the library streams the sequence through the device
        # in time parts and overlaps the copies with the parts' scans
        hA, hb, hh0 = s.A.pin_memory(), s.b.pin_memory(), s.h0.pin_memory()
        hh = torch.empty(B, T, D).pin_memory()
        parts = max(1, min(E2E_PARTS, (T + 127) // 128))
        ws_host = binding.alloc_workspace(
            int(binding.lib().pararnn_affine_scan_host_workspace_size(B, T, D, 0, parts)), dev)
        e2e_run = lambda: binding.affine_scan_host(hA, hb, hh0, parts=parts, out=hh, workspace=ws_host,
                                                   stream=stream)
        e2e_run()
        e2e_steps = max(1, min(steps, 5))
        ea, eb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        ea.record(stream)
        for _ in range(e2e_steps):
            e2e_run()
        eb.record(stream)
        torch.cuda.synchronize()
        line["e2e"] = {"value": job_value(n, e2e_steps, world, max_over_ranks(ea.elapsed_time(eb), dev)),
                       "unit": "elements/s", "h2d_bytes_per_step": (2 * n + B * D) * 4, "d2h_bytes_per_step": n * 4 + 4 * parts,
                       "parts": parts, "split": "time", "copy_gbs": copy_bandwidth(dev)}
        del ws_host
        line["clocks"] = clk.summary()
    del ws, h, A, b
    torch.cuda.empty_cache()
    return line


# The default run also times these families on the same box, a few steps each,
# and reports them under "workloads" (value, roofline, iterations).
SIDE_FAMILIES = ("diag", "dense_deer", "quasi_elk", "elk")


def _summary(line: dict) -> dict:
    rf = line["roofline"]
    c = line["config"]
    return {"value": line["value"], "unit": line["unit"], "ms_per_step": line["ms_per_step"],
            "steps": line["steps"], "iters": c.get("iters"), "status": c.get("status", "OK"),
            "workload": c["workload"],
            "roofline": {"bound": rf["bound"], "achieved": rf["achieved"], "peak": rf["peak"], "unit": rf["unit"],
                         "frac": rf["frac"], "kernel": rf["kernel"], "algorithmic": rf["algorithmic"]}}


def run_ours(args):
    import torch.distributed as dist
    world, rank = int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0"))
    if args.workload == "scan":
        line = bench_scan(args, full=True)
    else:
        line = bench_solve(args, args.workload)
    if args.workload == "untrained" and not args.no_side and args.jac_every == 1 and not args.T:
        side = {}
        for name in SIDE_FAMILIES:
            side[name] = _summary(bench_solve(args, name, full=False, steps=min(args.steps, 5)))
        side["scan"] = _summary(bench_scan(args, steps=min(args.steps, 10)))
        line["workloads"] = side
        line["gpu_launches"] += sum(2 * v["steps"] for k, v in side.items() if k != "scan") + side["scan"]["steps"]
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1 and dist.is_initialized():
        dist.destroy_process_group()
    return 0


def plan_launch(gpus: int, env: dict, argv: list[str]):
    """How bench.py runs for --gpus N: ("run", None) in this process,
    ("exec", cmd) re-launched under torchrun with one rank per GPU, or
    ("error", why) when an outer launcher started a different rank count."""
    world = env.get("WORLD_SIZE")
    if world is None:
        if gpus <= 1:
            return "run", None
        port = env.get("MASTER_PORT") or "29517"
        cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={gpus}",
               "--master-addr=127.0.0.1", f"--master-port={port}", os.path.abspath(__file__), *argv]
        return "exec", cmd
    if int(world) != gpus:
        return "error", f"--gpus {gpus} but WORLD_SIZE={world}"
    return "run", None


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="untrained", choices=sorted(BENCHES) + ["scan"],
                    help="which solve to time (default: the untrained dense GRU headline)")
    ap.add_argument("--T", type=int, default=0, help="override the sequence length")
    ap.add_argument("--jac-every", type=int, default=1,
                    help="DEER workloads: recompute the Jacobian only every k iterations")
    ap.add_argument("--no-side", action="store_true",
                    help="default workload: skip the other families' entries under \"workloads\"")
    args = ap.parse_args()
    how, what = plan_launch(args.gpus, dict(os.environ), sys.argv[1:])
    if how == "error":
        log(what)
        return 2
    if how == "exec":
        log("launching: " + " ".join(what))
        return subprocess.call(what)
    if args.warmup < 3:
        log("warmup raised to 3 (timing rule)")
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args)
    if args.workload != "scan" and BENCHES[args.workload]["mode"] == "ADJOINT":
        return run_adjoint(args)
    if args.workload != "scan" and BENCHES[args.workload]["mode"] == "LSTM":
        return run_lstm(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
