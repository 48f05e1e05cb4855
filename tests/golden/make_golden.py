"""Write tests/golden/oracle_iters.json: the fp64 oracle's iteration counts and
statuses on every workload at full size.

    python tests/golden/make_golden.py [--only NAME]

Calls only ``oracle/`` and the seeded input generators (no CUDA code).  The
pages print no worked example, so these counts are the oracle's, not the
pages'.  The count rule is the oracle's: iters = the first i + 1 with
max |h^(i+1) - h^(i)| <= tol ("ParaRNN" summary, "Newton's Iteration", with
the convergence reading stated in ``oracle/newton.py``).  The GPU must land
within +-1 of these.
"""
from __future__ import annotations

import argparse
import ctypes
import json
import os
import sys
import time

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import oracle  # noqa: E402
from oracle.cells import GRU, rollout  # noqa: E402
from newton_solve_nonlinear_b200.inputs import make_workload  # noqa: E402

OUT = os.path.join(os.path.dirname(os.path.abspath(__file__)), "oracle_iters.json")

# (key, workload name, overrides, mode, lambda)
CASES = [
    ("tiny/DEER", "tiny", {}, "DEER", None),
    ("tiny/QUASI", "tiny", {}, "QUASI", None),
    ("untrained/T1024/QUASI", "untrained", {"T": 1024}, "QUASI", None),
    ("untrained/T4096/QUASI", "untrained", {"T": 4096}, "QUASI", None),
    ("untrained/T16384/QUASI", "untrained", {"T": 16384}, "QUASI", None),
    ("untrained/T65536/QUASI", "untrained", {"T": 65536}, "QUASI", None),
    ("diag/QUASI", "diag", {}, "QUASI", None),
    ("dense_deer/DEER", "dense_deer", {}, "DEER", None),
    ("near_unstable/QUASI_ELK/0.01", "near_unstable", {}, "QUASI_ELK", 0.01),
    ("near_unstable/QUASI_ELK/0.1", "near_unstable", {}, "QUASI_ELK", 0.1),
    ("near_unstable/QUASI_ELK/1", "near_unstable", {}, "QUASI_ELK", 1.0),
    ("near_unstable/QUASI", "near_unstable", {}, "QUASI", None),
    ("near_unstable/DEER", "near_unstable", {}, "DEER", None),
    ("near_unstable/ELK/0.01", "near_unstable", {}, "ELK", 0.01),
    ("near_unstable/ELK/0.1", "near_unstable", {}, "ELK", 0.1),
    ("near_unstable/ELK/1", "near_unstable", {}, "ELK", 1.0),
    # radius 3: undamped DEER fails (capped at 40 iterations), the others converge
    ("unstable/DEER", "unstable", {}, "DEER", None, 40),
    ("unstable/QUASI", "unstable", {}, "QUASI", None),
    ("unstable/QUASI_ELK/0.01", "unstable", {}, "QUASI_ELK", 0.01),
    ("unstable/QUASI_ELK/0.1", "unstable", {}, "QUASI_ELK", 0.1),
    ("unstable/QUASI_ELK/1", "unstable", {}, "QUASI_ELK", 1.0),
    # full-Jacobian ELK stalls on it (max |dh| levels off near 7e-3 at lambda 1):
    # the first 100 damped steps are stored, capped
    ("unstable/ELK/1", "unstable", {}, "ELK", 1.0, 100),
]


def run_case(name, over, mode, lam, max_iters=None):
    w = make_workload(name, **over)
    c = GRU.from_workload(w)
    x = w.x.double().numpy()
    h0 = w.h0.double().numpy()
    t0 = time.time()
    if mode in ("DEER", "QUASI"):
        r = oracle.newton_solve(c, x, h0, mode, w.tol, max_iters=max_iters)
    else:
        r = oracle.elk_solve(c, x, h0, mode, lam, w.tol, max_iters=max_iters)
    secs = time.time() - t0
    ref = rollout(c, x, h0)
    err = float(np.max(np.abs(r["h"] - ref))) if np.all(np.isfinite(r["h"])) else float("nan")
    out = dict(iters=r["iters"], status=r["status"], tol=w.tol, deltas=r["deltas"],
               max_abs_vs_rollout=err, B=w.B, T=w.T, D=w.d, din=w.din, seconds=round(secs, 1))
    if max_iters is not None:
        out["max_iters"] = max_iters
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--only", default=None)
    args = ap.parse_args()
    try:  # keep freed memory in the heap: the oracle allocates large temporaries
        libc = ctypes.CDLL("libc.so.6")
        libc.mallopt(-3, 32 * 1024 * 1024)
        libc.mallopt(-1, 2 ** 31 - 1)
    except OSError:
        pass
    data = json.load(open(OUT)) if os.path.exists(OUT) else {}
    data.setdefault("_about", "fp64 oracle iteration counts at full workload sizes; written by "
                    "tests/golden/make_golden.py (oracle only)")
    for key, name, over, mode, lam, *cap in CASES:
        if args.only and not key.startswith(args.only):
            continue
        res = run_case(name, over, mode, lam, *cap)
        data[key] = res
        print(key, res["iters"], res["status"], res["max_abs_vs_rollout"], res["seconds"], flush=True)
        with open(OUT, "w") as f:
            json.dump(data, f, indent=1, sort_keys=True)


if __name__ == "__main__":
    main()
