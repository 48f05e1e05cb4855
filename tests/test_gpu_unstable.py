"""The near-unstable GRU at spectral radius 3, where undamped Newton fails.

The damped methods exist because DEER is unstable on such recurrences: its
full-Jacobian steps overshoot and the iteration does not settle, while the
Levenberg-Marquardt step (ELK, quasi-ELK) keeps every iterate bounded and
converges ("Towards Scalable and Stable Parallelization of Nonlinear RNNs",
atlas summary, "Problem" and "Key results").  The workload ``unstable`` (each
recurrent block rescaled to spectral radius 3; B = 2, T = 1000) is the seeded
case where the fp64 oracle shows exactly that (tests/golden/oracle_iters.json,
keys ``unstable/...``): DEER's max |dh| grows past 1e10 by its third iteration
and it has not converged after 40; quasi-DEER and quasi-ELK at lambda 0.01,
0.1 and 1 converge.  (At radius 1.5 the GRU's gates keep the Jacobians
contractive enough that DEER converges in 5 iterations.)

Full-Jacobian ELK with a fixed damping does not converge on it either: its
max |dh| falls from 0.57 and levels off near 7e-3 at lambda 1 (the oracle's
first 100 steps are stored); the GPU must follow that trajectory.

Gates: DEER stops without converging (NOT_CONVERGED at the cap, or DIVERGED
when its fp32 iterates overflow) and its first two iterations -- before the
overshoot -- match the oracle's deltas; every converging mode within +-1 of
the oracle's count, its delta trajectory matching the oracle's at every
iteration, and its converged states within 1e-4 of the oracle's final iterate;
ELK at lambda 1 NOT_CONVERGED after the same 100 steps along the oracle's
trajectory.
"""
import json
import os

import numpy as np
import pytest

import oracle
from oracle.cells import GRU, rollout
from newton_solve_nonlinear_b200 import binding
from newton_solve_nonlinear_b200.inputs import make_workload

pytestmark = pytest.mark.gpu

GOLDEN = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "oracle_iters.json")))


def _close(gpu, ref):
    n = min(len(gpu), len(ref))
    gpu, ref = np.asarray(gpu[:n], np.float64), np.asarray(ref[:n], np.float64)
    return np.abs(gpu - ref) <= 1e-3 * ref + 1e-5


def test_undamped_deer_fails():
    g = GOLDEN["unstable/DEER"]
    assert g["status"] == "NOT_CONVERGED" and g["iters"] == g["max_iters"] == 40
    assert max(g["deltas"][:3]) > 1e10  # the oracle's overshoot
    w = make_workload("unstable")
    r = binding.solve_workload(w, "DEER", max_iters=40, trace=True)
    assert r.status in ("NOT_CONVERGED", "DIVERGED"), r.status
    d = r.trace[:, 0].numpy()
    assert len(d) >= 2 and np.all(_close(d[:2], g["deltas"][:2])), (d[:3], g["deltas"][:3])


@pytest.mark.parametrize("mode,lam", [("QUASI", 0.0), ("QUASI_ELK", 0.01), ("QUASI_ELK", 0.1),
                                      ("QUASI_ELK", 1.0)])
def test_damped_and_quasi_modes_converge(mode, lam):
    key = "unstable/QUASI" if mode == "QUASI" else f"unstable/QUASI_ELK/{lam:g}"
    g = GOLDEN[key]
    assert g["status"] == "OK"
    w = make_workload("unstable")
    r = binding.solve_workload(w, mode, lam=lam, trace=True)
    assert r.status == "OK"
    assert abs(r.iters - g["iters"]) <= 1, (r.iters, g["iters"])
    ok = _close(r.trace[:, 0].numpy(), g["deltas"])
    assert np.all(ok), np.nonzero(~ok)[0][:10]
    c = GRU.from_workload(w)
    x, h0 = w.x.double().numpy(), w.h0.double().numpy()
    if mode == "QUASI":
        ref = oracle.newton_solve(c, x, h0, mode, w.tol)
    else:
        ref = oracle.elk_solve(c, x, h0, mode, lam, w.tol)
    h = r.h.double().cpu().numpy()
    if r.iters == ref["iters"]:
        assert np.max(np.abs(h - ref["h"])) <= 1e-4
    if mode == "QUASI":  # undamped: it stops next to the fixed point, the rollout itself
        assert np.max(np.abs(h - rollout(c, x, h0))) <= 1e-4


def test_full_jacobian_elk_stalls_along_the_oracle_trajectory():
    g = GOLDEN["unstable/ELK/1"]
    assert g["status"] == "NOT_CONVERGED" and g["iters"] == g["max_iters"] == 100
    w = make_workload("unstable")
    r = binding.solve_workload(w, "ELK", lam=1.0, max_iters=100, trace=True)
    assert r.status == "NOT_CONVERGED" and r.iters == 100
    ok = _close(r.trace[:, 0].numpy(), g["deltas"])
    assert np.all(ok), (np.nonzero(~ok)[0][:10], r.trace[:, 0].numpy()[:12], g["deltas"][:12])
