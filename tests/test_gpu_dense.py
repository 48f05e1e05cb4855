"""GPU parity of the dense-Jacobian path (DEER, dense affine scan) vs the oracle.

Tolerances:
  * dense affine scan vs serial fp64: ||h - h_ref||_inf / ||h_ref||_inf <= 1e-5;
  * single DEER iterations vs the oracle's iterates: max-abs <= 5e-5 (the
    chunk products J_L ... J_1 are accumulated in fp32 over up to a few
    hundred steps per chunk, so rounding grows by that factor over the cell's
    ~1e-7);
  * converged states vs the fp64 rollout: max-abs <= 1e-4; iteration counts
    within +-1 of the oracle's.
"""
import json
import os

import numpy as np
import pytest
import torch

import oracle
from oracle.cells import GRU, rollout
from newton_solve_nonlinear_b200 import binding
from newton_solve_nonlinear_b200.inputs import make_scan_input, make_workload

pytestmark = pytest.mark.gpu


def _oracle(w):
    return GRU.from_workload(w), w.x.double().numpy(), w.h0.double().numpy()


def _make(name, over):
    kw = {k: over[k] for k in ("bias_std", "h0_std") if k in over}
    return make_workload(name, **{k: v for k, v in over.items() if k not in kw}, **kw)


@pytest.mark.parametrize("B,T,D", [(1, 1, 4), (2, 100, 4), (2, 333, 32), (3, 1000, 64),
                                   (1, 5000, 8), (2, 2000, 16), (2, 700, 12)])
def test_affine_scan_dense(B, T, D):
    s = make_scan_input(B, T, D, dense=True, seed=T + D, h0_std=1.0)
    want = oracle.affine_scan(s.A.double().numpy(), s.b.double().numpy(), s.h0.double().numpy())
    got = binding.affine_scan(s.A.cuda(), s.b.cuda(), s.h0.cuda(), check=True).double().cpu().numpy()
    rel = np.max(np.abs(got - want)) / np.max(np.abs(want))
    assert rel <= 1e-5, rel


@pytest.mark.parametrize("name,over", [
    ("tiny", dict(T=1000, bias_std=0.3, h0_std=0.5)),
    ("dense_deer", dict(B=2, T=700, bias_std=0.2)),
    ("near_unstable", dict(B=2, T=300)),
    ("dense_deer", dict(B=3, T=257, d=12, din=5, h0_std=0.5)),
])
def test_each_deer_iteration_matches_oracle(name, over):
    w = _make(name, over)
    c, x, h0 = _oracle(w)
    ref = oracle.newton_solve(c, x, h0, "DEER", 0.0, max_iters=3, record=True)
    for n in (1, 2, 3):
        r = binding.solve_workload(w, "DEER", tol=0.0, max_iters=n)
        assert r.iters == n and r.status == "NOT_CONVERGED"
        err = np.max(np.abs(r.h.double().cpu().numpy() - ref["iterates"][n - 1]))
        assert err <= 5e-5, (n, err)


@pytest.mark.parametrize("name,over", [
    ("tiny", {}),
    ("dense_deer", dict(B=2, T=4096)),
    ("near_unstable", dict(B=2, T=500)),
    ("dense_deer", dict(B=1, T=999, d=20, din=7, h0_std=1.0, bias_std=0.3)),
])
def test_deer_converges_to_rollout(name, over):
    w = _make(name, over)
    c, x, h0 = _oracle(w)
    r = binding.solve_workload(w, "DEER")
    assert r.status == "OK"
    assert np.max(np.abs(r.h.double().cpu().numpy() - rollout(c, x, h0))) <= 1e-4
    ref = oracle.newton_solve(c, x, h0, "DEER", w.tol)
    assert abs(r.iters - ref["iters"]) <= 1, (r.iters, ref["iters"])


def test_deer_full_size_sampled():
    w = make_workload("dense_deer")
    r = binding.solve_workload(w, "DEER")
    assert r.status == "OK"
    c = GRU.from_workload(w)
    h = r.h.cpu()
    for b in (0, 3):
        want = rollout(c, w.x[b:b + 1].double().numpy(), w.h0[b:b + 1].double().numpy())
        assert np.max(np.abs(h[b:b + 1].double().numpy() - want)) <= 1e-4
    p = os.path.join(os.path.dirname(__file__), "golden", "oracle_iters.json")
    g = json.load(open(p)).get("dense_deer/DEER") if os.path.exists(p) else None
    if g is not None:
        assert abs(r.iters - g["iters"]) <= 1


def test_deer_nan_input_diverges():
    w = make_workload("dense_deer", B=2, T=300)
    w.x[0, 17, 3] = float("nan")
    r = binding.solve_workload(w, "DEER")
    assert r.status == "DIVERGED" and r.iters == 1
