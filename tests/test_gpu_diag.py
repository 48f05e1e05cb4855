"""GPU parity of the diagonal-Jacobian path against the fp64 oracle.

Covers the standalone diagonal scan, quasi-DEER on the dense GRU, exact Newton
on the diagonal-recurrence GRU, and quasi-ELK.  Every case calls the CUDA
library through the C ABI (``newton_solve_nonlinear_b200.binding``) and the
oracle on the same seeded inputs.

Tolerances (stated by the workloads, or derived here):
  * converged states vs the fp64 sequential rollout: max-abs <= 1e-4;
  * affine scan vs serial fp64: ||h - h_ref||_inf / ||h_ref||_inf <= 1e-5;
  * iteration counts: within +-1 of the oracle's;
  * single iterations (max_iters = 1, 2, 3) vs the oracle's iterates:
    max-abs <= 2e-5.  The GPU evaluates the cell in fp32 (relative error of a
    few 1e-7 per state after the fp32 gate arithmetic) and the scan
    accumulates products of a_t in (-1.5, 1.5); a few hundred ulps of 1.0 is
    the expected spread, so 2e-5 leaves a margin of ~10x.
"""
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


def _gpu(w, mode, **kw):
    return binding.solve_workload(w, mode, **kw)


# --------------------------------------------------------------- the scan ---
@pytest.mark.parametrize("B,T,D", [(1, 1, 4), (2, 3, 8), (3, 257, 64), (2, 1000, 100),
                                   (16, 4096, 64), (1, 5000, 12), (2, 333, 2048)])
def test_affine_scan_diag(B, T, D):
    s = make_scan_input(B, T, D, seed=B * 1000 + T, h0_std=1.0)
    want = oracle.affine_scan(s.A.double().numpy(), s.b.double().numpy(), s.h0.double().numpy())
    got = binding.affine_scan(s.A.cuda(), s.b.cuda(), s.h0.cuda(), check=True).double().cpu().numpy()
    rel = np.max(np.abs(got - want)) / np.max(np.abs(want))
    assert rel <= 1e-5, rel


@pytest.mark.parametrize("B,T,D,dense,parts", [(3, 1000, 100, 0, 3), (2, 1, 4, 0, 1), (16, 4096, 64, 0, 7),
                                                 (2, 333, 12, 1, 3), (1, 777, 32, 1, 5), (2, 5000, 12, 0, 9)])
def test_affine_scan_host_streamed(B, T, D, dense, parts):
    """The scan from and to host memory in time parts, each started from the
    last states of the part before (exact for a linear recurrence): normwise
    within 1e-5 of the serial fp64 scan, as the device scan."""
    s = make_scan_input(B, T, D, dense=bool(dense), seed=B * 1000 + T + parts, h0_std=1.0)
    want = oracle.affine_scan(s.A.double().numpy(), s.b.double().numpy(), s.h0.double().numpy())
    got = binding.affine_scan_host(s.A.pin_memory(), s.b.pin_memory(), s.h0.pin_memory(), parts=parts)
    assert not got.is_cuda
    rel = np.max(np.abs(got.double().numpy() - want)) / np.max(np.abs(want))
    assert rel <= 1e-5, rel
    assert binding.lib().pararnn_affine_scan_host_workspace_size(B, T, D, dense, (T + 127) // 128 + 1) == 0


def _same_run(a, b, atol=1e-6):
    """Two launches of the same solve agree to within fp32 rounding: the
    decoupled look-back composes the later tiles' maps in an order set by
    timing (how far back the first finished prefix lies), so the last bits
    may differ from one launch to the next."""
    return float((a.double().cpu() - b.double().cpu()).abs().max()) <= atol


def test_affine_scan_diag_in_place_and_repeat():
    s = make_scan_input(2, 777, 64, seed=5)
    A, b, h0 = s.A.cuda(), s.b.cuda(), s.h0.cuda()
    want = oracle.affine_scan(s.A.double().numpy(), s.b.double().numpy(), s.h0.double().numpy())
    ws = binding.alloc_workspace(binding.lib().pararnn_affine_scan_workspace_size(2, 777, 64, 0))
    first = binding.affine_scan(A, b, h0, workspace=ws, check=True).clone()
    second = binding.affine_scan(A, b, h0, workspace=ws, check=True)  # reused workspace
    assert _same_run(first, second)
    bb = b.clone()
    binding.affine_scan(A, bb, h0, out=bb, workspace=ws, check=True)  # h aliases b
    assert _same_run(first, bb)
    assert np.max(np.abs(first.double().cpu().numpy() - want)) / np.max(np.abs(want)) <= 1e-5


def test_affine_scan_closed_forms():
    B, T, D = 2, 3000, 64
    b = torch.randn(B, T, D, generator=torch.Generator().manual_seed(1))
    ones = torch.ones(B, T, D)
    h0 = torch.zeros(B, D)
    got = binding.affine_scan(ones.cuda(), b.cuda(), h0.cuda()).double().cpu()
    want = torch.cumsum(b.double(), 1)
    assert float((got - want).abs().max() / want.abs().max()) <= 1e-5
    got0 = binding.affine_scan(torch.zeros(B, T, D).cuda(), b.cuda(), h0.cuda()).cpu()
    assert torch.equal(got0, b)


# --------------------------------------------------- single iterations -------
@pytest.mark.parametrize("name,over,mode,lam", [
    ("untrained", dict(B=3, T=700, bias_std=0.3, h0_std=0.5), "QUASI", 0.0),
    ("tiny", dict(T=1000, bias_std=0.3, h0_std=0.5), "QUASI", 0.0),
    ("diag", dict(B=2, T=300, d=256, din=96, bias_std=0.3, h0_std=0.5), "QUASI", 0.0),
    ("diag", dict(B=2, T=130, d=100, din=40), "DEER", 0.0),
    ("diag", dict(B=3, T=129, d=192, din=64, bias_std=0.3, h0_std=1.0), "DEER", 0.0),
    ("near_unstable", dict(B=2, T=600), "QUASI_ELK", 0.1),
    ("near_unstable", dict(B=2, T=333, d=32, din=16, h0_std=0.5), "QUASI_ELK", 1.0),
    ("diag", dict(B=2, T=260, d=64, din=64), "QUASI_ELK", 0.01),
    ("untrained", dict(B=2, T=500, d=16, din=16, bias_std=0.3), "QUASI", 0.0),
    ("untrained", dict(B=2, T=333, d=8, din=8, h0_std=0.5), "QUASI", 0.0),
    ("untrained", dict(B=2, T=200, d=12, din=12), "QUASI", 0.0),
    ("untrained", dict(B=1, T=301, d=32, din=32, bias_std=0.3), "QUASI_ELK", 0.1),
])
def test_each_iteration_matches_oracle(name, over, mode, lam):
    kw = {k: over[k] for k in ("bias_std", "h0_std") if k in over}
    w = make_workload(name, **{k: v for k, v in over.items() if k not in kw}, **kw)
    c, x, h0 = _oracle(w)
    if mode in ("QUASI", "DEER"):
        ref = oracle.newton_solve(c, x, h0, mode, 0.0, max_iters=3, record=True)
    else:
        ref = oracle.elk_solve(c, x, h0, mode, lam, 0.0, max_iters=3, record=True)
    for n in (1, 2, 3):
        r = _gpu(w, mode, lam=lam, tol=0.0, max_iters=n)
        assert r.iters == n and r.status == "NOT_CONVERGED"
        err = np.max(np.abs(r.h.double().cpu().numpy() - ref["iterates"][n - 1]))
        assert err <= 2e-5, (n, err)
        assert abs(r.delta - ref["deltas"][n - 1]) <= 2e-5 + 1e-5 * ref["deltas"][n - 1]


# --------------------------------------------------------- converged ---------
@pytest.mark.parametrize("name,over,mode", [
    ("tiny", {}, "QUASI"),
    ("untrained", dict(T=1024), "QUASI"),
    ("untrained", dict(B=3, T=2049, bias_std=0.2, h0_std=0.5), "QUASI"),
    ("diag", dict(B=2, T=513, d=512, din=128), "QUASI"),
    ("diag", dict(B=1, T=100, d=68, din=20, h0_std=1.0), "DEER"),
    ("diag", dict(B=5, T=1000, d=128, din=64, h0_std=1.0, bias_std=0.2), "DEER"),
    ("diag", dict(B=2, T=1, d=64, din=32, h0_std=1.0), "QUASI"),
    ("near_unstable", dict(B=2, T=1000), "QUASI"),
])
def test_converged_matches_rollout_and_counts(name, over, mode):
    kw = {k: over[k] for k in ("bias_std", "h0_std") if k in over}
    w = make_workload(name, **{k: v for k, v in over.items() if k not in kw}, **kw)
    c, x, h0 = _oracle(w)
    want = rollout(c, x, h0)
    r = _gpu(w, mode)
    assert r.status == "OK"
    assert np.max(np.abs(r.h.double().cpu().numpy() - want)) <= 1e-4
    ref = oracle.newton_solve(c, x, h0, mode, w.tol)
    assert abs(r.iters - ref["iters"]) <= 1, (r.iters, ref["iters"])


@pytest.mark.parametrize("lam", [0.01, 0.1, 1.0])
def test_quasi_elk_matches_oracle_iterates(lam):
    """Damped steps converge linearly, so at tol 1e-4 both solvers stop while
    still up to ~1e-3 from the fixed point (the oracle too).  Gate: the count
    within +-1 of the oracle's, and -- when the counts agree -- the final
    iterate equal to the oracle's final iterate within 1e-4."""
    w = make_workload("near_unstable", B=2, T=1000)
    c, x, h0 = _oracle(w)
    r = _gpu(w, "QUASI_ELK", lam=lam)
    ref = oracle.elk_solve(c, x, h0, "QUASI_ELK", lam, w.tol)
    assert r.status == "OK" and ref["status"] == "OK"
    assert abs(r.iters - ref["iters"]) <= 1, (r.iters, ref["iters"])
    if r.iters == ref["iters"]:
        assert np.max(np.abs(r.h.double().cpu().numpy() - ref["h"])) <= 1e-4


def test_quasi_elk_tight_tolerance_reaches_rollout():
    """With heavy damping (lambda = 1) quasi-ELK stops at tol 1e-4 while still
    ~1e-3 from the fixed point (slow linear rate); at tol 1e-6 it reaches it."""
    w = make_workload("near_unstable", B=2, T=800)
    c, x, h0 = _oracle(w)
    r = _gpu(w, "QUASI_ELK", lam=1.0, tol=1e-6)
    assert r.status == "OK"
    assert np.max(np.abs(r.h.double().cpu().numpy() - rollout(c, x, h0))) <= 1e-4
    ref = oracle.elk_solve(c, x, h0, "QUASI_ELK", 1.0, w.tol)
    r2 = _gpu(w, "QUASI_ELK", lam=1.0)
    assert abs(r2.iters - ref["iters"]) <= 1


# ----------------------------------------------------------- statuses --------
def test_statuses_and_edges():
    w = make_workload("untrained", B=2, T=300)
    r = _gpu(w, "QUASI", max_iters=2)
    assert r.status == "NOT_CONVERGED" and r.iters == 2
    w.x[1, 123, 5] = float("nan")
    r = _gpu(w, "QUASI")
    assert r.status == "DIVERGED" and r.iters == 1
    for T in (1, 2, 3, 63, 64, 65):
        w = make_workload("untrained", B=1, T=T, h0_std=1.0)
        c, x, h0 = _oracle(w)
        r = _gpu(w, "QUASI")
        assert r.status == "OK"
        assert np.max(np.abs(r.h.double().cpu().numpy() - rollout(c, x, h0))) <= 1e-4
        assert r.iters <= T + 1


def test_async_entry_and_report():
    w = make_workload("untrained", B=2, T=500)
    dev = lambda t: t.cuda().contiguous()
    info = torch.zeros(4, dtype=torch.int32, device="cuda")
    out = binding.newton_solve(dev(w.w_ih), dev(w.b_ih), dev(w.w_hh), dev(w.b_hh), dev(w.x),
                               dev(w.h0), kind="dense", mode="QUASI", tol=w.tol, sync=False,
                               info_dev=info)
    torch.cuda.synchronize()
    iters, status = int(info[0]), int(info[1])
    delta = float(info[2:3].view(torch.float32))
    assert status == 0 and delta <= w.tol
    r = _gpu(w, "QUASI")
    assert abs(r.iters - iters) <= 1 and _same_run(r.h, out, atol=1e-6 if r.iters == iters else w.tol)


# --------------------------------------------- full-size, sampled outputs ----
def _golden():
    import json, os
    p = os.path.join(os.path.dirname(__file__), "golden", "oracle_iters.json")
    return json.load(open(p)) if os.path.exists(p) else {}


@pytest.mark.parametrize("key,name,over,mode,lam,samples", [
    ("untrained/T65536/QUASI", "untrained", dict(T=65536), "QUASI", 0.0, (0, 15)),
    ("untrained/T16384/QUASI", "untrained", dict(T=16384), "QUASI", 0.0, (0, 15)),
    ("untrained/T4096/QUASI", "untrained", dict(T=4096), "QUASI", 0.0, (0, 9)),
    ("untrained/T1024/QUASI", "untrained", dict(T=1024), "QUASI", 0.0, (2,)),
    ("diag/QUASI", "diag", {}, "QUASI", 0.0, (3,)),
    ("near_unstable/QUASI_ELK/0.1", "near_unstable", {}, "QUASI_ELK", 0.1, (0, 7)),
    ("near_unstable/QUASI_ELK/0.01", "near_unstable", {}, "QUASI_ELK", 0.01, (1, 6)),
    ("tiny/QUASI", "tiny", {}, "QUASI", 0.0, (0,)),
])
def test_full_size_sampled(key, name, over, mode, lam, samples):
    """Full workload sizes in the launch configuration the benchmark times.
    States are compared on whole sampled sequences (rollout of one sequence is
    cheap for the oracle); iteration counts against the stored oracle counts."""
    w = make_workload(name, **over)
    r = _gpu(w, mode, lam=lam)
    assert r.status == "OK"
    c = GRU.from_workload(w)
    h = r.h.cpu()
    for b in samples:
        want = rollout(c, w.x[b:b + 1].double().numpy(), w.h0[b:b + 1].double().numpy())
        assert np.max(np.abs(h[b:b + 1].double().numpy() - want)) <= 1e-4
    g = _golden().get(key)
    if g is not None:
        assert abs(r.iters - g["iters"]) <= 1, (r.iters, g["iters"])
