"""Pins of the fp64 oracle to things other than itself (CPU only).

Each test ties one oracle function to a library routine, a closed form, a
brute-force dense solve, finite differences, or an invariant the pages state.
Together they are chosen so that a dropped term, a wrong sign, an off-by-one
shift or a transposed operand in the oracle fails at least one of them.
"""
import numpy as np
import pytest
import torch

import oracle
from oracle import brute, elk, newton
from oracle.cells import GRU, residual, rollout
from oracle.scan import affine_scan
from newton_solve_nonlinear_b200.inputs import make_workload


def _rand_gru(kind, din, d, seed, scale=0.5):
    rng = np.random.default_rng(seed)
    w_hh = rng.normal(0, scale, (3 * d, d)) if kind == "dense" else rng.uniform(-1, 1, 3 * d)
    return GRU(kind=kind, w_ih=rng.normal(0, scale, (3 * d, din)), b_ih=rng.normal(0, 0.3, 3 * d),
               w_hh=w_hh, b_hh=rng.normal(0, 0.3, 3 * d))


def _torch_cell(c: GRU, din):
    d = c.d
    m = torch.nn.GRUCell(din, d).double()
    with torch.no_grad():
        m.weight_ih.copy_(torch.from_numpy(c.w_ih))
        m.bias_ih.copy_(torch.from_numpy(c.b_ih))
        m.bias_hh.copy_(torch.from_numpy(c.b_hh))
        if c.kind == "dense":
            m.weight_hh.copy_(torch.from_numpy(c.w_hh))
        else:
            W = np.concatenate([np.diag(c.w_hh[g * d:(g + 1) * d]) for g in range(3)], 0)
            m.weight_hh.copy_(torch.from_numpy(W))
    return m


# ---------------------------------------------------------------- the cell --
@pytest.mark.parametrize("kind", ["dense", "diag"])
def test_cell_equals_torch_grucell(kind):
    """The oracle cell is torch.nn.GRUCell (gate order r, z, n; reset gate
    applied after the recurrent bias), widened to fp64."""
    din, d = 5, 7
    c = _rand_gru(kind, din, d, seed=1)
    rng = np.random.default_rng(2)
    x = rng.normal(size=(11, din))
    h = rng.normal(size=(11, d))
    with torch.no_grad():
        ref = _torch_cell(c, din)(torch.from_numpy(x), torch.from_numpy(h)).numpy()
    np.testing.assert_allclose(c.step(h, x), ref, rtol=0, atol=1e-14)


def test_rollout_equals_torch_loop():
    din, d, B, T = 3, 6, 2, 40
    c = _rand_gru("dense", din, d, seed=3)
    rng = np.random.default_rng(4)
    x = rng.normal(size=(B, T, din))
    h0 = rng.normal(size=(B, d))
    m = _torch_cell(c, din)
    h = torch.from_numpy(h0)
    outs = []
    with torch.no_grad():
        for t in range(T):
            h = m(torch.from_numpy(x[:, t]), h)
            outs.append(h)
    np.testing.assert_allclose(rollout(c, x, h0), torch.stack(outs, 1).numpy(), rtol=0, atol=1e-13)


@pytest.mark.parametrize("kind", ["dense", "diag"])
def test_jacobian_central_differences(kind):
    """df/dh against fp64 central differences, every entry (dense) / the
    diagonal (diag cell, whose Jacobian is exactly diagonal)."""
    din, d = 4, 6
    c = _rand_gru(kind, din, d, seed=5, scale=0.9)
    rng = np.random.default_rng(6)
    h = rng.normal(size=d)
    x = rng.normal(size=din)
    p = c.project(x)
    eps = 1e-6
    fd = np.empty((d, d))
    for k in range(d):
        e = np.zeros(d)
        e[k] = eps
        fd[:, k] = (c.gates(h + e, p)[4] - c.gates(h - e, p)[4]) / (2 * eps)
    f, J = c.jacobian(h, p)
    np.testing.assert_allclose(J, fd, rtol=0, atol=1e-8)
    f2, a = c.jacobian_diag(h, p)
    np.testing.assert_allclose(a, np.diagonal(fd), rtol=0, atol=1e-8)
    np.testing.assert_allclose(f, f2, rtol=0, atol=0)
    if kind == "diag":
        np.testing.assert_allclose(fd - np.diag(np.diagonal(fd)), 0.0, atol=1e-9)


# ---------------------------------------------------------------- the scan --
def test_scan_closed_forms_diagonal():
    rng = np.random.default_rng(7)
    B, T, D = 2, 50, 3
    b = rng.normal(size=(B, T, D))
    h0 = rng.normal(size=(B, D))
    # a == 1: running sum
    np.testing.assert_allclose(affine_scan(np.ones((B, T, D)), b, h0),
                               h0[:, None] + np.cumsum(b, axis=1), atol=1e-12)
    # a == 0: h_t = b_t
    np.testing.assert_allclose(affine_scan(np.zeros((B, T, D)), b, h0), b, atol=0)
    # constant a, constant b: geometric series h_t = a^t h0 + beta (1 - a^t) / (1 - a)
    a, beta = 0.9, 0.37
    t = np.arange(1, T + 1)[None, :, None]
    want = a ** t * h0[:, None] + beta * (1 - a ** t) / (1 - a)
    np.testing.assert_allclose(affine_scan(np.full((B, T, D), a), np.full((B, T, D), beta), h0),
                               want, atol=1e-12)


def test_scan_closed_forms_dense():
    rng = np.random.default_rng(8)
    T, D = 30, 4
    # A_t = R (a rotation, not symmetric), b = 0: h_t = R^t h0 -- catches A vs A^T
    th = 0.3
    R = np.eye(D)
    R[:2, :2] = [[np.cos(th), -np.sin(th)], [np.sin(th), np.cos(th)]]
    R = R @ np.diag([1.0, 1.0, 0.5, 0.8])
    R[2, 3] = 0.7
    h0 = rng.normal(size=(1, D))
    A = np.broadcast_to(R, (1, T, D, D))
    got = affine_scan(A, np.zeros((1, T, D)), h0)
    want = np.stack([np.linalg.matrix_power(R, k) @ h0[0] for k in range(1, T + 1)])[None]
    np.testing.assert_allclose(got, want, atol=1e-12)
    # diagonal matrices agree with the diagonal scan
    a = rng.uniform(-1, 1, (2, T, D))
    b = rng.normal(size=(2, T, D))
    h0 = rng.normal(size=(2, D))
    Ad = np.zeros((2, T, D, D))
    Ad[..., np.arange(D), np.arange(D)] = a
    np.testing.assert_allclose(affine_scan(Ad, b, h0), affine_scan(a, b, h0), atol=1e-13)


# ------------------------------------------------------------------ Newton --
class LinearCell:
    """f(h, x) = A h + x: Newton on an affine map is exact in one step."""

    def __init__(self, A):
        self.A = A
        self.kind = "dense"

    @property
    def d(self):
        return self.A.shape[0]

    def project(self, x):
        return x

    def jacobian(self, h, p):
        f = h @ self.A.T + p
        return f, np.broadcast_to(self.A, h.shape[:-1] + self.A.shape)

    def jacobian_diag(self, h, p):
        f = h @ self.A.T + p
        return f, np.broadcast_to(np.diagonal(self.A), h.shape)


def test_newton_exact_on_linear_cell():
    """The pages' Newton step solves the linearised system; on an affine cell the
    linearisation is exact, so iteration 1 lands on the solution and iteration
    2 observes delta = 0 (iters = 2 under the counting rule)."""
    rng = np.random.default_rng(9)
    D, B, T = 5, 3, 64
    A = rng.normal(0, 0.4, (D, D))
    A *= 0.9 / np.max(np.abs(np.linalg.eigvals(A)))
    x = rng.normal(size=(B, T, D))
    h0 = rng.normal(size=(B, D))
    exact = affine_scan(np.broadcast_to(A, (B, T, D, D)), x, h0)
    r = newton.newton_solve(LinearCell(A), x, h0, "DEER", tol=1e-12, record=True)
    np.testing.assert_allclose(r["iterates"][0], exact, atol=1e-12)
    assert r["iters"] == 2 and r["status"] == "OK"
    # quasi-DEER is exact too when A is diagonal
    Ad = np.diag(rng.uniform(-0.9, 0.9, D))
    r = newton.newton_solve(LinearCell(Ad), x, h0, "QUASI", tol=1e-12, record=True)
    np.testing.assert_allclose(r["iterates"][0],
                               affine_scan(np.broadcast_to(np.diagonal(Ad), (B, T, D)), x, h0),
                               atol=1e-12)
    assert r["iters"] == 2


@pytest.mark.parametrize("mode", ["DEER", "QUASI"])
def test_undamped_newton_recovers_one_state_per_iteration(mode):
    """For any A_t, once h^(i)_{t-1} is exact the update gives
    h^(i+1)_t = f(h*_{t-1}, x_t) = h*_t; with h_0 fixed, iteration i makes
    h_1..h_i exact, so undamped (quasi-)Newton converges within T iterations.
    Pins the shift by one step and the h_0 boundary."""
    c = _rand_gru("dense", 3, 4, seed=10, scale=1.5)
    rng = np.random.default_rng(11)
    B, T = 2, 14
    x = rng.normal(size=(B, T, 3)) * 2
    h0 = rng.normal(size=(B, 4))
    ref = rollout(c, x, h0)
    r = newton.newton_solve(c, x, h0, mode, tol=0.0, max_iters=T, record=True)
    for i, h in enumerate(r["iterates"], start=1):
        np.testing.assert_allclose(h[:, :i], ref[:, :i], rtol=0, atol=1e-12)
    np.testing.assert_allclose(r["h"], ref, atol=1e-12)


@pytest.mark.parametrize("diagonal_only", [False, True])
def test_newton_step_equals_dense_solve(diagonal_only):
    """One structured step (linearise + forward substitution) equals
    h - Jac^{-1} R(h) with the whole (T*D)^2 system Jacobian assembled and
    solved densely; and the assembled Jacobian equals finite differences of
    the residual (full Jacobian case)."""
    c = _rand_gru("dense", 2, 3, seed=12, scale=0.8)
    rng = np.random.default_rng(13)
    T, D = 6, 3
    x = rng.normal(size=(1, T, 2))
    h0 = rng.normal(size=(1, D))
    guess = rng.normal(size=(1, T, D))
    A, b, _ = newton.linearise(c, guess, c.project(x), h0, dense=not diagonal_only)
    step = affine_scan(A, b, h0)
    dense = brute.newton_step_dense(c, guess[0].ravel(), x[0], h0[0], diagonal_only)
    np.testing.assert_allclose(step[0].ravel(), dense, atol=1e-11)
    if not diagonal_only:
        Jfd = brute.system_jacobian_fd(c, guess[0].ravel(), x[0], h0[0])
        np.testing.assert_allclose(brute.system_jacobian(c, guess[0].ravel(), x[0], h0[0]),
                                   Jfd, atol=1e-8)


def test_diag_cell_quasi_is_exact_newton():
    """For the diagonal-recurrence GRU, diag(J) = J: quasi-DEER and DEER
    produce the same iterates and the same count."""
    w = make_workload("diag", B=2, T=97, d=48, din=40, bias_std=0.2)
    c = GRU.from_workload(w)
    x, h0 = w.x.double().numpy(), w.h0.double().numpy()
    r1 = newton.newton_solve(c, x, h0, "DEER", w.tol, record=True)
    r2 = newton.newton_solve(c, x, h0, "QUASI", w.tol, record=True)
    assert r1["iters"] == r2["iters"]
    for a, b in zip(r1["iterates"], r2["iterates"]):
        np.testing.assert_allclose(a, b, atol=1e-14)
    np.testing.assert_allclose(r1["h"], rollout(c, x, h0), atol=1e-6)


@pytest.mark.parametrize("name,mode", [("tiny", "DEER"), ("tiny", "QUASI"),
                                       ("dense_deer", "DEER")])
def test_newton_converges_to_rollout(name, mode):
    w = make_workload(name, T=300, B=2)
    c = GRU.from_workload(w)
    x, h0 = w.x.double().numpy(), w.h0.double().numpy()
    r = newton.newton_solve(c, x, h0, mode, w.tol)
    assert r["status"] == "OK"
    np.testing.assert_allclose(r["h"], rollout(c, x, h0), atol=10 * w.tol)
    assert np.max(np.abs(residual(c, r["h"], x, h0))) < 10 * w.tol


def test_newton_counts_and_statuses():
    w = make_workload("tiny", T=200)
    c = GRU.from_workload(w)
    x, h0 = w.x.double().numpy(), w.h0.double().numpy()
    r = newton.newton_solve(c, x, h0, "QUASI", w.tol, max_iters=2)
    assert r["status"] == "NOT_CONVERGED" and r["iters"] == 2 and len(r["deltas"]) == 2
    x_bad = x.copy()
    x_bad[0, 50, 0] = np.nan
    r = newton.newton_solve(c, x_bad, h0, "QUASI", w.tol)
    assert r["status"] == "DIVERGED" and r["iters"] == 1
    # default cap T + 1: T = 1 is exact after one iteration, observed by the second
    w1 = make_workload("tiny", T=1, h0_std=1.0)
    r1 = newton.newton_solve(GRU.from_workload(w1), w1.x.double().numpy(),
                             w1.h0.double().numpy(), "QUASI", 1e-12)
    assert r1["status"] == "OK" and r1["iters"] == 2 and r1["deltas"][-1] == 0.0
    # the counting rule: iters is the first i+1 with delta_i <= tol
    r = newton.newton_solve(c, x, h0, "DEER", w.tol)
    assert r["deltas"][-1] <= w.tol and all(d > w.tol for d in r["deltas"][:-1])
    assert r["iters"] == len(r["deltas"])


# --------------------------------------------------------------------- ELK --
def _lm_dense_from_operands(A, b, y, h0, lam):
    """(Jac^T Jac + lam I) h = Jac^T c + lam y with Jac = I - (sub-diagonal A_t),
    c = b with A_1 h0 added: the minimiser of |Jac h - c|^2 + lam |h - y|^2."""
    B, T, D = b.shape
    out = np.empty((B, T, D))
    for k in range(B):
        Jac = np.eye(T * D)
        for t in range(1, T):
            At = A[k, t] if A.ndim == 4 else np.diag(A[k, t])
            Jac[t * D:(t + 1) * D, (t - 1) * D:t * D] = -At
        c = b[k].copy()
        A1 = A[k, 0] if A.ndim == 4 else np.diag(A[k, 0])
        c[0] += A1 @ h0[k]
        H = Jac.T @ Jac + lam * np.eye(T * D)
        out[k] = np.linalg.solve(H, Jac.T @ c.ravel() + lam * y[k].ravel()).reshape(T, D)
    return out


@pytest.mark.parametrize("dense", [False, True])
@pytest.mark.parametrize("lam", [1e-2, 0.3, 5.0])
def test_lm_step_three_ways(dense, lam):
    """Normal equations (block Thomas) == Kalman filter + RTS smoother == a dense
    assembled least-squares solve."""
    rng = np.random.default_rng(14)
    B, T, D = 2, 9, 3
    A = rng.normal(0, 0.9, (B, T, D, D)) if dense else rng.uniform(-1.5, 1.5, (B, T, D))
    b = rng.normal(size=(B, T, D))
    y = rng.normal(size=(B, T, D))
    h0 = rng.normal(size=(B, D))
    want = _lm_dense_from_operands(A, b, y, h0, lam)
    np.testing.assert_allclose(elk.lm_step_normal(A, b, y, h0, lam), want, atol=1e-10)
    np.testing.assert_allclose(elk.lm_step_kalman(A, b, y, h0, lam), want, atol=1e-10)


@pytest.mark.parametrize("diagonal_only", [False, True])
def test_lm_step_equals_dense_cell_assembly(diagonal_only):
    """The oracle's ELK step on a GRU equals h - (Jac^T Jac + lam I)^{-1} Jac^T R."""
    c = _rand_gru("dense", 2, 3, seed=15, scale=0.8)
    rng = np.random.default_rng(16)
    T, D, lam = 7, 3, 0.25
    x = rng.normal(size=(1, T, 2))
    h0 = rng.normal(size=(1, D))
    guess = rng.normal(size=(1, T, D))
    A, b, _ = newton.linearise(c, guess, c.project(x), h0, dense=not diagonal_only)
    step = elk.lm_step_normal(A, b, guess, h0, lam)
    dense = brute.lm_step_dense(c, guess[0].ravel(), x[0], h0[0], lam, diagonal_only)
    np.testing.assert_allclose(step[0].ravel(), dense, atol=1e-11)


@pytest.mark.parametrize("dense", [False, True])
def test_lm_limits(dense):
    rng = np.random.default_rng(17)
    B, T, D = 2, 12, 3
    A = rng.normal(0, 0.5, (B, T, D, D)) if dense else rng.uniform(-0.9, 0.9, (B, T, D))
    b = rng.normal(size=(B, T, D))
    y = rng.normal(size=(B, T, D))
    h0 = rng.normal(size=(B, D))
    exact = affine_scan(A, b, h0)
    # lambda -> 0: the DEER step (the undamped linear solve)
    np.testing.assert_allclose(elk.lm_step_normal(A, b, y, h0, 1e-12), exact, atol=1e-9)
    np.testing.assert_allclose(elk.lm_step_kalman(A, b, y, h0, 1e-12), exact, atol=1e-9)
    # lambda -> inf: no step
    np.testing.assert_allclose(elk.lm_step_normal(A, b, y, h0, 1e12), y, atol=1e-9)
    # the exact solution is a fixed point for every lambda
    for lam in (0.01, 1.0, 100.0):
        np.testing.assert_allclose(elk.lm_step_normal(A, b, exact, h0, lam), exact, atol=1e-11)
    # T = 1 closed form: h_1 = (A_1 h0 + b_1 + lam y_1) / (1 + lam)
    lam = 0.7
    A1 = A[:, :1]
    c1 = (np.einsum("bij,bj->bi", A1[:, 0], h0) if dense else A1[:, 0] * h0) + b[:, 0]
    np.testing.assert_allclose(elk.lm_step_normal(A1, b[:, :1], y[:, :1], h0, lam)[:, 0],
                               (c1 + lam * y[:, 0]) / (1 + lam), atol=1e-13)


@pytest.mark.parametrize("mode", ["ELK", "QUASI_ELK"])
def test_elk_converges_on_near_unstable(mode):
    w = make_workload("near_unstable", B=2, T=120, d=12, din=12)
    c = GRU.from_workload(w)
    x, h0 = w.x.double().numpy(), w.h0.double().numpy()
    r = elk.elk_solve(c, x, h0, mode, 0.1, 1e-9)
    assert r["status"] == "OK"
    np.testing.assert_allclose(r["h"], rollout(c, x, h0), atol=1e-7)


def test_public_names():
    assert oracle.newton_solve is newton.newton_solve
    assert oracle.elk_solve is elk.elk_solve
