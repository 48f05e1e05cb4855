"""ELK / quasi-ELK: the Levenberg-Marquardt-damped Newton step (fp64).

ELK stabilises DEER by adding a Levenberg-Marquardt trust region to each
Newton step and observes that the damped step is the posterior mean of a
linear-Gaussian state-space model, so it can be computed by a (parallel)
Kalman filter and smoother ("Towards Scalable and Stable Parallelization of
Nonlinear RNNs", abstract; atlas summary, "Approach" and "Builds on": iterated
extended Kalman smoother).  Quasi-ELK uses the diagonal Jacobian, making the
smoother D independent scalar problems (atlas summary, "Approach").

Reading of the LM parameterisation (the pages give no formula): with the
linearisation at the current guess y = h^(i) (A_t, b_t as in ``newton``),
the step minimises over h_1..h_T (h_0 = h0 fixed)

    sum_t |h_t - A_t h_{t-1} - b_t|^2  +  lambda * sum_t |h_t - y_t|^2 .

This is the Gauss-Newton model |r + J dh|^2 + lambda |dh|^2 written in terms of
h = y + dh.  As a state-space model: dynamics h_t = A_t h_{t-1} + b_t + w_t,
w_t ~ N(0, I); observations y_t = h_t + v_t, v_t ~ N(0, I / lambda); prior
h_0 = h0 exactly.  lambda -> 0 gives the DEER step; lambda -> inf gives no
step.

Two independent solvers of the same quadratic problem are written here:
  * ``lm_step_normal``  -- the block-tridiagonal normal equations solved by
                           block Gaussian elimination (Thomas; the system is
                           symmetric positive definite for lambda > 0);
  * ``lm_step_kalman``  -- the sequential Kalman filter and Rauch-Tung-Striebel
                           smoother of the state-space model above.
``elk_solve`` iterates with the first; tests cross-check the two.
"""
from __future__ import annotations

import numpy as np

from .cells import GRU
from .newton import (STATUS_DIVERGED, STATUS_NOT_CONVERGED, STATUS_OK, linearise)


# ---------------------------------------------------------------------------
# normal equations
# ---------------------------------------------------------------------------
def lm_step_normal(A, b, y, h0, lam):
    """Minimiser of sum |h_t - A_t h_{t-1} - b_t|^2 + lam sum |h_t - y_t|^2.

    Setting the gradient with respect to h_t to zero gives, for t = 1..T
    (terms with index T+1 absent):
        ((1+lam) I + A_{t+1}^T A_{t+1}) h_t - A_t h_{t-1} - A_{t+1}^T h_{t+1}
            = b_t - A_{t+1}^T b_{t+1} + lam y_t,
    with A_1 h_0 moved to the right-hand side of t = 1.

    A: [B,T,D] (diagonal) or [B,T,D,D] (dense); b, y [B,T,D]; h0 [B,D]."""
    A = np.asarray(A, np.float64)
    if A.ndim == 3:
        return _tridiag_scalar(A, np.asarray(b, np.float64), np.asarray(y, np.float64),
                               np.asarray(h0, np.float64), lam)
    return _tridiag_block(A, np.asarray(b, np.float64), np.asarray(y, np.float64),
                          np.asarray(h0, np.float64), lam)


def _tridiag_scalar(a, b, y, h0, lam):
    B, T, D = b.shape
    diag = np.full((B, T, D), 1.0 + lam)
    diag[:, :-1] += a[:, 1:] ** 2
    rhs = b + lam * y
    rhs[:, :-1] -= a[:, 1:] * b[:, 1:]
    rhs[:, 0] += a[:, 0] * h0
    # coupling of h_t with h_{t-1} is -a_t; of h_t with h_{t+1} is -a_{t+1}
    cp = np.empty((B, T, D))
    dp = np.empty((B, T, D))
    cp[:, 0] = -a[:, 1] / diag[:, 0] if T > 1 else 0.0
    dp[:, 0] = rhs[:, 0] / diag[:, 0]
    for t in range(1, T):
        sub = -a[:, t]
        m = diag[:, t] - sub * cp[:, t - 1]
        cp[:, t] = (-a[:, t + 1] / m) if t < T - 1 else 0.0
        dp[:, t] = (rhs[:, t] - sub * dp[:, t - 1]) / m
    h = np.empty((B, T, D))
    h[:, T - 1] = dp[:, T - 1]
    for t in range(T - 2, -1, -1):
        h[:, t] = dp[:, t] - cp[:, t] * h[:, t + 1]
    return h


def _tridiag_block(A, b, y, h0, lam):
    B, T, D = b.shape
    eye = np.eye(D)
    At = np.swapaxes(A, -1, -2)
    M = np.broadcast_to((1.0 + lam) * eye, (B, T, D, D)).copy()
    M[:, :-1] += At[:, 1:] @ A[:, 1:]
    rhs = b + lam * y
    rhs[:, :-1] -= np.einsum("btij,btj->bti", At[:, 1:], b[:, 1:])
    rhs[:, 0] += np.einsum("bij,bj->bi", A[:, 0], h0)
    # block Gaussian elimination: sub-diagonal block of row t is -A_t,
    # super-diagonal block is -A_{t+1}^T.
    Cp = np.zeros((B, T, D, D))
    dp = np.empty((B, T, D))
    S = M[:, 0]
    if T > 1:
        Cp[:, 0] = np.linalg.solve(S, -At[:, 1])
    dp[:, 0] = np.linalg.solve(S, rhs[:, 0][..., None])[..., 0]
    for t in range(1, T):
        sub = -A[:, t]
        S = M[:, t] - sub @ Cp[:, t - 1]
        r = rhs[:, t] - np.einsum("bij,bj->bi", sub, dp[:, t - 1])
        if t < T - 1:
            Cp[:, t] = np.linalg.solve(S, -At[:, t + 1])
        dp[:, t] = np.linalg.solve(S, r[..., None])[..., 0]
    h = np.empty((B, T, D))
    h[:, T - 1] = dp[:, T - 1]
    for t in range(T - 2, -1, -1):
        h[:, t] = dp[:, t] - np.einsum("bij,bj->bi", Cp[:, t], h[:, t + 1])
    return h


# ---------------------------------------------------------------------------
# Kalman filter + RTS smoother (independent cross-check)
# ---------------------------------------------------------------------------
def lm_step_kalman(A, b, y, h0, lam):
    """The same minimiser as the posterior mean of the state-space model.

    Filter (t = 1..T, m_0 = h0, P_0 = 0):
        m-_t = A_t m_{t-1} + b_t,   P-_t = A_t P_{t-1} A_t^T + I,
        K_t  = P-_t (P-_t + I/lam)^{-1} = lam P-_t (I + lam P-_t)^{-1},
        m_t  = m-_t + K_t (y_t - m-_t),   P_t = (I - K_t) P-_t.
    Smoother (s_T = m_T, t = T-1..1):
        G_t = P_t A_{t+1}^T (P-_{t+1})^{-1},   s_t = m_t + G_t (s_{t+1} - m-_{t+1}).
    Returns s [B,T,D]."""
    A = np.asarray(A, np.float64)
    b = np.asarray(b, np.float64)
    y = np.asarray(y, np.float64)
    B, T, D = b.shape
    if A.ndim == 3:
        m = np.array(h0, np.float64, copy=True)
        P = np.zeros((B, D))
        ms, Ps, mps, Pps = (np.empty((B, T, D)) for _ in range(4))
        for t in range(T):
            mp = A[:, t] * m + b[:, t]
            Pp = A[:, t] ** 2 * P + 1.0
            K = lam * Pp / (1.0 + lam * Pp)
            m = mp + K * (y[:, t] - mp)
            P = (1.0 - K) * Pp
            ms[:, t], Ps[:, t], mps[:, t], Pps[:, t] = m, P, mp, Pp
        s = np.empty((B, T, D))
        s[:, T - 1] = ms[:, T - 1]
        for t in range(T - 2, -1, -1):
            G = Ps[:, t] * A[:, t + 1] / Pps[:, t + 1]
            s[:, t] = ms[:, t] + G * (s[:, t + 1] - mps[:, t + 1])
        return s
    eye = np.eye(D)
    m = np.array(h0, np.float64, copy=True)
    P = np.zeros((B, D, D))
    ms, mps = np.empty((B, T, D)), np.empty((B, T, D))
    Ps, Pps = np.empty((B, T, D, D)), np.empty((B, T, D, D))
    for t in range(T):
        At = A[:, t]
        mp = np.einsum("bij,bj->bi", At, m) + b[:, t]
        Pp = At @ P @ np.swapaxes(At, -1, -2) + eye
        # K = lam Pp (I + lam Pp)^{-1}; Pp and (I + lam Pp) commute.
        K = np.swapaxes(np.linalg.solve(eye + lam * Pp, lam * np.swapaxes(Pp, -1, -2)), -1, -2)
        m = mp + np.einsum("bij,bj->bi", K, y[:, t] - mp)
        P = (eye - K) @ Pp
        P = 0.5 * (P + np.swapaxes(P, -1, -2))
        ms[:, t], mps[:, t], Ps[:, t], Pps[:, t] = m, mp, P, Pp
    s = np.empty((B, T, D))
    s[:, T - 1] = ms[:, T - 1]
    for t in range(T - 2, -1, -1):
        # G = P_t A_{t+1}^T Pp_{t+1}^{-1}  ->  G^T = Pp^{-1} A_{t+1} P_t (symmetric P, Pp)
        Gt = np.linalg.solve(Pps[:, t + 1], A[:, t + 1] @ Ps[:, t])
        G = np.swapaxes(Gt, -1, -2)
        s[:, t] = ms[:, t] + np.einsum("bij,bj->bi", G, s[:, t + 1] - mps[:, t + 1])
    return s


# ---------------------------------------------------------------------------
# the damped iteration
# ---------------------------------------------------------------------------
def elk_solve(cell: GRU, x: np.ndarray, h0: np.ndarray, mode: str, lam: float, tol: float,
              max_iters: int | None = None, record: bool = False) -> dict:
    """Iterate the LM step: ELK (full Jacobian) or quasi-ELK (diagonal Jacobian).

    Each iteration linearises at the current guess exactly as DEER does (see
    ``newton.linearise``), takes y = h^(i) as the observations, and replaces
    the guess by the damped step.  Initial guess, convergence test and
    statuses are those of ``newton.newton_solve``."""
    if mode not in ("ELK", "QUASI_ELK"):
        raise ValueError(mode)
    x = np.asarray(x, np.float64)
    h0 = np.asarray(h0, np.float64)
    B, T, _ = x.shape
    max_iters = T + 1 if max_iters is None or max_iters <= 0 else max_iters
    dense = mode == "ELK" and cell.kind == "dense"
    p = cell.project(x)
    h = np.zeros((B, T, cell.d))
    deltas, iterates = [], []
    status, iters = STATUS_NOT_CONVERGED, max_iters
    for i in range(max_iters):
        with np.errstate(all="ignore"):
            A, b, _ = linearise(cell, h, p, h0, dense)
            h_new = lm_step_normal(A, b, h, h0, lam)
            delta = float(np.max(np.abs(h_new - h)))
        h = h_new
        deltas.append(delta)
        if record:
            iterates.append(h.copy())
        if not np.all(np.isfinite(h)) or not np.isfinite(delta):
            status, iters = STATUS_DIVERGED, i + 1
            break
        if delta <= tol:
            status, iters = STATUS_OK, i + 1
            break
    out = dict(h=h, iters=iters, status=status, delta=deltas[-1] if deltas else 0.0,
               deltas=deltas)
    if record:
        out["iterates"] = iterates
    return out
