"""Dense assemblies of the whole unrolled system, for tiny T only (fp64).

These do not use the structure the fast solvers rely on (bidiagonal system
Jacobian, tridiagonal normal equations); they assemble the full
(T*D) x (T*D) matrices and call a dense solver.  Tests use them to pin the
structured steps in ``newton`` and ``elk`` ("ParaRNN" summary, "Newton's
Iteration": residual, Jacobian, linearised solve).
"""
from __future__ import annotations

import numpy as np

from .cells import GRU


def system_residual(cell: GRU, hflat: np.ndarray, x1: np.ndarray, h01: np.ndarray) -> np.ndarray:
    """R(h) = [h_t - f(h_{t-1}, x_t)]_t for ONE sequence, flattened to T*D."""
    T = x1.shape[0]
    D = cell.d
    h = hflat.reshape(T, D)
    out = np.empty((T, D))
    prev = h01
    for t in range(T):
        out[t] = h[t] - cell.step(prev, x1[t])
        prev = h[t]
    return out.reshape(-1)


def system_jacobian_fd(cell: GRU, hflat, x1, h01, eps: float = 1e-6) -> np.ndarray:
    """dR/dh by central finite differences over all T*D unknowns."""
    n = hflat.size
    Jac = np.empty((n, n))
    for k in range(n):
        e = np.zeros(n)
        e[k] = eps
        Jac[:, k] = (system_residual(cell, hflat + e, x1, h01)
                     - system_residual(cell, hflat - e, x1, h01)) / (2 * eps)
    return Jac


def system_jacobian(cell: GRU, hflat, x1, h01, diagonal_only: bool = False) -> np.ndarray:
    """dR/dh assembled from the cell Jacobians: identity blocks on the diagonal,
    -J_t at block (t, t-1).  ``diagonal_only`` keeps only diag(J_t) (quasi)."""
    T = x1.shape[0]
    D = cell.d
    h = hflat.reshape(T, D)
    p = cell.project(x1)
    Jac = np.eye(T * D)
    for t in range(1, T):
        _, J = cell.jacobian(h[t - 1], p[t])
        if diagonal_only:
            J = np.diag(np.diagonal(J))
        Jac[t * D:(t + 1) * D, (t - 1) * D:t * D] = -J
    return Jac


def newton_step_dense(cell: GRU, hflat, x1, h01, diagonal_only: bool = False) -> np.ndarray:
    """One (quasi-)Newton step h - Jac^{-1} R(h) by a dense LU solve."""
    R = system_residual(cell, hflat, x1, h01)
    Jac = system_jacobian(cell, hflat, x1, h01, diagonal_only)
    return hflat - np.linalg.solve(Jac, R)


def lm_step_dense(cell: GRU, hflat, x1, h01, lam: float, diagonal_only: bool = False) -> np.ndarray:
    """One Levenberg-Marquardt step h - (Jac^T Jac + lam I)^{-1} Jac^T R(h), dense."""
    R = system_residual(cell, hflat, x1, h01)
    Jac = system_jacobian(cell, hflat, x1, h01, diagonal_only)
    H = Jac.T @ Jac + lam * np.eye(Jac.shape[0])
    return hflat - np.linalg.solve(H, Jac.T @ R)
