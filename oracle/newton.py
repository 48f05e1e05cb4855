"""DEER (Newton) and quasi-DEER (diagonal Jacobian) on the unrolled GRU (fp64).

The method, as the pages state it:
  * the T hidden states are the unknowns of one system of nonlinear equations,
    one equation per step, h_t - f(h_{t-1}, x_t) = 0 ("ParaRNN" summary, "Core
    Idea"; "Federico Danieli" abstract; DEER poses the same states as a
    fixed-point problem, "Towards Scalable and Stable Parallelization of
    Nonlinear RNNs", abstract);
  * each Newton iteration computes the residual and the Jacobian and solves
    the linearised system ("ParaRNN" summary, "Newton's Iteration"); the
    system Jacobian is block lower-triangular (in fact block bidiagonal:
    identity on the diagonal, -J_t just below), so the solve is forward
    substitution, i.e. the linear recurrence of ``scan.affine_scan``;
  * quasi-DEER replaces each J_t by its diagonal (atlas summary, "Approach"),
    giving O(TD) memory and work per iteration at the price of more
    iterations (atlas summary, "Limitations").

Readings of what the pages leave open (also listed in the design notes):
  * initial guess h^(0)_t = 0 for every t;
  * update in absolute form: with A_t = J_t (or diag J_t) evaluated at the
    shifted guess h^(i)_{t-1} (h^(i)_0 = h0) and
    b_t = f(h^(i)_{t-1}, x_t) - A_t h^(i)_{t-1},
    the next guess is h^(i+1)_t = A_t h^(i+1)_{t-1} + b_t, h^(i+1)_0 = h0;
  * convergence: delta = max over (b, t, d) of |h^(i+1) - h^(i)|; stop with
    iters = i + 1 when delta <= tol; a non-finite value anywhere stops with
    DIVERGED; otherwise NOT_CONVERGED after max_iters iterations.  The default
    cap is T + 1: undamped Newton is exact after T iterations (each iteration
    fixes one more leading state), and one more iteration observes delta = 0.

Jacobian reuse (approximate Newton: the Jacobian recomputed only every few
steps, "ParaRNN" summary, "Newton's Iteration").  Reading: with period k,
iteration i keeps the A_t of iteration k floor(i / k) and forms b_t from the
new guess, b_t = f(h^(i)_{t-1}, x_t) - A_t h^(i)_{t-1} (the chord method in
between refreshes).  The fixed point is unchanged, and since h_0 is fixed the
first i states are still exact after i iterations.
"""
from __future__ import annotations

import numpy as np

from .cells import GRU
from .scan import affine_scan

STATUS_OK = "OK"
STATUS_NOT_CONVERGED = "NOT_CONVERGED"
STATUS_DIVERGED = "DIVERGED"


def shifted(h: np.ndarray, h0: np.ndarray) -> np.ndarray:
    """The guess moved one step later: row t holds h_{t-1} (row 0 holds h0)."""
    return np.concatenate([np.asarray(h0, np.float64)[:, None], h[:, :-1]], axis=1)


def linearise(cell: GRU, h: np.ndarray, p: np.ndarray, h0: np.ndarray, dense: bool):
    """Scan operands of one iteration at guess h.

    Returns (A, b, f): A_t = J_t ([B,T,D,D], dense) or diag J_t ([B,T,D]),
    b_t = f_t - A_t h_{t-1}, f_t = f(h_{t-1}, x_t)."""
    hp = shifted(h, h0)
    if dense:
        f, A = cell.jacobian(hp, p)
        b = f - np.einsum("btij,btj->bti", A, hp)
    else:
        f, A = cell.jacobian_diag(hp, p)
        b = f - A * hp
    return A, b, f


def kept_operands(A_kept: np.ndarray, f: np.ndarray, hp: np.ndarray, dense: bool):
    """Scan operands with a kept Jacobian: A_t = A_kept_t and
    b_t = f_t - A_kept_t h_{t-1}, f and h_{t-1} from the current guess."""
    b = f - (np.einsum("btij,btj->bti", A_kept, hp) if dense else A_kept * hp)
    return A_kept, b


def newton_solve(cell: GRU, x: np.ndarray, h0: np.ndarray, mode: str, tol: float,
                 max_iters: int | None = None, h_init: np.ndarray | None = None,
                 record: bool = False, jac_every: int = 1) -> dict:
    """Solve the unrolled system with DEER (mode 'DEER') or quasi-DEER ('QUASI').

    For the diagonal cell the Jacobian is diagonal, so both modes are exact
    Newton and produce identical iterates.  jac_every = k > 1 recomputes the
    Jacobian only at iterations 0, k, 2k, ... (see the module notes).

    Returns a dict: h [B,T,D], iters, status, delta (last max |dh|),
    deltas (every iteration's delta) and, when ``record``, the list of iterates.
    """
    if mode not in ("DEER", "QUASI"):
        raise ValueError(mode)
    if jac_every < 1:
        raise ValueError(jac_every)
    x = np.asarray(x, np.float64)
    h0 = np.asarray(h0, np.float64)
    B, T, _ = x.shape
    D = cell.d
    max_iters = T + 1 if max_iters is None or max_iters <= 0 else max_iters
    dense = mode == "DEER" and cell.kind == "dense"
    p = cell.project(x)
    h = np.zeros((B, T, D)) if h_init is None else np.array(h_init, np.float64, copy=True)
    deltas, iterates = [], []
    status, iters = STATUS_NOT_CONVERGED, max_iters
    A_kept = None
    for i in range(max_iters):
        with np.errstate(all="ignore"):
            A, b, f = linearise(cell, h, p, h0, dense)
            if i % jac_every == 0:
                A_kept = A
            else:
                A, b = kept_operands(A_kept, f, shifted(h, h0), dense)
            h_new = affine_scan(A, b, h0)
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
