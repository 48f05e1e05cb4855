"""Gradients through an evaluated sequence: the backward pass of training.

TEST INFRASTRUCTURE ONLY (see the package docstring): the product path never
imports this file.

The pages evaluate the GRU in order to train it (the ParaRNN talk page,
"Federico Danieli", Abstract; "Towards Scalable and Stable Parallelization of
Nonlinear RNNs", atlas summary, table "Measured effects reported in the paper":
training with the diagonal Jacobian approximation in the backward pass as
well).  The pages print no backward equations; this file states the plain
chain rule on the unrolled system.

The evaluated states solve h_t = f(h_{t-1}, p_t), t = 1..T, with h_0 given and
p_t = W_ih x_t + b_ih.  For a loss with upstream gradients g_t = dL/dh_t (the
partial derivatives, holding the other states fixed), the total derivatives
lam_t = dL/dh_t obey, backwards in time,

    lam_T = g_T,    lam_t = g_t + J_{t+1}^T lam_{t+1},

where J_{t+1} = df/dh at step t+1 (evaluated at h_t, p_{t+1}).  Then, with the
per-step partials of f (all of them diagonal in the lane index i):

    df_i/dp_{r,i} = (1 - z_i)(1 - n_i^2) g_i r_i (1 - r_i)
    df_i/dp_{z,i} = (h_{t-1,i} - n_i) z_i (1 - z_i)
    df_i/dp_{n,i} = (1 - z_i)(1 - n_i^2)           (g = U_n h_{t-1} + b_hn)

    dL/dp_t      = those three times lam_t                  [3D per step]
    dL/dh_0      = J_1^T lam_1
    dL/db_hh     = sum_t (dL/dp_{r,t}, dL/dp_{z,t}, dL/dp_{n,t} * r_t)
    dL/dU_g      = sum_t (the same three) (outer) h_{t-1}   (dense: [D, D] per gate;
                   diagonal cell: the elementwise product, [D] per gate)
    dL/dW_ih     = sum_t dL/dp_t (outer) x_t,   dL/db_ih = sum_t dL/dp_t,
    dL/dx_t      = W_ih^T dL/dp_t.

``jacobian='diag'`` replaces J_{t+1}^T by its diagonal in the lam recurrence
(the pages' quasi backward pass); for the diagonal-recurrence cell the two are
the same, since its Jacobian is diagonal.
"""
from __future__ import annotations

import numpy as np

from .cells import GRU


def step_partials(cell: GRU, h_prev: np.ndarray, p: np.ndarray):
    """Partials of one step at (h_prev, p), each [..., D]: df/dp_r, df/dp_z,
    df/dp_n, the reset gate r, and the step's value f."""
    r, z, g, n, f = cell.gates(h_prev, p)
    dn = (1.0 - z) * (1.0 - n * n)
    return dn * g * r * (1.0 - r), (h_prev - n) * z * (1.0 - z), dn, r, f


def adjoint(cell: GRU, x: np.ndarray, h0: np.ndarray, h: np.ndarray, g: np.ndarray,
            jacobian: str = "exact") -> dict:
    """Gradients of a loss through the evaluated states h (the rollout, or a
    converged Newton solve) given its upstream gradients g = dL/dh.

    x [B, T, Din], h0 [B, D], h [B, T, D], g [B, T, D] (float64).  Returns a dict:
    lam [B,T,D], dP [B,T,3D], dh0 [B,D], dw_hh (dense [3D,D], diagonal [3D]),
    db_hh [3D], dw_ih [3D,Din], db_ih [3D], dx [B,T,Din]."""
    if jacobian not in ("exact", "diag"):
        raise ValueError(jacobian)
    B, T, _ = x.shape
    d = cell.d
    P = cell.project(x)
    h_prev = np.concatenate([h0[:, None, :], h[:, :-1, :]], axis=1)  # h_{t-1}, t = 1..T
    lam = np.zeros_like(h)
    # backwards in time: lam_t = g_t + J_{t+1}^T lam_{t+1}
    carry = np.zeros((B, d))
    for t in range(T - 1, -1, -1):
        lam[:, t] = g[:, t] + carry
        if jacobian == "exact":
            _, J = cell.jacobian(h_prev[:, t], P[:, t])          # J_t [B, D, D]
            carry = np.einsum("bij,bi->bj", J, lam[:, t])        # J_t^T lam_t
        else:
            _, a = cell.jacobian_diag(h_prev[:, t], P[:, t])
            carry = a * lam[:, t]
    dh0 = carry  # J_1^T lam_1
    fr, fz, fn, r, _ = step_partials(cell, h_prev, P)
    dP = np.concatenate([fr * lam, fz * lam, fn * lam], axis=-1)
    grow = np.concatenate([fr * lam, fz * lam, fn * r * lam], axis=-1)  # d/d(recurrent pre-activation)
    db_hh = grow.sum(axis=(0, 1))
    if cell.kind == "dense":
        dw_hh = np.einsum("btk,btj->kj", grow, h_prev)
    else:
        dw_hh = (grow * np.concatenate([h_prev] * 3, axis=-1)).sum(axis=(0, 1))
    dw_ih = np.einsum("btk,bti->ki", dP, x)
    db_ih = dP.sum(axis=(0, 1))
    dx = dP @ cell.w_ih
    return dict(lam=lam, dP=dP, dh0=dh0, dw_hh=dw_hh, db_hh=db_hh, dw_ih=dw_ih, db_ih=db_ih, dx=dx)
