"""GRU cells in float64: value, Jacobian, and the sequential rollout.

The pages run GRUs throughout ("Towards Scalable and Stable Parallelization of
Nonlinear RNNs", abstract and atlas summary "Key results"; "Parallelizing
non-linear sequential models over the sequence length", abstract; ParaRNN
summary, "Experimental Results") but print no cell equations.  This file takes
the standard GRU (Cho et al. 2014, which the DEER page cites) in the layout of
``torch.nn.GRUCell``: gate rows ordered (r, z, n), the reset gate applied to the
recurrent term of the candidate after its bias:

    r = sigmoid(W_r x + b_ir + U_r h + b_hr)
    z = sigmoid(W_z x + b_iz + U_z h + b_hz)
    g = U_n h + b_hn
    n = tanh(W_n x + b_in + r * g)
    f(h, x) = (1 - z) * n + z * h

The diagonal-recurrence variant (the "adapted" GRU of the ParaRNN abstract)
replaces every U_g h by the elementwise product u_g * h, so its Jacobian is
exactly diagonal.

Jacobian with respect to h (chain rule on the lines above):

    df/dh = diag(z)
          + diag((h - n) * z(1-z))            U_z
          + diag((1-z)(1-n^2) * r)            U_n
          + diag((1-z)(1-n^2) * g * r(1-r))   U_r
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np


def sigmoid(v):
    return 1.0 / (1.0 + np.exp(-v))


@dataclass
class GRU:
    """GRU parameters widened to float64.

    kind  'dense': w_hh is [3D, D] (blocks U_r, U_z, U_n stacked by rows).
          'diag' : w_hh is [3D]    (vectors u_r, u_z, u_n).
    """

    kind: str
    w_ih: np.ndarray  # [3D, Din]
    b_ih: np.ndarray  # [3D]
    w_hh: np.ndarray
    b_hh: np.ndarray  # [3D]

    @property
    def d(self) -> int:
        return self.b_hh.shape[0] // 3

    @classmethod
    def from_workload(cls, w) -> "GRU":
        f64 = lambda t: t.double().numpy() if hasattr(t, "double") else np.asarray(t, np.float64)
        return cls(kind=w.kind, w_ih=f64(w.w_ih), b_ih=f64(w.b_ih),
                   w_hh=f64(w.w_hh), b_hh=f64(w.b_hh))

    # -- recurrent blocks ---------------------------------------------------
    def U(self, gate: int) -> np.ndarray:
        """Recurrent block of gate 0=r, 1=z, 2=n as a D x D matrix."""
        d = self.d
        if self.kind == "dense":
            return self.w_hh[gate * d:(gate + 1) * d]
        return np.diag(self.w_hh[gate * d:(gate + 1) * d])

    def U_diag(self, gate: int) -> np.ndarray:
        """Diagonal of the recurrent block of a gate (length D)."""
        d = self.d
        if self.kind == "dense":
            return np.diagonal(self.w_hh[gate * d:(gate + 1) * d]).copy()
        return self.w_hh[gate * d:(gate + 1) * d]

    # -- the cell -------------------------------------------------------------
    def project(self, x: np.ndarray) -> np.ndarray:
        """Input pre-activations W x + b_ih for every step: [..., Din] -> [..., 3D]."""
        return x @ self.w_ih.T + self.b_ih

    def recurrent(self, h: np.ndarray) -> np.ndarray:
        """Recurrent pre-activations U h + b_hh: [..., D] -> [..., 3D]."""
        if self.kind == "dense":
            return h @ self.w_hh.T + self.b_hh
        return np.concatenate([h * self.U_diag(0), h * self.U_diag(1), h * self.U_diag(2)],
                              axis=-1) + self.b_hh

    def gates(self, h: np.ndarray, p: np.ndarray):
        """Gate values at previous state h with input pre-activations p.

        Returns r, z, g, n and f = f(h, x), each [..., D]."""
        d = self.d
        q = self.recurrent(h)
        r = sigmoid(p[..., 0:d] + q[..., 0:d])
        z = sigmoid(p[..., d:2 * d] + q[..., d:2 * d])
        g = q[..., 2 * d:3 * d]
        n = np.tanh(p[..., 2 * d:3 * d] + r * g)
        f = (1.0 - z) * n + z * h
        return r, z, g, n, f

    def step(self, h: np.ndarray, x: np.ndarray) -> np.ndarray:
        """f(h, x) for one step."""
        return self.gates(h, self.project(x))[4]

    def _row_scales(self, h, r, z, g, n):
        cz = (h - n) * z * (1.0 - z)
        cn = (1.0 - z) * (1.0 - n * n) * r
        cr = (1.0 - z) * (1.0 - n * n) * g * r * (1.0 - r)
        return cz, cn, cr

    def jacobian(self, h: np.ndarray, p: np.ndarray):
        """f and the full Jacobian df/dh at (h, p): returns f [..., D], J [..., D, D]."""
        r, z, g, n, f = self.gates(h, p)
        cz, cn, cr = self._row_scales(h, r, z, g, n)
        d = self.d
        J = (z[..., :, None] * np.eye(d)
             + cz[..., :, None] * self.U(1)
             + cn[..., :, None] * self.U(2)
             + cr[..., :, None] * self.U(0))
        return f, J

    def jacobian_diag(self, h: np.ndarray, p: np.ndarray):
        """f and the diagonal of df/dh at (h, p): returns f, a, both [..., D].

        For the diagonal cell this is the whole Jacobian; for the dense cell it
        is the quasi-Newton approximation diag(J)."""
        r, z, g, n, f = self.gates(h, p)
        cz, cn, cr = self._row_scales(h, r, z, g, n)
        a = z + cz * self.U_diag(1) + cn * self.U_diag(2) + cr * self.U_diag(0)
        return f, a


def rollout(cell: GRU, x: np.ndarray, h0: np.ndarray) -> np.ndarray:
    """Sequential evaluation h_t = f(h_{t-1}, x_t), t = 1..T, from h_0 = h0.

    x [B, T, Din], h0 [B, D] -> h [B, T, D].  This is the unique solution of the
    unrolled system every parallel solver must reach (ParaRNN summary, "Core
    Idea": the recurrence written as one equation per step)."""
    x = np.asarray(x, np.float64)
    B, T, _ = x.shape
    p = cell.project(x)
    h = np.array(h0, np.float64, copy=True)
    out = np.empty((B, T, cell.d))
    for t in range(T):
        h = cell.gates(h, p[:, t])[4]
        out[:, t] = h
    return out


def residual(cell: GRU, h: np.ndarray, x: np.ndarray, h0: np.ndarray) -> np.ndarray:
    """r_t = h_t - f(h_{t-1}, x_t) for every t (with h_0 = h0): [B, T, D]."""
    p = cell.project(np.asarray(x, np.float64))
    h = np.asarray(h, np.float64)
    h_prev = np.concatenate([np.asarray(h0, np.float64)[:, None], h[:, :-1]], axis=1)
    return h - cell.gates(h_prev, p)[4]
