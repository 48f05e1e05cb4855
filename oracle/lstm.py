"""The diagonal-recurrence LSTM in float64: cell, 2x2-per-lane Jacobian,
sequential rollout and exact Newton (DEER) on the unrolled system.

TEST INFRASTRUCTURE ONLY (see the package docstring).

The pages apply the parallel Newton solve to "adaptations" of LSTM and GRU
(ParaLSTM, ParaGRU: the ParaRNN talk page "Federico Danieli", Abstract; the
ParaRNN summary page, "Experimental Results") but print no cell equations.
Reading: the standard LSTM in the layout of ``torch.nn.LSTMCell`` (gate rows
i, f, g, o), with the recurrent matrices replaced by vectors, as the adapted
GRU does (u_k * h instead of U_k h):

    i = sigmoid(p_i + u_i h + b_i)      f = sigmoid(p_f + u_f h + b_f)
    g = tanh(p_g + u_g h + b_g)         o = sigmoid(p_o + u_o h + b_o)
    c' = f c + i g                      h' = o tanh(c')

with p = W_ih x + b_ih and b = b_hh.  The state is s = (c, h); lane j of s'
depends only on lane j of s, so the Jacobian is a 2x2 block per lane:

    dc'/dc = f
    dc'/dh = c f(1-f) u_f + g i(1-i) u_i + i (1-g^2) u_g
    dh'/dc = o (1 - tanh(c')^2) f
    dh'/dh = tanh(c') o(1-o) u_o + o (1 - tanh(c')^2) dc'/dh

Newton's step on the unrolled system s_t = F(s_{t-1}, x_t) (the ParaRNN
summary page, "Core Idea" and "Newton's Iteration") is then the linear
recurrence s_t = A_t s_{t-1} + b_t with 2x2 blocks A_t (exact Newton).
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

from .cells import sigmoid


@dataclass
class LSTM:
    """Diagonal-recurrence LSTM parameters in float64: w_ih [4D, Din], b_ih [4D],
    u [4D] (recurrent vectors of the gates i, f, g, o), b_hh [4D]."""

    w_ih: np.ndarray
    b_ih: np.ndarray
    u: np.ndarray
    b_hh: np.ndarray

    @property
    def d(self) -> int:
        return self.b_hh.shape[0] // 4

    def project(self, x: np.ndarray) -> np.ndarray:
        """Input pre-activations W x + b_ih for every step: [..., Din] -> [..., 4D]."""
        return x @ self.w_ih.T + self.b_ih

    def gates(self, c: np.ndarray, h: np.ndarray, p: np.ndarray):
        """Gates at state (c, h) with input pre-activations p: i, f, g, o, c', h'."""
        d = self.d
        u, b = self.u, self.b_hh
        i = sigmoid(p[..., 0:d] + u[0:d] * h + b[0:d])
        f = sigmoid(p[..., d:2 * d] + u[d:2 * d] * h + b[d:2 * d])
        g = np.tanh(p[..., 2 * d:3 * d] + u[2 * d:3 * d] * h + b[2 * d:3 * d])
        o = sigmoid(p[..., 3 * d:4 * d] + u[3 * d:4 * d] * h + b[3 * d:4 * d])
        c2 = f * c + i * g
        h2 = o * np.tanh(c2)
        return i, f, g, o, c2, h2

    def step(self, c, h, p):
        """F(s, x): the next state (c', h')."""
        return self.gates(c, h, p)[4:]

    def jacobian(self, c, h, p):
        """The next state and its 2x2 Jacobian per lane: returns c', h', and
        A [..., D, 2, 2] with rows (c', h') and columns (c, h)."""
        d = self.d
        u = self.u
        i, f, g, o, c2, h2 = self.gates(c, h, p)
        tc = np.tanh(c2)
        dcc = f
        dch = c * f * (1 - f) * u[d:2 * d] + g * i * (1 - i) * u[0:d] + i * (1 - g * g) * u[2 * d:3 * d]
        dhc = o * (1 - tc * tc) * f
        dhh = tc * o * (1 - o) * u[3 * d:4 * d] + o * (1 - tc * tc) * dch
        A = np.stack([np.stack([dcc, dch], -1), np.stack([dhc, dhh], -1)], -2)
        return c2, h2, A


def lstm_rollout(cell: LSTM, x: np.ndarray, c0: np.ndarray, h0: np.ndarray):
    """Sequential evaluation s_t = F(s_{t-1}, x_t): x [B,T,Din], c0, h0 [B,D] ->
    c, h [B,T,D].  The unique answer every solver must reach."""
    P = cell.project(x)
    B, T, _ = x.shape
    c, h = c0, h0
    cs, hs = np.empty((B, T, cell.d)), np.empty((B, T, cell.d))
    for t in range(T):
        c, h = cell.step(c, h, P[:, t])
        cs[:, t], hs[:, t] = c, h
    return cs, hs


def lstm_newton_solve(cell: LSTM, x: np.ndarray, c0: np.ndarray, h0: np.ndarray, tol: float,
                      max_iters: int | None = None, record: bool = False) -> dict:
    """Exact Newton (DEER) on the unrolled LSTM.

    The guess starts at zero (c = h = 0 for every step).  Iteration i linearises
    F at the guess shifted by one step (s_0 fixed), A_t = dF/ds and
    b_t = F(s^(i)_{t-1}) - A_t s^(i)_{t-1}, then solves s^(i+1)_t =
    A_t s^(i+1)_{t-1} + b_t by forward substitution.  It stops when
    max |s^(i+1) - s^(i)| over both halves of the state, every lane, step and
    sequence is at most tol (OK), or on a non-finite value (DIVERGED), or after
    max_iters (default T + 1) iterations (NOT_CONVERGED).
    Returns dict(c, h, iters, status, deltas[, iterates (c, h) per iteration])."""
    P = cell.project(x)
    B, T, _ = x.shape
    d = cell.d
    max_iters = T + 1 if not max_iters or max_iters <= 0 else max_iters
    c = np.zeros((B, T, d))
    h = np.zeros((B, T, d))
    deltas, iterates = [], []
    status = "NOT_CONVERGED"
    it = 0
    for it in range(1, max_iters + 1):
        cp = np.concatenate([c0[:, None], c[:, :-1]], 1)  # s^(i)_{t-1}
        hp = np.concatenate([h0[:, None], h[:, :-1]], 1)
        fc, fh, A = cell.jacobian(cp, hp, P)
        bc = fc - (A[..., 0, 0] * cp + A[..., 0, 1] * hp)
        bh = fh - (A[..., 1, 0] * cp + A[..., 1, 1] * hp)
        nc, nh = np.empty_like(c), np.empty_like(h)
        sc, sh = c0, h0
        for t in range(T):  # forward substitution, 2x2 per lane
            sc, sh = (A[:, t, :, 0, 0] * sc + A[:, t, :, 0, 1] * sh + bc[:, t],
                      A[:, t, :, 1, 0] * sc + A[:, t, :, 1, 1] * sh + bh[:, t])
            nc[:, t], nh[:, t] = sc, sh
        if not (np.all(np.isfinite(nc)) and np.all(np.isfinite(nh))):
            c, h = nc, nh
            status = "DIVERGED"
            deltas.append(float("inf"))
            break
        delta = float(max(np.max(np.abs(nc - c)), np.max(np.abs(nh - h))))
        c, h = nc, nh
        deltas.append(delta)
        if record:
            iterates.append((c.copy(), h.copy()))
        if delta <= tol:
            status = "OK"
            break
    out = dict(c=c, h=h, iters=it, status=status, deltas=deltas)
    if record:
        out["iterates"] = iterates
    return out
