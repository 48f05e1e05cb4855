"""Pins of the oracle's diagonal-recurrence LSTM (CPU only).

The cell is tied to torch.nn.LSTMCell in fp64 (a library routine, with the
recurrent matrices set to diagonal blocks), the 2x2 lane Jacobian to central
differences, and one Newton iteration to a brute-force Newton step on the
whole unrolled system (its Jacobian by finite differences of the residual,
solved densely), so a wrong entry or a transposed 2x2 block in the
substitution fails; the converged solve equals the rollout.
"""
import numpy as np
import pytest
import torch

from oracle.lstm import LSTM, lstm_newton_solve, lstm_rollout


def _rand_lstm(din, d, seed, scale=0.5):
    rng = np.random.default_rng(seed)
    return LSTM(w_ih=rng.normal(0, scale, (4 * d, din)), b_ih=rng.normal(0, 0.3, 4 * d),
                u=rng.uniform(-1, 1, 4 * d), b_hh=rng.normal(0, 0.3, 4 * d))


def _torch_cell(c: LSTM, din):
    d = c.d
    m = torch.nn.LSTMCell(din, d).double()
    with torch.no_grad():
        m.weight_ih.copy_(torch.from_numpy(c.w_ih))
        m.bias_ih.copy_(torch.from_numpy(c.b_ih))
        m.bias_hh.copy_(torch.from_numpy(c.b_hh))
        m.weight_hh.copy_(torch.from_numpy(np.concatenate([np.diag(c.u[k * d:(k + 1) * d]) for k in range(4)], 0)))
    return m


def test_cell_equals_torch_lstmcell():
    din, d = 5, 7
    c = _rand_lstm(din, d, seed=1)
    rng = np.random.default_rng(2)
    x = rng.normal(size=(11, din))
    cc = rng.normal(size=(11, d))
    hh = rng.normal(size=(11, d))
    with torch.no_grad():
        h_ref, c_ref = _torch_cell(c, din)(torch.from_numpy(x), (torch.from_numpy(hh), torch.from_numpy(cc)))
    c2, h2 = c.step(cc, hh, c.project(x))
    np.testing.assert_allclose(c2, c_ref.numpy(), rtol=0, atol=1e-14)
    np.testing.assert_allclose(h2, h_ref.numpy(), rtol=0, atol=1e-14)


def test_jacobian_central_differences():
    din, d = 3, 6
    c = _rand_lstm(din, d, seed=3)
    rng = np.random.default_rng(4)
    p = c.project(rng.normal(size=(4, din)))
    cc, hh = rng.normal(size=(4, d)), rng.normal(size=(4, d))
    _, _, A = c.jacobian(cc, hh, p)
    eps = 1e-6
    for col, (dc, dh) in enumerate([(eps, 0.0), (0.0, eps)]):
        cp, hp = c.step(cc + dc, hh + dh, p)
        cm, hm = c.step(cc - dc, hh - dh, p)
        np.testing.assert_allclose(A[..., 0, col], (cp - cm) / (2 * eps), rtol=1e-6, atol=1e-8)
        np.testing.assert_allclose(A[..., 1, col], (hp - hm) / (2 * eps), rtol=1e-6, atol=1e-8)


def test_one_newton_iteration_equals_brute_force_step():
    """From the zero guess, one iteration equals s - J_R^{-1} R(s) for the whole
    system R(s)_t = s_t - F(s_{t-1}), J_R by central differences of R."""
    din, d, T = 2, 3, 5
    c = _rand_lstm(din, d, seed=5)
    rng = np.random.default_rng(6)
    x = rng.normal(size=(1, T, din))
    c0, h0 = rng.normal(size=(1, d)), rng.normal(size=(1, d))
    P = c.project(x)[0]

    def residual(s):  # s: [T, 2, d] = (c_t, h_t), flattened
        s = s.reshape(T, 2, d)
        r = np.empty_like(s)
        pc, ph = c0[0], h0[0]
        for t in range(T):
            fc, fh = c.step(pc, ph, P[t])
            r[t, 0], r[t, 1] = s[t, 0] - fc, s[t, 1] - fh
            pc, ph = s[t, 0], s[t, 1]
        return r.ravel()

    s0 = np.zeros((T, 2, d))
    n = s0.size
    J = np.empty((n, n))
    eps = 1e-6
    for k in range(n):
        e = np.zeros(n)
        e[k] = eps
        J[:, k] = (residual(s0.ravel() + e) - residual(s0.ravel() - e)) / (2 * eps)
    s1 = s0.ravel() - np.linalg.solve(J, residual(s0.ravel()))
    s1 = s1.reshape(T, 2, d)
    r = lstm_newton_solve(c, x, c0, h0, 0.0, max_iters=1, record=True)
    ci, hi = r["iterates"][0]
    np.testing.assert_allclose(ci[0], s1[:, 0], rtol=1e-7, atol=1e-8)
    np.testing.assert_allclose(hi[0], s1[:, 1], rtol=1e-7, atol=1e-8)


def test_newton_recovers_steps_and_converges_to_rollout():
    din, d, B, T = 3, 4, 2, 30
    c = _rand_lstm(din, d, seed=7)
    rng = np.random.default_rng(8)
    x = rng.normal(size=(B, T, din))
    c0, h0 = rng.normal(0, 0.5, (B, d)), rng.normal(0, 0.5, (B, d))
    cr, hr = lstm_rollout(c, x, c0, h0)
    r = lstm_newton_solve(c, x, c0, h0, 0.0, max_iters=4, record=True)
    for i, (ci, hi) in enumerate(r["iterates"], start=1):  # steps 1..i are exact after i iterations
        np.testing.assert_allclose(ci[:, :i], cr[:, :i], rtol=0, atol=1e-12)
        np.testing.assert_allclose(hi[:, :i], hr[:, :i], rtol=0, atol=1e-12)
    r = lstm_newton_solve(c, x, c0, h0, 1e-12)
    assert r["status"] == "OK" and r["iters"] <= T + 1
    np.testing.assert_allclose(r["c"], cr, rtol=0, atol=1e-10)
    np.testing.assert_allclose(r["h"], hr, rtol=0, atol=1e-10)


def test_newton_diverges_on_nan_and_stops_at_cap():
    c = _rand_lstm(2, 3, seed=9)
    x = np.random.default_rng(10).normal(size=(1, 20, 2))
    x[0, 5, 1] = np.nan
    r = lstm_newton_solve(c, x, np.zeros((1, 3)), np.zeros((1, 3)), 1e-6)
    assert r["status"] == "DIVERGED" and r["iters"] == 1
    x[0, 5, 1] = 0.0
    r = lstm_newton_solve(c, x, np.zeros((1, 3)), np.zeros((1, 3)), 0.0, max_iters=3)
    assert r["status"] == "NOT_CONVERGED" and r["iters"] == 3
