"""GPU parity of the diagonal-recurrence LSTM solve (exact Newton over 2x2
lane blocks) against the fp64 oracle.

Tolerances (as for the GRU paths): single iterations element by element
within 2e-5 of the oracle's iterates (fp32 cell, 2x2 scan over <= 32-step tiles
and look-back); converged (c, h) within 1e-4 of the fp64 rollout; iteration
counts within 1 of the oracle's.
"""
import numpy as np
import pytest
import torch

from oracle.lstm import LSTM, lstm_newton_solve, lstm_rollout
from newton_solve_nonlinear_b200 import binding
from newton_solve_nonlinear_b200.inputs import make_lstm_workload

pytestmark = pytest.mark.gpu


def _same_run(a, b, atol=1e-6):
    """Two launches of the same solve agree to within fp32 rounding: the
    decoupled look-back composes the later tiles' maps in an order set by
    timing (how far back the first finished prefix lies), so the last bits
    may differ from one launch to the next."""
    return float((a.double().cpu() - b.double().cpu()).abs().max()) <= atol


def _oracle(w):
    c = LSTM(w_ih=w.w_ih.double().numpy(), b_ih=w.b_ih.double().numpy(), u=w.u.double().numpy(),
             b_hh=w.b_hh.double().numpy())
    return c, w.x.double().numpy(), w.c0.double().numpy(), w.h0.double().numpy()


def _solve(w, **kw):
    dev = lambda t: t.cuda().contiguous()
    return binding.lstm_solve(dev(w.w_ih), dev(w.b_ih), dev(w.u), dev(w.b_hh), dev(w.x), dev(w.c0), dev(w.h0),
                              tol=kw.pop("tol", w.tol), **kw)


@pytest.mark.parametrize("B,T,d,din", [(2, 300, 64, 16), (1, 1, 4, 3), (3, 100, 96, 8), (2, 257, 128, 64)])
def test_each_iteration_matches_oracle(B, T, d, din):
    w = make_lstm_workload(B=B, T=T, d=d, din=din, x_dtype=torch.float32, bias_std=0.3, state_std=0.5,
                           seed=B + T + d)
    cell, x, c0, h0 = _oracle(w)
    ref = lstm_newton_solve(cell, x, c0, h0, 0.0, max_iters=3, record=True)
    for n in (1, 2, 3):
        c, h, r = _solve(w, tol=0.0, max_iters=n)
        if T > 1 or n == 1:
            assert r.iters == n, (r.iters, n)
        rc, rh = ref["iterates"][min(n, len(ref["iterates"])) - 1]
        assert np.max(np.abs(c.double().cpu().numpy() - rc)) <= 2e-5
        assert np.max(np.abs(h.double().cpu().numpy() - rh)) <= 2e-5


@pytest.mark.parametrize("B,T,d,din,dtype", [(2, 2000, 64, 32, torch.float32), (4, 1000, 128, 128, torch.bfloat16),
                                             (1, 777, 68, 12, torch.float32)])
def test_converges_to_rollout(B, T, d, din, dtype):
    w = make_lstm_workload(B=B, T=T, d=d, din=din, x_dtype=dtype, bias_std=0.3, state_std=0.5, seed=T)
    cell, x, c0, h0 = _oracle(w)
    c, h, r = _solve(w)
    assert r.status == "OK"
    cr, hr = lstm_rollout(cell, x, c0, h0)
    assert np.max(np.abs(c.double().cpu().numpy() - cr)) <= 1e-4
    assert np.max(np.abs(h.double().cpu().numpy() - hr)) <= 1e-4
    ref = lstm_newton_solve(cell, x, c0, h0, w.tol)
    assert abs(r.iters - ref["iters"]) <= 1, (r.iters, ref["iters"])


def test_full_size_sampled():
    """The benchmark size (B = 8, T = 4096, D = 2048, bf16 x and W_ih): every
    state against the rollout on 64 lanes (the cell is separable by lane)."""
    w = make_lstm_workload()
    c, h, r = _solve(w)
    assert r.status == "OK"
    lanes = np.arange(0, 2048, 32)
    idx4 = np.concatenate([lanes + k * 2048 for k in range(4)])
    sub = LSTM(w_ih=w.w_ih.double().numpy()[idx4], b_ih=w.b_ih.double().numpy()[idx4],
               u=w.u.double().numpy()[idx4], b_hh=w.b_hh.double().numpy()[idx4])
    cr, hr = lstm_rollout(sub, w.x.double().numpy(), w.c0.double().numpy()[:, lanes], w.h0.double().numpy()[:, lanes])
    assert np.max(np.abs(c.double().cpu().numpy()[..., lanes] - cr)) <= 1e-4
    assert np.max(np.abs(h.double().cpu().numpy()[..., lanes] - hr)) <= 1e-4


def test_statuses_and_rejections():
    w = make_lstm_workload(B=1, T=50, d=8, din=4, x_dtype=torch.float32)
    w.x[0, 10, 1] = float("nan")
    c, h, r = _solve(w)
    assert r.status == "DIVERGED" and r.iters == 1
    w = make_lstm_workload(B=1, T=50, d=8, din=4, x_dtype=torch.float32)
    c, h, r = _solve(w, tol=0.0, max_iters=2)
    assert r.status == "NOT_CONVERGED" and r.iters == 2
    assert binding.lstm_workspace_size(4, 6, 1, 50) == 0  # d % 4 != 0


@pytest.mark.parametrize("B,T,d,din,parts", [(5, 400, 64, 32, 3), (4, 300, 128, 64, 4), (3, 200, 64, 16, 1)])
def test_host_buffer_solve(B, T, d, din, parts):
    """From and to host memory in ramped parts: with one part the states equal
    the device solve's to fp32 rounding; in any split the parts are independent
    solves, so the converged (c, h) match the fp64 rollout within 1e-4."""
    w = make_lstm_workload(B=B, T=T, d=d, din=din, x_dtype=torch.float32, bias_std=0.3, state_std=0.5, seed=B * T)
    dev = lambda t: t.cuda().contiguous()
    pin = lambda t: t.contiguous().pin_memory()
    c, h, r = binding.lstm_solve_host(dev(w.w_ih), dev(w.b_ih), dev(w.u), dev(w.b_hh), pin(w.x), pin(w.c0),
                                      pin(w.h0), tol=w.tol, parts=parts)
    assert r.status == "OK" and not c.is_cuda and not h.is_cuda
    cell, x, c0, h0 = _oracle(w)
    cr, hr = lstm_rollout(cell, x, c0, h0)
    assert np.max(np.abs(c.double().numpy() - cr)) <= 1e-4
    assert np.max(np.abs(h.double().numpy() - hr)) <= 1e-4
    if parts == 1:
        cd, hd, rd = _solve(w)
        assert abs(rd.iters - r.iters) <= 1
        tol = 1e-6 if rd.iters == r.iters else w.tol
        assert _same_run(cd, c, tol) and _same_run(hd, h, tol)
