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


def _time_parts(T, parts):
    """The documented split of the streamed calls: 128-step units weighted
    min(p + 1, parts - p, 4), largest remainder (ties to the earlier part), at
    least one unit each, the last part ending at T."""
    units = (T + 127) // 128
    w = [min(p + 1, parts - p, 4) for p in range(parts)]
    W = sum(w)
    n = [units * v // W for v in w]
    rem = sorted(range(parts), key=lambda i: (-(units * w[i] % W), i))
    for r in range(units - sum(n)):
        n[rem[r % parts]] += 1
    n = [v * 128 for v in n]
    n[-1] -= units * 128 - T
    return n


def _streamed(w, parts, **kw):
    dev = lambda t: t.cuda().contiguous()
    pin = lambda t: t.contiguous().pin_memory()
    return binding.lstm_solve_host_streamed(dev(w.w_ih), dev(w.b_ih), dev(w.u), dev(w.b_hh), pin(w.x), pin(w.c0),
                                            pin(w.h0), tol=kw.pop("tol", w.tol), parts=parts, **kw)


@pytest.mark.parametrize("B,T,d,din,dtype,parts", [(3, 1000, 64, 32, torch.float32, 3),
                                                   (2, 777, 128, 128, torch.bfloat16, 5),
                                                   (4, 300, 68, 12, torch.float32, 1)])
def test_streamed_host_solve_converges_to_rollout(B, T, d, din, dtype, parts):
    """Time parts, every sequence in each, each part started from the (c, h)
    the part before it left: converged (c, h) within 1e-4 of the fp64 rollout;
    with one part the call is the device solve (fp32 rounding)."""
    w = make_lstm_workload(B=B, T=T, d=d, din=din, x_dtype=dtype, bias_std=0.3, state_std=0.5, seed=T + parts)
    c, h, r = _streamed(w, parts)
    assert r.status == "OK" and not c.is_cuda
    cell, x, c0, h0 = _oracle(w)
    cr, hr = lstm_rollout(cell, x, c0, h0)
    assert np.max(np.abs(c.double().numpy() - cr)) <= 1e-4
    assert np.max(np.abs(h.double().numpy() - hr)) <= 1e-4
    if parts == 1:
        cd, hd, rd = _solve(w)
        assert abs(rd.iters - r.iters) <= 1
        tol = 1e-6 if rd.iters == r.iters else w.tol
        assert _same_run(cd, c, tol) and _same_run(hd, h, tol)


def test_streamed_host_solve_fixed_iterations_per_part():
    """tol 0, two iterations: each part equals the oracle's two-iteration solve
    of its window from the (c, h) the result holds at the part's start."""
    w = make_lstm_workload(B=2, T=600, d=64, din=16, x_dtype=torch.float32, bias_std=0.3, state_std=0.5, seed=9)
    parts = 4
    c, h, r = _streamed(w, parts, tol=0.0, max_iters=2)
    assert r.iters == 2 * parts and r.status == "NOT_CONVERGED"
    cell, x, c0, h0 = _oracle(w)
    gc, gh = c.double().numpy(), h.double().numpy()
    t0, cin, hin = 0, c0, h0
    for n in _time_parts(w.T, parts):
        ref = lstm_newton_solve(cell, x[:, t0:t0 + n], cin, hin, 0.0, max_iters=2, record=True)
        rc, rh = ref["iterates"][1]
        assert np.max(np.abs(gc[:, t0:t0 + n] - rc)) <= 2e-5
        assert np.max(np.abs(gh[:, t0:t0 + n] - rh)) <= 2e-5
        cin, hin = gc[:, t0 + n - 1], gh[:, t0 + n - 1]
        t0 += n
