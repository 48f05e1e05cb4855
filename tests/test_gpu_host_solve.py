"""GPU parity of the host-buffer solve (inputs and states in page-locked host
memory, the batch solved in parts with the copies overlapped) vs the oracle.

The parts are independent solves, so:
  * with one part the call runs the device solve on the same batch and its
    states equal the device call's to fp32 rounding (the look-back's
    association order follows timing);
  * with a fixed iteration count (tol 0) every sequence's iterate depends on
    that sequence alone and matches the oracle's iterate within the family's
    tolerance (5e-5 max-abs, as for the device path);
  * converged states match the fp64 rollout within 1e-4 whatever the split.
"""
import numpy as np
import pytest
import torch

import oracle
from oracle.cells import GRU, rollout
from newton_solve_nonlinear_b200 import binding
from newton_solve_nonlinear_b200.inputs import make_workload

pytestmark = pytest.mark.gpu


def _same_run(a, b, atol=1e-6):
    """Two launches of the same solve agree to within fp32 rounding: the
    decoupled look-back composes the later tiles' maps in an order set by
    timing (how far back the first finished prefix lies), so the last bits
    may differ from one launch to the next."""
    return float((a.double().cpu() - b.double().cpu()).abs().max()) <= atol


def _weights(w):
    dev = lambda t: t.cuda().contiguous()
    return dev(w.w_ih), dev(w.b_ih), dev(w.w_hh), dev(w.b_hh)


def _host_solve(w, mode, parts, **kw):
    x = w.x.contiguous().pin_memory()
    h0 = w.h0.float().contiguous().pin_memory()
    kw.setdefault("tol", w.tol)
    return binding.newton_solve_host(*_weights(w), x, h0, kind=w.kind, mode=mode, parts=parts, **kw)


def _oracle(w):
    return GRU.from_workload(w), w.x.double().numpy(), w.h0.double().numpy()


def test_one_part_equals_device_solve():
    w = make_workload("untrained", B=3, T=2500, h0_std=0.5)
    r_host = _host_solve(w, "QUASI", 1)
    r_dev = binding.solve_workload(w, "QUASI")
    assert r_host.status == r_dev.status == "OK"
    assert abs(r_host.iters - r_dev.iters) <= 1
    assert not r_host.h.is_cuda
    assert _same_run(r_host.h, r_dev.h, atol=1e-6 if r_host.iters == r_dev.iters else w.tol)


@pytest.mark.parametrize("name,over,mode,lam", [
    ("untrained", dict(B=5, T=3000, h0_std=0.5), "QUASI", 0.0),
    ("untrained", dict(B=4, T=1000, x_dtype=torch.bfloat16, w_dtype=torch.bfloat16), "DEER", 0.0),
    ("dense_deer", dict(B=3, T=1500, bias_std=0.2), "DEER", 0.0),
    ("near_unstable", dict(B=3, T=400), "QUASI_ELK", 0.5),
    ("near_unstable", dict(B=3, T=200), "ELK", 0.3),
])
@pytest.mark.parametrize("parts", [2, 3])
def test_fixed_iterations_match_oracle(name, over, mode, lam, parts):
    w = make_workload(name, **over)
    c, x, h0 = _oracle(w)
    if mode in ("ELK", "QUASI_ELK"):
        ref = oracle.elk_solve(c, x, h0, mode, lam, 0.0, max_iters=2, record=True)
    else:
        ref = oracle.newton_solve(c, x, h0, mode, 0.0, max_iters=2, record=True)
    r = _host_solve(w, mode, parts, tol=0.0, max_iters=2, lam=lam)
    assert r.iters == 2 and r.status == "NOT_CONVERGED"
    err = np.max(np.abs(r.h.double().numpy() - ref["iterates"][1]))
    assert err <= 5e-5, err


@pytest.mark.parametrize("name,over,mode,parts", [
    ("untrained", dict(B=5, T=3000, h0_std=0.5), "QUASI", 5),
    ("untrained", dict(B=7, T=777, bias_std=0.3), "DEER", 3),
    ("diag", dict(B=3, T=500, d=128, din=128), "DEER", 2),
    ("diag", dict(B=2, T=300, d=256, din=256), "QUASI", 2),
    ("dense_deer", dict(B=3, T=2000), "DEER", 3),
])
def test_converged_states_match_rollout(name, over, mode, parts):
    w = make_workload(name, **over)
    c, x, h0 = _oracle(w)
    r = _host_solve(w, mode, parts)
    assert r.status == "OK"
    assert np.max(np.abs(r.h.double().numpy() - rollout(c, x, h0))) <= 1e-4


def test_parts_clamped_and_caller_buffer_used():
    w = make_workload("untrained", B=2, T=300)
    out = torch.full((2, 300, 64), float("nan")).pin_memory()
    r = _host_solve(w, "QUASI", 9, out=out)
    assert r.h.data_ptr() == out.data_ptr() and r.status == "OK"
    c, x, h0 = _oracle(w)
    assert np.max(np.abs(out.double().numpy() - rollout(c, x, h0))) <= 1e-4


def test_device_tensor_rejected():
    w = make_workload("untrained", B=2, T=64)
    with pytest.raises(ValueError):
        binding.newton_solve_host(*_weights(w), w.x.cuda(), w.h0.float(), kind=w.kind,
                                  mode="QUASI", tol=w.tol)


# ---- the streamed solve: time parts, every sequence in each part ----------

def _time_parts(T, parts):
    """The documented split: 128-step units weighted min(p + 1, parts - p, 4),
    largest remainder (ties to the earlier part), at least one unit each, the
    last part ending at T."""
    units = (T + 127) // 128
    w = [min(p + 1, parts - p, 4) for p in range(parts)]
    W = sum(w)
    n = [units * v // W for v in w]
    rem = sorted(range(parts), key=lambda i: (-(units * w[i] % W), i))
    for r in range(units - sum(n)):
        n[rem[r % parts]] += 1
    for i in range(parts):
        while n[i] == 0:
            j = max(range(parts), key=lambda q: (n[q], -q))
            n[j] -= 1
            n[i] += 1
    n = [v * 128 for v in n]
    n[-1] -= units * 128 - T
    return n


def _streamed(w, mode, parts, **kw):
    x = w.x.contiguous().pin_memory()
    h0 = w.h0.float().contiguous().pin_memory()
    kw.setdefault("tol", w.tol)
    return binding.newton_solve_host_streamed(*_weights(w), x, h0, kind=w.kind, mode=mode, parts=parts, **kw)


def test_streamed_one_part_equals_device_solve():
    w = make_workload("untrained", B=3, T=2500, h0_std=0.5)
    r = _streamed(w, "QUASI", 1)
    r_dev = binding.solve_workload(w, "QUASI")
    assert r.status == r_dev.status == "OK" and abs(r.iters - r_dev.iters) <= 1
    assert _same_run(r.h, r_dev.h, atol=1e-6 if r.iters == r_dev.iters else w.tol)


@pytest.mark.parametrize("name,over,mode,lam,parts", [
    ("untrained", dict(B=3, T=1000, h0_std=0.5), "QUASI", 0.0, 3),
    ("dense_deer", dict(B=2, T=1500, bias_std=0.2), "DEER", 0.0, 4),
    ("near_unstable", dict(B=2, T=700), "QUASI_ELK", 0.5, 3),
    ("diag", dict(B=2, T=900, d=128, din=128), "QUASI", 0.0, 5),
])
def test_streamed_fixed_iterations_match_oracle_per_part(name, over, mode, lam, parts):
    """tol 0, two iterations: each part is the oracle's two-iteration solve of
    its window, started from the state the part before it left (read from the
    result, so that each part is checked on its own)."""
    w = make_workload(name, **over)
    c, x, h0 = _oracle(w)
    r = _streamed(w, mode, parts, tol=0.0, max_iters=2, lam=lam)
    sizes = _time_parts(w.T, parts)
    assert sum(sizes) == w.T and r.iters == 2 * parts and r.status == "NOT_CONVERGED"
    got = r.h.double().numpy()
    t0, hin = 0, h0
    for n in sizes:
        if mode in ("ELK", "QUASI_ELK"):
            ref = oracle.elk_solve(c, x[:, t0:t0 + n], hin, mode, lam, 0.0, max_iters=2, record=True)
        else:
            ref = oracle.newton_solve(c, x[:, t0:t0 + n], hin, mode, 0.0, max_iters=2, record=True)
        err = np.max(np.abs(got[:, t0:t0 + n] - ref["iterates"][1]))
        assert err <= 5e-5, (t0, n, err)
        hin = got[:, t0 + n - 1]
        t0 += n


@pytest.mark.parametrize("name,over,mode,lam,parts", [
    ("untrained", dict(B=5, T=3000, h0_std=0.5), "QUASI", 0.0, 7),
    ("untrained", dict(B=4, T=1000, x_dtype=torch.bfloat16, w_dtype=torch.bfloat16), "DEER", 0.0, 3),
    ("diag", dict(B=3, T=777, d=128, din=128), "DEER", 0.0, 4),
    ("dense_deer", dict(B=3, T=2000), "DEER", 0.0, 6),
    ("near_unstable", dict(B=2, T=600), "ELK", 0.3, 2),
])
def test_streamed_converged_states_match_rollout(name, over, mode, lam, parts):
    w = make_workload(name, **over)
    c, x, h0 = _oracle(w)
    tol = 1e-6 if mode in ("ELK", "QUASI_ELK") else w.tol
    r = _streamed(w, mode, parts, lam=lam, tol=tol)
    assert r.status == "OK"
    assert np.max(np.abs(r.h.double().numpy() - rollout(c, x, h0))) <= 1e-4


def test_streamed_parts_bounds():
    w = make_workload("untrained", B=2, T=300)
    out = torch.full((2, 300, 64), float("nan")).pin_memory()
    r = _streamed(w, "QUASI", 99, out=out)  # clamped to ceil(300 / 128) = 3 parts
    assert r.h.data_ptr() == out.data_ptr() and r.status == "OK"
    c, x, h0 = _oracle(w)
    assert np.max(np.abs(out.double().numpy() - rollout(c, x, h0))) <= 1e-4
    assert binding.host_streamed_workspace_size("dense", 64, 64, 2, 300, "QUASI", 4) == 0
    assert binding.host_streamed_workspace_size("dense", 64, 64, 2, 300, "QUASI", 3) > 0


@pytest.mark.parametrize("name,over,mode,parts", [("untrained", {}, "QUASI", 7),
                                                  ("diag", {}, "QUASI", 7)])
def test_streamed_full_size_sampled(name, over, mode, parts):
    """The streamed host-buffer solve at the benchmark's full size and part
    count (the call the end-to-end number goes through): every part converged,
    whole sampled sequences within 1e-4 of the fp64 rollout."""
    w = make_workload(name, **over)
    r = _streamed(w, mode, parts)
    assert r.status == "OK"
    c = GRU.from_workload(w)
    for b in (0, w.B - 1):
        want = rollout(c, w.x[b:b + 1].double().numpy(), w.h0[b:b + 1].double().numpy())
        assert np.max(np.abs(r.h[b:b + 1].double().numpy() - want)) <= 1e-4


def test_concurrent_host_calls_on_two_streams():
    """Two host-buffer solves running at once from two host threads on two
    streams: each call takes its own set of helper streams (the per-device
    cache hands a set to one call at a time) and both results are right."""
    import threading
    ws_ = [make_workload("untrained", B=2, T=1500, h0_std=0.5, seed=s) for s in (1, 2)]
    outs, errs = [None, None], []

    def run(i):
        try:
            with torch.cuda.stream(torch.cuda.Stream()):
                s = torch.cuda.current_stream()
                outs[i] = _streamed(ws_[i], "QUASI", 3, stream=s) if i == 0 else _host_solve(ws_[i], "QUASI", 2,
                                                                                           stream=s)
        except Exception as e:  # reported on the main thread
            errs.append(e)

    th = [threading.Thread(target=run, args=(i,)) for i in (0, 1)]
    for t in th:
        t.start()
    for t in th:
        t.join()
    assert not errs, errs
    for w, r in zip(ws_, outs):
        assert r.status == "OK"
        c, x, h0 = _oracle(w)
        assert np.max(np.abs(r.h.double().numpy() - rollout(c, x, h0))) <= 1e-4
