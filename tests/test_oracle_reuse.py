"""Pins of the oracle's Jacobian reuse (CPU only).

Approximate Newton with the Jacobian recomputed only every k iterations (the
"ParaRNN" summary, "Newton's Iteration") is, on the whole unrolled system
R(h)_t = h_t - f(h_{t-1}, x_t), the chord method between refreshes:
h^(i+1) = h^(i) - J_R(h^(i0))^{-1} R(h^(i)), i0 = k floor(i / k).  The pin
builds J_R by central differences of R (the quasi variant keeps only the
diagonal of each sub-diagonal block), solves densely, and compares every
iterate; a mistake in which Jacobian or which guess enters b_t fails it.
"""
import numpy as np
import pytest

from oracle import brute, newton
from oracle.cells import GRU, rollout


def _rand_gru(kind, din, d, seed, scale=0.8):
    rng = np.random.default_rng(seed)
    w_hh = rng.normal(0, scale, (3 * d, d)) if kind == "dense" else rng.uniform(-1, 1, 3 * d)
    return GRU(kind=kind, w_ih=rng.normal(0, scale, (3 * d, din)), b_ih=rng.normal(0, 0.3, 3 * d),
               w_hh=w_hh, b_hh=rng.normal(0, 0.3, 3 * d))


def _chord_iterates(c, x, h0, k, n, diagonal_only):
    T, D = x.shape[1], c.d
    h = np.zeros(T * D)
    out, J = [], None
    for i in range(n):
        if i % k == 0:
            J = brute.system_jacobian_fd(c, h, x[0], h0[0])
            if diagonal_only:  # sub-diagonal blocks: their diagonals only
                for t in range(1, T):
                    blk = J[t * D:(t + 1) * D, (t - 1) * D:t * D]
                    J[t * D:(t + 1) * D, (t - 1) * D:t * D] = np.diag(np.diag(blk))
        h = h - np.linalg.solve(J, brute.system_residual(c, h, x[0], h0[0]))
        out.append(h.reshape(1, T, D).copy())
    return out


@pytest.mark.parametrize("mode,k", [("DEER", 2), ("DEER", 3), ("DEER", 100), ("QUASI", 2), ("QUASI", 100)])
def test_reuse_iterates_equal_chord_method(mode, k):
    c = _rand_gru("dense", 2, 3, seed=31)
    rng = np.random.default_rng(32)
    T = 6
    x = rng.normal(size=(1, T, 2))
    h0 = rng.normal(0, 0.5, (1, 3))
    r = newton.newton_solve(c, x, h0, mode, 0.0, max_iters=5, record=True, jac_every=k)
    want = _chord_iterates(c, x, h0, k, 5, diagonal_only=mode == "QUASI")
    for i, (got, ref) in enumerate(zip(r["iterates"], want)):
        np.testing.assert_allclose(got, ref, rtol=0, atol=1e-8, err_msg=f"iteration {i}")


def test_reuse_period_one_is_plain_newton_and_period_changes_iterates():
    c = _rand_gru("dense", 3, 4, seed=33)
    rng = np.random.default_rng(34)
    x = rng.normal(size=(2, 12, 3))
    h0 = rng.normal(0, 0.5, (2, 4))
    r0 = newton.newton_solve(c, x, h0, "DEER", 0.0, max_iters=4, record=True)
    r1 = newton.newton_solve(c, x, h0, "DEER", 0.0, max_iters=4, record=True, jac_every=1)
    r2 = newton.newton_solve(c, x, h0, "DEER", 0.0, max_iters=4, record=True, jac_every=2)
    for a, b in zip(r0["iterates"], r1["iterates"]):
        assert np.array_equal(a, b)
    assert np.array_equal(r0["iterates"][0], r2["iterates"][0])  # iteration 0 refreshes
    assert np.max(np.abs(r0["iterates"][1] - r2["iterates"][1])) > 1e-6


@pytest.mark.parametrize("k", [2, 4])
def test_reuse_fixes_one_state_per_iteration_and_converges(k):
    c = _rand_gru("dense", 3, 4, seed=35, scale=0.5)
    rng = np.random.default_rng(36)
    B, T = 2, 25
    x = rng.normal(size=(B, T, 3))
    h0 = rng.normal(0, 0.5, (B, 4))
    ref = rollout(c, x, h0)
    r = newton.newton_solve(c, x, h0, "DEER", 0.0, max_iters=6, record=True, jac_every=k)
    for i, h in enumerate(r["iterates"], start=1):
        np.testing.assert_allclose(h[:, :i], ref[:, :i], rtol=0, atol=1e-12)
    r = newton.newton_solve(c, x, h0, "DEER", 1e-12, jac_every=k)
    assert r["status"] == "OK" and r["iters"] <= T + 1
    np.testing.assert_allclose(r["h"], ref, rtol=0, atol=1e-10)
    with pytest.raises(ValueError):
        newton.newton_solve(c, x, h0, "DEER", 1e-6, jac_every=0)
