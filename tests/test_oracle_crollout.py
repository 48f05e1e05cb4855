"""The host rollout in C (fp64 and fp32, OpenMP over the batch) against the
oracle's numpy rollout, which is pinned to torch.nn.GRUCell (CPU only)."""
import numpy as np
import pytest

from oracle import crollout
from oracle.cells import GRU, rollout


def _cell(kind, din, d, seed):
    rng = np.random.default_rng(seed)
    w_hh = rng.normal(0, 0.5 / np.sqrt(d), (3 * d, d)) if kind == "dense" else rng.uniform(-1, 1, 3 * d)
    return GRU(kind=kind, w_ih=rng.normal(0, 0.5, (3 * d, din)), b_ih=rng.normal(0, 0.3, 3 * d),
               w_hh=w_hh, b_hh=rng.normal(0, 0.3, 3 * d))


@pytest.mark.parametrize("kind,B,T,din,d", [("dense", 3, 200, 5, 7), ("diag", 2, 300, 4, 9), ("dense", 1, 1, 1, 1)])
def test_c_rollout_equals_oracle(kind, B, T, din, d):
    c = _cell(kind, din, d, seed=B + T + d)
    rng = np.random.default_rng(1)
    x = rng.normal(size=(B, T, din))
    h0 = rng.normal(0, 0.5, (B, d))
    want = rollout(c, x, h0)
    np.testing.assert_allclose(crollout.rollout(c, x, h0, np.float64, threads=2), want, rtol=0, atol=1e-12)
    got32 = crollout.rollout(c, x, h0, np.float32, threads=1)
    assert got32.dtype == np.float32
    assert np.max(np.abs(got32 - want)) <= 1e-4
    assert crollout.max_threads() >= 1


def test_c_lstm_rollout_equals_oracle():
    from oracle.lstm import LSTM, lstm_rollout
    rng = np.random.default_rng(3)
    din, d, B, T = 5, 6, 3, 150
    cell = LSTM(w_ih=rng.normal(0, 0.5, (4 * d, din)), b_ih=rng.normal(0, 0.3, 4 * d), u=rng.uniform(-1, 1, 4 * d),
                b_hh=rng.normal(0, 0.3, 4 * d))
    x = rng.normal(size=(B, T, din))
    c0, h0 = rng.normal(0, 0.5, (B, d)), rng.normal(0, 0.5, (B, d))
    cw, hw = lstm_rollout(cell, x, c0, h0)
    c, h = crollout.lstm_rollout(cell, x, c0, h0, np.float64, threads=2)
    np.testing.assert_allclose(c, cw, rtol=0, atol=1e-12)
    np.testing.assert_allclose(h, hw, rtol=0, atol=1e-12)
    c32, h32 = crollout.lstm_rollout(cell, x, c0, h0, np.float32, threads=1)
    assert max(np.max(np.abs(c32 - cw)), np.max(np.abs(h32 - hw))) <= 1e-4
