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
