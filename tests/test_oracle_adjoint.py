"""Pins of the oracle's backward pass (gradients through the evaluated sequence).

The exact adjoint is tied to torch autograd through an fp64 rollout of
``torch.nn.GRUCell`` (a library routine; the diagonal cell as a GRUCell whose
recurrent blocks are diagonal matrices).  The quasi (diagonal-Jacobian)
backward pass has no library counterpart: it is pinned by the two cases in
which it must equal the exact one (T = 1, and a dense cell whose recurrent
blocks happen to be diagonal) and by its recurrence on a hand-checkable case.
"""
import numpy as np
import pytest
import torch

from oracle.adjoint import adjoint
from oracle.cells import GRU, rollout


def _rand_gru(kind, din, d, seed, scale=0.5):
    rng = np.random.default_rng(seed)
    w_hh = rng.normal(0, scale, (3 * d, d)) if kind == "dense" else rng.uniform(-1, 1, 3 * d)
    return GRU(kind=kind, w_ih=rng.normal(0, scale, (3 * d, din)), b_ih=rng.normal(0, 0.3, 3 * d),
               w_hh=w_hh, b_hh=rng.normal(0, 0.3, 3 * d))


def _torch_grads(c: GRU, x, h0, g):
    """Autograd of L = sum(h * g) through an fp64 torch.nn.GRUCell rollout."""
    B, T, din = x.shape
    d = c.d
    m = torch.nn.GRUCell(din, d).double()
    with torch.no_grad():
        m.weight_ih.copy_(torch.from_numpy(c.w_ih))
        m.bias_ih.copy_(torch.from_numpy(c.b_ih))
        m.bias_hh.copy_(torch.from_numpy(c.b_hh))
        if c.kind == "dense":
            m.weight_hh.copy_(torch.from_numpy(c.w_hh))
        else:
            m.weight_hh.copy_(torch.from_numpy(
                np.concatenate([np.diag(c.w_hh[k * d:(k + 1) * d]) for k in range(3)], 0)))
    xt = torch.from_numpy(x).requires_grad_(True)
    ht = torch.from_numpy(h0).requires_grad_(True)
    hs, h = [], ht
    for t in range(T):
        h = m(xt[:, t], h)
        h.retain_grad()
        hs.append(h)
    loss = sum((hs[t] * torch.from_numpy(g[:, t])).sum() for t in range(T))
    loss.backward()
    lam = np.stack([hs[t].grad.numpy() for t in range(T)], 1)
    w_hh_grad = m.weight_hh.grad.numpy()
    if c.kind == "diag":  # d/du_g is the diagonal of the gate's block
        w_hh_grad = np.concatenate([np.diagonal(w_hh_grad[k * d:(k + 1) * d]) for k in range(3)])
    return dict(lam=lam, dx=xt.grad.numpy(), dh0=ht.grad.numpy(), dw_ih=m.weight_ih.grad.numpy(),
                db_ih=m.bias_ih.grad.numpy(), dw_hh=w_hh_grad, db_hh=m.bias_hh.grad.numpy())


@pytest.mark.parametrize("kind", ["dense", "diag"])
def test_exact_adjoint_equals_autograd(kind):
    din, d, B, T = 3, 5, 2, 17
    c = _rand_gru(kind, din, d, seed=11)
    rng = np.random.default_rng(12)
    x = rng.normal(size=(B, T, din))
    h0 = rng.normal(0, 0.5, size=(B, d))
    g = rng.normal(size=(B, T, d))
    h = rollout(c, x, h0)
    got = adjoint(c, x, h0, h, g, jacobian="exact")
    want = _torch_grads(c, x, h0, g)
    for k in ("lam", "dx", "dh0", "dw_ih", "db_ih", "dw_hh", "db_hh"):
        np.testing.assert_allclose(got[k], want[k], rtol=1e-10, atol=1e-12, err_msg=k)
    # dP is the gradient w.r.t. the input pre-activations: dx = dP W_ih
    np.testing.assert_allclose(got["dP"] @ c.w_ih, want["dx"], rtol=1e-10, atol=1e-12)


def test_diag_cell_quasi_backward_is_exact():
    """The diagonal cell's Jacobian is diagonal: its quasi backward pass is the
    exact gradient (the case the GPU kernel computes)."""
    din, d, B, T = 4, 6, 3, 23
    c = _rand_gru("diag", din, d, seed=21)
    rng = np.random.default_rng(22)
    x = rng.normal(size=(B, T, din))
    h0 = rng.normal(0, 0.5, size=(B, d))
    g = rng.normal(size=(B, T, d))
    h = rollout(c, x, h0)
    got = adjoint(c, x, h0, h, g, jacobian="diag")
    want = _torch_grads(c, x, h0, g)
    for k in ("lam", "dx", "dh0", "dw_ih", "db_ih", "dw_hh", "db_hh"):
        np.testing.assert_allclose(got[k], want[k], rtol=1e-10, atol=1e-12, err_msg=k)


def test_quasi_backward_limits():
    din, d, B = 3, 4, 2
    rng = np.random.default_rng(31)
    # T = 1: no recurrence to approximate
    c = _rand_gru("dense", din, d, seed=32)
    x = rng.normal(size=(B, 1, din))
    h0 = rng.normal(size=(B, d))
    g = rng.normal(size=(B, 1, d))
    h = rollout(c, x, h0)
    q = adjoint(c, x, h0, h, g, jacobian="diag")
    e = adjoint(c, x, h0, h, g, jacobian="exact")
    for k in ("lam", "dP", "dw_hh", "db_hh", "dx"):
        np.testing.assert_allclose(q[k], e[k], rtol=1e-12, atol=1e-14, err_msg=k)
    # only dh0 sees J_1, and there the quasi pass keeps its diagonal
    _, a = c.jacobian_diag(h0, c.project(x[:, 0]))
    np.testing.assert_allclose(q["dh0"], a * g[:, 0], rtol=1e-12, atol=1e-14)
    # a dense cell whose recurrent blocks are diagonal: quasi == exact
    cd = _rand_gru("dense", din, d, seed=33)
    cd.w_hh = np.concatenate([np.diag(rng.uniform(-1, 1, d)) for _ in range(3)], 0)
    x = rng.normal(size=(B, 9, din))
    g = rng.normal(size=(B, 9, d))
    h = rollout(cd, x, h0)
    q = adjoint(cd, x, h0, h, g, jacobian="diag")
    e = adjoint(cd, x, h0, h, g, jacobian="exact")
    for k in ("lam", "dP", "dh0", "dw_hh", "db_hh"):
        np.testing.assert_allclose(q[k], e[k], rtol=1e-12, atol=1e-14, err_msg=k)


def test_adjoint_of_linear_readout_closed_form():
    """A cell that copies its state (z = 1 exactly is out of reach, so take the
    limit numerically): with b_hz large, f = h and J = I, so lam_t is the
    suffix sum of g and dh0 = lam_1."""
    din, d, B, T = 2, 3, 1, 6
    c = _rand_gru("diag", din, d, seed=41, scale=0.1)
    c.b_hh[d:2 * d] = 60.0  # z = sigmoid(60) = 1 - 1e-26: f = h, J = I to fp64 precision
    rng = np.random.default_rng(42)
    x = rng.normal(size=(B, T, din))
    h0 = rng.normal(size=(B, d))
    g = rng.normal(size=(B, T, d))
    h = rollout(c, x, h0)
    got = adjoint(c, x, h0, h, g)
    suffix = np.cumsum(g[:, ::-1], axis=1)[:, ::-1]
    np.testing.assert_allclose(got["lam"], suffix, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(got["dh0"], suffix[:, 0], rtol=1e-12, atol=1e-12)
