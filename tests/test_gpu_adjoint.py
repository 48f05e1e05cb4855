"""GPU parity of the backward pass vs the fp64 oracle: the diagonal-recurrence
GRU (exact) and the dense GRU with the Jacobian's diagonal (the quasi backward).

Inputs: a random diagonal cell, synthetic fp32 pre-activations P, the fp64
rollout of the cell from P (rounded to fp32), and random upstream gradients.
The oracle sees exactly the same (fp32-valued) arrays: it runs with an
identity input projection, so its x is P.

Tolerance: normwise, ||got - want||_inf <= 1e-4 ||want||_inf for dP and dh0
(lam accumulates T fp32 steps of a_t lam + g) and 1e-4 for the parameter sums
over B*T terms; the kernel's exponentials carry ~1e-7 relative error.
"""
import ctypes

import numpy as np
import pytest
import torch

from oracle.adjoint import adjoint as oracle_adjoint
from oracle.cells import GRU
from newton_solve_nonlinear_b200 import binding

pytestmark = pytest.mark.gpu


def _case(B, T, D, seed, u_range=0.9):
    g = torch.Generator().manual_seed(seed)
    u = (torch.rand(3 * D, generator=g) * 2 - 1) * u_range
    b_hh = torch.randn(3 * D, generator=g) * 0.3
    P = torch.randn(B, T, 3 * D, generator=g)
    h0 = torch.randn(B, D, generator=g) * 0.5
    dh = torch.randn(B, T, D, generator=g)
    # the oracle's own cell, fed P directly (identity input projection)
    cell = GRU(kind="diag", w_ih=np.zeros((3 * D, 0)), b_ih=np.zeros(3 * D), w_hh=u.double().numpy(),
               b_hh=b_hh.double().numpy())
    Pd = P.double().numpy()
    hs, hv = [], h0.double().numpy()
    for t in range(T):  # the rollout h_t = f(h_{t-1}, p_t) through the oracle's gates
        hv = cell.gates(hv, Pd[:, t])[4]
        hs.append(hv)
    h = torch.from_numpy(np.stack(hs, 1)).float()
    return cell, u, b_hh, P, h0, h, dh


def _identity_cell(cell, idx3=None):
    w = cell.w_hh if idx3 is None else cell.w_hh[idx3]
    b = cell.b_hh if idx3 is None else cell.b_hh[idx3]
    return GRU(kind="diag", w_ih=np.eye(len(w)), b_ih=np.zeros(len(w)), w_hh=w, b_hh=b)


def _same_run(a, b, atol=1e-6):
    """Two launches of the same solve agree to within fp32 rounding: the
    decoupled look-back composes the later tiles' maps in an order set by
    timing (how far back the first finished prefix lies), so the last bits
    may differ from one launch to the next."""
    return float((a.double().cpu() - b.double().cpu()).abs().max()) <= atol


def _rel(got, want):
    return float(np.max(np.abs(got - want)) / max(np.max(np.abs(want)), 1e-30))


def _check(B, T, D, seed, lanes=None):
    cell, u, b_hh, P, h0, h, dh = _case(B, T, D, seed)
    r = binding.adjoint(u.cuda(), b_hh.cuda(), P.cuda(), h0.cuda(), h.cuda(), dh.cuda(), check=True)
    f64 = lambda t: t.double().numpy()
    if lanes is None:
        ref = oracle_adjoint(_identity_cell(cell), f64(P), f64(h0), f64(h), f64(dh), jacobian="diag")
        sel, sel3 = slice(None), slice(None)
    else:  # the diagonal cell is separable by lane: the oracle on a subset of lanes
        idx = np.asarray(lanes)
        idx3 = np.concatenate([idx, D + idx, 2 * D + idx])
        ref = oracle_adjoint(_identity_cell(cell, idx3), f64(P)[..., idx3], f64(h0)[:, idx], f64(h)[..., idx], f64(dh)[..., idx],
                             jacobian="diag")
        sel, sel3 = idx, idx3
    got = {k: v.double().cpu().numpy() for k, v in r.items()}
    assert _rel(got["dP"][..., sel3], ref["dP"]) <= 1e-4
    assert _rel(got["dh0"][:, sel], ref["dh0"]) <= 1e-4
    assert _rel(got["dw_hh"][sel3], ref["dw_hh"]) <= 1e-4
    assert _rel(got["db_hh"][sel3], ref["db_hh"]) <= 1e-4


@pytest.mark.parametrize("B,T,D", [(2, 100, 64), (3, 257, 96), (1, 1, 5), (2, 33, 130), (1, 64, 64),
                                   (4, 1000, 128)])
def test_adjoint_matches_oracle(B, T, D):
    _check(B, T, D, seed=B * 1000 + T + D)


def test_adjoint_full_size_sampled_lanes():
    """The diagonal workload's size (B = 8, T = 4096, D = 2048), the oracle on 96 lanes."""
    _check(8, 4096, 2048, seed=7, lanes=list(range(0, 2048, 64)) + list(range(1000, 1064)))


def test_adjoint_repeatable_and_rejects_wide_dense():
    cell, u, b_hh, P, h0, h, dh = _case(2, 300, 64, seed=3)
    args = [t.cuda() for t in (u, b_hh, P, h0, h, dh)]
    r1 = binding.adjoint(*args)
    r2 = binding.adjoint(*args)
    for k in r1:
        assert _rel(r1[k].double().cpu().numpy(), r2[k].double().cpu().numpy()) <= 1e-6, k
    assert binding.adjoint_workspace_size(64, 2, 300, kind="dense") > 0
    assert binding.adjoint_workspace_size(65, 2, 300, kind="dense") == 0


def _dense_case(B, T, D, seed, scale=0.9):
    """A random dense GRU (U [3D, D] with entries of std scale/sqrt(D)), P, h0,
    the fp64 rollout from P (rounded to fp32) and upstream gradients."""
    g = torch.Generator().manual_seed(seed)
    w_hh = torch.randn(3 * D, D, generator=g) * (scale / D ** 0.5)
    b_hh = torch.randn(3 * D, generator=g) * 0.3
    P = torch.randn(B, T, 3 * D, generator=g)
    h0 = torch.randn(B, D, generator=g) * 0.5
    dh = torch.randn(B, T, D, generator=g)
    cell = GRU(kind="dense", w_ih=np.eye(3 * D), b_ih=np.zeros(3 * D), w_hh=w_hh.double().numpy(),
               b_hh=b_hh.double().numpy())
    Pd = P.double().numpy()
    hs, hv = [], h0.double().numpy()
    for t in range(T):
        hv = cell.gates(hv, Pd[:, t])[4]
        hs.append(hv)
    h = torch.from_numpy(np.stack(hs, 1)).float()
    return cell, w_hh, b_hh, P, h0, h, dh


@pytest.mark.parametrize("B,T,D", [(2, 100, 64), (3, 257, 32), (1, 1, 5), (2, 1030, 64), (1, 64, 48),
                                   (4, 700, 12)])
def test_dense_adjoint_matches_oracle_diag_jacobian(B, T, D):
    """The dense cell's backward with the Jacobian's diagonal in the lam
    recurrence, against the oracle's jacobian='diag' pass; dW_hh [3D, D] is
    a sum over B*T outer products (normwise 1e-4 as above)."""
    cell, w_hh, b_hh, P, h0, h, dh = _dense_case(B, T, D, seed=B * 7 + T + D)
    r = binding.adjoint(w_hh.cuda(), b_hh.cuda(), P.cuda(), h0.cuda(), h.cuda(), dh.cuda(), check=True)
    f64 = lambda t: t.double().numpy()
    ref = oracle_adjoint(cell, f64(P), f64(h0), f64(h), f64(dh), jacobian="diag")
    got = {k: v.double().cpu().numpy() for k, v in r.items()}
    assert got["dw_hh"].shape == (3 * D, D)
    for k in ("dP", "dh0", "dw_hh", "db_hh"):
        assert _rel(got[k], ref[k]) <= 1e-4, k


def test_dense_adjoint_full_size_deterministic():
    """The dense workloads' size (B = 16, T = 65536, D = 64): two runs agree
    to fp32 rounding; dP and dh0 of sequence 0 match the oracle run on that
    sequence alone (sequences are independent); db_hh and dW_hh match fp64
    sums formed from the returned dP over all sequences."""
    B, T, D = 16, 65536, 64
    g = torch.Generator().manual_seed(11)
    w_hh = torch.randn(3 * D, D, generator=g) * (0.9 / D ** 0.5)
    b_hh = torch.randn(3 * D, generator=g) * 0.3
    P = torch.randn(B, T, 3 * D, generator=g)
    h0 = torch.randn(B, D, generator=g) * 0.5
    dh = torch.randn(B, T, D, generator=g)
    cell = GRU(kind="dense", w_ih=np.eye(3 * D), b_ih=np.zeros(3 * D), w_hh=w_hh.double().numpy(),
               b_hh=b_hh.double().numpy())
    # states: an fp32 rollout on the CPU (torch ops); the oracle reads the same h
    h = torch.empty(B, T, D)
    hv = h0.clone()
    Pc = P
    for t in range(T):
        q = hv @ w_hh.T + b_hh
        r_ = torch.sigmoid(Pc[:, t, :D] + q[:, :D])
        z_ = torch.sigmoid(Pc[:, t, D:2 * D] + q[:, D:2 * D])
        n_ = torch.tanh(Pc[:, t, 2 * D:] + r_ * q[:, 2 * D:])
        hv = (1 - z_) * n_ + z_ * hv
        h[:, t] = hv
    args = [t.cuda() for t in (w_hh, b_hh, P, h0, h, dh)]
    r1 = binding.adjoint(*args, check=True)
    r2 = binding.adjoint(*args)
    for k in r1:
        assert _rel(r1[k].double().cpu().numpy(), r2[k].double().cpu().numpy()) <= 1e-6, k
    f64 = lambda t: t.double().numpy()
    ref = oracle_adjoint(cell, f64(P[:1]), f64(h0[:1]), f64(h[:1]), f64(dh[:1]), jacobian="diag")
    got = {k: v.double().cpu().numpy() for k, v in r1.items()}
    assert _rel(got["dP"][:1], ref["dP"]) <= 1e-4
    assert _rel(got["dh0"][:1], ref["dh0"]) <= 1e-4
    # the parameter sums from the kernel's own dP, in fp64: db_hh exactly
    # from dP and r; dW_hh from grow (outer) h_{t-1}
    Pd, hd = f64(P), f64(h)
    hp = np.concatenate([f64(h0)[:, None], hd[:, :-1]], 1)
    q = hp @ f64(w_hh).T + f64(b_hh)
    rg = 1 / (1 + np.exp(-(Pd[..., :D] + q[..., :D])))
    dP = got["dP"]
    grow = np.concatenate([dP[..., :2 * D], dP[..., 2 * D:] * rg], -1)
    assert _rel(got["db_hh"], grow.sum((0, 1))) <= 1e-4
    assert _rel(got["dw_hh"], np.einsum("btk,btj->kj", grow, hp)) <= 1e-4


def test_dense_adjoint_with_diagonal_u_equals_diagonal_cell():
    """A dense U that is diagonal per gate is the diagonal cell: the two paths
    give the same dP, dh0, db_hh, and dW_hh's diagonal blocks equal du."""
    B, T, D = 2, 500, 64
    cell, u, b_hh, P, h0, h, dh = _case(B, T, D, seed=21)
    U = torch.cat([torch.diag(u[k * D:(k + 1) * D]) for k in range(3)], 0)
    rd = binding.adjoint(u.cuda(), b_hh.cuda(), P.cuda(), h0.cuda(), h.cuda(), dh.cuda())
    rD = binding.adjoint(U.cuda(), b_hh.cuda(), P.cuda(), h0.cuda(), h.cuda(), dh.cuda())
    for k in ("dP", "dh0", "db_hh"):
        assert _rel(rD[k].double().cpu().numpy(), rd[k].double().cpu().numpy()) <= 1e-5, k
    diag = torch.cat([torch.diagonal(rD["dw_hh"][k * D:(k + 1) * D]) for k in range(3)])
    assert _rel(diag.double().cpu().numpy(), rd["dw_hh"].double().cpu().numpy()) <= 1e-5


def test_adjoint_gives_autograd_gradients_of_a_solve():
    """End to end on the GPU: solve the diagonal GRU with exact Newton, take the
    backward pass, and form the input gradients with plain GEMMs; compare with
    torch autograd of an fp64 rollout on the CPU (a library routine)."""
    from newton_solve_nonlinear_b200.inputs import make_workload
    w = make_workload("diag", B=2, T=300, d=64, din=48, x_dtype=torch.float32, w_dtype=torch.float32,
                      bias_std=0.2, h0_std=0.5)
    dev = lambda t: t.cuda().contiguous()
    sol = binding.solve_workload(w, "QUASI", tol=1e-6)
    assert sol.status == "OK"
    P = binding.input_projection(dev(w.x), dev(w.w_ih), dev(w.b_ih), d=64, kind="diag")
    gen = torch.Generator().manual_seed(5)
    dh = torch.randn(2, 300, 64, generator=gen)
    r = binding.adjoint(dev(w.w_hh), dev(w.b_hh), P, dev(w.h0), sol.h, dh.cuda())
    dx = (r["dP"] @ dev(w.w_ih)).double().cpu()
    # autograd reference: GRUCell with diagonal recurrent blocks, fp64
    d = 64
    m = torch.nn.GRUCell(48, d).double()
    with torch.no_grad():
        m.weight_ih.copy_(w.w_ih.double())
        m.bias_ih.copy_(w.b_ih.double())
        m.bias_hh.copy_(w.b_hh.double())
        m.weight_hh.copy_(torch.cat([torch.diag(w.w_hh[k * d:(k + 1) * d].double()) for k in range(3)], 0))
    x = w.x.double().requires_grad_(True)
    h0 = w.h0.double().requires_grad_(True)
    h, loss = h0, 0.0
    for t in range(300):
        h = m(x[:, t], h)
        loss = loss + (h * dh[:, t].double()).sum()
    loss.backward()
    assert _rel(dx.numpy(), x.grad.numpy()) <= 1e-4
    assert _rel(r["dh0"].double().cpu().numpy(), h0.grad.numpy()) <= 1e-4
    gw = m.weight_hh.grad
    du = torch.cat([torch.diagonal(gw[k * d:(k + 1) * d]) for k in range(3)])
    assert _rel(r["dw_hh"].double().cpu().numpy(), du.numpy()) <= 1e-4
    assert _rel(r["db_hh"].double().cpu().numpy(), m.bias_hh.grad.numpy()) <= 1e-4


@pytest.mark.parametrize("kind,B,T,D,parts", [("diag", 5, 300, 64, 3), ("diag", 3, 100, 130, 1),
                                              ("dense", 4, 500, 64, 4), ("dense", 2, 77, 12, 2)])
def test_host_buffer_adjoint_matches_device(kind, B, T, D, parts):
    """From and to host memory in ramped parts: dL/dP and dL/dh0 are per
    sequence, so they equal the device pass's to fp32 rounding; dW_hh and db_hh
    are the parts' sums added in part order (the device pass adds the same
    terms in another order): normwise within 1e-5."""
    if kind == "diag":
        cell, w, b_hh, P, h0, h, dh = _case(B, T, D, seed=B + T)
    else:
        cell, w, b_hh, P, h0, h, dh = _dense_case(B, T, D, seed=B + T)
    ref = binding.adjoint(w.cuda(), b_hh.cuda(), P.cuda(), h0.cuda(), h.cuda(), dh.cuda())
    pin = lambda t: t.contiguous().pin_memory()
    got = binding.adjoint_host(w.cuda(), b_hh.cuda(), pin(P), pin(h0), pin(h), pin(dh), parts=parts)
    assert _same_run(got["dP"], ref["dP"]) and _same_run(got["dh0"], ref["dh0"])
    for k in ("dw_hh", "db_hh"):
        assert _rel(got[k].double().numpy(), ref[k].double().cpu().numpy()) <= 1e-5, k


# ---- the dense cell's exact backward pass (full transposed Jacobian) ----

@pytest.mark.parametrize("B,T,D", [(2, 100, 64), (3, 257, 32), (1, 1, 8), (2, 300, 12), (1, 64, 48)])
def test_exact_dense_adjoint_matches_oracle(B, T, D):
    """pararnn_adjoint_exact against the oracle's jacobian='exact' pass (whose
    reverse recurrence is J_{t+1}^T lam_{t+1} with the full Jacobian; the
    oracle itself equals torch autograd through an fp64 GRUCell rollout):
    normwise 1e-4 as the other backward passes.  The diagonal pass differs from
    it (checked too), so the test tells the two apart."""
    cell, w_hh, b_hh, P, h0, h, dh = _dense_case(B, T, D, seed=B * 5 + T + D)
    r = binding.adjoint_exact(w_hh.cuda(), b_hh.cuda(), P.cuda(), h0.cuda(), h.cuda(), dh.cuda())
    f64 = lambda t: t.double().numpy()
    ref = oracle_adjoint(cell, f64(P), f64(h0), f64(h), f64(dh), jacobian="exact")
    got = {k: v.double().cpu().numpy() for k, v in r.items()}
    for k in ("dP", "dh0", "dw_hh", "db_hh"):
        assert _rel(got[k], ref[k]) <= 1e-4, k
    if T > 1:
        quasi = oracle_adjoint(cell, f64(P), f64(h0), f64(h), f64(dh), jacobian="diag")
        assert _rel(got["dP"], quasi["dP"]) > 1e-3


def test_exact_dense_adjoint_with_diagonal_u_equals_diagonal_pass():
    """With every recurrent block diagonal the Jacobian is diagonal, so the
    exact pass equals the diagonal-Jacobian pass."""
    B, T, D = 2, 400, 32
    cell, u, b_hh, P, h0, h, dh = _case(B, T, D, seed=33)
    U = torch.cat([torch.diag(u[k * D:(k + 1) * D]) for k in range(3)], 0)
    args = [U.cuda(), b_hh.cuda(), P.cuda(), h0.cuda(), h.cuda(), dh.cuda()]
    rx = binding.adjoint_exact(*args)
    rq = binding.adjoint(*args)
    for k in ("dP", "dh0", "dw_hh", "db_hh"):
        assert _rel(rx[k].double().cpu().numpy(), rq[k].double().cpu().numpy()) <= 1e-5, k


def test_exact_dense_adjoint_rejects_other_cells():
    L = binding.lib()
    assert L.pararnn_adjoint_exact_workspace_size(ctypes.byref(binding.make_cell("diag", 1, 64, torch.float32)),
                                                  2, 10) == 0
    assert L.pararnn_adjoint_exact_workspace_size(ctypes.byref(binding.make_cell("dense", 1, 68, torch.float32)),
                                                  2, 10) == 0
    assert L.pararnn_adjoint_exact_workspace_size(ctypes.byref(binding.make_cell("dense", 1, 30, torch.float32)),
                                                  2, 10) == 0
