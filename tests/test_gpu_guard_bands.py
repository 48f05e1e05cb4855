"""Guard-band checks of every entry point on small and ragged shapes.

A memory checker without a device-side fault: each input, output and
workspace array is placed inside a larger allocation whose bands before and
after it are filled with 0xFF bytes (NaN as fp32 and bf16), and every output
array itself starts as NaN.  After the call:

  * the bands are byte-for-byte unchanged (no write left its array);
  * no output holds a NaN (every element was written, and no read beyond an
    input's end -- which would fetch NaN -- reached a result);
  * the results equal those of the same call on ordinary allocations (fp32
    rounding: the look-back composes maps in an order set by timing).

The workspace starts all 0xFF, so a kernel that relied on workspace contents
it did not set itself would also show here.  Shapes: B, T and D chosen off the
tile sizes (T = 1, 65, 257, ...; D = 5, 12, 48, 60, 100, 130) so that every
kernel's ragged tile, lane group and chunk tails are taken.
"""
import ctypes
import math

import pytest
import torch

from newton_solve_nonlinear_b200 import binding
from newton_solve_nonlinear_b200.inputs import make_lstm_workload, make_scan_input, make_workload

pytestmark = pytest.mark.gpu

BAND = 4096  # bytes before and after each array (keeps the array 256-byte aligned)


class Guarded:
    """An array of ``shape`` and ``dtype`` inside a banded allocation."""

    def __init__(self, shape, dtype, device="cuda", init=None, pinned=False):
        esize = torch.empty((), dtype=dtype).element_size()
        self.n = math.prod(shape) * esize
        raw = torch.empty(self.n + 2 * BAND + 256, dtype=torch.uint8, device=device)
        if pinned:
            raw = raw.pin_memory()
        off = (-raw.data_ptr()) % 256
        self.raw = raw[off:off + self.n + 2 * BAND]
        self.raw.fill_(0xFF)
        self.t = self.raw[BAND:BAND + self.n].view(dtype).view(shape)
        if init is not None:
            self.t.copy_(init)

    def bands_intact(self) -> bool:
        lo = self.raw[:BAND]
        hi = self.raw[BAND + self.n:]
        return bool((lo == 0xFF).all()) and bool((hi == 0xFF).all())


def _ws(nbytes):
    return Guarded((nbytes,), torch.uint8)


def _close(a, b, tol=1e-5):
    a, b = a.double().cpu(), b.double().cpu()
    scale = max(float(b.abs().max()), 1.0)
    return float((a - b).abs().max()) <= tol * scale


def _finite(*ts):
    return all(bool(torch.isfinite(t.float()).all()) for t in ts)


def _solve_cases():
    # (workload, overrides, mode, lam): each line reaches a different kernel
    return [
        ("untrained", dict(B=3, T=257), "QUASI", 0.0),               # tcgen05 quasi kernel, D = 64
        ("near_unstable", dict(B=2, T=130, d=32, din=32), "QUASI_ELK", 0.1),  # tcgen05 quasi-ELK, D = 32
        ("dense_deer", dict(B=3, T=257, d=12, din=5), "QUASI", 0.0),  # diagonal-Jacobian kernel, dense cell
        ("near_unstable", dict(B=2, T=65, d=60, din=7), "QUASI_ELK", 0.1),
        ("dense_deer", dict(B=3, T=257, d=12, din=5), "DEER", 0.0),   # mma.sync DEER, D <= 32
        ("dense_deer", dict(B=2, T=65, d=48, din=8), "DEER", 0.0),    # CUDA-core DEER, D = 48
        ("near_unstable", dict(B=2, T=65, d=8, din=3), "ELK", 0.1),   # dense ELK
        ("diag", dict(B=2, T=257, d=128, din=64, x_dtype=torch.float32, w_dtype=torch.float32), "DEER", 0.0),
        ("diag", dict(B=3, T=65, d=100, din=12, x_dtype=torch.float32, w_dtype=torch.float32), "QUASI_ELK", 0.1),
        ("diag", dict(B=2, T=1, d=64, din=64, x_dtype=torch.float32, w_dtype=torch.float32), "ELK", 1.0),
        ("diag", dict(B=2, T=65, d=256, din=64), "QUASI", 0.0),       # bf16 tcgen05 projection
    ]


@pytest.mark.parametrize("name,over,mode,lam", _solve_cases())
def test_solve_guard_bands(name, over, mode, lam):
    w = make_workload(name, seed=3, bias_std=0.2, h0_std=0.5, **over)
    dev = lambda t: t.cuda().contiguous()
    ins = {k: Guarded(tuple(getattr(w, k).shape), getattr(w, k).dtype, init=dev(getattr(w, k)))
           for k in ("w_ih", "b_ih", "w_hh", "b_hh", "x", "h0")}
    out = Guarded((w.B, w.T, w.d), torch.float32)
    need = binding.workspace_size(w.kind, w.din, w.d, w.B, w.T, mode, w.x_dtype)
    ws = _ws(need)
    # damped steps on short sequences need more iterations than the default cap of T + 1
    cap = 400
    r = binding.newton_solve(*(ins[k].t for k in ("w_ih", "b_ih", "w_hh", "b_hh", "x", "h0")),
                             kind=w.kind, mode=mode, tol=w.tol, lam=lam, max_iters=cap,
                             out=out.t, workspace=ws.t)
    ref = binding.solve_workload(w, mode, lam=lam, max_iters=cap)
    torch.cuda.synchronize()
    assert r.status == ref.status == "OK", (r.status, ref.status)
    assert abs(r.iters - ref.iters) <= 1
    assert _finite(out.t)
    assert _close(out.t, ref.h, 1e-4)
    for g in (*ins.values(), out, ws):
        assert g.bands_intact()


def test_reuse_and_trace_guard_bands():
    w = make_workload("dense_deer", seed=5, bias_std=0.2, B=2, T=257, d=16, din=5)
    dev = lambda t: t.cuda().contiguous()
    args = [dev(getattr(w, k)) for k in ("w_ih", "b_ih", "w_hh", "b_hh", "x", "h0")]
    out = Guarded((w.B, w.T, w.d), torch.float32)
    cell = binding.make_cell("dense", w.din, w.d, torch.float32)
    ws = _ws(int(binding.lib().pararnn_reuse_workspace_size(ctypes.byref(cell), w.B, w.T)))
    r = binding.newton_solve(*args, kind="dense", mode="DEER", tol=w.tol, jac_every=2, out=out.t, workspace=ws.t)
    ref = binding.newton_solve(*args, kind="dense", mode="DEER", tol=w.tol, jac_every=2)
    assert r.status == ref.status == "OK" and _finite(out.t) and _close(out.t, ref.h, 1e-4)
    assert out.bands_intact() and ws.bands_intact()

    out2 = Guarded((w.B, w.T, w.d), torch.float32)
    ws2 = _ws(binding.workspace_size("dense", w.din, w.d, w.B, w.T, "QUASI"))
    r2 = binding.newton_solve(*args, kind="dense", mode="QUASI", tol=w.tol, out=out2.t, workspace=ws2.t,
                              trace=True)
    assert r2.status == "OK" and r2.trace.shape == (r2.iters, 2) and _finite(r2.trace, out2.t)
    assert out2.bands_intact() and ws2.bands_intact()


@pytest.mark.parametrize("B,T,D,dense", [(3, 1000, 100, False), (2, 1, 4, False), (2, 333, 12, True),
                                         (1, 65, 48, True)])
def test_affine_scan_guard_bands(B, T, D, dense):
    s = make_scan_input(B, T, D, dense=dense, seed=B + T, h0_std=1.0)
    A = Guarded(tuple(s.A.shape), torch.float32, init=s.A.cuda())
    b = Guarded(tuple(s.b.shape), torch.float32, init=s.b.cuda())
    h0 = Guarded(tuple(s.h0.shape), torch.float32, init=s.h0.cuda())
    h = Guarded((B, T, D), torch.float32)
    need = int(binding.lib().pararnn_affine_scan_workspace_size(B, T, D, int(dense)))
    ws = _ws(need)
    binding.affine_scan(A.t, b.t, h0.t, out=h.t, workspace=ws.t, check=True)
    ref = binding.affine_scan(s.A.cuda(), s.b.cuda(), s.h0.cuda(), check=True)
    assert _finite(h.t) and _close(h.t, ref)
    for g in (A, b, h0, h, ws):
        assert g.bands_intact()

    # the same from and to host memory, streamed in time parts
    parts = min(3, (T + 127) // 128)
    hA = Guarded(tuple(s.A.shape), torch.float32, device="cpu", init=s.A, pinned=True)
    hb = Guarded(tuple(s.b.shape), torch.float32, device="cpu", init=s.b, pinned=True)
    hh0 = Guarded(tuple(s.h0.shape), torch.float32, device="cpu", init=s.h0, pinned=True)
    hh = Guarded((B, T, D), torch.float32, device="cpu", pinned=True)
    wsh = _ws(int(binding.lib().pararnn_affine_scan_host_workspace_size(B, T, D, int(dense), parts)))
    binding.affine_scan_host(hA.t, hb.t, hh0.t, parts=parts, out=hh.t, workspace=wsh.t)
    assert _finite(hh.t) and _close(hh.t, ref)
    for g in (hA, hb, hh0, hh, wsh):
        assert g.bands_intact()


def _adjoint_inputs(B, T, D, dense, seed):
    g = torch.Generator().manual_seed(seed)
    w_hh = torch.randn(3 * D, D, generator=g) / D if dense else (torch.rand(3 * D, generator=g) * 2 - 1) * 0.9
    b_hh = torch.randn(3 * D, generator=g) * 0.3
    P = torch.randn(B, T, 3 * D, generator=g)
    h0 = torch.randn(B, D, generator=g) * 0.5
    h = torch.tanh(torch.randn(B, T, D, generator=g))
    dh = torch.randn(B, T, D, generator=g)
    return w_hh, b_hh, P, h0, h, dh


@pytest.mark.parametrize("B,T,D,kind", [(2, 257, 130, "diag"), (1, 1, 5, "diag"), (2, 65, 48, "dense"),
                                        (3, 100, 12, "exact"), (1, 33, 64, "exact")])
def test_adjoint_guard_bands(B, T, D, kind):
    arrs = _adjoint_inputs(B, T, D, kind != "diag", seed=B * T + D)
    ins = [Guarded(tuple(a.shape), torch.float32, init=a.cuda()) for a in arrs]
    w_hh, b_hh, P, h0 = arrs[:4]
    outs = {"dP": Guarded(tuple(P.shape), torch.float32), "dh0": Guarded(tuple(h0.shape), torch.float32),
            "dw_hh": Guarded(tuple(w_hh.shape), torch.float32), "db_hh": Guarded(tuple(b_hh.shape), torch.float32)}
    o = {k: v.t for k, v in outs.items()}
    if kind == "exact":
        cell = binding.make_cell("dense", 1, D, torch.float32)
        ws = _ws(int(binding.lib().pararnn_adjoint_exact_workspace_size(ctypes.byref(cell), B, T)))
        binding.adjoint_exact(*(g.t for g in ins), workspace=ws.t, out=o)
        ref = binding.adjoint_exact(*(a.cuda() for a in arrs))
    else:
        ws = _ws(binding.adjoint_workspace_size(D, B, T, "dense" if kind == "dense" else "diag"))
        binding.adjoint(*(g.t for g in ins), workspace=ws.t, out=o, check=True)
        ref = binding.adjoint(*(a.cuda() for a in arrs), check=True)
    torch.cuda.synchronize()
    for k, g in outs.items():
        assert _finite(g.t), k
        assert _close(g.t, ref[k], 1e-5), k
    for g in (*ins, *outs.values(), ws):
        assert g.bands_intact()


@pytest.mark.parametrize("B,T,d,din,dtype", [(2, 257, 96, 8, torch.float32), (2, 65, 128, 128, torch.bfloat16),
                                             (1, 1, 4, 3, torch.float32)])
def test_lstm_guard_bands(B, T, d, din, dtype):
    w = make_lstm_workload(B=B, T=T, d=d, din=din, seed=7, x_dtype=dtype)
    names = ("w_ih", "b_ih", "u", "b_hh", "x", "c0", "h0")
    ins = {k: Guarded(tuple(getattr(w, k).shape), getattr(w, k).dtype, init=getattr(w, k).cuda()) for k in names}
    c = Guarded((B, T, d), torch.float32)
    h = Guarded((B, T, d), torch.float32)
    ws = _ws(binding.lstm_workspace_size(din, d, B, T, dtype))
    _, _, r = binding.lstm_solve(*(ins[k].t for k in names), tol=1e-4, out=(c.t, h.t), workspace=ws.t)
    rc, rh, ref = binding.lstm_solve(*(getattr(w, k).cuda() for k in names), tol=1e-4)
    torch.cuda.synchronize()
    assert r.status == ref.status == "OK"
    assert _finite(c.t, h.t) and _close(c.t, rc, 1e-4) and _close(h.t, rh, 1e-4)
    for g in (*ins.values(), c, h, ws):
        assert g.bands_intact()


@pytest.mark.parametrize("M,din,d,kind,dtype", [(1031, 64, 64, "dense", torch.float32),  # TF32 tcgen05
                                               (333, 7, 12, "dense", torch.float32),     # CUDA cores
                                               (300, 64, 256, "diag", torch.bfloat16)])  # bf16 tcgen05
def test_projection_guard_bands(M, din, d, kind, dtype):
    g = torch.Generator().manual_seed(M)
    x = torch.randn(1, M, din, generator=g).to(dtype)
    w = (torch.randn(3 * d, din, generator=g) / math.sqrt(din)).to(dtype)
    b = torch.randn(3 * d, generator=g)
    gx, gw, gb = (Guarded(tuple(t.shape), t.dtype, init=t.cuda()) for t in (x, w, b))
    out = Guarded((1, M, 3 * d), torch.float32)
    binding.input_projection(gx.t, gw.t, gb.t, d=d, kind=kind, out=out.t)
    ref = binding.input_projection(x.cuda(), w.cuda(), b.cuda(), d=d, kind=kind)
    torch.cuda.synchronize()
    assert _finite(out.t) and _close(out.t, ref, 1e-6)
    for gg in (gx, gw, gb, out):
        assert gg.bands_intact()


def test_chunked_and_host_guard_bands():
    w = make_workload("untrained", seed=11, bias_std=0.2, h0_std=0.5, B=3, T=300)
    dev = lambda t: t.cuda().contiguous()
    wts = [dev(getattr(w, k)) for k in ("w_ih", "b_ih", "w_hh", "b_hh")]
    ref = binding.solve_workload(w, "QUASI")

    out = Guarded((w.B, w.T, w.d), torch.float32)
    ws = _ws(binding.chunked_workspace_size("dense", w.din, w.d, w.B, w.T, 97, "QUASI"))
    r = binding.newton_solve_chunked(*wts, dev(w.x), dev(w.h0), kind="dense", mode="QUASI", tol=w.tol,
                                     t_chunk=97, out=out.t, workspace=ws.t)
    assert r.status == "OK" and _finite(out.t) and _close(out.t, ref.h, 1e-4)
    assert out.bands_intact() and ws.bands_intact()

    xh = Guarded(tuple(w.x.shape), torch.float32, device="cpu", init=w.x, pinned=True)
    h0h = Guarded(tuple(w.h0.shape), torch.float32, device="cpu", init=w.h0, pinned=True)
    oh = Guarded((w.B, w.T, w.d), torch.float32, device="cpu", pinned=True)
    wsh = _ws(binding.host_workspace_size("dense", w.din, w.d, w.B, w.T, "QUASI", 2))
    r = binding.newton_solve_host(*wts, xh.t, h0h.t, kind="dense", mode="QUASI", tol=w.tol, parts=2,
                                  out=oh.t, workspace=wsh.t)
    assert r.status == "OK" and _finite(oh.t) and _close(oh.t, ref.h, 1e-4)
    for g in (xh, h0h, oh, wsh):
        assert g.bands_intact()

    oh2 = Guarded((w.B, w.T, w.d), torch.float32, device="cpu", pinned=True)
    wss = _ws(binding.host_streamed_workspace_size("dense", w.din, w.d, w.B, w.T, "QUASI", 3))
    r = binding.newton_solve_host_streamed(*wts, xh.t, h0h.t, kind="dense", mode="QUASI", tol=w.tol, parts=3,
                                           out=oh2.t, workspace=wss.t)
    assert r.status == "OK" and _finite(oh2.t) and _close(oh2.t, ref.h, 1e-4)
    for g in (xh, h0h, oh2, wss):
        assert g.bands_intact()


def test_host_lstm_and_adjoint_guard_bands():
    """The host-buffer LSTM calls (batch parts and time parts) and the
    host-buffer backward pass, with banded host and device arrays."""
    w = make_lstm_workload(B=3, T=300, d=64, din=16, seed=13, x_dtype=torch.float32, bias_std=0.3, state_std=0.5)
    dev = [getattr(w, k).cuda().contiguous() for k in ("w_ih", "b_ih", "u", "b_hh")]
    hin = {k: Guarded(tuple(getattr(w, k).shape), torch.float32, device="cpu", init=getattr(w, k), pinned=True)
           for k in ("x", "c0", "h0")}
    rc, rh, _ = binding.lstm_solve(*dev, w.x.cuda(), w.c0.cuda(), w.h0.cuda(), tol=w.tol)
    for streamed in (False, True):
        c = Guarded((w.B, w.T, w.d), torch.float32, device="cpu", pinned=True)
        h = Guarded((w.B, w.T, w.d), torch.float32, device="cpu", pinned=True)
        if streamed:
            ws = _ws(binding.lstm_host_streamed_workspace_size(w.din, w.d, w.B, w.T, 3, torch.float32))
            _, _, r = binding.lstm_solve_host_streamed(*dev, hin["x"].t, hin["c0"].t, hin["h0"].t, tol=w.tol,
                                                       parts=3, out=(c.t, h.t), workspace=ws.t)
        else:
            cell = binding.make_cell("lstm_diag", w.din, w.d, torch.float32)
            ws = _ws(int(binding.lib().pararnn_lstm_host_workspace_size(ctypes.byref(cell), w.B, w.T, 2)))
            _, _, r = binding.lstm_solve_host(*dev, hin["x"].t, hin["c0"].t, hin["h0"].t, tol=w.tol, parts=2,
                                              out=(c.t, h.t), workspace=ws.t)
        assert r.status == "OK" and _finite(c.t, h.t)
        assert _close(c.t, rc, 1e-4) and _close(h.t, rh, 1e-4)
        for g in (*hin.values(), c, h, ws):
            assert g.bands_intact()

    B, T, D = 3, 200, 48
    arrs = _adjoint_inputs(B, T, D, True, seed=21)
    w_hh, b_hh = arrs[0].cuda(), arrs[1].cuda()
    hP, hh0, hh, hdh = (Guarded(tuple(a.shape), torch.float32, device="cpu", init=a, pinned=True)
                        for a in (arrs[2], arrs[3], arrs[4], arrs[5]))
    outs = {"dP": Guarded(tuple(arrs[2].shape), torch.float32, device="cpu", pinned=True),
            "dh0": Guarded(tuple(arrs[3].shape), torch.float32, device="cpu", pinned=True),
            "dw_hh": Guarded(tuple(arrs[0].shape), torch.float32, device="cpu", pinned=True),
            "db_hh": Guarded(tuple(arrs[1].shape), torch.float32, device="cpu", pinned=True)}
    cell = binding.make_cell("dense", 1, D, torch.float32)
    ws = _ws(int(binding.lib().pararnn_adjoint_host_workspace_size(ctypes.byref(cell), B, T, 2)))
    binding.adjoint_host(w_hh, b_hh, hP.t, hh0.t, hh.t, hdh.t, parts=2, out={k: g.t for k, g in outs.items()},
                         workspace=ws.t)
    ref = binding.adjoint(*(a.cuda() for a in arrs), check=True)
    for k, g in outs.items():
        assert _finite(g.t), k
        assert _close(g.t, ref[k], 1e-5), k
    for g in (hP, hh0, hh, hdh, *outs.values(), ws):
        assert g.bands_intact()
