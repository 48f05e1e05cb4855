"""Thin ctypes binding of ``libpararnn.so`` (the C ABI in ``include/pararnn.h``).

Argument marshalling only: every step of the solve runs in the library's CUDA
kernels.  PyTorch supplies device memory and the current stream.  There is no
CPU path: if the library is missing or a tensor is not on a CUDA device, the
call raises.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libpararnn.so")

DEER, QUASI, ELK, QUASI_ELK = 0, 1, 2, 3
MODES = {"DEER": DEER, "QUASI": QUASI, "ELK": ELK, "QUASI_ELK": QUASI_ELK}
GRU_DENSE, GRU_DIAG, LSTM_DIAG = 0, 1, 2
F32, BF16 = 0, 1
STATUS = {0: "OK", 1: "NOT_CONVERGED", 2: "DIVERGED", 3: "INVALID_ARG", 4: "CUDA_ERROR",
          5: "TIMEOUT"}
EXPORTS = ("pararnn_workspace_size", "pararnn_newton_solve", "pararnn_newton_solve_async",
           "pararnn_input_projection", "pararnn_newton_iterate_async",
           "pararnn_affine_scan_workspace_size", "pararnn_affine_scan",
           "pararnn_affine_scan_status", "pararnn_status_string", "pararnn_newton_solve_host",
           "pararnn_host_workspace_size", "pararnn_adjoint", "pararnn_adjoint_workspace_size",
           "pararnn_adjoint_status", "pararnn_newton_solve_guess_async", "pararnn_newton_solve_chunked",
           "pararnn_chunked_workspace_size", "pararnn_lstm_solve", "pararnn_lstm_workspace_size",
           "pararnn_newton_solve_reuse", "pararnn_reuse_workspace_size", "pararnn_lstm_solve_host",
           "pararnn_lstm_host_workspace_size", "pararnn_adjoint_host", "pararnn_adjoint_host_workspace_size",
           "pararnn_newton_solve_trace", "pararnn_test_withheld_publish", "pararnn_adjoint_exact",
           "pararnn_adjoint_exact_workspace_size", "pararnn_newton_solve_host_streamed",
           "pararnn_host_streamed_workspace_size", "pararnn_lstm_solve_host_streamed",
           "pararnn_lstm_host_streamed_workspace_size", "pararnn_affine_scan_host",
           "pararnn_affine_scan_host_workspace_size")


class Cell(ctypes.Structure):
    _fields_ = [("kind", ctypes.c_int), ("din", ctypes.c_int), ("d", ctypes.c_int),
                ("x_dtype", ctypes.c_int), ("w_dtype", ctypes.c_int)]


class Params(ctypes.Structure):
    _fields_ = [("w_ih", ctypes.c_void_p), ("b_ih", ctypes.c_void_p),
                ("w_hh", ctypes.c_void_p), ("b_hh", ctypes.c_void_p)]


class Info(ctypes.Structure):
    _fields_ = [("iters", ctypes.c_int), ("status", ctypes.c_int),
                ("delta", ctypes.c_float), ("residual", ctypes.c_float)]


_lib = None


def lib() -> ctypes.CDLL:
    """Load the library once; raise if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            raise RuntimeError(
                f"{_LIB_PATH} is missing: build it with `python -m newton_solve_nonlinear_b200.build`")
        L = ctypes.CDLL(_LIB_PATH)
        vp, ci, cf, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
        L.pararnn_workspace_size.argtypes = [ctypes.POINTER(Cell), ci, ci, ci]
        L.pararnn_workspace_size.restype = sz
        solve_args = [ctypes.POINTER(Cell), ctypes.POINTER(Params), vp, vp, ci, ci, ci, cf, cf, ci,
                      vp, vp, vp, sz, vp]
        L.pararnn_newton_solve.argtypes = solve_args
        L.pararnn_newton_solve.restype = ci
        L.pararnn_newton_solve_async.argtypes = solve_args
        L.pararnn_newton_solve_async.restype = ci
        L.pararnn_input_projection.argtypes = [ctypes.POINTER(Cell), ctypes.POINTER(Params), vp, ci,
                                               ci, vp, vp]
        L.pararnn_input_projection.restype = ci
        L.pararnn_newton_iterate_async.argtypes = solve_args
        L.pararnn_newton_iterate_async.restype = ci
        L.pararnn_affine_scan_workspace_size.argtypes = [ci, ci, ci, ci]
        L.pararnn_affine_scan_workspace_size.restype = sz
        L.pararnn_affine_scan.argtypes = [vp, vp, vp, ci, ci, ci, ci, vp, vp, sz, vp]
        L.pararnn_affine_scan.restype = ci
        L.pararnn_affine_scan_status.argtypes = [vp, vp]
        L.pararnn_affine_scan_status.restype = ci
        L.pararnn_affine_scan_host.argtypes = [vp, vp, vp, ci, ci, ci, ci, vp, ci, vp, sz, vp]
        L.pararnn_affine_scan_host.restype = ci
        L.pararnn_affine_scan_host_workspace_size.argtypes = [ci, ci, ci, ci, ci]
        L.pararnn_affine_scan_host_workspace_size.restype = sz
        L.pararnn_newton_solve_host.argtypes = [ctypes.POINTER(Cell), ctypes.POINTER(Params), vp, vp,
                                                ci, ci, ci, cf, cf, ci, vp, vp, ci, vp, sz, vp]
        L.pararnn_newton_solve_host.restype = ci
        L.pararnn_host_workspace_size.argtypes = [ctypes.POINTER(Cell), ci, ci, ci, ci]
        L.pararnn_host_workspace_size.restype = sz
        L.pararnn_newton_solve_host_streamed.argtypes = L.pararnn_newton_solve_host.argtypes
        L.pararnn_newton_solve_host_streamed.restype = ci
        L.pararnn_host_streamed_workspace_size.argtypes = [ctypes.POINTER(Cell), ci, ci, ci, ci]
        L.pararnn_host_streamed_workspace_size.restype = sz
        L.pararnn_adjoint.argtypes = [ctypes.POINTER(Cell), ctypes.POINTER(Params), vp, vp, vp, vp, ci, ci,
                                      vp, vp, vp, vp, vp, sz, vp]
        L.pararnn_adjoint.restype = ci
        L.pararnn_adjoint_workspace_size.argtypes = [ctypes.POINTER(Cell), ci, ci]
        L.pararnn_adjoint_workspace_size.restype = sz
        L.pararnn_adjoint_status.argtypes = [vp, vp]
        L.pararnn_adjoint_status.restype = ci
        L.pararnn_newton_solve_guess_async.argtypes = [ctypes.POINTER(Cell), ctypes.POINTER(Params), vp, vp, vp,
                                                       ci, ci, ci, cf, cf, ci, vp, vp, vp, sz, vp]
        L.pararnn_newton_solve_guess_async.restype = ci
        L.pararnn_newton_solve_chunked.argtypes = [ctypes.POINTER(Cell), ctypes.POINTER(Params), vp, vp, ci, ci,
                                                   ci, ci, cf, cf, ci, vp, ctypes.POINTER(Info), vp, sz, vp]
        L.pararnn_newton_solve_chunked.restype = ci
        L.pararnn_chunked_workspace_size.argtypes = [ctypes.POINTER(Cell), ci, ci, ci, ci]
        L.pararnn_chunked_workspace_size.restype = sz
        L.pararnn_lstm_solve.argtypes = [ctypes.POINTER(Cell), ctypes.POINTER(Params), vp, vp, vp, ci, ci, cf, ci,
                                         vp, vp, ctypes.POINTER(Info), vp, sz, vp]
        L.pararnn_lstm_solve.restype = ci
        L.pararnn_lstm_workspace_size.argtypes = [ctypes.POINTER(Cell), ci, ci]
        L.pararnn_lstm_workspace_size.restype = sz
        L.pararnn_newton_solve_reuse.argtypes = [ctypes.POINTER(Cell), ctypes.POINTER(Params), vp, vp, ci, ci, ci,
                                                 cf, ci, vp, ctypes.POINTER(Info), vp, sz, vp]
        L.pararnn_newton_solve_reuse.restype = ci
        L.pararnn_reuse_workspace_size.argtypes = [ctypes.POINTER(Cell), ci, ci]
        L.pararnn_reuse_workspace_size.restype = sz
        L.pararnn_lstm_solve_host.argtypes = [ctypes.POINTER(Cell), ctypes.POINTER(Params), vp, vp, vp, ci, ci, cf, ci,
                                              vp, vp, ctypes.POINTER(Info), ci, vp, sz, vp]
        L.pararnn_lstm_solve_host.restype = ci
        L.pararnn_lstm_host_workspace_size.argtypes = [ctypes.POINTER(Cell), ci, ci, ci]
        L.pararnn_lstm_host_workspace_size.restype = sz
        L.pararnn_lstm_solve_host_streamed.argtypes = L.pararnn_lstm_solve_host.argtypes
        L.pararnn_lstm_solve_host_streamed.restype = ci
        L.pararnn_lstm_host_streamed_workspace_size.argtypes = [ctypes.POINTER(Cell), ci, ci, ci]
        L.pararnn_lstm_host_streamed_workspace_size.restype = sz
        L.pararnn_adjoint_host.argtypes = [ctypes.POINTER(Cell), ctypes.POINTER(Params), vp, vp, vp, vp, ci, ci,
                                           vp, vp, vp, vp, ci, vp, sz, vp]
        L.pararnn_adjoint_host.restype = ci
        L.pararnn_adjoint_host_workspace_size.argtypes = [ctypes.POINTER(Cell), ci, ci, ci]
        L.pararnn_adjoint_host_workspace_size.restype = sz
        L.pararnn_newton_solve_trace.argtypes = [ctypes.POINTER(Cell), ctypes.POINTER(Params), vp, vp, ci, ci, ci,
                                                 cf, cf, ci, vp, ctypes.POINTER(Info), vp, ci, vp, sz, vp]
        L.pararnn_newton_solve_trace.restype = ci
        L.pararnn_test_withheld_publish.argtypes = [ctypes.POINTER(Cell), ctypes.POINTER(Params), vp, vp, ci, ci,
                                                    ci, cf, vp, ctypes.POINTER(Info), ctypes.c_longlong, vp, sz, vp]
        L.pararnn_test_withheld_publish.restype = ci
        L.pararnn_adjoint_exact.argtypes = [ctypes.POINTER(Cell), ctypes.POINTER(Params), vp, vp, vp, vp, ci, ci,
                                            vp, vp, vp, vp, vp, sz, vp]
        L.pararnn_adjoint_exact.restype = ci
        L.pararnn_adjoint_exact_workspace_size.argtypes = [ctypes.POINTER(Cell), ci, ci]
        L.pararnn_adjoint_exact_workspace_size.restype = sz
        L.pararnn_status_string.argtypes = [ci]
        L.pararnn_status_string.restype = ctypes.c_char_p
        _lib = L
    return _lib


def _dtype_code(t: torch.dtype) -> int:
    if t == torch.float32:
        return F32
    if t == torch.bfloat16:
        return BF16
    raise TypeError(f"unsupported dtype {t}")


def _dev(t: torch.Tensor, name: str) -> int:
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


def _stream(stream) -> int:
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


def make_cell(kind: str, din: int, d: int, dtype: torch.dtype) -> Cell:
    code = {"dense": GRU_DENSE, "diag": GRU_DIAG, "lstm_diag": LSTM_DIAG}[kind]
    return Cell(code, din, d, _dtype_code(dtype), _dtype_code(dtype))


def lstm_workspace_size(din: int, d: int, B: int, T: int, dtype: torch.dtype = torch.float32) -> int:
    cell = make_cell("lstm_diag", din, d, dtype)
    return int(lib().pararnn_lstm_workspace_size(ctypes.byref(cell), B, T))


def lstm_solve(w_ih, b_ih, u, b_hh, x, c0, h0, *, tol: float, max_iters: int = 0, out=None, workspace=None,
               stream=None):
    """Evaluate the diagonal-recurrence LSTM over x [B, T, Din] by exact Newton.
    Weights: w_ih [4D, Din] (x's dtype), b_ih, u, b_hh [4D] fp32; c0, h0 [B, D].
    Returns (c, h, SolveResult) with c, h [B, T, D] fp32 CUDA tensors."""
    B, T, din = x.shape
    d = h0.shape[1]
    cell = make_cell("lstm_diag", din, d, x.dtype)
    L = lib()
    need = int(L.pararnn_lstm_workspace_size(ctypes.byref(cell), B, T))
    if need == 0:
        raise ValueError("arguments rejected by pararnn_lstm_workspace_size")
    if workspace is None:
        workspace = alloc_workspace(need, x.device)
    c, h = out if out is not None else (torch.empty(B, T, d, dtype=torch.float32, device=x.device),
                                        torch.empty(B, T, d, dtype=torch.float32, device=x.device))
    params = Params(_dev(w_ih, "w_ih"), _dev(b_ih, "b_ih"), _dev(u, "u"), _dev(b_hh, "b_hh"))
    info = Info()
    rc = L.pararnn_lstm_solve(ctypes.byref(cell), ctypes.byref(params), _dev(x, "x"), _dev(c0, "c0"), _dev(h0, "h0"),
                              B, T, float(tol), int(max_iters), _dev(c, "c"), _dev(h, "h"), ctypes.byref(info),
                              _dev(workspace, "workspace"), workspace.numel(), _stream(stream))
    if rc in (3, 4):
        raise RuntimeError(f"pararnn_lstm_solve: {L.pararnn_status_string(rc).decode()}")
    return c, h, SolveResult(h, info.iters, STATUS[info.status], info.delta, info.residual)


def workspace_size(kind: str, din: int, d: int, B: int, T: int, mode: str,
                   dtype: torch.dtype = torch.float32) -> int:
    cell = make_cell(kind, din, d, dtype)
    return int(lib().pararnn_workspace_size(ctypes.byref(cell), B, T, MODES[mode]))


def alloc_workspace(nbytes: int, device=None) -> torch.Tensor:
    """A 256-byte aligned device buffer of at least ``nbytes`` bytes."""
    buf = torch.empty(nbytes + 256, dtype=torch.uint8, device=device or "cuda")
    off = (-buf.data_ptr()) % 256
    return buf[off:off + nbytes]


@dataclass
class SolveResult:
    h: torch.Tensor
    iters: int
    status: str
    delta: float
    residual: float
    trace: object = None  # [iters, 2] host tensor: max |dh| and max |r| per iteration (trace=True)


def newton_solve(w_ih, b_ih, w_hh, b_hh, x, h0, *, kind: str, mode: str, tol: float,
                 lam: float = 0.0, max_iters: int = 0, out=None, workspace=None,
                 stream=None, sync: bool = True, info_dev=None, h_init=None, jac_every: int = 1,
                 trace: bool = False):
    """Evaluate the GRU over x [B, T, Din] with the chosen Newton mode.

    All tensors must be contiguous CUDA tensors (x and w_ih fp32 or bf16, the
    rest fp32).  With ``sync`` the call waits and returns a SolveResult; with
    ``sync=False`` it only enqueues, writing the report into ``info_dev`` (an
    int32 CUDA tensor of 4 elements) and returns ``out``.  ``h_init`` [B, T, D]
    (fp32 CUDA) starts the iteration from that guess instead of zero.
    ``jac_every`` > 1 (mode DEER, dense cell, d <= 32) recomputes the Jacobian
    only every jac_every iterations (synchronous; no h_init).  ``trace`` (sync
    only) also returns every iteration's max |dh| and max |r| (SolveResult.trace)."""
    B, T, din = x.shape
    d = h0.shape[1]
    cell = make_cell(kind, din, d, x.dtype)
    if w_ih.dtype != x.dtype:
        raise TypeError("x and w_ih must have the same dtype")
    L = lib()
    if jac_every != 1:
        if mode != "DEER" or h_init is not None or not sync:
            raise ValueError("jac_every > 1 takes mode DEER, sync=True and no h_init")
        need = int(L.pararnn_reuse_workspace_size(ctypes.byref(cell), B, T))
        if need == 0:
            raise ValueError("arguments rejected by pararnn_reuse_workspace_size")
        if workspace is None:
            workspace = alloc_workspace(need, x.device)
        if out is None:
            out = torch.empty(B, T, d, dtype=torch.float32, device=x.device)
        params = Params(_dev(w_ih, "w_ih"), _dev(b_ih, "b_ih"), _dev(w_hh, "w_hh"), _dev(b_hh, "b_hh"))
        info = Info()
        rc = L.pararnn_newton_solve_reuse(ctypes.byref(cell), ctypes.byref(params), _dev(x, "x"), _dev(h0, "h0"),
                                          B, T, int(jac_every), float(tol), int(max_iters), _dev(out, "out"),
                                          ctypes.byref(info), _dev(workspace, "workspace"), workspace.numel(),
                                          _stream(stream))
        if rc in (3, 4):
            raise RuntimeError(f"pararnn_newton_solve_reuse: {L.pararnn_status_string(rc).decode()}")
        return SolveResult(out, info.iters, STATUS[info.status], info.delta, info.residual)
    m = MODES[mode]
    need = int(L.pararnn_workspace_size(ctypes.byref(cell), B, T, m))
    if need == 0:
        raise ValueError("arguments rejected by pararnn_workspace_size")
    if workspace is None:
        workspace = alloc_workspace(need, x.device)
    if out is None:
        out = torch.empty(B, T, d, dtype=torch.float32, device=x.device)
    params = Params(_dev(w_ih, "w_ih"), _dev(b_ih, "b_ih"), _dev(w_hh, "w_hh"), _dev(b_hh, "b_hh"))
    args = (ctypes.byref(cell), ctypes.byref(params), _dev(x, "x"), _dev(h0, "h0"), B, T, m,
            float(lam), float(tol), int(max_iters), _dev(out, "out"))
    if h_init is not None:
        own = info_dev is None
        if own:
            info_dev = torch.zeros(4, dtype=torch.int32, device=x.device)
        rc = L.pararnn_newton_solve_guess_async(ctypes.byref(cell), ctypes.byref(params), _dev(x, "x"),
                                                _dev(h0, "h0"), _dev(h_init, "h_init"), B, T, m, float(lam),
                                                float(tol), int(max_iters), _dev(out, "out"),
                                                _dev(info_dev, "info_dev"), _dev(workspace, "workspace"),
                                                workspace.numel(), _stream(stream))
        if rc != 0:
            raise RuntimeError(f"pararnn_newton_solve_guess_async: {L.pararnn_status_string(rc).decode()}")
        if not sync:
            return out
        rep = info_dev.cpu()  # waits for the solve
        return SolveResult(out, int(rep[0]), STATUS[int(rep[1])], float(rep[2:3].view(torch.float32)),
                           float(rep[3:4].view(torch.float32)))
    if sync and trace:
        cap = int(max_iters) if max_iters > 0 else T + 1
        tr = torch.full((cap, 2), float("nan"), dtype=torch.float32, device=x.device)
        info = Info()
        rc = L.pararnn_newton_solve_trace(*args, ctypes.byref(info), _dev(tr, "trace"), cap,
                                          _dev(workspace, "workspace"), workspace.numel(), _stream(stream))
        if rc in (3, 4):
            raise RuntimeError(f"pararnn_newton_solve_trace: {L.pararnn_status_string(rc).decode()}")
        return SolveResult(out, info.iters, STATUS[info.status], info.delta, info.residual,
                           tr[:info.iters].cpu())
    if sync:
        info = Info()
        rc = L.pararnn_newton_solve(*args, ctypes.byref(info), _dev(workspace, "workspace"),
                                    workspace.numel(), _stream(stream))
        if rc in (3, 4):
            raise RuntimeError(f"pararnn_newton_solve: {L.pararnn_status_string(rc).decode()}")
        return SolveResult(out, info.iters, STATUS[info.status], info.delta, info.residual)
    if info_dev is None:
        raise ValueError("sync=False needs info_dev (int32 CUDA tensor with 4 elements)")
    rc = L.pararnn_newton_solve_async(*args, _dev(info_dev, "info_dev"),
                                      _dev(workspace, "workspace"), workspace.numel(),
                                      _stream(stream))
    if rc != 0:
        raise RuntimeError(f"pararnn_newton_solve_async: {L.pararnn_status_string(rc).decode()}")
    return out


def _host(t: torch.Tensor, name: str) -> int:
    if t.is_cuda:
        raise ValueError(f"{name} must be a host tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


def newton_solve_chunked(w_ih, b_ih, w_hh, b_hh, x, h0, *, kind: str, mode: str, tol: float, t_chunk: int,
                         lam: float = 0.0, max_iters: int = 0, out=None, workspace=None,
                         stream=None) -> "SolveResult":
    """The solve over consecutive time chunks of at most ``t_chunk`` steps (device
    memory grows with t_chunk, not T); the report sums iterations over chunks."""
    B, T, din = x.shape
    d = h0.shape[1]
    cell = make_cell(kind, din, d, x.dtype)
    L = lib()
    m = MODES[mode]
    need = int(L.pararnn_chunked_workspace_size(ctypes.byref(cell), B, T, int(t_chunk), m))
    if need == 0:
        raise ValueError("arguments rejected by pararnn_chunked_workspace_size")
    if workspace is None:
        workspace = alloc_workspace(need, x.device)
    if out is None:
        out = torch.empty(B, T, d, dtype=torch.float32, device=x.device)
    params = Params(_dev(w_ih, "w_ih"), _dev(b_ih, "b_ih"), _dev(w_hh, "w_hh"), _dev(b_hh, "b_hh"))
    info = Info()
    rc = L.pararnn_newton_solve_chunked(ctypes.byref(cell), ctypes.byref(params), _dev(x, "x"), _dev(h0, "h0"),
                                        B, T, int(t_chunk), m, float(lam), float(tol), int(max_iters),
                                        _dev(out, "out"), ctypes.byref(info), _dev(workspace, "workspace"),
                                        workspace.numel(), _stream(stream))
    if rc in (3, 4):
        raise RuntimeError(f"pararnn_newton_solve_chunked: {L.pararnn_status_string(rc).decode()}")
    return SolveResult(out, info.iters, STATUS[info.status], info.delta, info.residual)


def chunked_workspace_size(kind: str, din: int, d: int, B: int, T: int, t_chunk: int, mode: str,
                           dtype: torch.dtype = torch.float32) -> int:
    cell = make_cell(kind, din, d, dtype)
    return int(lib().pararnn_chunked_workspace_size(ctypes.byref(cell), B, T, int(t_chunk), MODES[mode]))


def host_workspace_size(kind: str, din: int, d: int, B: int, T: int, mode: str, parts: int,
                        dtype: torch.dtype = torch.float32) -> int:
    cell = make_cell(kind, din, d, dtype)
    return int(lib().pararnn_host_workspace_size(ctypes.byref(cell), B, T, MODES[mode], parts))


def newton_solve_host(w_ih, b_ih, w_hh, b_hh, x_host, h0_host, *, kind: str, mode: str, tol: float,
                      lam: float = 0.0, max_iters: int = 0, parts: int = 4, out=None,
                      workspace=None, device=None, stream=None) -> "SolveResult":
    """The solve from and to HOST tensors (x_host [B,T,Din], h0_host [B,D];
    ``out`` a host [B,T,D] fp32 tensor, page-locked for overlap).  The batch is
    solved in ``parts`` parts with copies overlapped with compute; weights are
    CUDA tensors.  Returns a SolveResult whose h is the host tensor and whose
    report is the worst part's."""
    B, T, din = x_host.shape
    d = h0_host.shape[1]
    parts = max(1, min(int(parts), B))
    cell = make_cell(kind, din, d, x_host.dtype)
    L = lib()
    m = MODES[mode]
    need = int(L.pararnn_host_workspace_size(ctypes.byref(cell), B, T, m, parts))
    if need == 0:
        raise ValueError("arguments rejected by pararnn_host_workspace_size")
    if workspace is None:
        workspace = alloc_workspace(need, w_hh.device if device is None else device)
    if out is None:
        out = torch.empty(B, T, d, dtype=torch.float32).pin_memory()
    params = Params(_dev(w_ih, "w_ih"), _dev(b_ih, "b_ih"), _dev(w_hh, "w_hh"), _dev(b_hh, "b_hh"))
    info = Info()
    rc = L.pararnn_newton_solve_host(ctypes.byref(cell), ctypes.byref(params), _host(x_host, "x_host"),
                                     _host(h0_host, "h0_host"), B, T, m, float(lam), float(tol),
                                     int(max_iters), _host(out, "out"), ctypes.byref(info), parts,
                                     _dev(workspace, "workspace"), workspace.numel(), _stream(stream))
    if rc in (3, 4):
        raise RuntimeError(f"pararnn_newton_solve_host: {L.pararnn_status_string(rc).decode()}")
    return SolveResult(out, info.iters, STATUS[info.status], info.delta, info.residual)


def host_streamed_workspace_size(kind: str, din: int, d: int, B: int, T: int, mode: str, parts: int,
                                 dtype: torch.dtype = torch.float32) -> int:
    cell = make_cell(kind, din, d, dtype)
    return int(lib().pararnn_host_streamed_workspace_size(ctypes.byref(cell), B, T, MODES[mode], parts))


def newton_solve_host_streamed(w_ih, b_ih, w_hh, b_hh, x_host, h0_host, *, kind: str, mode: str, tol: float,
                               lam: float = 0.0, max_iters: int = 0, parts: int = 7, out=None,
                               workspace=None, device=None, stream=None) -> "SolveResult":
    """The solve from and to HOST tensors with the sequence streamed through
    the device in ``parts`` time parts (whole batch in each; clamped to
    1 .. ceil(T / 128)), each part solved from the previous part's last states
    while the next part's inputs are copied in and the previous part's states
    out.  The report sums iterations over the parts."""
    B, T, din = x_host.shape
    d = h0_host.shape[1]
    parts = max(1, min(int(parts), (T + 127) // 128))
    cell = make_cell(kind, din, d, x_host.dtype)
    L = lib()
    m = MODES[mode]
    need = int(L.pararnn_host_streamed_workspace_size(ctypes.byref(cell), B, T, m, parts))
    if need == 0:
        raise ValueError("arguments rejected by pararnn_host_streamed_workspace_size")
    if workspace is None:
        workspace = alloc_workspace(need, w_hh.device if device is None else device)
    if out is None:
        out = torch.empty(B, T, d, dtype=torch.float32).pin_memory()
    params = Params(_dev(w_ih, "w_ih"), _dev(b_ih, "b_ih"), _dev(w_hh, "w_hh"), _dev(b_hh, "b_hh"))
    info = Info()
    rc = L.pararnn_newton_solve_host_streamed(ctypes.byref(cell), ctypes.byref(params), _host(x_host, "x_host"),
                                              _host(h0_host, "h0_host"), B, T, m, float(lam), float(tol),
                                              int(max_iters), _host(out, "out"), ctypes.byref(info), parts,
                                              _dev(workspace, "workspace"), workspace.numel(), _stream(stream))
    if rc in (3, 4):
        raise RuntimeError(f"pararnn_newton_solve_host_streamed: {L.pararnn_status_string(rc).decode()}")
    return SolveResult(out, info.iters, STATUS[info.status], info.delta, info.residual)


def lstm_solve_host(w_ih, b_ih, u, b_hh, x_host, c0_host, h0_host, *, tol: float, max_iters: int = 0,
                    parts: int = 4, out=None, workspace=None, device=None, stream=None):
    """The LSTM solve from and to HOST tensors (x_host [B,T,Din], c0_host and
    h0_host [B,D]; ``out`` a pair of host [B,T,D] fp32 tensors, page-locked for
    overlap), in ``parts`` parts with the copies overlapped with compute;
    weights are CUDA tensors.  Returns (c, h, SolveResult) with host c, h."""
    B, T, din = x_host.shape
    d = h0_host.shape[1]
    parts = max(1, min(int(parts), B))
    cell = make_cell("lstm_diag", din, d, x_host.dtype)
    L = lib()
    need = int(L.pararnn_lstm_host_workspace_size(ctypes.byref(cell), B, T, parts))
    if need == 0:
        raise ValueError("arguments rejected by pararnn_lstm_host_workspace_size")
    if workspace is None:
        workspace = alloc_workspace(need, u.device if device is None else device)
    c, h = out if out is not None else (torch.empty(B, T, d, dtype=torch.float32).pin_memory(),
                                        torch.empty(B, T, d, dtype=torch.float32).pin_memory())
    params = Params(_dev(w_ih, "w_ih"), _dev(b_ih, "b_ih"), _dev(u, "u"), _dev(b_hh, "b_hh"))
    info = Info()
    rc = L.pararnn_lstm_solve_host(ctypes.byref(cell), ctypes.byref(params), _host(x_host, "x_host"),
                                   _host(c0_host, "c0_host"), _host(h0_host, "h0_host"), B, T, float(tol),
                                   int(max_iters), _host(c, "c"), _host(h, "h"), ctypes.byref(info), parts,
                                   _dev(workspace, "workspace"), workspace.numel(), _stream(stream))
    if rc in (3, 4):
        raise RuntimeError(f"pararnn_lstm_solve_host: {L.pararnn_status_string(rc).decode()}")
    return c, h, SolveResult(h, info.iters, STATUS[info.status], info.delta, info.residual)


def lstm_solve_host_streamed(w_ih, b_ih, u, b_hh, x_host, c0_host, h0_host, *, tol: float, max_iters: int = 0,
                             parts: int = 7, out=None, workspace=None, device=None, stream=None):
    """The LSTM solve from and to HOST tensors with the sequence streamed
    through the device in ``parts`` time parts (clamped to 1 .. ceil(T / 128));
    the report sums iterations over the parts.  Returns (c, h, SolveResult)."""
    B, T, din = x_host.shape
    d = h0_host.shape[1]
    parts = max(1, min(int(parts), (T + 127) // 128))
    cell = make_cell("lstm_diag", din, d, x_host.dtype)
    L = lib()
    need = int(L.pararnn_lstm_host_streamed_workspace_size(ctypes.byref(cell), B, T, parts))
    if need == 0:
        raise ValueError("arguments rejected by pararnn_lstm_host_streamed_workspace_size")
    if workspace is None:
        workspace = alloc_workspace(need, u.device if device is None else device)
    c, h = out if out is not None else (torch.empty(B, T, d, dtype=torch.float32).pin_memory(),
                                        torch.empty(B, T, d, dtype=torch.float32).pin_memory())
    params = Params(_dev(w_ih, "w_ih"), _dev(b_ih, "b_ih"), _dev(u, "u"), _dev(b_hh, "b_hh"))
    info = Info()
    rc = L.pararnn_lstm_solve_host_streamed(ctypes.byref(cell), ctypes.byref(params), _host(x_host, "x_host"),
                                            _host(c0_host, "c0_host"), _host(h0_host, "h0_host"), B, T, float(tol),
                                            int(max_iters), _host(c, "c"), _host(h, "h"), ctypes.byref(info), parts,
                                            _dev(workspace, "workspace"), workspace.numel(), _stream(stream))
    if rc in (3, 4):
        raise RuntimeError(f"pararnn_lstm_solve_host_streamed: {L.pararnn_status_string(rc).decode()}")
    return c, h, SolveResult(h, info.iters, STATUS[info.status], info.delta, info.residual)


def lstm_host_streamed_workspace_size(din: int, d: int, B: int, T: int, parts: int,
                                      dtype: torch.dtype = torch.bfloat16) -> int:
    cell = make_cell("lstm_diag", din, d, dtype)
    return int(lib().pararnn_lstm_host_streamed_workspace_size(ctypes.byref(cell), B, T, parts))


def adjoint_workspace_size(d: int, B: int, T: int, kind: str = "diag") -> int:
    cell = make_cell(kind, 1, d, torch.float32)
    return int(lib().pararnn_adjoint_workspace_size(ctypes.byref(cell), B, T))


def adjoint_exact(w_hh, b_hh, P, h0, h, dh, *, workspace=None, out=None, stream=None) -> dict:
    """The exact backward pass of the dense GRU (full transposed Jacobian):
    w_hh [3D, D], b_hh [3D], P [B,T,3D], h0 [B,D], h and dh [B,T,D], all fp32
    CUDA.  Returns dict(dP, dh0, dw_hh, db_hh)."""
    B, T, d = h.shape
    cell = make_cell("dense", 1, d, torch.float32)
    L = lib()
    need = int(L.pararnn_adjoint_exact_workspace_size(ctypes.byref(cell), B, T))
    if need == 0:
        raise ValueError("arguments rejected by pararnn_adjoint_exact_workspace_size")
    if workspace is None:
        workspace = alloc_workspace(need, h.device)
    o = out or {}
    dP = o["dP"] if "dP" in o else torch.empty_like(P)
    dh0 = o["dh0"] if "dh0" in o else torch.empty_like(h0)
    dw = o["dw_hh"] if "dw_hh" in o else torch.empty_like(w_hh)
    db = o["db_hh"] if "db_hh" in o else torch.empty_like(b_hh)
    params = Params(None, None, _dev(w_hh, "w_hh"), _dev(b_hh, "b_hh"))
    rc = L.pararnn_adjoint_exact(ctypes.byref(cell), ctypes.byref(params), _dev(P, "P"), _dev(h0, "h0"),
                                 _dev(h, "h"), _dev(dh, "dh"), B, T, _dev(dP, "dP"), _dev(dh0, "dh0"),
                                 _dev(dw, "dw_hh"), _dev(db, "db_hh"), _dev(workspace, "workspace"),
                                 workspace.numel(), _stream(stream))
    if rc != 0:
        raise RuntimeError(f"pararnn_adjoint_exact: {L.pararnn_status_string(rc).decode()}")
    return dict(dP=dP, dh0=dh0, dw_hh=dw, db_hh=db)


def adjoint(w_hh, b_hh, P, h0, h, dh, *, workspace=None, out=None, stream=None, check: bool = False) -> dict:
    """Backward pass of the GRU through the states h: gradients w.r.t. the
    pre-activations P [B,T,3D], h0 [B,D], w_hh and b_hh [3D], given
    dh = dL/dh [B,T,D] (all fp32 CUDA).  w_hh [3D] is the diagonal cell (exact
    gradients); w_hh [3D, D] the dense cell, whose adjoint runs with the
    Jacobian's diagonal (D <= 64).  Returns dict(dP, dh0, dw_hh, db_hh)."""
    B, T, d = h.shape
    cell = make_cell("dense" if w_hh.dim() == 2 else "diag", 1, d, torch.float32)
    L = lib()
    need = int(L.pararnn_adjoint_workspace_size(ctypes.byref(cell), B, T))
    if need == 0:
        raise ValueError("arguments rejected by pararnn_adjoint_workspace_size")
    if workspace is None:
        workspace = alloc_workspace(need, h.device)
    o = out or {}
    dP = o["dP"] if "dP" in o else torch.empty_like(P)
    dh0 = o["dh0"] if "dh0" in o else torch.empty_like(h0)
    dw = o["dw_hh"] if "dw_hh" in o else torch.empty_like(w_hh)
    db = o["db_hh"] if "db_hh" in o else torch.empty_like(b_hh)
    params = Params(None, None, _dev(w_hh, "w_hh"), _dev(b_hh, "b_hh"))
    rc = L.pararnn_adjoint(ctypes.byref(cell), ctypes.byref(params), _dev(P, "P"), _dev(h0, "h0"), _dev(h, "h"),
                           _dev(dh, "dh"), B, T, _dev(dP, "dP"), _dev(dh0, "dh0"), _dev(dw, "dw_hh"),
                           _dev(db, "db_hh"), _dev(workspace, "workspace"), workspace.numel(), _stream(stream))
    if rc != 0:
        raise RuntimeError(f"pararnn_adjoint: {L.pararnn_status_string(rc).decode()}")
    if check:
        st = L.pararnn_adjoint_status(_dev(workspace, "workspace"), _stream(stream))
        if st != 0:
            raise RuntimeError(f"pararnn_adjoint: {STATUS.get(st, st)}")
    return dict(dP=dP, dh0=dh0, dw_hh=dw, db_hh=db)


def adjoint_host(w_hh, b_hh, P_host, h0_host, h_host, dh_host, *, parts: int = 4, out=None, workspace=None,
                 stream=None) -> dict:
    """The backward pass from and to HOST tensors (P_host [B,T,3D], h0_host
    [B,D], h_host and dh_host [B,T,D], page-locked for overlap), in ``parts``
    parts with the copies overlapped with compute; w_hh, b_hh CUDA tensors
    (w_hh [3D]: diagonal cell, [3D, D]: dense cell).  Returns dict(dP, dh0,
    dw_hh, db_hh) of host tensors."""
    B, T, d = h_host.shape
    parts = max(1, min(int(parts), B))
    cell = make_cell("dense" if w_hh.dim() == 2 else "diag", 1, d, torch.float32)
    L = lib()
    need = int(L.pararnn_adjoint_host_workspace_size(ctypes.byref(cell), B, T, parts))
    if need == 0:
        raise ValueError("arguments rejected by pararnn_adjoint_host_workspace_size")
    if workspace is None:
        workspace = alloc_workspace(need, w_hh.device)
    o = out or {}
    pinned = lambda key, shape: o[key] if key in o else torch.empty(shape, dtype=torch.float32).pin_memory()
    dP = pinned("dP", P_host.shape)
    dh0 = pinned("dh0", h0_host.shape)
    dw = pinned("dw_hh", w_hh.shape)
    db = pinned("db_hh", b_hh.shape)
    params = Params(None, None, _dev(w_hh, "w_hh"), _dev(b_hh, "b_hh"))
    rc = L.pararnn_adjoint_host(ctypes.byref(cell), ctypes.byref(params), _host(P_host, "P_host"),
                                _host(h0_host, "h0_host"), _host(h_host, "h_host"), _host(dh_host, "dh_host"), B, T,
                                _host(dP, "dP"), _host(dh0, "dh0"), _host(dw, "dw_hh"), _host(db, "db_hh"), parts,
                                _dev(workspace, "workspace"), workspace.numel(), _stream(stream))
    if rc != 0:
        raise RuntimeError(f"pararnn_adjoint_host: {L.pararnn_status_string(rc).decode()}")
    return dict(dP=dP, dh0=dh0, dw_hh=dw, db_hh=db)


def input_projection(x, w_ih, b_ih, *, d: int, kind: str = "dense", out=None, stream=None):
    """P = x W_ih^T + b_ih for every step: x [B,T,Din] -> P [B,T,3D] fp32."""
    B, T, din = x.shape
    cell = make_cell(kind, din, d, x.dtype)
    if out is None:
        out = torch.empty(B, T, 3 * d, dtype=torch.float32, device=x.device)
    params = Params(_dev(w_ih, "w_ih"), _dev(b_ih, "b_ih"), 0, 0)
    rc = lib().pararnn_input_projection(ctypes.byref(cell), ctypes.byref(params), _dev(x, "x"),
                                        B, T, _dev(out, "out"), _stream(stream))
    if rc != 0:
        raise RuntimeError(f"pararnn_input_projection: {STATUS.get(rc, rc)}")
    return out


def newton_iterate(P, w_hh, b_hh, h0, *, kind: str, din: int, mode: str, tol: float,
                   info_dev, lam: float = 0.0, max_iters: int = 0, out=None, workspace=None,
                   dtype=torch.float32, stream=None):
    """Enqueue the Newton loop on precomputed P [B,T,3D]; report into info_dev."""
    B, T, _ = P.shape
    d = h0.shape[1]
    cell = make_cell(kind, din, d, dtype)
    L = lib()
    m = MODES[mode]
    if workspace is None:
        workspace = alloc_workspace(int(L.pararnn_workspace_size(ctypes.byref(cell), B, T, m)),
                                    P.device)
    if out is None:
        out = torch.empty(B, T, d, dtype=torch.float32, device=P.device)
    params = Params(0, 0, _dev(w_hh, "w_hh"), _dev(b_hh, "b_hh"))
    rc = L.pararnn_newton_iterate_async(ctypes.byref(cell), ctypes.byref(params), _dev(P, "P"),
                                        _dev(h0, "h0"), B, T, m, float(lam), float(tol),
                                        int(max_iters), _dev(out, "out"), _dev(info_dev, "info"),
                                        _dev(workspace, "workspace"), workspace.numel(),
                                        _stream(stream))
    if rc != 0:
        raise RuntimeError(f"pararnn_newton_iterate_async: {STATUS.get(rc, rc)}")
    return out


def solve_workload(w, mode: str, *, lam: float = 0.0, tol=None, max_iters: int = 0,
                   device="cuda", **kw) -> SolveResult:
    """Move a ``inputs.Workload`` to the device and solve it."""
    dev = lambda t: t.to(device).contiguous()
    return newton_solve(dev(w.w_ih), dev(w.b_ih), dev(w.w_hh), dev(w.b_hh), dev(w.x), dev(w.h0),
                        kind=w.kind, mode=mode, tol=w.tol if tol is None else tol, lam=lam,
                        max_iters=max_iters, **kw)


def withheld_publish(w, mode: str, tile: int, *, out=None, workspace=None, device="cuda",
                     stream=None) -> SolveResult:
    """The testing hook pararnn_test_withheld_publish on a ``inputs.Workload``:
    the solve with look-back tile ``tile`` silent in the first iteration."""
    dev = lambda t: t.to(device).contiguous()
    x, h0 = dev(w.x), dev(w.h0)
    B, T, din = x.shape
    d = h0.shape[1]
    cell = make_cell(w.kind, din, d, x.dtype)
    L = lib()
    m = MODES[mode]
    need = int(L.pararnn_workspace_size(ctypes.byref(cell), B, T, m))
    if workspace is None:
        workspace = alloc_workspace(need, x.device)
    if out is None:
        out = torch.empty(B, T, d, dtype=torch.float32, device=x.device)
    w_ih, b_ih, w_hh, b_hh = dev(w.w_ih), dev(w.b_ih), dev(w.w_hh), dev(w.b_hh)
    params = Params(_dev(w_ih, "w_ih"), _dev(b_ih, "b_ih"), _dev(w_hh, "w_hh"), _dev(b_hh, "b_hh"))
    info = Info()
    rc = L.pararnn_test_withheld_publish(ctypes.byref(cell), ctypes.byref(params), _dev(x, "x"), _dev(h0, "h0"),
                                         B, T, m, float(w.tol), _dev(out, "out"), ctypes.byref(info), int(tile),
                                         _dev(workspace, "workspace"), workspace.numel(), _stream(stream))
    if rc in (3, 4):
        raise RuntimeError(f"pararnn_test_withheld_publish: {L.pararnn_status_string(rc).decode()}")
    return SolveResult(out, info.iters, STATUS[info.status], info.delta, info.residual)


def affine_scan(A, b, h0, *, out=None, workspace=None, stream=None, check: bool = False):
    """h_t = A_t h_{t-1} + b_t over t for every sequence.  A is [B,T,D]
    (diagonal) or [B,T,D,D] (dense); b [B,T,D]; h0 [B,D]; all fp32 CUDA."""
    B, T, D = b.shape
    dense = 1 if A.dim() == 4 else 0
    L = lib()
    need = int(L.pararnn_affine_scan_workspace_size(B, T, D, dense))
    if need == 0:
        raise ValueError("arguments rejected by pararnn_affine_scan_workspace_size")
    if workspace is None:
        workspace = alloc_workspace(need, b.device)
    if out is None:
        out = torch.empty_like(b)
    rc = L.pararnn_affine_scan(_dev(A, "A"), _dev(b, "b"), _dev(h0, "h0"), B, T, D, dense,
                               _dev(out, "out"), _dev(workspace, "workspace"), workspace.numel(),
                               _stream(stream))
    if rc != 0:
        raise RuntimeError(f"pararnn_affine_scan: {L.pararnn_status_string(rc).decode()}")
    if check:
        st = L.pararnn_affine_scan_status(_dev(workspace, "workspace"), _stream(stream))
        if st != 0:
            raise RuntimeError(f"pararnn_affine_scan: {STATUS.get(st, st)}")
    return out


def affine_scan_host(A_host, b_host, h0_host, *, parts: int = 7, out=None, workspace=None, device=None,
                     stream=None):
    """The affine scan from and to HOST tensors (A [B,T,D] or [B,T,D,D], b
    [B,T,D], h0 [B,D], fp32; page-locked for overlap), streamed through the
    device in ``parts`` time parts (clamped to 1 .. ceil(T / 128)), each part
    started from the previous part's last states.  Returns the host h."""
    B, T, D = b_host.shape
    dense = 1 if A_host.dim() == 4 else 0
    parts = max(1, min(int(parts), (T + 127) // 128))
    L = lib()
    need = int(L.pararnn_affine_scan_host_workspace_size(B, T, D, dense, parts))
    if need == 0:
        raise ValueError("arguments rejected by pararnn_affine_scan_host_workspace_size")
    if workspace is None:
        workspace = alloc_workspace(need, device or "cuda")
    if out is None:
        out = torch.empty(B, T, D, dtype=torch.float32).pin_memory()
    rc = L.pararnn_affine_scan_host(_host(A_host, "A_host"), _host(b_host, "b_host"), _host(h0_host, "h0_host"),
                                    B, T, D, dense, _host(out, "out"), parts, _dev(workspace, "workspace"),
                                    workspace.numel(), _stream(stream))
    if rc != 0:
        raise RuntimeError(f"pararnn_affine_scan_host: {L.pararnn_status_string(rc).decode()}")
    return out
