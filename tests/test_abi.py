"""The C ABI library loads and exports every entry point the header declares.

CPU only: these call host-side functions of the library (size queries and
status names), never a kernel.
"""
import ctypes
import os
import re

import pytest

from newton_solve_nonlinear_b200 import binding

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = []
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            names += re.findall(r"PARARNN_API\s+[\w\s\*]+?\b(pararnn_\w+)\s*\(", src)
    return names


@pytest.fixture(scope="module")
def L():
    if not os.path.exists(binding._LIB_PATH):
        from newton_solve_nonlinear_b200 import build
        build.build()
    return binding.lib()


def test_every_declared_symbol_is_exported(L):
    names = _declared()
    assert set(names) >= set(binding.EXPORTS)
    for n in names:
        assert hasattr(L, n), n


def test_status_strings(L):
    for code, name in binding.STATUS.items():
        assert L.pararnn_status_string(code).decode() == "PARARNN_" + name
    assert L.pararnn_status_string(99).decode() == "PARARNN_UNKNOWN_STATUS"


def test_workspace_sizes(L):
    ws = lambda *a, **k: binding.workspace_size(*a, **k)
    # valid problems need at least the projection and a second iterate buffer
    n = ws("dense", 64, 64, 16, 1024, "QUASI")
    assert n >= 16 * 1024 * 64 * 4 * 4
    assert ws("diag", 2048, 2048, 8, 4096, "QUASI") >= 8 * 4096 * 2048 * 16
    # quasi-ELK keeps its forward results
    assert ws("dense", 64, 64, 8, 1000, "QUASI_ELK") > ws("dense", 64, 64, 8, 1000, "QUASI")
    # ELK on the dense cell keeps three D x D blocks per step for the reduction
    assert ws("dense", 64, 64, 8, 10000, "ELK") >= 3 * 8 * 10000 * 64 * 64 * 4
    assert ws("dense", 4, 12, 2, 33, "ELK") >= 3 * 2 * 33 * 16 * 16 * 4
    # rejected: D not a multiple of 4, dense D > 64, bad mode, empty sizes
    assert ws("dense", 4, 6, 1, 10, "QUASI") == 0
    assert ws("dense", 4, 128, 1, 10, "QUASI") == 0
    assert ws("diag", 4, 128, 1, 10, "QUASI") > 0
    assert ws("dense", 4, 8, 0, 10, "QUASI") == 0
    assert ws("dense", 4, 8, 1, 0, "QUASI") == 0
    cell = binding.make_cell("dense", 4, 8, __import__("torch").float32)
    assert L.pararnn_workspace_size(ctypes.byref(cell), 1, 10, 7) == 0


def test_scan_workspace_sizes(L):
    assert L.pararnn_affine_scan_workspace_size(16, 1024, 64, 0) > 0
    assert L.pararnn_affine_scan_workspace_size(16, 1024, 62, 0) == 0
    assert L.pararnn_affine_scan_workspace_size(0, 1024, 64, 0) == 0


def test_invalid_arguments_are_rejected_without_a_gpu(L):
    """Argument checks run on the host before anything is enqueued."""
    cell = binding.make_cell("dense", 4, 8, __import__("torch").float32)
    params = binding.Params(0, 0, 0, 0)
    rc = L.pararnn_newton_solve(ctypes.byref(cell), ctypes.byref(params), None, None, 1, 10, 1,
                                0.0, 1e-5, 0, None, None, None, 0, None)
    assert rc == 3
    rc = L.pararnn_affine_scan(None, None, None, 1, 10, 8, 0, None, None, 0, None)
    assert rc == 3


def _al(n):
    return (n + 255) // 256 * 256


@pytest.mark.parametrize("B,parts,largest", [(16, 7, 4), (16, 6, 4), (16, 1, 16), (8, 7, 2), (5, 5, 1), (4, 3, 2)])
def test_host_pipeline_part_sizes(L, B, parts, largest):
    """The host-buffer solve ramps its parts (weights 1, 2, 3, 4, ..., 4, 3, 2, 1,
    largest remainder, at least one sequence each); its workspace is one solve
    workspace for the largest part, three staging buffers (fewer when there are
    fewer parts) of that part's x and h, h0 for the batch and one report per part."""
    T, din, d = 1000, 64, 64
    cell = binding.make_cell("dense", din, d, binding.torch.float32)
    m = binding.MODES["QUASI"]
    solve = L.pararnn_workspace_size(ctypes.byref(cell), largest, T, m)
    nbuf = min(parts, 3)
    want = (_al(solve) + nbuf * _al(largest * T * din * 4) + nbuf * _al(largest * T * d * 4) + _al(B * d * 4)
            + _al(parts * 16))
    assert L.pararnn_host_workspace_size(ctypes.byref(cell), B, T, m, parts) == want
    assert L.pararnn_host_workspace_size(ctypes.byref(cell), B, T, m, B + 1) == 0


def test_reuse_and_adjoint_size_queries(L):
    dense32 = binding.make_cell("dense", 16, 32, binding.torch.float32)
    dense64 = binding.make_cell("dense", 64, 64, binding.torch.float32)
    m = binding.MODES["DEER"]
    assert L.pararnn_reuse_workspace_size(ctypes.byref(dense32), 4, 1000) == \
        L.pararnn_workspace_size(ctypes.byref(dense32), 4, 1000, m) + _al(4 * 1000 * 512)
    assert L.pararnn_reuse_workspace_size(ctypes.byref(dense64), 4, 1000) == 0
    assert L.pararnn_adjoint_workspace_size(ctypes.byref(dense64), 2, 100) > 0
    assert L.pararnn_adjoint_workspace_size(ctypes.byref(binding.make_cell("dense", 65, 65, binding.torch.float32)),
                                            2, 100) == 0
    assert L.pararnn_adjoint_host_workspace_size(ctypes.byref(dense64), 4, 100, 3) > 0
    assert L.pararnn_adjoint_host_workspace_size(ctypes.byref(dense64), 4, 100, 5) == 0


@pytest.mark.parametrize("T,parts,largest", [(65536, 7, 16384), (1000, 3, 512), (300, 3, 128), (129, 2, 128),
                                             (4096, 7, 1024), (1, 1, 1)])
def test_streamed_host_part_sizes(L, T, parts, largest):
    """The streamed calls split T in 128-step units with the ramped weights
    (T = 65536 in 7 parts: 4096, 8192, 12288, 16384, ...); their workspace is
    one solve (or scan) workspace for the longest part, three staging buffers
    (fewer when there are fewer parts) of that part for every sequence, h0 and
    the carry for the batch, and one report per part.  parts > ceil(T / 128)
    is rejected."""
    B, din, d = 4, 64, 64
    cell = binding.make_cell("dense", din, d, binding.torch.float32)
    m = binding.MODES["QUASI"]
    solve = L.pararnn_workspace_size(ctypes.byref(cell), B, largest, m)
    nbuf = min(parts, 3)
    want = (_al(solve) + nbuf * _al(B * largest * din * 4) + nbuf * _al(B * largest * d * 4) + 2 * _al(B * d * 4)
            + _al(parts * 16))
    assert L.pararnn_host_streamed_workspace_size(ctypes.byref(cell), B, T, m, parts) == want
    assert L.pararnn_host_streamed_workspace_size(ctypes.byref(cell), B, T, m, (T + 127) // 128 + 1) == 0
    # the scan from host memory: A, b and h staged per part, h0 and the carry, a status word per part
    scan = L.pararnn_affine_scan_workspace_size(B, largest, d, 0)
    want_scan = (_al(scan) + 3 * nbuf * _al(B * largest * d * 4) + 2 * _al(B * d * 4) + _al(parts * 4))
    assert L.pararnn_affine_scan_host_workspace_size(B, T, d, 0, parts) == want_scan
    assert L.pararnn_affine_scan_host_workspace_size(B, T, d, 0, (T + 127) // 128 + 1) == 0
    lstm = binding.make_cell("lstm_diag", din, d, binding.torch.float32)
    assert L.pararnn_lstm_host_streamed_workspace_size(ctypes.byref(lstm), B, T, parts) > 0
    assert L.pararnn_lstm_host_streamed_workspace_size(ctypes.byref(lstm), B, T, (T + 127) // 128 + 1) == 0
