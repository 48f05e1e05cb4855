"""The scan entry point for callers that cannot allocate device memory.

Some callers cannot call cudaMalloc when they need the scan (plugins handed
only their input and output buffers, code running where an allocator must not
be entered).  ``pararnn_affine_scan_noalloc`` keeps the scan's scratch in a
device array inside the library instead of a caller workspace.  These tests
call it through the C ABI: twice in a row (the array is shared and reused),
checking each result against the ordinary entry point, ``pararnn_affine_scan``,
and against the fp64 serial recurrence of the oracle, with the scan tolerance
the other tests use (normwise 1e-5); at the largest size the array admits;
with h aliasing b or A; and the rejections (a size just above the array, a
partial overlap).  The file is collected last, so a run that stops at the
first failure has already run every other test; it passes alone in a fresh
process as well.
"""
import ctypes

import numpy as np
import pytest
import torch

from newton_solve_nonlinear_b200 import binding
from newton_solve_nonlinear_b200.inputs import make_scan_input
from oracle.scan import affine_scan as serial_scan

pytestmark = pytest.mark.gpu

NOALLOC_BYTES = 16 << 20  # the library's scratch array


def _entry():
    fn = binding.lib().pararnn_affine_scan_noalloc
    vp, ci = ctypes.c_void_p, ctypes.c_int
    fn.argtypes = [vp, vp, vp, ci, ci, ci, vp, vp, vp]
    fn.restype = ci
    return fn


def _call(fn, A, b, h0, out, status=None):
    B, T, D = b.shape
    return fn(A.data_ptr(), b.data_ptr(), h0.data_ptr(), B, T, D, out.data_ptr(),
              None if status is None else status.data_ptr(), torch.cuda.current_stream().cuda_stream)


def _normwise(got, ref):
    return float(np.max(np.abs(got - ref)) / np.max(np.abs(ref)))


def test_noalloc_scan_matches_workspace_scan_and_oracle_twice():
    fn = _entry()
    for call, (B, T, D) in enumerate([(3, 1500, 100), (2, 4099, 64)]):
        s = make_scan_input(B, T, D, seed=100 + call, h0_std=1.0)
        A, b, h0 = s.A.cuda(), s.b.cuda(), s.h0.cuda()
        want = binding.affine_scan(A, b, h0, check=True)
        out = torch.full_like(b, float("nan"))
        status = torch.full((1,), 7, dtype=torch.int32, device="cuda")
        assert _call(fn, A, b, h0, out, status) == 0
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        got = out.double().cpu().numpy()
        assert np.all(np.isfinite(got))
        assert _normwise(got, want.double().cpu().numpy()) <= 1e-5
        ref = serial_scan(s.A.double().numpy(), s.b.double().numpy(), s.h0.double().numpy())
        assert _normwise(got, ref) <= 1e-5


def test_noalloc_scan_at_the_largest_admitted_size():
    """[31, 65536, 64] needs 15.5 MiB + 256 B of scratch, just under the array."""
    fn = _entry()
    B, T, D = 31, 65536, 64
    assert binding.lib().pararnn_affine_scan_workspace_size(B, T, D, 0) <= NOALLOC_BYTES
    s = make_scan_input(B, T, D, seed=7)
    A, b, h0 = s.A.cuda(), s.b.cuda(), s.h0.cuda()
    want = binding.affine_scan(A, b, h0, check=True)
    out = torch.full_like(b, float("nan"))
    status = torch.full((1,), 7, dtype=torch.int32, device="cuda")
    assert _call(fn, A, b, h0, out, status) == 0
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    assert _normwise(out.double().cpu().numpy(), want.double().cpu().numpy()) <= 1e-5
    # sampled sequences against the serial fp64 recurrence
    for q in (0, 30):
        ref = serial_scan(s.A[q:q + 1].double().numpy(), s.b[q:q + 1].double().numpy(),
                          s.h0[q:q + 1].double().numpy())
        assert _normwise(out[q:q + 1].double().cpu().numpy(), ref) <= 1e-5


def test_noalloc_scan_in_place():
    """h may be b itself or A itself."""
    fn = _entry()
    s = make_scan_input(2, 3000, 64, seed=11, h0_std=1.0)
    A, b, h0 = s.A.cuda(), s.b.cuda(), s.h0.cuda()
    want = binding.affine_scan(A, b, h0, check=True).double().cpu().numpy()
    for alias in ("b", "A"):
        A2, b2 = A.clone(), b.clone()
        out = b2 if alias == "b" else A2
        assert _call(fn, A2, b2, h0, out) == 0
        torch.cuda.synchronize()
        assert _normwise(out.double().cpu().numpy(), want) <= 1e-5, alias


def test_noalloc_scan_rejects_sizes_beyond_its_array_and_partial_overlap():
    fn = _entry()
    # [32, 65536, 64] needs 16 MiB + 256 B of scratch, above the array.  The
    # four buffers are distinct and do not overlap, so only the size can be
    # what is rejected (the size check reads no buffer).
    B, T, D = 32, 65536, 64
    assert binding.lib().pararnn_affine_scan_workspace_size(B, T, D, 0) > NOALLOC_BYTES
    bufs = [torch.zeros(4, device="cuda") for _ in range(4)]
    rc = fn(*(t.data_ptr() for t in bufs[:3]), B, T, D, bufs[3].data_ptr(), None,
            torch.cuda.current_stream().cuda_stream)
    assert rc == 3  # PARARNN_INVALID_ARG, nothing enqueued
    # h overlapping b partly (shifted by one step) is rejected
    s = make_scan_input(1, 64, 8, seed=3)
    A, h0 = s.A.cuda(), s.h0.cuda()
    big = torch.zeros(65 * 8, device="cuda")
    b, h = big[:64 * 8].view(1, 64, 8), big[8:].view(1, 64, 8)
    assert _call(fn, A, b, h0, h) == 3
