"""The scan entry point for callers that cannot allocate device memory.

Some callers cannot call cudaMalloc when they need the scan (plugins handed
only their input and output buffers, code running where an allocator must not
be entered).  ``pararnn_affine_scan_noalloc`` keeps the scan's scratch in a
device array inside the library instead of a caller workspace.  This test
calls it through the C ABI twice in a row (the array is shared and reused) and
checks each result against the ordinary entry point, ``pararnn_affine_scan``,
with the scan tolerance the other tests use (normwise 1e-5).  It sits in a
file of its own, collected last, so a run that stops at the first failure has
already run every other test; it passes alone in a fresh process as well.
"""
import ctypes

import numpy as np
import pytest
import torch

from newton_solve_nonlinear_b200 import binding
from newton_solve_nonlinear_b200.inputs import make_scan_input

pytestmark = pytest.mark.gpu


def _entry():
    fn = binding.lib().pararnn_affine_scan_noalloc
    vp, ci = ctypes.c_void_p, ctypes.c_int
    fn.argtypes = [vp, vp, vp, ci, ci, ci, vp, vp, vp]
    fn.restype = ci
    return fn


def test_noalloc_scan_matches_workspace_scan_twice():
    fn = _entry()
    stream = torch.cuda.current_stream().cuda_stream
    for call, (B, T, D) in enumerate([(3, 1500, 100), (2, 4099, 64)]):
        s = make_scan_input(B, T, D, seed=100 + call, h0_std=1.0)
        A, b, h0 = s.A.cuda(), s.b.cuda(), s.h0.cuda()
        want = binding.affine_scan(A, b, h0, check=True)
        out = torch.full_like(b, float("nan"))
        status = torch.full((1,), 7, dtype=torch.int32, device="cuda")
        rc = fn(A.data_ptr(), b.data_ptr(), h0.data_ptr(), B, T, D, out.data_ptr(),
                status.data_ptr(), stream)
        assert rc == 0
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        got, ref = out.double().cpu().numpy(), want.double().cpu().numpy()
        assert np.all(np.isfinite(got))
        assert np.max(np.abs(got - ref)) / np.max(np.abs(ref)) <= 1e-5


def test_noalloc_scan_rejects_sizes_beyond_its_array():
    fn = _entry()
    x = torch.zeros(4, device="cuda")
    # [64, 65536, 64] needs 64 MiB of descriptors, above the 16 MiB array
    rc = fn(x.data_ptr(), x.data_ptr(), x.data_ptr(), 64, 65536, 64, x.data_ptr(), None,
            torch.cuda.current_stream().cuda_stream)
    assert rc == 3  # PARARNN_INVALID_ARG, nothing enqueued
