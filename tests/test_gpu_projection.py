"""GPU parity of the input projection P = x W_ih^T + b_ih (pararnn_input_projection).

bf16 operands with Din % 64 == 0 and 3D % 256 == 0 run on the tcgen05 kernel;
fp32 operands with Din = 32 or 64 and 3D = 96 or 192 on the tcgen05 3 x TF32
kernel; other shapes on the CUDA-core kernel.  Reference: the same bf16 (or
fp32) values widened to fp64 and multiplied exactly.  Tolerance: the kernels
accumulate Din products in fp32, so |P - P_ref| <= 1e-5 * sqrt(Din) * max|x||w| is
a loose bound of the rounding; the check uses max-abs <= 2e-5 * sqrt(Din) relative
to the scale of P.
"""
import numpy as np
import pytest
import torch

from newton_solve_nonlinear_b200 import binding

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("M,din,d,dtype", [
    (4096, 2048, 2048, torch.bfloat16),   # tcgen05, the diagonal-layer shape (reduced M)
    (1000, 128, 256, torch.bfloat16),     # tcgen05, ragged M (not a multiple of 128)
    (77, 64, 512, torch.bfloat16),        # tcgen05, a single partial row tile
    (33001, 128, 256, torch.bfloat16),    # tcgen05, several tiles per CTA (both accumulators), ragged M
    (333, 96, 256, torch.bfloat16),       # CUDA-core (Din not a multiple of 64)
    (2000, 64, 64, torch.float32),        # tcgen05 3 x TF32 (N = 192, K = 64)
    (1000, 32, 32, torch.float32),        # tcgen05 3 x TF32 (N = 96, K = 32), ragged M
    (129, 64, 32, torch.float32),         # tcgen05 3 x TF32 (N = 96, K = 64), one row past a tile
    (7, 32, 64, torch.float32),           # tcgen05 3 x TF32 (N = 192, K = 32), a partial tile
    (300001, 64, 64, torch.float32),      # tcgen05 3 x TF32, several tiles per CTA
    (517, 2, 4, torch.float32),           # CUDA-core fp32
    (999, 48, 64, torch.float32),         # CUDA-core fp32 (K not 32 or 64)
])
def test_projection_matches_fp64(M, din, d, dtype):
    g = torch.Generator().manual_seed(M + din)
    x = (torch.randn(1, M, din, generator=g)).to(dtype)
    w = (torch.randn(3 * d, din, generator=g) / din ** 0.5).to(dtype)
    b = torch.randn(3 * d, generator=g)
    P = binding.input_projection(x.cuda(), w.cuda(), b.cuda(), d=d).cpu().double().numpy()[0]
    ref = x[0].double().numpy() @ w.double().numpy().T + b.double().numpy()
    scale = np.max(np.abs(ref))
    err = np.max(np.abs(P - ref))
    assert np.all(np.isfinite(P))
    assert err <= 2e-5 * np.sqrt(din) * scale, (err, scale)
