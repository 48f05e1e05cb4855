"""The linear recurrence h_t = A_t h_{t-1} + b_t by forward substitution (fp64).

Each Newton iteration of the pages solves a linear system whose matrix is the
Jacobian of the unrolled recurrence: identity blocks on the diagonal and -A_t
just below it ("ParaRNN" summary, "Newton's Iteration": block lower-triangular,
solved by forward substitution).  Written out, that solve is this recurrence;
the GPU evaluates it as a parallel associative scan ("Towards Scalable and
Stable Parallelization of Nonlinear RNNs", atlas summary, "Builds on").  Here it
is the plain serial loop.
"""
from __future__ import annotations

import numpy as np


def affine_scan(A: np.ndarray, b: np.ndarray, h0: np.ndarray) -> np.ndarray:
    """Serial h_t = A_t h_{t-1} + b_t for t = 1..T, h_0 = h0.

    A: diagonal [B, T, D] (elementwise) or dense [B, T, D, D]; b [B, T, D];
    h0 [B, D].  Returns h [B, T, D] (h[:, 0] is h_1)."""
    A = np.asarray(A, np.float64)
    b = np.asarray(b, np.float64)
    B, T, D = b.shape
    dense = A.ndim == 4
    h = np.array(h0, np.float64, copy=True)
    out = np.empty((B, T, D))
    for t in range(T):
        if dense:
            h = np.einsum("bij,bj->bi", A[:, t], h) + b[:, t]
        else:
            h = A[:, t] * h + b[:, t]
        out[:, t] = h
    return out
