"""Seeded synthetic workloads for the parallel-Newton GRU solver.

This module draws random numbers and nothing else: it holds no GRU, Newton,
scan or Kalman arithmetic.  Both sides of every parity check consume the same
arrays it returns -- the CUDA path (through the C-ABI binding) and the fp64
CPU oracle (which widens them to float64).

Distributions follow the workloads the pages time: an untrained GRU evaluated
from a zero state ("Towards Scalable and Stable Parallelization of Nonlinear
RNNs", atlas summary, "Key results" and "Experimental setup"), and a GRU whose
recurrence is near-unstable, where undamped Newton diverges (same page,
"Problem" and "Surprising findings").  The pages name datasets (C. elegans
eigenworms, a noisy sine wave) and trained weights that are not available
here; the seeded draws below stand in for them.

Readings (the pages fix none of these):
  * ``N(0, s)`` means variance ``s`` (standard deviation ``sqrt(s)``).
  * Biases are zero and ``h0`` is zero unless a workload says otherwise.
  * The draw order is W_ih, W_hh (or the diagonal vectors u), b_ih, b_hh, x, h0,
    all from one ``torch.Generator('cpu')`` seeded with ``seed``.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np
import torch

__all__ = [
    "Workload",
    "ScanInput",
    "make_workload",
    "make_scan_input",
    "WORKLOADS",
]

# Solver modes and cell kinds, by name (the C-ABI enums use the same order).
MODES = ("DEER", "QUASI", "ELK", "QUASI_ELK")
CELLS = ("dense", "diag")


@dataclass
class Workload:
    """One GRU evaluation problem: parameters, inputs and solver settings.

    Tensors live on the CPU; callers move them to the device themselves.
    Layouts (row-major, contiguous):
      w_ih [3D, Din]   rows in gate order (r, z, n)
      b_ih [3D]
      w_hh dense: [3D, D]; diag: [3D] = the three vectors u_r, u_z, u_n
      b_hh [3D]
      x    [B, T, Din]  (x[:, 0] is x_1)
      h0   [B, D]
    """

    name: str
    kind: str
    din: int
    d: int
    B: int
    T: int
    x_dtype: torch.dtype
    w_dtype: torch.dtype
    w_ih: torch.Tensor
    b_ih: torch.Tensor
    w_hh: torch.Tensor
    b_hh: torch.Tensor
    x: torch.Tensor
    h0: torch.Tensor
    tol: float
    modes: tuple
    lambdas: tuple = ()
    meta: dict = field(default_factory=dict)

    @property
    def states(self) -> int:
        return self.B * self.T * self.d


@dataclass
class ScanInput:
    """Operands of a linear recurrence h_t = A_t h_{t-1} + b_t."""

    A: torch.Tensor  # diag: [B, T, D]; dense: [B, T, D, D]
    b: torch.Tensor  # [B, T, D]
    h0: torch.Tensor  # [B, D]
    dense: bool


def _normal(g, shape, var):
    return torch.randn(*shape, generator=g, dtype=torch.float32) * math.sqrt(var)


def _uniform(g, shape, lo, hi):
    return torch.rand(*shape, generator=g, dtype=torch.float32) * (hi - lo) + lo


def _rescale_spectral_radius(m: torch.Tensor, radius: float) -> torch.Tensor:
    """Scale a square matrix so that its spectral radius equals ``radius``.

    The eigenvalues are taken in float64; the scaled matrix is returned as
    float32 (the precision the solver receives)."""
    m64 = m.double().numpy()
    rho = float(np.max(np.abs(np.linalg.eigvals(m64))))
    return torch.from_numpy(m64 * (radius / rho)).float()


# name -> default settings.  Every field can be overridden in make_workload so
# that tests can run the same distributions at sizes the oracle finishes fast.
WORKLOADS = {
    # Tiny dense GRU: full Jacobian (DEER) and its diagonal (quasi-DEER).
    "tiny": dict(kind="dense", din=2, d=4, B=1, T=1024, w_var=lambda din, d: 1.0 / d,
                 whh_var=lambda d: 1.0 / d, x_dtype=torch.float32,
                 w_dtype=torch.float32, tol=1e-6, modes=("DEER", "QUASI")),
    # Untrained dense GRU swept over T; quasi-DEER.  Also the scan-alone case.
    "untrained": dict(kind="dense", din=64, d=64, B=16, T=65536,
                      w_var=lambda din, d: 1.0 / d, whh_var=lambda d: 1.0 / d,
                      x_dtype=torch.float32, w_dtype=torch.float32, tol=1e-5,
                      modes=("QUASI",)),
    # GRU layer whose recurrent weights are elementwise vectors (diagonal
    # Jacobian, so quasi-DEER is exact Newton); bf16 inputs and projection.
    "diag": dict(kind="diag", din=2048, d=2048, B=8, T=4096,
                 w_var=lambda din, d: 1.0 / din, u_range=(-1.0, 1.0),
                 x_dtype=torch.bfloat16, w_dtype=torch.bfloat16, tol=1e-4,
                 modes=("QUASI",)),
    # Dense DEER with full 32x32 Jacobians over a long sequence.
    "dense_deer": dict(kind="dense", din=16, d=32, B=4, T=65536,
                       w_var=lambda din, d: 0.8 / d, whh_var=lambda d: 0.8 / d,
                       x_dtype=torch.float32, w_dtype=torch.float32, tol=1e-5,
                       modes=("DEER",)),
    # Near-unstable GRU: each recurrent block N(0,1) rescaled to spectral
    # radius 1.5; undamped Newton diverges, ELK / quasi-ELK damp it.
    "near_unstable": dict(kind="dense", din=64, d=64, B=8, T=10000,
                          w_var=lambda din, d: 1.0 / din, whh_var=None,
                          radius=1.5, x_dtype=torch.float32,
                          w_dtype=torch.float32, tol=1e-4,
                          modes=("ELK", "QUASI_ELK", "DEER"),
                          lambdas=(1e-2, 1e-1, 1.0)),
    # The near-unstable GRU with each recurrent block at spectral radius 3:
    # the setting in which undamped Newton (DEER) actually fails -- its steps
    # overshoot by many orders of magnitude and it does not converge -- while
    # the damped methods (ELK, quasi-ELK) and quasi-DEER do.  At radius 1.5
    # the GRU's gates keep the Jacobians contractive enough that DEER converges.
    "unstable": dict(kind="dense", din=64, d=64, B=2, T=1000,
                     w_var=lambda din, d: 1.0 / din, whh_var=None,
                     radius=3.0, x_dtype=torch.float32,
                     w_dtype=torch.float32, tol=1e-4,
                     modes=("ELK", "QUASI_ELK", "QUASI", "DEER"),
                     lambdas=(1e-2, 1e-1, 1.0)),
}


def make_workload(name: str, *, seed: int = 0, bias_std: float = 0.0,
                  h0_std: float = 0.0, **overrides) -> Workload:
    """Draw the parameters and inputs of workload ``name``.

    ``overrides`` may change B, T, d, din, tol, x_dtype, w_dtype, kind.  Sizes
    change the shapes drawn, not the distributions.  ``bias_std`` and
    ``h0_std`` (default 0, the workloads' own setting) let tests exercise the
    bias and initial-state paths with the same generator.
    """
    spec = dict(WORKLOADS[name])
    spec.update({k: v for k, v in overrides.items() if k in
                 ("B", "T", "d", "din", "tol", "x_dtype", "w_dtype", "kind")})
    kind, din, d, B, T = spec["kind"], spec["din"], spec["d"], spec["B"], spec["T"]
    g = torch.Generator("cpu").manual_seed(seed)

    w_ih = _normal(g, (3 * d, din), spec["w_var"](din, d))
    if kind == "diag":
        lo, hi = spec.get("u_range", (-1.0, 1.0))
        w_hh = _uniform(g, (3 * d,), lo, hi)
    elif spec.get("radius") is not None:
        blocks = [_normal(g, (d, d), 1.0) for _ in range(3)]
        w_hh = torch.cat([_rescale_spectral_radius(m, spec["radius"]) for m in blocks], 0)
    else:
        w_hh = _normal(g, (3 * d, d), spec["whh_var"](d))
    b_ih = _normal(g, (3 * d,), 1.0) * bias_std
    b_hh = _normal(g, (3 * d,), 1.0) * bias_std
    x = _normal(g, (B, T, din), 1.0)
    h0 = _normal(g, (B, d), 1.0) * h0_std

    x = x.to(spec["x_dtype"]).contiguous()
    w_ih = w_ih.to(spec["w_dtype"]).contiguous()
    return Workload(name=name, kind=kind, din=din, d=d, B=B, T=T,
                    x_dtype=spec["x_dtype"], w_dtype=spec["w_dtype"],
                    w_ih=w_ih, b_ih=b_ih.contiguous(), w_hh=w_hh.contiguous(),
                    b_hh=b_hh.contiguous(), x=x, h0=h0.contiguous(),
                    tol=spec["tol"], modes=spec["modes"],
                    lambdas=spec.get("lambdas", ()),
                    meta=dict(seed=seed, bias_std=bias_std, h0_std=h0_std))


def make_scan_input(B: int, T: int, D: int, *, dense: bool = False, seed: int = 0,
                    a_range=(0.5, 1.0), dense_var: float = 0.8,
                    h0_std: float = 0.0) -> ScanInput:
    """Operands for the affine scan alone.

    Diagonal: a ~ U(a_range), b ~ N(0,1), h0 = 0 (the scan-alone case of the
    untrained-GRU workload).  Dense (no workload fixes one): A_t ~ N(0,
    dense_var / D) entrywise, b ~ N(0, 1).
    """
    g = torch.Generator("cpu").manual_seed(seed)
    if dense:
        A = _normal(g, (B, T, D, D), dense_var / D)
    else:
        A = _uniform(g, (B, T, D), *a_range)
    b = _normal(g, (B, T, D), 1.0)
    h0 = _normal(g, (B, D), 1.0) * h0_std
    return ScanInput(A=A.contiguous(), b=b.contiguous(), h0=h0.contiguous(), dense=dense)



@dataclass
class LstmWorkload:
    """A diagonal-recurrence LSTM problem (layouts row-major, contiguous):
    w_ih [4D, Din] rows in gate order (i, f, g, o); b_ih [4D]; u [4D] the
    recurrent vectors; b_hh [4D]; x [B, T, Din]; c0, h0 [B, D]."""

    din: int
    d: int
    B: int
    T: int
    x_dtype: torch.dtype
    w_ih: torch.Tensor
    b_ih: torch.Tensor
    u: torch.Tensor
    b_hh: torch.Tensor
    x: torch.Tensor
    c0: torch.Tensor
    h0: torch.Tensor
    tol: float

    @property
    def states(self) -> int:
        return self.B * self.T * self.d


def make_lstm_workload(*, B: int = 8, T: int = 4096, d: int = 2048, din: int = 2048, seed: int = 0,
                       x_dtype: torch.dtype = torch.bfloat16, tol: float = 1e-4, bias_std: float = 0.0,
                       state_std: float = 0.0) -> LstmWorkload:
    """The diagonal-recurrence LSTM with the diagonal GRU workload's
    distributions: W_ih ~ N(0, 1/Din), u ~ U(-1, 1), x ~ N(0, 1), biases and
    initial state 0 unless ``bias_std`` / ``state_std`` say otherwise; x and
    W_ih in ``x_dtype`` (bf16 by default, as the diagonal GRU workload)."""
    g = torch.Generator("cpu").manual_seed(seed)
    w_ih = _normal(g, (4 * d, din), 1.0 / din)
    u = _uniform(g, (4 * d,), -1.0, 1.0)
    b_ih = _normal(g, (4 * d,), 1.0) * bias_std
    b_hh = _normal(g, (4 * d,), 1.0) * bias_std
    x = _normal(g, (B, T, din), 1.0)
    c0 = _normal(g, (B, d), 1.0) * state_std
    h0 = _normal(g, (B, d), 1.0) * state_std
    return LstmWorkload(din=din, d=d, B=B, T=T, x_dtype=x_dtype, w_ih=w_ih.to(x_dtype).contiguous(),
                        b_ih=b_ih.contiguous(), u=u.contiguous(), b_hh=b_hh.contiguous(),
                        x=x.to(x_dtype).contiguous(), c0=c0.contiguous(), h0=h0.contiguous(), tol=tol)
