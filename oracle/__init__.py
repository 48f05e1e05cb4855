"""fp64 CPU oracle for the parallel-Newton evaluation of a GRU.

TEST INFRASTRUCTURE ONLY.  Only the test suite, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py`` may import this package.  The product
path (the CUDA library and its binding) never imports it, calls it, or falls
back to it; the two share no code.

What it states, plainly and slowly, in float64:
  * ``cells``   -- the GRU cell (dense and diagonal recurrence), its Jacobian
                   with respect to the previous state, and the sequential
                   rollout h_t = f(h_{t-1}, x_t), which is the unique answer
                   every solver must reach.
  * ``scan``    -- the linear recurrence h_t = A_t h_{t-1} + b_t solved by
                   forward substitution (diagonal or dense A_t).
  * ``newton``  -- DEER (Newton) and quasi-DEER (diagonal Jacobian) iterations
                   on the unrolled system, with the convergence rule.
  * ``elk``     -- the Levenberg-Marquardt step of ELK / quasi-ELK solved two
                   independent ways: the block-tridiagonal normal equations,
                   and a sequential Kalman filter + RTS smoother.
  * ``brute``   -- dense (T*D) x (T*D) assemblies for tiny T, used only to pin
                   the structured solvers above.
  * ``lstm``    -- the diagonal-recurrence LSTM: cell, 2x2-per-lane Jacobian,
                   rollout and exact Newton on the unrolled system.
  * ``adjoint`` -- the backward pass: gradients of a loss through the evaluated
                   states (reverse-time recurrence with J^T, exact or with the
                   diagonal of J), and the parameter and input gradients.

Pins (tests marked "not gpu") tie each part to something other than itself:
``torch.nn.GRUCell`` (a library routine), central finite differences, closed
forms of the linear recurrence and of the one-step LM problem, brute-force
dense solves, and invariants the pages state (Newton is exact on an affine
cell; undamped Newton recovers one more exact state per iteration).  The pages
print no worked numeric example, so nothing here is pinned to printed values.
"""
from . import cells, scan, newton, elk, brute, adjoint, lstm  # noqa: F401
from .cells import GRU, rollout  # noqa: F401
from .newton import newton_solve, STATUS_OK, STATUS_NOT_CONVERGED, STATUS_DIVERGED  # noqa: F401
from .elk import elk_solve  # noqa: F401
from .scan import affine_scan  # noqa: F401
