"""Plant plausible mistakes in the oracle (CPU only) and check a pin catches each.

This is evidence that the pins in ``test_oracle_pins`` are strong enough: a
dropped term, a flipped sign, a transposed operand, a missing shift or a wrong
damping convention must each make some pin fail.
"""
import numpy as np
import pytest

from oracle import cells, elk, newton, scan
import tests.test_oracle_pins as pins
import tests.test_oracle_reuse as reuse_pins


def _fails(fn, *args):
    with pytest.raises(AssertionError):
        fn(*args)


def test_flipped_sign_in_jacobian(monkeypatch):
    orig = cells.GRU._row_scales

    def bad(self, h, r, z, g, n):
        cz, cn, cr = orig(self, h, r, z, g, n)
        return -cz, cn, cr
    monkeypatch.setattr(cells.GRU, "_row_scales", bad)
    _fails(pins.test_jacobian_central_differences, "dense")


def test_dropped_reset_gate_term(monkeypatch):
    orig = cells.GRU._row_scales

    def bad(self, h, r, z, g, n):
        cz, cn, cr = orig(self, h, r, z, g, n)
        return cz, cn, 0.0 * cr
    monkeypatch.setattr(cells.GRU, "_row_scales", bad)
    _fails(pins.test_jacobian_central_differences, "dense")
    _fails(pins.test_jacobian_central_differences, "diag")


def test_transposed_recurrent_block(monkeypatch):
    orig = cells.GRU.U
    monkeypatch.setattr(cells.GRU, "U", lambda self, gate: orig(self, gate).T)
    _fails(pins.test_jacobian_central_differences, "dense")


def test_reset_gate_before_bias(monkeypatch):
    def bad(self, h, p):
        d = self.d
        q = self.recurrent(h) - self.b_hh
        r = cells.sigmoid(p[..., 0:d] + q[..., 0:d] + self.b_hh[0:d])
        z = cells.sigmoid(p[..., d:2 * d] + q[..., d:2 * d] + self.b_hh[d:2 * d])
        g = q[..., 2 * d:]
        n = np.tanh(p[..., 2 * d:] + r * g + self.b_hh[2 * d:])
        return r, z, g, n, (1 - z) * n + z * h
    monkeypatch.setattr(cells.GRU, "gates", bad)
    _fails(pins.test_cell_equals_torch_grucell, "dense")


def test_missing_shift(monkeypatch):
    monkeypatch.setattr(newton, "shifted", lambda h, h0: h)
    _fails(pins.test_undamped_newton_recovers_one_state_per_iteration, "QUASI")


def test_transposed_dense_scan(monkeypatch):
    orig = scan.affine_scan

    def bad(A, b, h0):
        A = np.asarray(A)
        return orig(np.swapaxes(A, -1, -2) if A.ndim == 4 else A, b, h0)
    monkeypatch.setattr(pins, "affine_scan", bad)
    _fails(pins.test_scan_closed_forms_dense)


def test_inverted_damping_convention(monkeypatch):
    orig = elk.lm_step_normal
    monkeypatch.setattr(elk, "lm_step_normal", lambda A, b, y, h0, lam: orig(A, b, y, h0, 1.0 / lam))
    _fails(pins.test_lm_limits, False)


# ---------------------------------------------------------- backward pass --
import oracle.adjoint as adj  # noqa: E402
import tests.test_oracle_adjoint as adj_pins  # noqa: E402


def test_adjoint_without_transpose(monkeypatch):
    """J_t instead of J_t^T in the lam recurrence."""
    orig = cells.GRU.jacobian

    def bad(self, h, p):
        f, J = orig(self, h, p)
        return f, np.swapaxes(J, -1, -2)
    monkeypatch.setattr(cells.GRU, "jacobian", bad)
    _fails(adj_pins.test_exact_adjoint_equals_autograd, "dense")


def test_adjoint_dropped_reset_factor(monkeypatch):
    """The n gate's recurrent gradient without its reset-gate factor."""
    orig = adj.step_partials

    def bad(cell, h_prev, p):
        fr, fz, fn, r, f = orig(cell, h_prev, p)
        return fr, fz, fn, np.ones_like(r), f
    monkeypatch.setattr(adj, "step_partials", bad)
    _fails(adj_pins.test_exact_adjoint_equals_autograd, "diag")


def test_adjoint_unshifted_previous_state(monkeypatch):
    """Partials evaluated at h_t instead of h_{t-1}."""
    def bad(cell, x, h0, h, g, jacobian="exact"):
        B, T, _ = x.shape
        P = cell.project(x)
        lam = np.zeros_like(h)
        carry = np.zeros((B, cell.d))
        for t in range(T - 1, -1, -1):
            lam[:, t] = g[:, t] + carry
            _, a = cell.jacobian_diag(h[:, t], P[:, t])
            carry = a * lam[:, t]
        out = dict(lam=lam, dh0=carry)
        for k in ("dx", "dw_ih", "db_ih", "dw_hh", "db_hh", "dP"):
            out[k] = np.zeros(1)
        return out
    monkeypatch.setattr(adj_pins, "adjoint", bad)
    _fails(adj_pins.test_diag_cell_quasi_backward_is_exact)


# ------------------------------------------------------------------ LSTM --
import oracle.lstm as lstm  # noqa: E402
import tests.test_oracle_lstm as lstm_pins  # noqa: E402


def test_lstm_dropped_candidate_term(monkeypatch):
    """dc'/dh without its candidate-gate term."""
    orig = lstm.LSTM.jacobian

    def bad(self, c, h, p):
        d = self.d
        u = self.u.copy()
        self.u = u.copy()
        self.u[2 * d:3 * d] = 0.0
        try:
            _, _, A_wrong = orig(self, c, h, p)
        finally:
            self.u = u
        c2, h2, A = orig(self, c, h, p)
        A = A.copy()
        A[..., 0, 1] = A_wrong[..., 0, 1]
        return c2, h2, A
    monkeypatch.setattr(lstm.LSTM, "jacobian", bad)
    _fails(lstm_pins.test_jacobian_central_differences)


def test_lstm_transposed_block(monkeypatch):
    """The substitution with each 2x2 block transposed."""
    orig = lstm.LSTM.jacobian

    def bad(self, c, h, p):
        c2, h2, A = orig(self, c, h, p)
        return c2, h2, np.swapaxes(A, -1, -2)
    monkeypatch.setattr(lstm.LSTM, "jacobian", bad)
    _fails(lstm_pins.test_one_newton_iteration_equals_brute_force_step)


def test_reuse_with_offset_from_the_new_jacobian(monkeypatch):
    """Jacobian reuse that keeps A but forms b_t with the new guess's Jacobian."""
    def bad(A_kept, f, hp, dense):
        return A_kept, f - (np.einsum("btij,btj->bti", A_kept, hp) * 0.0 if dense else 0.0 * hp)
    monkeypatch.setattr(newton, "kept_operands", bad)
    _fails(reuse_pins.test_reuse_iterates_equal_chord_method, "DEER", 2)
    _fails(reuse_pins.test_reuse_iterates_equal_chord_method, "QUASI", 2)


def test_reuse_ignored(monkeypatch):
    """Jacobian reuse that silently recomputes the Jacobian every iteration."""
    orig = newton.linearise
    latest = {}

    def lin(cell, h, p, h0, dense):
        A, b, f = orig(cell, h, p, h0, dense)
        latest["A"] = A
        return A, b, f

    def fresh(A_kept, f, hp, dense):
        A = latest["A"]
        return A, f - (np.einsum("btij,btj->bti", A, hp) if dense else A * hp)
    monkeypatch.setattr(newton, "linearise", lin)
    monkeypatch.setattr(newton, "kept_operands", fresh)
    _fails(reuse_pins.test_reuse_iterates_equal_chord_method, "DEER", 3)
    _fails(reuse_pins.test_reuse_iterates_equal_chord_method, "QUASI", 100)
