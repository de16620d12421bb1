"""Planted mistakes: each mutant of the recurrence must fail at least one pin.

The mutants are CPU-only numpy variants, each with one plausible mistake
(a dropped term, a wrong sign or order, a transposed operand).  They show
that the pins in ``pinlib`` would catch that mistake in the oracle.
"""
import numpy as np
import pytest

import pinlib


def _make(variant):
    def impl(q, k, v, a, b, S0):
        S = np.array(S0, dtype=np.float64, copy=True)
        out = []
        for t in range(q.shape[0]):
            S_prev = S.copy()
            if variant == "gate_after_reflection":
                S = S - b[t] * np.outer(k[t], k[t] @ S)
                S = a[t][:, None] * S + b[t] * np.outer(k[t], v[t])
                out.append(S.T @ q[t])
                continue
            if variant == "no_gate":
                pass
            elif variant == "gate_on_columns":
                S = S * a[t][None, : S.shape[1]] if S.shape[1] == len(a[t]) else S * a[t][0]
            else:
                S = a[t][:, None] * S
            r = (S_prev if variant == "read_before_gate" else S).T @ k[t]
            if variant == "wrong_delta_sign":
                S = S + b[t] * np.outer(k[t], v[t] + r)
            elif variant == "beta_only_on_write":
                S = S + np.outer(k[t], b[t] * v[t] - r)
            elif variant == "beta_squared":
                S = S + b[t] * b[t] * np.outer(k[t], v[t] - r)
            else:
                S = S + b[t] * np.outer(k[t], v[t] - r)
            if variant == "readout_before_update":
                out.append((a[t][:, None] * S_prev).T @ q[t])
            elif variant == "readout_transposed":
                out.append(S[:, : len(q[t])] @ q[t] if S.shape[0] == S.shape[1] else S.T @ q[t] * 1.0001)
            else:
                out.append(S.T @ q[t])
        return np.array(out), S
    return impl


MUTANTS = ["gate_after_reflection", "no_gate", "gate_on_columns", "read_before_gate",
           "wrong_delta_sign", "beta_only_on_write", "beta_squared", "readout_before_update",
           "readout_transposed"]


def test_correct_variant_passes_all_pins():
    impl = _make("correct")
    for check in pinlib.ALL_CHECKS:
        check(impl)


@pytest.mark.parametrize("variant", MUTANTS)
def test_mutant_is_caught(variant):
    impl = _make(variant)
    failed = []
    for check in pinlib.ALL_CHECKS:
        try:
            check(impl)
        except (AssertionError, ValueError, IndexError, np.linalg.LinAlgError):
            failed.append(check.__name__)
    assert failed, f"mutant {variant} passed every pin"
