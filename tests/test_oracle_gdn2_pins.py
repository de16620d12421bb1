"""The fp64 Gated DeltaNet-2 oracle against its pins, and planted mistakes
that the pins must catch (CPU only).

The mutants are numpy variants of the recurrence with one plausible mistake
each (a gate on the wrong axis, a dropped gate, the erase read taken before
the decay, the write gate applied to the erase read); every one of them must
fail at least one pin in ``pinlib_gdn2``.
"""
import numpy as np
import pytest

import pinlib_gdn2 as pg


@pytest.mark.parametrize("check", pg.ALL_CHECKS, ids=lambda c: c.__name__)
def test_oracle_passes(check):
    check(pg.oracle_unit)


def _make(variant):
    def impl(q, k, v, a, b, w, S0):
        S = np.array(S0, dtype=np.float64, copy=True)
        out = []
        for t in range(q.shape[0]):
            S_prev = S.copy()
            S = a[t][:, None] * S
            e = k[t] if variant == "erase_gate_dropped" else b[t] * k[t]
            z = v[t] if variant == "write_gate_dropped" else w[t] * v[t]
            if variant == "read_before_decay":
                r = S_prev.T @ e
            elif variant == "write_gate_on_read":
                r = w[t] * (S.T @ k[t])
            else:
                r = S.T @ e
            if variant == "erase_gate_on_key_written":
                S = S + np.outer(b[t] * k[t], z) - np.outer(k[t], r)
            else:
                S = S + np.outer(k[t], z - r)
            out.append(S.T @ q[t])
        return np.array(out), S
    return impl


MUTANTS = ["erase_gate_dropped", "write_gate_dropped", "read_before_decay",
           "write_gate_on_read", "erase_gate_on_key_written"]


def test_correct_variant_passes_all_pins():
    impl = _make("correct")
    for check in pg.ALL_CHECKS:
        check(impl)


@pytest.mark.parametrize("variant", MUTANTS)
def test_every_mutant_fails_a_pin(variant):
    impl = _make(variant)
    failed = []
    for check in pg.ALL_CHECKS:
        try:
            check(impl)
        except AssertionError:
            failed.append(check.__name__)
    assert failed, f"mutant {variant} passes every pin"
