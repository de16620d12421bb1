"""The fp64 SFDA oracle against its pins, and planted mistakes that the pins
must catch (CPU only).

The mutants are numpy variants of the recurrence with one plausible mistake
each (the phase sign flipped, the phase dropped, channels paired as
(p, p + dk/2) instead of (2p, 2p+1), the gate applied after the delta
correction, the read taken before the gate, the decay applied to one row of
each pair only); every one of them must fail at least one pin in
``pinlib_sfda``.
"""
import math

import numpy as np
import pytest

import pinlib_sfda as ps


@pytest.mark.parametrize("check", ps.ALL_CHECKS, ids=lambda c: c.__name__)
def test_oracle_passes(check):
    check(ps.oracle_unit)


def _gate(variant, a, th):
    m = a.shape[0]
    L = np.zeros((2 * m, 2 * m))
    for p in range(m):
        s = -1.0 if variant == "phase_sign_flipped" else 1.0
        x = 0.0 if variant == "phase_dropped" else s * th[p]
        blk = np.array([[math.cos(x), -math.sin(x)], [math.sin(x), math.cos(x)]])
        if variant == "decay_on_real_row_only":
            blk = np.diag([a[p], 1.0]) @ blk
        else:
            blk = a[p] * blk
        if variant == "half_split_pairs":
            idx = [p, p + m]
        else:
            idx = [2 * p, 2 * p + 1]
        L[np.ix_(idx, idx)] = blk
    return L


def _make(variant):
    def impl(q, k, v, a, th, b, S0):
        S = np.array(S0, dtype=np.float64, copy=True)
        out = []
        for t in range(q.shape[0]):
            L = _gate(variant, a[t], th[t])
            if variant == "gate_after_delta":
                S = L @ (S + b[t] * np.outer(k[t], v[t] - S.T @ k[t]))
            elif variant == "read_before_gate":
                r = S.T @ k[t]
                S = L @ S + b[t] * np.outer(k[t], v[t] - r)
            else:
                S = L @ S
                S = S + b[t] * np.outer(k[t], v[t] - S.T @ k[t])
            out.append(S.T @ q[t])
        return np.array(out), S
    return impl


MUTANTS = ["phase_sign_flipped", "phase_dropped", "half_split_pairs", "gate_after_delta",
           "read_before_gate", "decay_on_real_row_only"]


def test_correct_variant_passes_all_pins():
    impl = _make("correct")
    for check in ps.ALL_CHECKS:
        check(impl)


@pytest.mark.parametrize("variant", MUTANTS)
def test_every_mutant_fails_a_pin(variant):
    impl = _make(variant)
    failed = []
    for check in ps.ALL_CHECKS:
        try:
            check(impl)
        except AssertionError:
            failed.append(check.__name__)
    assert failed, f"mutant {variant} passes every pin"
