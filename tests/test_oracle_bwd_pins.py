"""The fp64 backward oracle against its pins, and planted mistakes that the
pins must catch (CPU only).

The mutants are numpy variants of the reverse-time adjoint with one plausible
mistake each (the gate gradient taken with the gated state instead of the
previous one, the read term of dk dropped, dbeta without the read, the state
gradient not passed back through the gate, dq taken from the previous state,
the sign of dr flipped); every one of them must fail at least one pin in
``pinlib_bwd``.
"""
import numpy as np
import pytest

import pinlib_bwd as pb


@pytest.mark.parametrize("check", pb.ALL_CHECKS, ids=lambda c: c.__name__)
def test_oracle_passes(check):
    check(pb.oracle_unit)


def _make(variant):
    def impl(q, k, v, a, b, S0, dO, dST):
        T, dk = q.shape
        states = [np.array(S0, dtype=np.float64)]
        rs, us = [], []
        for t in range(T):
            Sp = a[t][:, None] * states[-1]
            r = Sp.T @ k[t]
            u = b[t] * (v[t] - r)
            states.append(Sp + np.outer(k[t], u))
            rs.append(r)
            us.append(u)
        g = {"dq": np.zeros_like(q), "dk": np.zeros_like(k), "dv": np.zeros_like(v),
             "dalpha": np.zeros_like(a), "dbeta": np.zeros(T)}
        dS = np.array(dST, dtype=np.float64)
        for t in range(T - 1, -1, -1):
            S_prev, S_t = states[t], states[t + 1]
            g["dq"][t] = (S_prev if variant == "dq_from_previous_state" else S_t) @ dO[t]
            dS = dS + np.outer(q[t], dO[t])
            du = dS.T @ k[t]
            g["dk"][t] = dS @ us[t]
            g["dbeta"][t] = du @ (v[t] if variant == "dbeta_without_read" else v[t] - rs[t])
            g["dv"][t] = b[t] * du
            dr = (1.0 if variant == "dr_sign_flipped" else -1.0) * b[t] * du
            Sp = a[t][:, None] * S_prev
            dSp = dS + np.outer(k[t], dr)
            if variant != "dk_without_read_term":
                g["dk"][t] += Sp @ dr
            g["dalpha"][t] = np.sum(dSp * (Sp if variant == "dalpha_with_gated_state"
                                           else S_prev), axis=1)
            dS = dSp if variant == "dS_not_gated" else a[t][:, None] * dSp
        g["dS0"] = dS
        return g
    return impl


MUTANTS = ["dalpha_with_gated_state", "dk_without_read_term", "dbeta_without_read",
           "dS_not_gated", "dq_from_previous_state", "dr_sign_flipped"]


def test_correct_variant_passes_all_pins():
    impl = _make("correct")
    for check in pb.ALL_CHECKS:
        check(impl)


@pytest.mark.parametrize("variant", MUTANTS)
def test_every_mutant_fails_a_pin(variant):
    impl = _make(variant)
    failed = []
    for check in pb.ALL_CHECKS:
        try:
            check(impl)
        except AssertionError:
            failed.append(check.__name__)
    assert failed, f"mutant {variant} passes every pin"
