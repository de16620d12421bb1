"""Pins for the Gated DeltaNet-2 recurrence: checks that do not trust the implementation.

Each ``check_*`` takes an implementation ``impl(q, k, v, alpha, b, w, S0)`` of
ONE (sequence, head) unit -- q, k, alpha, b ``[T, dk]``, v, w ``[T, dv]``,
S0 ``[dk, dv]``, all fp64 numpy -- returning ``(out [T, dv], S_final
[dk, dv])``, and raises ``AssertionError`` when the implementation breaks a
fact fixed by the page or by the mathematics.

The recurrence ("Gated DeltaNet-2" technical summary, Methodology section 1):
    S_t = (I - k_t (b_t . k_t)^T) Diag(alpha_t) S_{t-1} + k_t (w_t . v_t)^T,
    o_t = S_t^T q_t,
with an erase gate b_t on the key side and a write gate w_t on the value side.

The facts, with their sources:
  G-1  tying b_t = w_t = beta_t gives back the (pinned) CKDA recurrence
       (Methodology section 1: "recovers KDA").
  G-2  b = 0 (nothing erased): the state is the gated sum of the written
       outer products, S_T = Gamma S_0 + sum_t P(T, t) k_t (w_t . v_t)^T.
  G-3  exact per-channel write: with alpha = 1, b = 1 and |k_t| = 1 the update
       replaces the read along k_t by the gated value, S_t^T k_t = w_t . v_t
       (the fast-weight reading of Methodology section 2: the old gated read
       is subtracted before the new gated value is added).
  G-4  w = 0 and S_0 = 0: nothing is ever written, the state and the output
       stay zero.
  G-5  value channels whose write gate is always 0 are never written: with
       S_0 = 0 those columns of S and of the output stay zero (the write gate
       acts on the value axis).
  G-6  a block of tokens acts on S_0 as an affine map, S_end = M S_0 + B.
  G-7  brute force on tiny inputs with explicit dk x dk transition matrices.
"""
from __future__ import annotations

import numpy as np

import pinlib


def _rng(seed):
    return np.random.default_rng(seed)


def _unit_rows(x):
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


def random_unit(T, dk, dv, seed):
    r = _rng(seed)
    q = _unit_rows(r.standard_normal((T, dk)))
    k = _unit_rows(r.standard_normal((T, dk)))
    v = r.standard_normal((T, dv))
    a = r.uniform(-1.0, 1.0, (T, dk))
    b = r.uniform(0.0, 1.0, (T, dk))
    w = r.uniform(0.0, 1.0, (T, dv))
    S0 = r.standard_normal((dk, dv))
    return q, k, v, a, b, w, S0


def _rel(x, y):
    return float(np.max(np.abs(x - y)) / max(1e-300, np.max(np.abs(y))))


def check_g1_reduces_to_ckda(impl, seed=21):
    q, k, v, a, _, _, S0 = random_unit(40, 6, 5, seed)
    beta = _rng(seed + 1).uniform(0.0, 2.0, 40)
    o, S = impl(q, k, v, a, np.repeat(beta[:, None], 6, 1), np.repeat(beta[:, None], 5, 1), S0)
    ro, rS = pinlib.oracle_unit(q, k, v, a, beta, S0)
    assert _rel(o, ro) < 1e-12 and _rel(S, rS) < 1e-12, "b = w = beta must give CKDA"


def check_g2_no_erase(impl, seed=22):
    q, k, v, a, _, w, S0 = random_unit(30, 5, 4, seed)
    T = q.shape[0]
    o, S = impl(q, k, v, a, np.zeros_like(k), w, S0)
    # closed form: S_t = diag(prod alpha_1..t) S0 + sum_{s<=t} diag(prod alpha_{s+1}..t) k_s z_s^T
    for t in range(T):
        St = np.prod(a[: t + 1], axis=0)[:, None] * S0
        for s in range(t + 1):
            P = np.prod(a[s + 1: t + 1], axis=0) if s < t else np.ones(a.shape[1])
            St = St + np.outer(P * k[s], w[s] * v[s])
        assert _rel(o[t], St.T @ q[t]) < 1e-12, f"output {t}"
    assert _rel(S, St) < 1e-12


def check_g3_exact_write(impl, seed=23):
    q, k, v, _, _, w, S0 = random_unit(25, 8, 6, seed)
    o, S = impl(k, k, v, np.ones_like(k), np.ones_like(k), w, S0)  # query with the key
    assert np.max(np.abs(o - w * v)) < 1e-12, "the gated value must be written exactly"


def check_g4_zero_write(impl, seed=24):
    q, k, v, a, b, _, _ = random_unit(20, 5, 4, seed)
    o, S = impl(q, k, v, a, b, np.zeros_like(v), np.zeros((5, 4)))
    assert np.max(np.abs(o)) == 0.0 and np.max(np.abs(S)) == 0.0


def check_g5_write_gate_on_value_axis(impl, seed=25):
    q, k, v, a, b, w, _ = random_unit(20, 5, 4, seed)
    w = w.copy()
    w[:, 1] = 0.0
    w[:, 3] = 0.0
    o, S = impl(q, k, v, a, b, w, np.zeros((5, 4)))
    assert np.max(np.abs(o[:, [1, 3]])) == 0.0 and np.max(np.abs(S[:, [1, 3]])) == 0.0
    assert np.max(np.abs(o[:, [0, 2]])) > 0.0


def check_g6_affine(impl, seed=26):
    q, k, v, a, b, w, S0 = random_unit(24, 4, 3, seed)
    _, B = impl(q, k, v, a, b, w, np.zeros_like(S0))
    cols = []
    for i in range(4):
        E = np.zeros((4, 3))
        E[i, 0] = 1.0
        _, Si = impl(q, k, np.zeros_like(v), a, b, w, E)
        cols.append(Si[:, 0])
    M = np.stack(cols, axis=1)
    _, S = impl(q, k, v, a, b, w, S0)
    assert _rel(S, M @ S0 + B) < 1e-12, "a block must act on S0 as an affine map"


def check_g7_bruteforce(impl, seed=27):
    q, k, v, a, b, w, S0 = random_unit(12, 3, 2, seed)
    o, S = impl(q, k, v, a, b, w, S0)
    X = S0.copy()
    for t in range(12):
        A_t = (np.eye(3) - np.outer(k[t], b[t] * k[t])) @ np.diag(a[t])
        X = A_t @ X + np.outer(k[t], w[t] * v[t])
        assert _rel(o[t], X.T @ q[t]) < 1e-12, f"output {t}"
    assert _rel(S, X) < 1e-12


ALL_CHECKS = [check_g1_reduces_to_ckda, check_g2_no_erase, check_g3_exact_write,
              check_g4_zero_write, check_g5_write_gate_on_value_axis, check_g6_affine,
              check_g7_bruteforce]


def oracle_unit(q, k, v, a, b, w, S0):
    """The fp64 oracle on one (sequence, head) unit, in the pin signature."""
    import oracle

    T, dk = q.shape
    dv = v.shape[1]
    out, S = oracle.forward_gdn2(q.reshape(1, T, 1, dk), k.reshape(1, T, 1, dk),
                                 v.reshape(1, T, 1, dv), a.reshape(1, T, 1, dk),
                                 b.reshape(1, T, 1, dk), w.reshape(1, T, 1, dv),
                                 S0=S0.reshape(1, 1, dk, dv), n_threads=1)
    return out.reshape(T, dv), S.reshape(dk, dv)
