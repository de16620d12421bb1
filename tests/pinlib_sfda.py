"""Pins for the SFDA recurrence: checks that do not trust the implementation.

Each ``check_*`` takes an implementation ``impl(q, k, v, alpha, theta, beta,
S0)`` of ONE (sequence, head) unit -- q, k ``[T, dk]`` (dk even), v
``[T, dv]``, alpha, theta ``[T, dk/2]``, beta ``[T]``, S0 ``[dk, dv]``, all
fp64 numpy -- returning ``(out [T, dv], S_final [dk, dv])``, and raises
``AssertionError`` when the implementation breaks a fact fixed by the page or
by the mathematics.

The recurrence ("Semidirect Fourier Delta Attention (SFDA)" technical
summary, "Arquitectura Central", in real coordinates):
    S_t = (I - beta_t k_t k_t^T) Lambda_t S_{t-1} + beta_t k_t v_t^T,
    o_t = S_t^T q_t,
with Lambda_t block diagonal, block p = alpha_p R(theta_p) acting on the state
rows (2p, 2p+1), R(x) = [[cos x, -sin x], [sin x, cos x]] (complex channel p
has its real part in row 2p and its imaginary part in row 2p+1).

The facts, with their sources:
  S-1  zero phases give back the (pinned) CKDA recurrence with the decay of
       channel p on both rows of its pair ("Principales Contribuciones" item
       1: KDA is recovered when the phases are zero).
  S-2  theta = pi gives CKDA with the negated decays (e^{i pi} = -1: a phase
       of pi is a negative real gate).
  S-3  beta = 0 (no delta correction) closed form: each row pair of the state
       is scaled by the product of its decays and rotated by the SUM of its
       phases, S_t = Gamma_t S_0, o_t = S_t^T q_t (the phase-decay blocks are
       complex scalars, so their product is the product of the moduli and the
       sum of the angles).
  S-4  the constructed mod-5 counter ("Resultados", constructed counter, and
       "Expresividad de Estado Finito": phase-only SFDA realises cyclic
       counters exactly): with dk = 2, alpha = 1, beta = 0 and
       theta_t = 2 pi x_t / 5 for input bits x_t, the state angle after any
       length from 27 to 213 decodes the count of ones mod 5 exactly; with a
       reset token (alpha = 0, beta = 1, k = e_0, v = 1: the delta correction
       writes a register, "Con Correccion Delta") it decodes the count since
       the last reset.
  S-5  with |alpha| = 1, beta in {0, 2} and |k| = 1 every transition is
       orthogonal -- a rotation when beta = 0, a reflection (det -1) when
       beta = 2 on a single pair ("Con Reflexiones": dihedral memory) -- so
       with v = 0 the Frobenius norm of the state is kept.
  S-6  brute force on tiny inputs with explicit dk x dk transition matrices.
  S-7  a block of tokens acts on S_0 as an affine map, S_end = M S_0 + B
       ("Principales Contribuciones" item 3).
  S-8  rotating q, k and S_0 by one fixed block rotation (the same angle per
       pair at every token) leaves the output unchanged and rotates the final
       state: the phase-decay blocks commute with block rotations.
"""
from __future__ import annotations

import math

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
    a = r.uniform(-1.0, 1.0, (T, dk // 2))
    th = r.uniform(-math.pi, math.pi, (T, dk // 2))
    b = r.uniform(0.0, 2.0, T)
    S0 = r.standard_normal((dk, dv))
    return q, k, v, a, th, b, S0


def _rel(x, y):
    return float(np.max(np.abs(x - y)) / max(1e-300, np.max(np.abs(y))))


def _rot(x):
    return np.array([[math.cos(x), -math.sin(x)], [math.sin(x), math.cos(x)]])


def block_gate(a, th):
    """The dk x dk real gate Lambda for one token: blocks a_p R(th_p)."""
    m = a.shape[0]
    L = np.zeros((2 * m, 2 * m))
    for p in range(m):
        L[2 * p:2 * p + 2, 2 * p:2 * p + 2] = a[p] * _rot(th[p])
    return L


def check_s1_zero_phase_is_ckda(impl, seed=31):
    q, k, v, a, _, b, S0 = random_unit(40, 6, 5, seed)
    o, S = impl(q, k, v, a, np.zeros_like(a), b, S0)
    ro, rS = pinlib.oracle_unit(q, k, v, np.repeat(a, 2, axis=1), b, S0)
    assert _rel(o, ro) < 1e-12 and _rel(S, rS) < 1e-12, "theta = 0 must give CKDA"


def check_s2_phase_pi_is_negative_gate(impl, seed=32):
    q, k, v, a, _, b, S0 = random_unit(40, 6, 5, seed)
    a = np.abs(a)
    o, S = impl(q, k, v, a, np.full_like(a, math.pi), b, S0)
    ro, rS = pinlib.oracle_unit(q, k, v, -np.repeat(a, 2, axis=1), b, S0)
    assert _rel(o, ro) < 1e-12 and _rel(S, rS) < 1e-12, "theta = pi must negate the gate"


def check_s3_beta_zero_closed_form(impl, seed=33):
    q, k, v, a, th, _, S0 = random_unit(30, 8, 3, seed)
    T, m = a.shape
    o, S = impl(q, k, v, a, th, np.zeros(T), S0)
    for t in range(T):
        St = np.zeros_like(S0)
        for p in range(m):
            g = np.prod(a[: t + 1, p]) * _rot(float(np.sum(th[: t + 1, p])))
            St[2 * p:2 * p + 2] = g @ S0[2 * p:2 * p + 2]
        assert _rel(o[t], St.T @ q[t]) < 1e-12, f"output {t}"
    assert _rel(S, St) < 1e-12, "state"


def _decode_angle(S, period=5):
    ang = math.atan2(S[1, 0], S[0, 0])
    return int(round(ang / (2 * math.pi / period))) % period


def check_s4_mod5_counter(impl, seed=34):
    r = _rng(seed)
    for L in (27, 64, 128, 213):
        x = r.integers(0, 2, L)
        th = (2 * math.pi / 5 * x)[:, None].astype(np.float64)
        a = np.ones((L, 1))
        k = np.tile([1.0, 0.0], (L, 1))
        q = k.copy()
        S0 = np.array([[1.0], [0.0]])
        o, S = impl(q, k, np.zeros((L, 1)), a, th, np.zeros(L), S0)
        count = np.cumsum(x)
        ang = 2 * math.pi / 5 * count[-1]
        assert np.max(np.abs(S[:, 0] - [math.cos(ang), math.sin(ang)])) < 1e-12
        assert _decode_angle(S) == count[-1] % 5, f"counter at length {L}"
        # the read-out along e_0 is cos(2 pi count_t / 5) at every position
        assert np.max(np.abs(o[:, 0] - np.cos(2 * math.pi / 5 * count))) < 1e-12
    # with resets written by the delta correction
    L = 200
    tok = r.choice(3, L, p=[0.45, 0.45, 0.10])  # 0: no-op, 1: increment, 2: reset
    a = np.where(tok == 2, 0.0, 1.0)[:, None]
    th = np.where(tok == 1, 2 * math.pi / 5, 0.0)[:, None]
    b = np.where(tok == 2, 1.0, 0.0)
    k = np.tile([1.0, 0.0], (L, 1))
    v = np.ones((L, 1))
    S = np.array([[1.0], [0.0]])
    c = 0
    for t0 in range(0, L, 25):  # read the state every 25 tokens through the affine chain
        sl = slice(t0, t0 + 25)
        _, S = impl(k[sl], k[sl], v[sl], a[sl], th[sl], b[sl], S)
        for t in tok[sl]:
            c = 0 if t == 2 else (c + (t == 1)) % 5
        assert _decode_angle(S) == c and abs(np.linalg.norm(S) - 1) < 1e-12, f"reset counter {t0}"


def check_s5_orthogonal(impl, seed=35):
    r = _rng(seed)
    # single transitions on a pair: rotation (beta = 0, det +1) or reflection (beta = 2, det -1)
    for beta, det in ((0.0, 1.0), (2.0, -1.0)):
        for _ in range(4):
            a = r.choice([-1.0, 1.0], (1, 1))
            th = r.uniform(-math.pi, math.pi, (1, 1))
            k = _unit_rows(r.standard_normal((1, 2)))
            _, A = impl(k, k, np.zeros((1, 2)), a, th, np.array([beta]), np.eye(2))
            assert np.max(np.abs(A.T @ A - np.eye(2))) < 1e-13, "transition must be orthogonal"
            assert abs(np.linalg.det(A) - det) < 1e-13, "rotation vs reflection"
    # long run: the norm of the state is kept
    T, dk, dv = 300, 8, 3
    k = _unit_rows(r.standard_normal((T, dk)))
    a = r.choice([-1.0, 1.0], (T, dk // 2))
    th = r.uniform(-math.pi, math.pi, (T, dk // 2))
    b = r.choice([0.0, 2.0], T)
    S0 = r.standard_normal((dk, dv))
    _, S = impl(k, k, np.zeros((T, dv)), a, th, b, S0)
    assert abs(np.linalg.norm(S) / np.linalg.norm(S0) - 1.0) < 1e-12, "norm must be kept"


def check_s6_bruteforce(impl, seed=36):
    q, k, v, a, th, b, S0 = random_unit(12, 4, 2, seed)
    o, S = impl(q, k, v, a, th, b, S0)
    X = S0.copy()
    for t in range(12):
        A_t = (np.eye(4) - b[t] * np.outer(k[t], k[t])) @ block_gate(a[t], th[t])
        X = A_t @ X + b[t] * np.outer(k[t], v[t])
        assert _rel(o[t], X.T @ q[t]) < 1e-12, f"output {t}"
    assert _rel(S, X) < 1e-12


def check_s7_affine(impl, seed=37):
    q, k, v, a, th, b, S0 = random_unit(24, 4, 3, seed)
    _, B = impl(q, k, v, a, th, b, np.zeros_like(S0))
    cols = []
    for i in range(4):
        E = np.zeros((4, 3))
        E[i, 0] = 1.0
        _, Si = impl(q, k, np.zeros_like(v), a, th, b, E)
        cols.append(Si[:, 0])
    M = np.stack(cols, axis=1)
    _, S = impl(q, k, v, a, th, b, S0)
    assert _rel(S, M @ S0 + B) < 1e-12, "a block must act on S0 as an affine map"


def check_s8_block_rotation_equivariance(impl, seed=38):
    q, k, v, a, th, b, S0 = random_unit(30, 6, 4, seed)
    phi = _rng(seed + 1).uniform(-math.pi, math.pi, 3)
    R = block_gate(np.ones(3), phi)
    o, S = impl(q, k, v, a, th, b, S0)
    o2, S2 = impl(q @ R.T, k @ R.T, v, a, th, b, R @ S0)
    assert _rel(o2, o) < 1e-12, "outputs must not change"
    assert _rel(S2, R @ S) < 1e-12, "the final state must rotate"


ALL_CHECKS = [check_s1_zero_phase_is_ckda, check_s2_phase_pi_is_negative_gate,
              check_s3_beta_zero_closed_form, check_s4_mod5_counter, check_s5_orthogonal,
              check_s6_bruteforce, check_s7_affine, check_s8_block_rotation_equivariance]


def oracle_unit(q, k, v, a, th, b, S0):
    """The fp64 oracle on one (sequence, head) unit, in the pin signature."""
    import oracle

    T, dk = q.shape
    dv = v.shape[1]
    out, S = oracle.forward_sfda(q.reshape(1, T, 1, dk), k.reshape(1, T, 1, dk),
                                 v.reshape(1, T, 1, dv), a.reshape(1, T, 1, dk // 2),
                                 th.reshape(1, T, 1, dk // 2), b.reshape(1, T, 1),
                                 S0=S0.reshape(1, 1, dk, dv), n_threads=1)
    return out.reshape(T, dv), S.reshape(dk, dv)
