"""Pins for the CKDA recurrence: checks that do not trust the implementation.

Each ``check_*`` takes an implementation ``impl(q, k, v, alpha, beta, S0)``
of ONE (sequence, head) unit -- q, k, alpha ``[T, dk]``, v ``[T, dv]``,
beta ``[T]``, S0 ``[dk, dv]``, all fp64 numpy -- returning
``(out [T, dv], S_final [dk, dv])``, and raises ``AssertionError`` when the
implementation breaks a fact fixed by the pages or by the mathematics.

The facts, with their sources:
  P-1  d=2 worked example: Diag(1, -1) followed by the beta=2 reflection about
       k = (cos phi, sin phi) is the rotation R(2 phi + pi); angles add along a
       chain ("Complex KDA" page, "Complex KDA (CKDA) Mimarisi ..." section;
       "Kimi Delta Attention enhanced ..." page, first section).
  P-2  beta=2, alpha in {+-1}^d, |k|=1: every transition is orthogonal, so with
       v=0 the Frobenius norm of the state is kept ("Complex KDA" page,
       "Teorik Cikarimlar ..." section: orthogonal DPR1 matrices).
  P-3  transitions are non-expansive: ||(I - b k k^T) Diag(a)||_2 <= max|a_i|
       for b in [0, 2], |k| = 1 ("Complex KDA" page, "Complex KDA (CKDA)
       Mimarisi ..." section).
  P-4  alpha = 1 gives DeltaNet, scalar alpha gives Gated DeltaNet ("Gated
       DeltaNet-2" page, Methodology section 1; "GPT-2'den Kimi K3'ye" page on
       DeltaNet / Gated DeltaNet).
  P-5  the chunkwise WY form equals the sequential loop ("SFDA" page,
       "El Teorema de Chunk-WY Constructivo" and "Resultados", residuals at
       working precision).
  P-6  a block of tokens acts on its start state as an exact affine map
       S_end = M S_start + B, B from the zero-initial-state run ("SFDA" page,
       "Principales Contribuciones" item 3).
  P-7..P-12 follow from the recurrence itself: beta=0 and alpha=0 closed
       forms, delta-rule retrieval, sign symmetry, linearity, and brute-force
       expansion with explicit transition matrices.
"""
from __future__ import annotations

import math
import os

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _rng(seed):
    return np.random.default_rng(seed)


def _unit_rows(x):
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


def random_unit(T, dk, dv, seed, alpha_lo=-1.0, alpha_hi=1.0):
    r = _rng(seed)
    q = _unit_rows(r.standard_normal((T, dk)))
    k = _unit_rows(r.standard_normal((T, dk)))
    v = r.standard_normal((T, dv))
    a = r.uniform(alpha_lo, alpha_hi, (T, dk))
    b = r.uniform(0.0, 2.0, T)
    S0 = r.standard_normal((dk, dv))
    return q, k, v, a, b, S0


def _rel(a, b):
    scale = max(1.0, float(np.max(np.abs(b))))
    return float(np.max(np.abs(np.asarray(a) - np.asarray(b)))) / scale


def load_p1_golden():
    rows = []
    with open(os.path.join(GOLDEN, "p1_rotation_d2.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            phi, r00, r01, r10, r11 = (float(x) for x in line.split())
            rows.append((phi, np.array([[r00, r01], [r10, r11]])))
    return rows


def check_p1_rotation(impl):
    """One step on S0 = I gives the transition matrix, which must be R(2 phi + pi)."""
    for phi, R in load_p1_golden():
        k = np.array([[math.cos(phi), math.sin(phi)]])
        a = np.array([[1.0, -1.0]])
        b = np.array([2.0])
        v = np.zeros((1, 2))
        q = np.array([[1.0, 0.0]])
        out, S = impl(q, k, v, a, b, np.eye(2))
        assert _rel(S, R) <= 1e-15 * 4, (phi, S, R)
        assert abs(np.linalg.det(S) - 1.0) <= 1e-14
        assert _rel(out[0], R[0]) <= 1e-15 * 4  # o = S^T e_0 = first row of S


def check_p1_chain(impl, T=64, seed=1):
    r = _rng(seed)
    phis = r.uniform(-math.pi, math.pi, T)
    k = np.stack([np.cos(phis), np.sin(phis)], axis=1)
    a = np.tile([1.0, -1.0], (T, 1))
    b = np.full(T, 2.0)
    v = np.zeros((T, 3))
    q = _unit_rows(r.standard_normal((T, 2)))
    S0 = r.standard_normal((2, 3))
    out, S = impl(q, k, v, a, b, S0)
    th = float(np.sum(2 * phis + math.pi))
    R = np.array([[math.cos(th), -math.sin(th)], [math.sin(th), math.cos(th)]])
    assert _rel(S, R @ S0) <= 1e-12
    # every intermediate output is the rotated state read by q_t
    th_t = np.cumsum(2 * phis + math.pi)
    for t in (0, T // 2, T - 1):
        Rt = np.array([[math.cos(th_t[t]), -math.sin(th_t[t])], [math.sin(th_t[t]), math.cos(th_t[t])]])
        assert _rel(out[t], (Rt @ S0).T @ q[t]) <= 1e-12


def check_p2_orthogonal(impl, d=8, seed=2):
    r = _rng(seed)
    for trial in range(8):
        k = _unit_rows(r.standard_normal((1, d)))
        a = np.where(r.random((1, d)) < 0.5, -1.0, 1.0)
        _, A = impl(np.zeros((1, d)), k, np.zeros((1, d)), a, np.array([2.0]), np.eye(d))
        assert _rel(A.T @ A, np.eye(d)) <= 1e-14
    T = 2000
    k = _unit_rows(r.standard_normal((T, d)))
    a = np.where(r.random((T, d)) < 0.5, -1.0, 1.0)
    S0 = r.standard_normal((d, 5))
    _, S = impl(np.zeros((T, d)), k, np.zeros((T, 5)), a, np.full(T, 2.0), S0)
    ratio = np.linalg.norm(S) / np.linalg.norm(S0)
    assert abs(ratio - 1.0) <= 1e-12, ratio


def check_p3_nonexpansive(impl, d=6, seed=3):
    r = _rng(seed)
    for trial in range(200):
        k = _unit_rows(r.standard_normal((1, d)))
        a = r.uniform(-1, 1, (1, d))
        b = np.array([r.uniform(0, 2)])
        if trial % 10 == 0:
            b[0] = 2.0
        _, A = impl(np.zeros((1, d)), k, np.zeros((1, d)), a, b, np.eye(d))
        bound = max(1.0, abs(1.0 - b[0])) * float(np.max(np.abs(a)))
        assert np.linalg.norm(A, 2) <= bound + 1e-12
        # the transition is diagonal-plus-rank-one: A - Diag(a) has rank <= 1
        sv = np.linalg.svd(A - np.diag(a[0]), compute_uv=False)
        assert sv[1] <= 1e-12 * max(1.0, sv[0])


def _deltanet(q, k, v, b, S0):
    """DeltaNet, written independently: S <- S - b k (k^T S) + b k v^T, o = S^T q."""
    S = S0.copy()
    out = []
    for t in range(q.shape[0]):
        S = S - b[t] * np.outer(k[t], k[t] @ S) + b[t] * np.outer(k[t], v[t])
        out.append(S.T @ q[t])
    return np.array(out), S


def _gated_deltanet(q, k, v, g, b, S0):
    """Gated DeltaNet with a scalar decay g_t: S <- g_t (I - b k k^T) S + b k v^T."""
    S = S0.copy()
    out = []
    for t in range(q.shape[0]):
        S = g[t] * (S - b[t] * np.outer(k[t], k[t] @ S)) + b[t] * np.outer(k[t], v[t])
        out.append(S.T @ q[t])
    return np.array(out), S


def check_p4_reductions(impl, seed=4):
    q, k, v, a, b, S0 = random_unit(40, 5, 4, seed)
    o1, S1 = impl(q, k, v, np.ones_like(a), b, S0)
    o2, S2 = _deltanet(q, k, v, b, S0)
    assert _rel(o1, o2) <= 1e-13 and _rel(S1, S2) <= 1e-13
    g = _rng(seed + 1).uniform(-1, 1, 40)
    o1, S1 = impl(q, k, v, np.repeat(g[:, None], 5, axis=1), b, S0)
    o2, S2 = _gated_deltanet(q, k, v, g, b, S0)
    assert _rel(o1, o2) <= 1e-13 and _rel(S1, S2) <= 1e-13


def check_p5_chunked(impl, seed=5):
    from oracle import chunked

    for C in (4, 8, 16):
        q, k, v, a, b, S0 = random_unit(37, 6, 5, seed + C)
        a[5] = 0.0          # a zero-gate row
        a[9, :3] = 0.0      # zero channels
        a[12] = -1.0        # a full reflection row
        o1, S1 = impl(q, k, v, a, b, S0)
        o2, S2 = chunked.forward_unit(q, k, v, a, b, S0, C)
        assert _rel(o2, o1) <= 1e-12 and _rel(S2, S1) <= 1e-12, (C, _rel(o2, o1), _rel(S2, S1))


def _transition(k, a, b):
    return (np.eye(len(k)) - b * np.outer(k, k)) @ np.diag(a)


def check_p6_affine(impl, seed=6):
    from oracle import chunked

    q, k, v, a, b, S0 = random_unit(24, 5, 3, seed)
    o_all, S_all = impl(q, k, v, a, b, S0)
    o_a, S_mid = impl(q[:11], k[:11], v[:11], a[:11], b[:11], S0)
    o_b, S_end = impl(q[11:], k[11:], v[11:], a[11:], b[11:], S_mid)
    assert _rel(np.concatenate([o_a, o_b]), o_all) <= 1e-13 and _rel(S_end, S_all) <= 1e-13
    # S_end = M S_start + B with M the product of transitions and B the zero-start run
    M = np.eye(5)
    for t in range(24):
        M = _transition(k[t], a[t], b[t]) @ M
    _, Bz = impl(q, k, v, a, b, np.zeros((5, 3)))
    assert _rel(S_all, M @ S0 + Bz) <= 1e-12
    # and the chunk-form summary agrees with both
    Mc, Bc = chunked.chunk_affine(q, k, v, a, b)
    assert _rel(Mc, M) <= 1e-12 and _rel(Bc, Bz) <= 1e-12


def check_p7_beta_zero(impl, seed=7):
    q, k, v, a, b, S0 = random_unit(30, 4, 3, seed)
    out, S = impl(q, k, v, a, np.zeros(30), S0)
    G = np.cumprod(a, axis=0)
    assert _rel(S, G[-1][:, None] * S0) <= 1e-14
    for t in range(30):
        assert _rel(out[t], (G[t][:, None] * S0).T @ q[t]) <= 1e-13


def check_p8_alpha_zero(impl, seed=8):
    q, k, v, a, b, S0 = random_unit(30, 4, 3, seed)
    out, S = impl(q, k, v, np.zeros_like(a), b, S0)
    assert _rel(S, b[-1] * np.outer(k[-1], v[-1])) <= 1e-14
    for t in range(30):
        assert _rel(out[t], b[t] * float(k[t] @ q[t]) * v[t]) <= 1e-14


def check_p9_retrieval(impl, seed=9):
    q, k, v, a, b, S0 = random_unit(20, 6, 4, seed)
    out, _ = impl(k, k, v, a, np.ones(20), S0)   # read with q_t = k_t, beta = 1
    assert _rel(out, v) <= 1e-13
    # general beta, one step: S_1^T k = (1 - b)(Diag(a) S0)^T k + b v
    out, _ = impl(k[:1], k[:1], v[:1], a[:1], b[:1], S0)
    expect = (1 - b[0]) * ((a[0][:, None] * S0).T @ k[0]) + b[0] * v[0]
    assert _rel(out[0], expect) <= 1e-13


def check_p10_sign_symmetry(impl, seed=10):
    q, k, v, a, b, S0 = random_unit(25, 5, 4, seed)
    o1, S1 = impl(q, k, v, a, b, S0)
    o2, S2 = impl(q, -k, -v, a, b, S0)
    assert np.array_equal(o1, o2) and np.array_equal(S1, S2)


def check_p11_linearity(impl, seed=11):
    q, k, v, a, b, S0 = random_unit(25, 5, 4, seed)
    r = _rng(seed + 100)
    v2 = r.standard_normal(v.shape)
    S02 = r.standard_normal(S0.shape)
    o1, S1 = impl(q, k, v, a, b, S0)
    o2, S2 = impl(q, k, v2, a, b, S02)
    o3, S3 = impl(q, k, 2.0 * v - 3.0 * v2, a, b, 2.0 * S0 - 3.0 * S02)
    assert _rel(o3, 2 * o1 - 3 * o2) <= 1e-12 and _rel(S3, 2 * S1 - 3 * S2) <= 1e-12


def check_p12_bruteforce(impl, seed=12):
    for d in (2, 3, 4):
        for T in (1, 3, 8):
            q, k, v, a, b, S0 = random_unit(T, d, d, seed + 10 * d + T)
            out, S = impl(q, k, v, a, b, S0)
            # S_T = (A_T ... A_1) S0 + sum_t (A_T ... A_{t+1}) b_t k_t v_t^T
            As = [_transition(k[t], a[t], b[t]) for t in range(T)]
            for t_end in range(T):
                P = np.eye(d)
                for t in range(t_end + 1):
                    P = As[t] @ P
                St = P @ S0
                for t in range(t_end + 1):
                    R = np.eye(d)
                    for j in range(t + 1, t_end + 1):
                        R = As[j] @ R
                    St = St + R @ (b[t] * np.outer(k[t], v[t]))
                assert _rel(out[t_end], St.T @ q[t_end]) <= 1e-13
            assert _rel(S, St) <= 1e-13


ALL_CHECKS = [
    check_p1_rotation, check_p1_chain, check_p2_orthogonal, check_p3_nonexpansive,
    check_p4_reductions, check_p5_chunked, check_p6_affine, check_p7_beta_zero,
    check_p8_alpha_zero, check_p9_retrieval, check_p10_sign_symmetry,
    check_p11_linearity, check_p12_bruteforce,
]


def oracle_unit(q, k, v, a, b, S0):
    """Adapter: the C oracle on one (sequence, head) unit."""
    import oracle

    out, S = oracle.forward(q[None, :, None, :], k[None, :, None, :], v[None, :, None, :],
                            a[None, :, None, :], b[None, :, None], S0=S0[None, None], n_threads=1)
    return out[0, :, 0, :], S[0, 0]
