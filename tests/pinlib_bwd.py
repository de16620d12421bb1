"""Pins for the backward of the CKDA recurrence: checks that do not trust the
implementation.

Each ``check_*`` takes an implementation ``impl(q, k, v, alpha, beta, S0, dO,
dS_T)`` of the gradient for ONE (sequence, head) unit -- q, k, alpha
``[T, dk]``, v, dO ``[T, dv]``, beta ``[T]``, S0, dS_T ``[dk, dv]``, all fp64
numpy -- returning a dict with ``dq, dk, dalpha [T, dk]``, ``dv [T, dv]``,
``dbeta [T]`` and ``dS0 [dk, dv]``: the gradient of the scalar
L = sum(dO * O) + sum(dS_T * S_T) with respect to each input, where
(O, S_T) is the CKDA forward ("Complex KDA ..." page, section "Complex KDA
(CKDA) Mimarisi ve Parametre Genislemesi"; the "Gated DeltaNet-2" page,
Methodology section 1, form with b = w = beta).  A check raises
``AssertionError`` when the implementation breaks a fact fixed by the
mathematics.

  B-1  central finite differences of the pinned forward oracle (pinlib):
       every gradient entry on a tiny unit (T = 9), and a random sample of
       entries on a unit longer than the oracle's 64-token recompute segment
       (T = 70).
  B-2  the gradient is linear in the upstream gradients (dO, dS_T).
  B-3  zero upstream gradients give exactly zero gradients.
  B-4  beta = 0 (nothing written): dk = dv = 0 exactly; dq, dS0 and dbeta
       in closed form through the products of the gates.
  B-5  alpha = 0 (memoryless, S_t = beta_t k_t v_t^T): every gradient in
       closed form.
  B-6  (k, v) -> (-k, -v) negates dk and dv and leaves the other gradients
       bit-identical.
"""
from __future__ import annotations

import numpy as np

import pinlib


def _rng(seed):
    return np.random.default_rng(seed)


def _unit_rows(x):
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


def random_case(T, dk, dv, seed):
    r = _rng(seed)
    q = _unit_rows(r.standard_normal((T, dk)))
    k = _unit_rows(r.standard_normal((T, dk)))
    v = r.standard_normal((T, dv))
    a = r.uniform(-1.0, 1.0, (T, dk))
    b = r.uniform(0.0, 2.0, T)
    S0 = r.standard_normal((dk, dv))
    dO = r.standard_normal((T, dv))
    dST = r.standard_normal((dk, dv))
    return q, k, v, a, b, S0, dO, dST


NAMES = ("q", "k", "v", "alpha", "beta", "S0")
GRAD = {"q": "dq", "k": "dk", "v": "dv", "alpha": "dalpha", "beta": "dbeta", "S0": "dS0"}


def _loss(inp, dO, dST):
    o, S = pinlib.oracle_unit(inp["q"], inp["k"], inp["v"], inp["alpha"], inp["beta"], inp["S0"])
    return float(np.sum(dO * o) + np.sum(dST * S))


def _fd_check(impl, case, entries=None, h=1e-6, tol=1e-7, seed=0):
    q, k, v, a, b, S0, dO, dST = case
    inp = {"q": q, "k": k, "v": v, "alpha": a, "beta": b, "S0": S0}
    g = impl(q, k, v, a, b, S0, dO, dST)
    r = _rng(seed)
    for name in NAMES:
        x = inp[name]
        idx = list(np.ndindex(x.shape))
        if entries is not None and len(idx) > entries:
            idx = [idx[i] for i in r.choice(len(idx), entries, replace=False)]
        grad = np.asarray(g[GRAD[name]])
        scale = max(1.0, float(np.max(np.abs(grad))))
        for ix in idx:
            xp = {kk: vv.copy() for kk, vv in inp.items()}
            xm = {kk: vv.copy() for kk, vv in inp.items()}
            xp[name][ix] += h
            xm[name][ix] -= h
            fd = (_loss(xp, dO, dST) - _loss(xm, dO, dST)) / (2 * h)
            assert abs(fd - grad[ix]) <= tol * scale, f"d{name}{ix}: {grad[ix]} vs {fd}"


def check_b1_finite_differences(impl, seed=41):
    _fd_check(impl, random_case(9, 3, 2, seed))
    _fd_check(impl, random_case(70, 3, 2, seed + 1), entries=12, seed=seed)


def check_b2_linear_in_upstream(impl, seed=42):
    q, k, v, a, b, S0, dO, dST = random_case(20, 4, 3, seed)
    r = _rng(seed + 1)
    dO2, dST2 = r.standard_normal(dO.shape), r.standard_normal(dST.shape)
    g1 = impl(q, k, v, a, b, S0, dO, dST)
    g2 = impl(q, k, v, a, b, S0, dO2, dST2)
    g3 = impl(q, k, v, a, b, S0, 2.0 * dO - 3.0 * dO2, 2.0 * dST - 3.0 * dST2)
    for n in GRAD.values():
        want = 2.0 * np.asarray(g1[n]) - 3.0 * np.asarray(g2[n])
        assert np.max(np.abs(np.asarray(g3[n]) - want)) <= 1e-11 * max(1.0, np.max(np.abs(want))), n


def check_b3_zero_upstream(impl, seed=43):
    q, k, v, a, b, S0, dO, dST = random_case(15, 4, 3, seed)
    g = impl(q, k, v, a, b, S0, np.zeros_like(dO), np.zeros_like(dST))
    for n in GRAD.values():
        assert np.max(np.abs(np.asarray(g[n]))) == 0.0, n


def check_b4_beta_zero(impl, seed=44):
    q, k, v, a, _, S0, dO, dST = random_case(12, 4, 3, seed)
    T = q.shape[0]
    g = impl(q, k, v, a, np.zeros(T), S0, dO, dST)
    assert np.max(np.abs(g["dk"])) == 0.0 and np.max(np.abs(g["dv"])) == 0.0
    Gam = np.cumprod(a, axis=0)                      # Gamma_t = prod_{s<=t} alpha_s
    for t in range(T):
        St = Gam[t][:, None] * S0
        assert np.allclose(g["dq"][t], St @ dO[t], rtol=0, atol=1e-12), f"dq {t}"
        # dL/dS_t: the outputs from t on and dS_T, carried back through the gates
        dSt = np.zeros_like(S0)
        for t2 in range(t, T):
            P = np.prod(a[t + 1:t2 + 1], axis=0)
            dSt += P[:, None] * np.outer(q[t2], dO[t2])
        dSt += np.prod(a[t + 1:], axis=0)[:, None] * dST
        r_t = St.T @ k[t]
        assert abs(g["dbeta"][t] - (dSt.T @ k[t]) @ (v[t] - r_t)) <= 1e-11, f"dbeta {t}"
    dS0 = sum(Gam[t][:, None] * np.outer(q[t], dO[t]) for t in range(T)) + Gam[-1][:, None] * dST
    assert np.allclose(g["dS0"], dS0, rtol=0, atol=1e-11)


def check_b5_alpha_zero(impl, seed=45):
    q, k, v, _, b, S0, dO, dST = random_case(10, 4, 3, seed)
    T, dk = q.shape
    g = impl(q, k, v, np.zeros((T, dk)), b, S0, dO, dST)
    for t in range(T):
        dS = np.outer(q[t], dO[t]) + (dST if t == T - 1 else 0.0)   # dL/dS_t
        assert np.allclose(g["dv"][t], b[t] * (dS.T @ k[t]), atol=1e-12), f"dv {t}"
        assert np.allclose(g["dq"][t], b[t] * k[t] * (v[t] @ dO[t]), atol=1e-12), f"dq {t}"
        assert np.allclose(g["dk"][t], b[t] * (dS @ v[t]), atol=1e-12), f"dk {t}"
        assert abs(g["dbeta"][t] - k[t] @ dS @ v[t]) <= 1e-12, f"dbeta {t}"
        S_prev = S0 if t == 0 else b[t - 1] * np.outer(k[t - 1], v[t - 1])
        # S_t = (I - b k k^T) Diag(alpha) S_prev + ...: dalpha = rowsum(((I - b k k^T)^T dS) * S_prev)
        dSp = dS - b[t] * np.outer(k[t], dS.T @ k[t])
        assert np.allclose(g["dalpha"][t], np.sum(dSp * S_prev, axis=1), atol=1e-12), f"da {t}"
    assert np.max(np.abs(g["dS0"])) == 0.0


def check_b6_sign_symmetry(impl, seed=46):
    q, k, v, a, b, S0, dO, dST = random_case(16, 4, 3, seed)
    g1 = impl(q, k, v, a, b, S0, dO, dST)
    g2 = impl(q, -k, -v, a, b, S0, dO, dST)
    assert np.array_equal(g2["dk"], -g1["dk"]) and np.array_equal(g2["dv"], -g1["dv"])
    for n in ("dq", "dalpha", "dbeta", "dS0"):
        assert np.array_equal(g2[n], g1[n]), n


ALL_CHECKS = [check_b1_finite_differences, check_b2_linear_in_upstream, check_b3_zero_upstream,
              check_b4_beta_zero, check_b5_alpha_zero, check_b6_sign_symmetry]


def oracle_unit(q, k, v, a, b, S0, dO, dST):
    """The fp64 backward oracle on one (sequence, head) unit, in the pin signature."""
    import oracle

    T, dk = q.shape
    dv = v.shape[1]
    g = oracle.backward(q.reshape(1, T, 1, dk), k.reshape(1, T, 1, dk), v.reshape(1, T, 1, dv),
                        a.reshape(1, T, 1, dk), b.reshape(1, T, 1), dO.reshape(1, T, 1, dv),
                        S0=S0.reshape(1, 1, dk, dv), dS_final=dST.reshape(1, 1, dk, dv),
                        n_threads=1)
    return {"dq": g["dq"].reshape(T, dk), "dk": g["dk"].reshape(T, dk),
            "dv": g["dv"].reshape(T, dv), "dalpha": g["dalpha"].reshape(T, dk),
            "dbeta": g["dbeta"].reshape(T), "dS0": g["dS0"].reshape(dk, dv)}
