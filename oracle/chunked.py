"""Chunkwise WY restatement of CKDA in numpy fp64 -- TEST INFRASTRUCTURE ONLY.

This is not the reference result (that is the sequential loop in
``ckda_oracle.c``); it restates the chunkwise-parallel form that the CUDA
kernels follow, plainly and without blocking tricks, so that tests can pin
the algebra of the chunk form against the sequential loop on tiny inputs.

Sources for the chunk form:
  * "Semidirect Fourier Delta Attention (SFDA)" summary, section "El Teorema
    de Chunk-WY Constructivo": within a block the product of transitions is a
    diagonal product minus a correction whose rank is bounded by the block
    size; and "Principales Contribuciones" item 3: the block acts on its start
    state as an exact affine map S_end = M S_start + B, where B is the result
    of the zero-initial-state recurrence.
  * "Gated DeltaNet-2" summary, Methodology section 3: the per-channel decay
    is absorbed into the erase/write factors, and the auxiliary matrices come
    from a lower-triangular solve (I + T)^-1.

Per chunk of positions r = 0..L-1 with start state S0, writing P(r, s) for the
channel-wise product alpha_{s+1} * ... * alpha_r (P(r, r) = 1):
  Gamma_r = alpha_0 * ... * alpha_r,   rho_s = P(L-1, s),   gamma = Gamma_{L-1}
  T[r, s] = beta_r sum_i k_ri k_si P_i(r, s)          (s < r)
  A[r, s] = sum_i q_ri k_si P_i(r, s)                 (s <= r)
  W = (I + T)^-1 diag(beta) (K * Gamma),  U~ = (I + T)^-1 diag(beta) V
  U = U~ - W S0
  O = (Q * Gamma) S0 + A U
  S_end = Diag(gamma) S0 + (K * rho)^T U
All gate products are explicit products of alphas: no division and no
logarithm, so zero and negative gates are handled exactly.
"""
from __future__ import annotations

import numpy as np


def pair_products(alpha: np.ndarray) -> np.ndarray:
    """P[r, s, :] = prod_{j=s+1..r} alpha[j, :] for s <= r (else 0)."""
    L, d = alpha.shape
    P = np.zeros((L, L, d))
    for s in range(L):
        acc = np.ones(d)
        P[s, s] = acc
        for r in range(s + 1, L):
            acc = acc * alpha[r]
            P[r, s] = acc
    return P


def chunk_factors(q, k, v, alpha, beta):
    """All chunk quantities for one (sequence, head) chunk of length L.

    q, k, alpha: [L, dk]; v: [L, dv]; beta: [L].  Returns a dict with
    T, A, W, Ut (= U~), Gamma, rho, gamma.
    """
    L, dk = k.shape
    P = pair_products(alpha)
    Gamma = np.ones((L, dk))
    acc = np.ones(dk)
    for r in range(L):
        acc = acc * alpha[r]
        Gamma[r] = acc
    rho = P[L - 1, :, :]  # rho[s] = P(L-1, s)
    gamma = Gamma[L - 1]
    T = np.zeros((L, L))
    A = np.zeros((L, L))
    for r in range(L):
        for s in range(r + 1):
            if s < r:
                T[r, s] = beta[r] * np.sum(k[r] * k[s] * P[r, s])
            A[r, s] = np.sum(q[r] * k[s] * P[r, s])
    IT = np.eye(L) + T
    W = np.linalg.solve(IT, beta[:, None] * (k * Gamma))
    Ut = np.linalg.solve(IT, beta[:, None] * v)
    return dict(T=T, A=A, W=W, Ut=Ut, Gamma=Gamma, rho=rho, gamma=gamma)


def chunk_step(q, k, v, alpha, beta, S0):
    """Apply one chunk to the start state S0: returns (O, S_end)."""
    f = chunk_factors(q, k, v, alpha, beta)
    U = f["Ut"] - f["W"] @ S0
    O = (q * f["Gamma"]) @ S0 + f["A"] @ U
    S_end = f["gamma"][:, None] * S0 + (k * f["rho"]).T @ U
    return O, S_end


def chunk_affine(q, k, v, alpha, beta):
    """The chunk's affine map S_end = M S_start + B (SFDA page, contribution 3).

    M = Diag(gamma) - (K * rho)^T W  and  B = (K * rho)^T U~.
    """
    f = chunk_factors(q, k, v, alpha, beta)
    Kr = k * f["rho"]
    M = np.diag(f["gamma"]) - Kr.T @ f["W"]
    B = Kr.T @ f["Ut"]
    return M, B


def forward_unit(q, k, v, alpha, beta, S0, chunk):
    """Chunked forward of one (sequence, head) unit, fp64.

    q, k, alpha: [T, dk]; v: [T, dv]; beta: [T]; S0: [dk, dv].
    The last chunk may be partial.  Returns (out [T, dv], S_final).
    """
    q, k, v, alpha, beta = (np.asarray(x, dtype=np.float64) for x in (q, k, v, alpha, beta))
    S = np.array(S0, dtype=np.float64, copy=True)
    T = q.shape[0]
    out = np.zeros((T, v.shape[1]))
    for c0 in range(0, T, chunk):
        c1 = min(T, c0 + chunk)
        O, S = chunk_step(q[c0:c1], k[c0:c1], v[c0:c1], alpha[c0:c1], beta[c0:c1], S)
        out[c0:c1] = O
    return out, S


def forward(q, k, v, alpha, beta, S0=None, chunk=16):
    """Chunked forward over a fixed-length batch [B, T, H, d] (fp64 numpy)."""
    q, k, v, alpha, beta = (np.asarray(x, dtype=np.float64) for x in (q, k, v, alpha, beta))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    out = np.zeros((B, T, H, dv))
    S_final = np.zeros((B, H, dk, dv))
    for b in range(B):
        for h in range(H):
            s0 = np.zeros((dk, dv)) if S0 is None else np.asarray(S0[b, h], dtype=np.float64)
            o, s = forward_unit(q[b, :, h], k[b, :, h], v[b, :, h], alpha[b, :, h],
                                beta[b, :, h], s0, chunk)
            out[b, :, h] = o
            S_final[b, h] = s
    return out, S_final
