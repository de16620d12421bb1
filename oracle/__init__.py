"""CKDA fp64 CPU oracle -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may import this package.  The
product path (``delta_rule_linear_ckda_b200``) never imports it, and it never
imports the product path: the two share no code.

Contents
--------
``forward`` / ``decode_step``
    Thin ctypes wrappers around ``ckda_oracle.c``: the sequential CKDA
    recurrence in fp64, token by token,
    ``S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T``,
    ``o_t = S_t^T q_t`` ("Complex KDA ..." page, section "Complex KDA (CKDA)
    Mimarisi ve Parametre Genislemesi"; "Gated DeltaNet-2" page, Methodology
    section 1 with b_t = w_t = beta_t).
``forward_gdn2``
    The Gated DeltaNet-2 recurrence ("Gated DeltaNet-2" page, Methodology
    section 1): the same loop with an erase gate b_t (key side) and a write
    gate w_t (value side) in place of beta_t,
    ``S_t = (I - k_t (b_t . k_t)^T) Diag(alpha_t) S_{t-1} + k_t (w_t . v_t)^T``;
    pinned by ``tests/pinlib_gdn2.py`` (G-1..G-7).
``forward_sfda``
    The SFDA recurrence ("Semidirect Fourier Delta Attention (SFDA)" page,
    "Arquitectura Central"): the real diagonal gate replaced by 2x2
    rotation-decay blocks ``alpha_p R(theta_p)`` on the state rows
    ``(2p, 2p+1)``,
    ``S_t = (I - beta_t k_t k_t^T) Lambda_t S_{t-1} + beta_t k_t v_t^T``;
    pinned by ``tests/pinlib_sfda.py`` (S-1..S-8).
``backward``
    The gradient of a scalar loss through the CKDA forward: given dL/do_t
    and dL/dS_final, dL/d(q, k, v, alpha, beta, S0), the adjoint of the
    per-token body taken step by step in reverse (states recomputed from
    checkpoints every 64 tokens); pinned by ``tests/pinlib_bwd.py`` (B-1..B-6:
    finite differences of the pinned forward, closed forms, symmetries).
``chunked`` (submodule)
    A plain numpy fp64 restatement of the chunkwise WY form, used only to pin
    the chunked algorithm against the sequential loop on tiny inputs.

Inputs are upcast exactly to fp64 (bf16 and fp32 values are representable),
so the oracle consumes bit-identical values to the CUDA path.  Parity
status of every function is listed in the test-suite module docstrings; all
functions here are pinned (no "parity unpinned" entries).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ckda_oracle.c")
_LIB = os.path.join(_HERE, "libckda_oracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile ``ckda_oracle.c`` with gcc into ``libckda_oracle.so``."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-std=c11", "-Wall", "-shared", "-fPIC", "-o", tmp, _SRC, "-lpthread", "-lm"]
        )
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            dp = ctypes.POINTER(ctypes.c_double)
            i64 = ctypes.c_int64
            lib.ckda_oracle_forward.argtypes = [
                i64, i64, i64, i64, ctypes.POINTER(ctypes.c_int64),
                dp, dp, dp, dp, dp, dp, dp, dp, ctypes.c_int,
            ]
            lib.ckda_oracle_forward.restype = ctypes.c_int
            lib.ckda_oracle_gdn2_forward.argtypes = [
                i64, i64, i64, i64, ctypes.POINTER(ctypes.c_int64),
                dp, dp, dp, dp, dp, dp, dp, dp, dp, ctypes.c_int,
            ]
            lib.ckda_oracle_gdn2_forward.restype = ctypes.c_int
            lib.ckda_oracle_sfda_forward.argtypes = [
                i64, i64, i64, i64, ctypes.POINTER(ctypes.c_int64),
                dp, dp, dp, dp, dp, dp, dp, dp, dp, ctypes.c_int,
            ]
            lib.ckda_oracle_sfda_forward.restype = ctypes.c_int
            lib.ckda_oracle_backward.argtypes = [
                i64, i64, i64, i64, ctypes.POINTER(ctypes.c_int64),
                dp, dp, dp, dp, dp, dp, dp, dp, dp, dp, dp, dp, dp, dp, ctypes.c_int,
            ]
            lib.ckda_oracle_backward.restype = ctypes.c_int
            lib.ckda_oracle_decode_step.argtypes = [
                i64, i64, i64, i64, dp, dp, dp, dp, dp, dp, dp, ctypes.c_int,
            ]
            lib.ckda_oracle_decode_step.restype = ctypes.c_int
            _lib = lib
    return _lib


def _f64(x) -> np.ndarray:
    """Exact upcast to a contiguous fp64 numpy array (torch or numpy input)."""
    if hasattr(x, "detach"):  # torch tensor
        x = x.detach().to("cpu")
        import torch

        x = x.to(torch.float64).numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def default_threads() -> int:
    return max(1, len(os.sched_getaffinity(0)))


def forward(q, k, v, alpha, beta, S0=None, cu_seqlens=None, n_threads=None):
    """Sequential fp64 CKDA forward.

    Fixed-length batch: q, k, alpha ``[B, T, H, dk]``, v ``[B, T, H, dv]``,
    beta ``[B, T, H]``.  Packed batch: pass ``cu_seqlens`` (``[N+1]``) and
    tensors ``[T_total, H, d]`` (a leading 1 is accepted).  ``S0`` is
    ``[N, H, dk, dv]`` or None (zero state).

    Returns ``(out, S_final)`` as fp64 numpy arrays, ``out`` shaped like ``v``.
    """
    qd, kd, vd, ad, bd = (_f64(t) for t in (q, k, v, alpha, beta))
    out_shape = vd.shape
    if cu_seqlens is None:
        if qd.ndim != 4:
            raise ValueError("fixed-length batch expects [B, T, H, d] tensors")
        B, T, H, dk = qd.shape
        cu = np.arange(B + 1, dtype=np.int64) * T
    else:
        cu = np.ascontiguousarray(np.asarray(
            cu_seqlens.cpu().numpy() if hasattr(cu_seqlens, "cpu") else cu_seqlens,
            dtype=np.int64))
        if qd.ndim == 4:
            if qd.shape[0] != 1:
                raise ValueError("packed batch expects a leading dimension of 1")
            qd, kd, vd, ad, bd = qd[0], kd[0], vd[0], ad[0], bd[0]
        H, dk = qd.shape[1], qd.shape[2]
    N = len(cu) - 1
    dv = vd.shape[-1]
    T_total = int(cu[-1])
    qd, kd, ad = (x.reshape(T_total, H, dk) for x in (qd, kd, ad))
    vd = vd.reshape(T_total, H, dv)
    bd = bd.reshape(T_total, H)
    S0d = None if S0 is None else _f64(S0).reshape(N, H, dk, dv)
    out = np.zeros((T_total, H, dv), dtype=np.float64)
    S_final = np.zeros((N, H, dk, dv), dtype=np.float64)
    rc = _load().ckda_oracle_forward(
        N, H, dk, dv, cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)),
        _ptr(qd), _ptr(kd), _ptr(vd), _ptr(ad), _ptr(bd), _ptr(S0d),
        _ptr(out), _ptr(S_final), int(n_threads or default_threads()),
    )
    if rc != 0:
        raise ValueError("ckda_oracle_forward rejected its arguments")
    return out.reshape(out_shape), S_final


def forward_gdn2(q, k, v, alpha, b, w, S0=None, cu_seqlens=None, n_threads=None):
    """Sequential fp64 Gated DeltaNet-2 forward ("Gated DeltaNet-2" summary,
    Methodology section 1): the CKDA recurrence with the scalar beta replaced
    by an erase gate ``b`` (shaped like ``k``) and a write gate ``w`` (shaped
    like ``v``).  Other arguments and the result as in ``forward``."""
    qd, kd, vd, ad, bgd, wgd = (_f64(t) for t in (q, k, v, alpha, b, w))
    out_shape = vd.shape
    if cu_seqlens is None:
        if qd.ndim != 4:
            raise ValueError("fixed-length batch expects [B, T, H, d] tensors")
        B, T, H, dk = qd.shape
        cu = np.arange(B + 1, dtype=np.int64) * T
    else:
        cu = np.ascontiguousarray(np.asarray(
            cu_seqlens.cpu().numpy() if hasattr(cu_seqlens, "cpu") else cu_seqlens,
            dtype=np.int64))
        if qd.ndim == 4:
            if qd.shape[0] != 1:
                raise ValueError("packed batch expects a leading dimension of 1")
            qd, kd, vd, ad, bgd, wgd = qd[0], kd[0], vd[0], ad[0], bgd[0], wgd[0]
        H, dk = qd.shape[1], qd.shape[2]
    N = len(cu) - 1
    dv = vd.shape[-1]
    T_total = int(cu[-1])
    qd, kd, ad, bgd = (x.reshape(T_total, H, dk) for x in (qd, kd, ad, bgd))
    vd, wgd = (x.reshape(T_total, H, dv) for x in (vd, wgd))
    S0d = None if S0 is None else _f64(S0).reshape(N, H, dk, dv)
    out = np.zeros((T_total, H, dv), dtype=np.float64)
    S_final = np.zeros((N, H, dk, dv), dtype=np.float64)
    rc = _load().ckda_oracle_gdn2_forward(
        N, H, dk, dv, cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)),
        _ptr(qd), _ptr(kd), _ptr(vd), _ptr(ad), _ptr(bgd), _ptr(wgd), _ptr(S0d),
        _ptr(out), _ptr(S_final), int(n_threads or default_threads()),
    )
    if rc != 0:
        raise ValueError("ckda_oracle_gdn2_forward rejected its arguments")
    return out.reshape(out_shape), S_final


def forward_sfda(q, k, v, alpha, theta, beta, S0=None, cu_seqlens=None, n_threads=None):
    """Sequential fp64 SFDA forward ("Semidirect Fourier Delta Attention
    (SFDA)" summary, "Arquitectura Central", real coordinates): the CKDA
    recurrence with Diag(alpha_t) replaced by the block-diagonal
    phase-decay gate whose block p is ``alpha_p R(theta_p)`` on state rows
    ``(2p, 2p+1)``.  ``alpha`` and ``theta`` are shaped like ``k`` with the
    last dimension halved; other arguments and the result as in
    ``forward``."""
    qd, kd, vd, ad, td, bd = (_f64(t) for t in (q, k, v, alpha, theta, beta))
    out_shape = vd.shape
    if cu_seqlens is None:
        if qd.ndim != 4:
            raise ValueError("fixed-length batch expects [B, T, H, d] tensors")
        B, T, H, dk = qd.shape
        cu = np.arange(B + 1, dtype=np.int64) * T
    else:
        cu = np.ascontiguousarray(np.asarray(
            cu_seqlens.cpu().numpy() if hasattr(cu_seqlens, "cpu") else cu_seqlens,
            dtype=np.int64))
        if qd.ndim == 4:
            if qd.shape[0] != 1:
                raise ValueError("packed batch expects a leading dimension of 1")
            qd, kd, vd, ad, td, bd = qd[0], kd[0], vd[0], ad[0], td[0], bd[0]
        H, dk = qd.shape[1], qd.shape[2]
    if dk % 2:
        raise ValueError("SFDA pairs the key channels: dk must be even")
    N = len(cu) - 1
    dv = vd.shape[-1]
    T_total = int(cu[-1])
    qd, kd = (x.reshape(T_total, H, dk) for x in (qd, kd))
    ad, td = (x.reshape(T_total, H, dk // 2) for x in (ad, td))
    vd = vd.reshape(T_total, H, dv)
    bd = bd.reshape(T_total, H)
    S0d = None if S0 is None else _f64(S0).reshape(N, H, dk, dv)
    out = np.zeros((T_total, H, dv), dtype=np.float64)
    S_final = np.zeros((N, H, dk, dv), dtype=np.float64)
    rc = _load().ckda_oracle_sfda_forward(
        N, H, dk, dv, cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)),
        _ptr(qd), _ptr(kd), _ptr(vd), _ptr(ad), _ptr(td), _ptr(bd), _ptr(S0d),
        _ptr(out), _ptr(S_final), int(n_threads or default_threads()),
    )
    if rc != 0:
        raise ValueError("ckda_oracle_sfda_forward rejected its arguments")
    return out.reshape(out_shape), S_final


def backward(q, k, v, alpha, beta, dO, S0=None, dS_final=None, cu_seqlens=None,
             n_threads=None):
    """fp64 gradients of the CKDA forward (see ``ckda_oracle_backward``).

    Inputs as in ``forward``; ``dO`` is shaped like ``v`` (the gradient of the
    loss with respect to the output), ``dS_final`` like the final state (or
    None = 0).  Returns a dict of fp64 numpy arrays ``dq, dk, dv, dalpha,
    dbeta, dS0`` shaped like ``q, k, v, alpha, beta`` and the state."""
    qd, kd, vd, ad, bd, dod = (_f64(t) for t in (q, k, v, alpha, beta, dO))
    shapes = {"dq": qd.shape, "dk": kd.shape, "dv": vd.shape, "dalpha": ad.shape,
              "dbeta": bd.shape}
    if cu_seqlens is None:
        if qd.ndim != 4:
            raise ValueError("fixed-length batch expects [B, T, H, d] tensors")
        B, T, H, dk = qd.shape
        cu = np.arange(B + 1, dtype=np.int64) * T
    else:
        cu = np.ascontiguousarray(np.asarray(
            cu_seqlens.cpu().numpy() if hasattr(cu_seqlens, "cpu") else cu_seqlens,
            dtype=np.int64))
        if qd.ndim == 4:
            if qd.shape[0] != 1:
                raise ValueError("packed batch expects a leading dimension of 1")
            qd, kd, vd, ad, bd, dod = qd[0], kd[0], vd[0], ad[0], bd[0], dod[0]
        H, dk = qd.shape[1], qd.shape[2]
    N = len(cu) - 1
    dv = vd.shape[-1]
    T_total = int(cu[-1])
    qd, kd, ad = (x.reshape(T_total, H, dk) for x in (qd, kd, ad))
    vd, dod = (x.reshape(T_total, H, dv) for x in (vd, dod))
    bd = bd.reshape(T_total, H)
    S0d = None if S0 is None else _f64(S0).reshape(N, H, dk, dv)
    dSf = None if dS_final is None else _f64(dS_final).reshape(N, H, dk, dv)
    g = {"dq": np.zeros((T_total, H, dk)), "dk": np.zeros((T_total, H, dk)),
         "dv": np.zeros((T_total, H, dv)), "dalpha": np.zeros((T_total, H, dk)),
         "dbeta": np.zeros((T_total, H)), "dS0": np.zeros((N, H, dk, dv))}
    rc = _load().ckda_oracle_backward(
        N, H, dk, dv, cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)),
        _ptr(qd), _ptr(kd), _ptr(vd), _ptr(ad), _ptr(bd), _ptr(S0d), _ptr(dod), _ptr(dSf),
        _ptr(g["dq"]), _ptr(g["dk"]), _ptr(g["dv"]), _ptr(g["dalpha"]), _ptr(g["dbeta"]),
        _ptr(g["dS0"]), int(n_threads or default_threads()),
    )
    if rc != 0:
        raise ValueError("ckda_oracle_backward rejected its arguments")
    for name, shp in shapes.items():
        g[name] = g[name].reshape(shp)
    return g


def _one_token(x):
    """[B, H, ...] -> [B, 1, H, ...] (one token per sequence)."""
    x = _f64(x)
    return x.reshape(x.shape[0], 1, *x.shape[1:])


def decode_step_gdn2(q, k, v, alpha, b, w, S, n_threads=None):
    """One fp64 Gated DeltaNet-2 step (``forward_gdn2`` on one token per
    sequence): q, k, alpha, b ``[B, H, dk]``, v, w ``[B, H, dv]``, S
    ``[B, H, dk, dv]``.  Returns ``(out, S_new)``."""
    out, Sn = forward_gdn2(*(_one_token(t) for t in (q, k, v, alpha, b, w)), S0=_f64(S),
                           n_threads=n_threads)
    return out[:, 0], Sn


def decode_step_sfda(q, k, v, alpha, theta, beta, S, n_threads=None):
    """One fp64 SFDA step (``forward_sfda`` on one token per sequence): q, k
    ``[B, H, dk]``, v ``[B, H, dv]``, alpha, theta ``[B, H, dk / 2]``, beta
    ``[B, H]``, S ``[B, H, dk, dv]``.  Returns ``(out, S_new)``."""
    out, Sn = forward_sfda(*(_one_token(t) for t in (q, k, v, alpha, theta, beta)), S0=_f64(S),
                           n_threads=n_threads)
    return out[:, 0], Sn


def decode_step(q, k, v, alpha, beta, S, n_threads=None):
    """One fp64 recurrent step: q, k, alpha ``[B, H, dk]``, v ``[B, H, dv]``,
    beta ``[B, H]``, S ``[B, H, dk, dv]``.  Returns ``(out, S_new)``."""
    qd, kd, vd, ad, bd = (_f64(t) for t in (q, k, v, alpha, beta))
    Sd = _f64(S).copy()
    B, H, dk = qd.shape
    dv = vd.shape[-1]
    out = np.zeros((B, H, dv), dtype=np.float64)
    rc = _load().ckda_oracle_decode_step(
        B, H, dk, dv, _ptr(qd), _ptr(kd), _ptr(vd), _ptr(ad), _ptr(bd), _ptr(Sd),
        _ptr(out), int(n_threads or default_threads()),
    )
    if rc != 0:
        raise ValueError("ckda_oracle_decode_step rejected its arguments")
    return out, Sd
