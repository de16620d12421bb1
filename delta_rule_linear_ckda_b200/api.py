"""Torch-tensor front end of the C ABI (argument marshalling only).

Every function checks dtypes, shapes and contiguity, passes ``data_ptr()``
values and the current CUDA stream to ``libckda.so`` and raises ``CKDAError``
on a non-zero status.  All arithmetic happens in the CUDA kernels.
"""
from __future__ import annotations

import math
from typing import Optional, Tuple

import torch

from . import _lib
from ._lib import CKDAError

_DT = {torch.float32: _lib.CKDA_F32, torch.bfloat16: _lib.CKDA_BF16}


def _stream_ptr(device) -> int:
    return torch.cuda.current_stream(device).cuda_stream


def _need(t: torch.Tensor, name: str, dtype=None, device=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")


def _p(t: Optional[torch.Tensor]):
    return None if t is None else t.data_ptr()


def fwd_chunked(q, k, v, alpha, beta, S0=None, cu_seqlens=None, chunk: int = 64,
                out=None, S_final=None, return_final: bool = True, fp32core: bool = False,
                out_dtype=None, workspace=None) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """Chunked CKDA forward.  Shapes as in ``ckda_fwd_chunked`` (include/ckda.h).

    Fixed-length: q, k, alpha ``[B, T, H, dk]``; v ``[B, T, H, dv]``; beta ``[B, T, H]``.
    Packed: ``cu_seqlens`` int32 ``[N+1]`` and tensors with a leading 1 or without it.
    ``out_dtype`` (float32 or bfloat16) defaults to the dtype of ``out`` if given,
    else to the input dtype.  ``workspace`` is an optional uint8 CUDA tensor of at
    least ``workspace_bytes(...)`` bytes; without it one is taken from torch's
    caching allocator for the call.
    Returns ``(out, S_final)``; ``S_final`` is None when ``return_final`` is False.
    """
    dev = q.device
    B, T, H, dk, dv, N = _inputs_shape(q, k, v, alpha, beta, cu_seqlens)
    if S0 is not None:
        _need(S0, "S0", torch.float32, dev)
        if tuple(S0.shape) != (N, H, dk, dv):
            raise ValueError(f"S0 must be [{N}, {H}, {dk}, {dv}]")
    if out_dtype is None:
        out_dtype = out.dtype if out is not None else q.dtype
    if out_dtype not in _DT:
        raise TypeError("out_dtype must be float32 or bfloat16")
    if out is None:
        out = torch.empty(v.shape, dtype=out_dtype, device=dev)
    else:
        _need(out, "out", out_dtype, dev)
        if out.shape != v.shape:
            raise ValueError("out must have v's shape")
    if return_final and S_final is None:
        S_final = torch.empty((N, H, dk, dv), dtype=torch.float32, device=dev)
    if S_final is not None:
        _need(S_final, "S_final", torch.float32, dev)
    lib = _lib.load()
    with torch.cuda.device(dev):
        if fp32core:
            rc = lib.ckda_fwd_chunked_fp32core(
                _p(q), _p(k), _p(v), _p(alpha), _p(beta), _p(S0), _p(cu_seqlens), _p(out),
                _p(S_final), B, T, H, dk, dv, chunk, _DT[q.dtype], _DT[out_dtype],
                _stream_ptr(dev))
        else:
            need = workspace_bytes(B, T, H, dk, dv, chunk, q.dtype, out_dtype,
                                   cu_seqlens is not None)
            if workspace is None and need > 0:
                workspace = torch.empty(need, dtype=torch.uint8, device=dev)
            if workspace is not None:
                _need(workspace, "workspace", torch.uint8, dev)
            rc = lib.ckda_fwd_chunked(
                _p(q), _p(k), _p(v), _p(alpha), _p(beta), _p(S0), _p(cu_seqlens), _p(out),
                _p(S_final), B, T, H, dk, dv, chunk, _DT[q.dtype], _DT[out_dtype],
                _p(workspace), 0 if workspace is None else workspace.numel(), _stream_ptr(dev))
    if rc != 0:
        raise CKDAError(rc, "ckda_fwd_chunked")
    return out, S_final


def fwd_chunked_static(q, k, v, alpha, beta, S0=None, cu_seqlens=None, chunk: int = 64,
                       out=None, S_final=None, return_final: bool = True, out_dtype=None):
    """``fwd_chunked`` through ``ckda_fwd_chunked_static``: no workspace is passed or
    allocated; the library's fixed device scratch (``CKDA_STATIC_SCRATCH_BYTES``)
    is used.  Calls that may run concurrently on one device race on that scratch."""
    dev = q.device
    B, T, H, dk, dv, N = _inputs_shape(q, k, v, alpha, beta, cu_seqlens)
    if S0 is not None:
        _need(S0, "S0", torch.float32, dev)
        if tuple(S0.shape) != (N, H, dk, dv):
            raise ValueError(f"S0 must be [{N}, {H}, {dk}, {dv}]")
    if out_dtype is None:
        out_dtype = out.dtype if out is not None else q.dtype
    if out_dtype not in _DT:
        raise TypeError("out_dtype must be float32 or bfloat16")
    if out is None:
        out = torch.empty(v.shape, dtype=out_dtype, device=dev)
    else:
        _need(out, "out", out_dtype, dev)
        if out.shape != v.shape:
            raise ValueError("out must have v's shape")
    if return_final and S_final is None:
        S_final = torch.empty((N, H, dk, dv), dtype=torch.float32, device=dev)
    if S_final is not None:
        _need(S_final, "S_final", torch.float32, dev)
    with torch.cuda.device(dev):
        rc = _lib.load().ckda_fwd_chunked_static(
            _p(q), _p(k), _p(v), _p(alpha), _p(beta), _p(S0), _p(cu_seqlens), _p(out),
            _p(S_final), B, T, H, dk, dv, chunk, _DT[q.dtype], _DT[out_dtype], _stream_ptr(dev))
    if rc != 0:
        raise CKDAError(rc, "ckda_fwd_chunked_static")
    return out, S_final


def _inputs_shape(q, k, v, alpha, beta, cu_seqlens, pair_gates=False):
    """Checks the forward inputs; returns (B, T, H, dk, dv, N) as passed to the ABI.
    ``pair_gates``: alpha holds one decay per channel pair (last dim dk / 2)."""
    dev = q.device
    if q.dtype not in _DT:
        raise TypeError("q, k, v must be float32 or bfloat16")
    for name, t in (("q", q), ("k", k), ("v", v)):
        _need(t, name, q.dtype, dev)
    _need(alpha, "alpha", torch.float32, dev)
    _need(beta, "beta", torch.float32, dev)
    if cu_seqlens is None:
        if q.dim() != 4:
            raise ValueError("q must be [B, T, H, dk]")
        B, T, H, dk = q.shape
        N = B
    else:
        _need(cu_seqlens, "cu_seqlens", torch.int32, dev)
        if q.dim() == 4:
            if q.shape[0] != 1:
                raise ValueError("packed inputs take a leading dimension of 1")
            T, H, dk = q.shape[1:]
        else:
            T, H, dk = q.shape
        N = cu_seqlens.numel() - 1
        B = N
    dv = v.shape[-1]
    a_shape = q.shape[:-1] + (dk // 2,) if pair_gates else q.shape
    if pair_gates and dk % 2:
        raise ValueError("the phase-decay gates pair the key channels: dk must be even")
    if k.shape != q.shape or alpha.shape != a_shape or v.shape[:-1] != q.shape[:-1]:
        raise ValueError("q, k, alpha must share a shape (alpha: last dim dk / 2 for paired "
                         "gates) and v must match it but for the last dim")
    if tuple(beta.shape) != tuple(q.shape[:-1]):
        raise ValueError("beta must have q's shape without the last dim")
    return B, T, H, dk, dv, N


def fwd_factors(q, k, v, alpha, beta, cu_seqlens=None, chunk: int = 64, workspace=None):
    """Phase 1 of the tensor-core forward: the S0-independent WY factors of every
    chunk, written to ``workspace`` (uint8 CUDA tensor; allocated if None).
    Returns the workspace, to be passed to ``fwd_carry`` with the same sizes."""
    B, T, H, dk, dv, N = _inputs_shape(q, k, v, alpha, beta, cu_seqlens)
    dev = q.device
    need = workspace_bytes(B, T, H, dk, dv, chunk, q.dtype, torch.float32, cu_seqlens is not None)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)
    _need(workspace, "workspace", torch.uint8, dev)
    with torch.cuda.device(dev):
        rc = _lib.load().ckda_fwd_factors(
            _p(q), _p(k), _p(v), _p(alpha), _p(beta), _p(cu_seqlens), B, T, H, dk, dv, chunk,
            _DT[q.dtype], _p(workspace), workspace.numel(), _stream_ptr(dev))
    if rc != 0:
        raise CKDAError(rc, "ckda_fwd_factors")
    return workspace


def fwd_carry(workspace, v, B, T, H, dk, dv, S0=None, cu_seqlens=None, chunk: int = 64,
              dtype=torch.bfloat16, out=None, S_final=None, out_dtype=torch.float32,
              return_final: bool = True):
    """Phase 2: apply the factors in ``workspace`` from ``S0``.  ``v`` is the value
    tensor of the ``fwd_factors`` call (the carry reads it); sizes (B, T, H as in
    ``ckda_fwd_chunked``) and ``dtype`` must be those of that call.
    Returns ``(out, S_final)``."""
    dev = workspace.device
    _need(workspace, "workspace", torch.uint8, dev)
    _need(v, "v", dtype, dev)
    N = B
    if out_dtype not in _DT:
        raise TypeError("out_dtype must be float32 or bfloat16")
    shape = (B, T, H, dv) if cu_seqlens is None else (T, H, dv)
    if out is None:
        out = torch.empty(shape, dtype=out_dtype, device=dev)
    else:
        _need(out, "out", out_dtype, dev)
        if out.numel() != math.prod(shape):
            raise ValueError(f"out must hold {shape}")
    if S0 is not None:
        _need(S0, "S0", torch.float32, dev)
        if tuple(S0.shape) != (N, H, dk, dv):
            raise ValueError(f"S0 must be [{N}, {H}, {dk}, {dv}]")
    if cu_seqlens is not None:
        _need(cu_seqlens, "cu_seqlens", torch.int32, dev)
    if return_final and S_final is None:
        S_final = torch.empty((N, H, dk, dv), dtype=torch.float32, device=dev)
    if S_final is not None:
        _need(S_final, "S_final", torch.float32, dev)
    with torch.cuda.device(dev):
        rc = _lib.load().ckda_fwd_carry(
            _p(v), _p(S0), _p(cu_seqlens), _p(out), _p(S_final), B, T, H, dk, dv, chunk, _DT[dtype],
            _DT[out_dtype], _p(workspace), workspace.numel(), _stream_ptr(dev))
    if rc != 0:
        raise CKDAError(rc, "ckda_fwd_carry")
    return out, S_final


def gdn2_fwd_chunked(q, k, v, alpha, b, w, S0=None, cu_seqlens=None, chunk: int = 64,
                     out=None, S_final=None, return_final: bool = True, out_dtype=None,
                     workspace=None):
    """Chunked Gated DeltaNet-2 forward (``ckda_gdn2_fwd_chunked``): CKDA with an
    erase gate ``b`` (fp32, shaped like ``k``) and a write gate ``w`` (fp32, shaped
    like ``v``) in place of beta.  Other arguments, the workspace and the result
    as in ``fwd_chunked``."""
    dev = q.device
    _need(b, "b", torch.float32, dev)
    _need(w, "w", torch.float32, dev)
    if b.shape != k.shape or w.shape != v.shape:
        raise ValueError("b must have k's shape and w v's shape")
    beta_like = b[..., 0]  # shape check only: [B, T, H] or [T, H]
    B, T, H, dk, dv, N = _inputs_shape(q, k, v, alpha, beta_like.contiguous(), cu_seqlens)
    if S0 is not None:
        _need(S0, "S0", torch.float32, dev)
        if tuple(S0.shape) != (N, H, dk, dv):
            raise ValueError(f"S0 must be [{N}, {H}, {dk}, {dv}]")
    if out_dtype is None:
        out_dtype = out.dtype if out is not None else q.dtype
    if out_dtype not in _DT:
        raise TypeError("out_dtype must be float32 or bfloat16")
    if out is None:
        out = torch.empty(v.shape, dtype=out_dtype, device=dev)
    else:
        _need(out, "out", out_dtype, dev)
        if out.shape != v.shape:
            raise ValueError("out must have v's shape")
    if return_final and S_final is None:
        S_final = torch.empty((N, H, dk, dv), dtype=torch.float32, device=dev)
    if S_final is not None:
        _need(S_final, "S_final", torch.float32, dev)
    need = workspace_bytes(B, T, H, dk, dv, chunk, q.dtype, out_dtype, cu_seqlens is not None)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    if workspace is not None:
        _need(workspace, "workspace", torch.uint8, dev)
    with torch.cuda.device(dev):
        rc = _lib.load().ckda_gdn2_fwd_chunked(
            _p(q), _p(k), _p(v), _p(alpha), _p(b), _p(w), _p(S0), _p(cu_seqlens), _p(out),
            _p(S_final), B, T, H, dk, dv, chunk, _DT[q.dtype], _DT[out_dtype], _p(workspace),
            0 if workspace is None else workspace.numel(), _stream_ptr(dev))
    if rc != 0:
        raise CKDAError(rc, "ckda_gdn2_fwd_chunked")
    return out, S_final


def sfda_fwd_chunked(q, k, v, alpha, theta, beta, S0=None, cu_seqlens=None, chunk: int = 64,
                     out=None, S_final=None, return_final: bool = True, out_dtype=None,
                     workspace=None, fp32core: bool = False):
    """Chunked SFDA forward (``ckda_sfda_fwd_chunked``): the CKDA recurrence with
    Diag(alpha) replaced by phase-decay blocks ``alpha_p R(theta_p)`` on the key
    channel pairs ``(2p, 2p+1)``.  ``alpha`` and ``theta`` are fp32 shaped like
    ``k`` with the last dim halved; beta, the workspace and the other arguments
    as in ``fwd_chunked`` (``fp32core`` forces the fp32 CUDA-core kernel)."""
    dev = q.device
    B, T, H, dk, dv, N = _inputs_shape(q, k, v, alpha, beta, cu_seqlens, pair_gates=True)
    _need(theta, "theta", torch.float32, dev)
    if theta.shape != alpha.shape:
        raise ValueError("theta must have alpha's shape")
    if S0 is not None:
        _need(S0, "S0", torch.float32, dev)
        if tuple(S0.shape) != (N, H, dk, dv):
            raise ValueError(f"S0 must be [{N}, {H}, {dk}, {dv}]")
    if out_dtype is None:
        out_dtype = out.dtype if out is not None else q.dtype
    if out_dtype not in _DT:
        raise TypeError("out_dtype must be float32 or bfloat16")
    if out is None:
        out = torch.empty(v.shape, dtype=out_dtype, device=dev)
    else:
        _need(out, "out", out_dtype, dev)
        if out.shape != v.shape:
            raise ValueError("out must have v's shape")
    if return_final and S_final is None:
        S_final = torch.empty((N, H, dk, dv), dtype=torch.float32, device=dev)
    if S_final is not None:
        _need(S_final, "S_final", torch.float32, dev)
    lib = _lib.load()
    if fp32core:
        with torch.cuda.device(dev):
            rc = lib.ckda_sfda_fwd_chunked_fp32core(
                _p(q), _p(k), _p(v), _p(alpha), _p(theta), _p(beta), _p(S0), _p(cu_seqlens),
                _p(out), _p(S_final), B, T, H, dk, dv, chunk, _DT[q.dtype], _DT[out_dtype],
                _stream_ptr(dev))
        if rc != 0:
            raise CKDAError(rc, "ckda_sfda_fwd_chunked_fp32core")
        return out, S_final
    need = workspace_bytes(B, T, H, dk, dv, chunk, q.dtype, out_dtype, cu_seqlens is not None)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    if workspace is not None:
        _need(workspace, "workspace", torch.uint8, dev)
    with torch.cuda.device(dev):
        rc = lib.ckda_sfda_fwd_chunked(
            _p(q), _p(k), _p(v), _p(alpha), _p(theta), _p(beta), _p(S0), _p(cu_seqlens),
            _p(out), _p(S_final), B, T, H, dk, dv, chunk, _DT[q.dtype], _DT[out_dtype],
            _p(workspace), 0 if workspace is None else workspace.numel(), _stream_ptr(dev))
    if rc != 0:
        raise CKDAError(rc, "ckda_sfda_fwd_chunked")
    return out, S_final


def scan_workspace_bytes(B, T, H, dk, dv, segments) -> int:
    """Scratch bytes ``fwd_chunked_scan`` needs for these sizes."""
    rc = _lib.load().ckda_fwd_chunked_scan_workspace_bytes(B, T, H, dk, dv, segments)
    if rc < 0:
        raise CKDAError(int(rc), "ckda_fwd_chunked_scan_workspace_bytes")
    return int(rc)


def fwd_chunked_scan(q, k, v, alpha, beta, segments: int, S0=None, chunk: int = 64, out=None,
                     S_final=None, return_final: bool = True, out_dtype=None, workspace=None):
    """``fwd_chunked`` for fixed-length batches as a chunk-parallel scan over
    ``segments`` segments of each sequence (``ckda_fwd_chunked_scan``): segment
    summaries [M | B] in parallel, a scan of the segment start states, then
    every segment's carry in parallel.  Same result up to rounding."""
    dev = q.device
    B, T, H, dk, dv, N = _inputs_shape(q, k, v, alpha, beta, None)
    if S0 is not None:
        _need(S0, "S0", torch.float32, dev)
        if tuple(S0.shape) != (N, H, dk, dv):
            raise ValueError(f"S0 must be [{N}, {H}, {dk}, {dv}]")
    if out_dtype is None:
        out_dtype = out.dtype if out is not None else q.dtype
    if out_dtype not in _DT:
        raise TypeError("out_dtype must be float32 or bfloat16")
    if out is None:
        out = torch.empty(v.shape, dtype=out_dtype, device=dev)
    else:
        _need(out, "out", out_dtype, dev)
        if out.shape != v.shape:
            raise ValueError("out must have v's shape")
    if return_final and S_final is None:
        S_final = torch.empty((N, H, dk, dv), dtype=torch.float32, device=dev)
    if S_final is not None:
        _need(S_final, "S_final", torch.float32, dev)
        if tuple(S_final.shape) != (N, H, dk, dv):
            raise ValueError(f"S_final must be [{N}, {H}, {dk}, {dv}]")
    if workspace is None:
        workspace = torch.empty(max(1, scan_workspace_bytes(B, T, H, dk, dv, segments)),
                                dtype=torch.uint8, device=dev)
    _need(workspace, "workspace", torch.uint8, dev)
    with torch.cuda.device(dev):
        rc = _lib.load().ckda_fwd_chunked_scan(
            _p(q), _p(k), _p(v), _p(alpha), _p(beta), _p(S0), _p(out), _p(S_final), B, T, H, dk,
            dv, chunk, _DT[q.dtype], _DT[out_dtype], segments, _p(workspace), workspace.numel(),
            _stream_ptr(dev))
    if rc != 0:
        raise CKDAError(rc, "ckda_fwd_chunked_scan")
    return out, S_final


def bwd_workspace_bytes(B, T, H, dk, dv, varlen=False) -> int:
    """Scratch bytes ``bwd_chunked`` needs for these sizes."""
    rc = _lib.load().ckda_bwd_chunked_workspace_bytes(B, T, H, dk, dv, 1 if varlen else 0)
    if rc < 0:
        raise CKDAError(int(rc), "ckda_bwd_chunked_workspace_bytes")
    return int(rc)


def bwd_chunked(q, k, v, alpha, beta, dO, S0=None, dS_final=None, cu_seqlens=None,
                grads=None, want_dS0: bool = True, workspace=None):
    """Backward of ``fwd_chunked`` (``ckda_bwd_chunked``): the gradients of a scalar
    loss with respect to q, k, v, alpha, beta and S0, given ``dO`` (dL/dout, fp32 or
    bf16, shaped like v) and ``dS_final`` (dL/dS_final, fp32, or None = 0).

    Returns a dict of fp32 tensors ``dq, dk, dv, dalpha, dbeta`` (shaped like the
    inputs) and ``dS0`` (``[N, H, dk, dv]``, or None when ``want_dS0`` is false).
    ``grads`` may supply preallocated output tensors under the same names."""
    dev = q.device
    B, T, H, dk, dv, N = _inputs_shape(q, k, v, alpha, beta, cu_seqlens)
    if dO.dtype not in _DT:
        raise TypeError("dO must be float32 or bfloat16")
    _need(dO, "dO", dO.dtype, dev)
    if dO.shape != v.shape:
        raise ValueError("dO must have v's shape")
    if S0 is not None:
        _need(S0, "S0", torch.float32, dev)
        if tuple(S0.shape) != (N, H, dk, dv):
            raise ValueError(f"S0 must be [{N}, {H}, {dk}, {dv}]")
    if dS_final is not None:
        _need(dS_final, "dS_final", torch.float32, dev)
        if tuple(dS_final.shape) != (N, H, dk, dv):
            raise ValueError(f"dS_final must be [{N}, {H}, {dk}, {dv}]")
    want = {"dq": q.shape, "dk": k.shape, "dv": v.shape, "dalpha": alpha.shape,
            "dbeta": beta.shape}
    if want_dS0:
        want["dS0"] = (N, H, dk, dv)
    g = dict(grads or {})
    for name, shp in want.items():
        if g.get(name) is None:
            g[name] = torch.empty(shp, dtype=torch.float32, device=dev)
        _need(g[name], name, torch.float32, dev)
        if tuple(g[name].shape) != tuple(shp):
            raise ValueError(f"{name} must be {tuple(shp)}")
    if not want_dS0:
        g["dS0"] = None
    need = bwd_workspace_bytes(B, T, H, dk, dv, cu_seqlens is not None)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    if workspace is not None:
        _need(workspace, "workspace", torch.uint8, dev)
    with torch.cuda.device(dev):
        rc = _lib.load().ckda_bwd_chunked(
            _p(q), _p(k), _p(v), _p(alpha), _p(beta), _p(S0), _p(cu_seqlens), _p(dO),
            _p(dS_final), _p(g["dq"]), _p(g["dk"]), _p(g["dv"]), _p(g["dalpha"]),
            _p(g["dbeta"]), _p(g["dS0"]), B, T, H, dk, dv, _DT[q.dtype], _DT[dO.dtype],
            _p(workspace), 0 if workspace is None else workspace.numel(), _stream_ptr(dev))
    if rc != 0:
        raise CKDAError(rc, "ckda_bwd_chunked")
    return g


def workspace_bytes(B, T, H, dk, dv, chunk=64, dtype=torch.bfloat16, out_dtype=torch.float32,
                    varlen=False) -> int:
    """Scratch bytes ``fwd_chunked`` needs for these sizes (0 on the fp32 CUDA-core path)."""
    rc = _lib.load().ckda_fwd_chunked_workspace_bytes(B, T, H, dk, dv, chunk, _DT[dtype],
                                                      _DT[out_dtype], 1 if varlen else 0)
    if rc < 0:
        raise CKDAError(int(rc), "ckda_fwd_chunked_workspace_bytes")
    return int(rc)


def fwd_path(B, T, H, dk, dv, chunk=64, dtype=torch.bfloat16, out_dtype=torch.float32,
             varlen=False) -> str:
    """Which kernel ``fwd_chunked`` runs for these sizes: "tcgen05" or "fp32core"."""
    rc = _lib.load().ckda_fwd_chunked_path(B, T, H, dk, dv, chunk, _DT[dtype], _DT[out_dtype],
                                           1 if varlen else 0)
    if rc < 0:
        raise CKDAError(rc, "ckda_fwd_chunked_path")
    return "tcgen05" if rc == 1 else "fp32core"


def _decode_out(q, v, out, out_dtype, dev):
    if out_dtype is None:
        out_dtype = out.dtype if out is not None else q.dtype
    if out_dtype not in _DT:
        raise TypeError("out_dtype must be float32 or bfloat16")
    B, H, _ = q.shape
    if out is None:
        out = torch.empty((B, H, v.shape[-1]), dtype=out_dtype, device=dev)
    else:
        _need(out, "out", out_dtype, dev)
    return out, out_dtype


def _decode_checks(q, k, v, S, gates):
    dev = q.device
    if q.dtype not in _DT:
        raise TypeError("q, k, v must be float32 or bfloat16")
    for name, t in (("q", q), ("k", k), ("v", v)):
        _need(t, name, q.dtype, dev)
    _need(S, "S", torch.float32, dev)
    B, H, dk = q.shape
    dv = v.shape[-1]
    if tuple(S.shape) != (B, H, dk, dv) or k.shape != q.shape or tuple(v.shape[:2]) != (B, H):
        raise ValueError("shape mismatch")
    for name, t, shape in gates:
        _need(t, name, torch.float32, dev)
        if tuple(t.shape) != tuple(shape):
            raise ValueError(f"{name} must be {tuple(shape)}")
    return dev, B, H, dk, dv


def decode_step(q, k, v, alpha, beta, S, out=None, out_dtype=None) -> torch.Tensor:
    """One recurrent step, in place on ``S`` ``[B, H, dk, dv]`` (fp32).

    q, k, alpha ``[B, H, dk]``; v ``[B, H, dv]``; beta ``[B, H]``.  Returns ``out``
    (``out_dtype`` defaults to the dtype of ``out`` if given, else the input dtype).
    """
    B, H, dk = q.shape
    dev, B, H, dk, dv = _decode_checks(q, k, v, S, (("alpha", alpha, (B, H, dk)),
                                                    ("beta", beta, (B, H))))
    out, out_dtype = _decode_out(q, v, out, out_dtype, dev)
    with torch.cuda.device(dev):
        rc = _lib.load().ckda_decode_step(_p(q), _p(k), _p(v), _p(alpha), _p(beta), _p(S), _p(out),
                                          B, H, dk, dv, _DT[q.dtype], _DT[out_dtype],
                                          _stream_ptr(dev))
    if rc != 0:
        raise CKDAError(rc, "ckda_decode_step")
    return out


def gdn2_decode_step(q, k, v, alpha, b, w, S, out=None, out_dtype=None) -> torch.Tensor:
    """One Gated DeltaNet-2 step in place on ``S`` (``ckda_gdn2_decode_step``):
    erase gate ``b`` ``[B, H, dk]`` and write gate ``w`` ``[B, H, dv]`` (fp32) in
    place of beta; otherwise as ``decode_step``."""
    B, H, dk = q.shape
    dv = v.shape[-1]
    dev, B, H, dk, dv = _decode_checks(q, k, v, S, (("alpha", alpha, (B, H, dk)),
                                                    ("b", b, (B, H, dk)), ("w", w, (B, H, dv))))
    out, out_dtype = _decode_out(q, v, out, out_dtype, dev)
    with torch.cuda.device(dev):
        rc = _lib.load().ckda_gdn2_decode_step(_p(q), _p(k), _p(v), _p(alpha), _p(b), _p(w),
                                               _p(S), _p(out), B, H, dk, dv, _DT[q.dtype],
                                               _DT[out_dtype], _stream_ptr(dev))
    if rc != 0:
        raise CKDAError(rc, "ckda_gdn2_decode_step")
    return out


def sfda_decode_step(q, k, v, alpha, theta, beta, S, out=None, out_dtype=None) -> torch.Tensor:
    """One SFDA step in place on ``S`` (``ckda_sfda_decode_step``): decays
    ``alpha`` and phases ``theta`` ``[B, H, dk / 2]`` (fp32) per channel pair,
    ``beta`` ``[B, H]``; otherwise as ``decode_step``."""
    B, H, dk = q.shape
    dev, B, H, dk, dv = _decode_checks(q, k, v, S, (("alpha", alpha, (B, H, dk // 2)),
                                                    ("theta", theta, (B, H, dk // 2)),
                                                    ("beta", beta, (B, H))))
    out, out_dtype = _decode_out(q, v, out, out_dtype, dev)
    with torch.cuda.device(dev):
        rc = _lib.load().ckda_sfda_decode_step(_p(q), _p(k), _p(v), _p(alpha), _p(theta),
                                               _p(beta), _p(S), _p(out), B, H, dk, dv,
                                               _DT[q.dtype], _DT[out_dtype], _stream_ptr(dev))
    if rc != 0:
        raise CKDAError(rc, "ckda_sfda_decode_step")
    return out


def device_status(device=None) -> int:
    """Synchronise the current stream and return (and clear) the device status word."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    with torch.cuda.device(dev):
        return _lib.load().ckda_device_status(_stream_ptr(dev))
