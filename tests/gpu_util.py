"""Helpers shared by the GPU parity tests (no method arithmetic here)."""
from __future__ import annotations

import numpy as np
import torch

import oracle

TOL_F32 = 1e-4   # max|o - o_ref| / rms(o_ref) for fp32-input workloads
TOL_BF16 = 2e-2  # the same metric for bf16-input workloads


def rel_max_err(got, ref) -> float:
    """max|got - ref| / rms(ref) over the whole tensor (fp64)."""
    g = got.detach().cpu().double().numpy() if hasattr(got, "detach") else np.asarray(got, np.float64)
    r = np.asarray(ref, dtype=np.float64)
    rms = float(np.sqrt(np.mean(r * r)))
    if rms == 0.0:
        return float(np.max(np.abs(g - r))) if g.size else 0.0
    return float(np.max(np.abs(g - r))) / rms


def oracle_fixed(case, b_idx=None, h_idx=None):
    """fp64 oracle on a subset of (batch, head) units of a fixed-length case."""
    B, T, H, dk = case.q.shape
    b_idx = list(range(B)) if b_idx is None else list(b_idx)
    h_idx = list(range(H)) if h_idx is None else list(h_idx)
    bi = torch.tensor(b_idx)
    hi = torch.tensor(h_idx)

    def sel(x):
        return x.detach().cpu()[bi][:, :, hi]

    S0 = None
    if case.S0 is not None:
        S0 = case.S0.detach().cpu()[bi][:, hi]
    out, S = oracle.forward(sel(case.q), sel(case.k), sel(case.v), sel(case.alpha),
                            sel(case.beta), S0=S0)
    return out, S, bi, hi


def oracle_packed(case, seq_idx=None, h_idx=None):
    """fp64 oracle on a subset of (sequence, head) units of a packed case.

    Returns (out [tokens_of_selected_seqs, H', dv], S [N', H', dk, dv], token_index, h_index).
    """
    cu = case.cu_seqlens.detach().cpu().to(torch.int64)
    N = cu.numel() - 1
    seq_idx = list(range(N)) if seq_idx is None else list(seq_idx)
    h_idx = list(range(case.H)) if h_idx is None else list(h_idx)
    tok = torch.cat([torch.arange(int(cu[n]), int(cu[n + 1])) for n in seq_idx]) if seq_idx else \
        torch.zeros(0, dtype=torch.int64)
    lens = torch.tensor([int(cu[n + 1] - cu[n]) for n in seq_idx], dtype=torch.int64)
    cu_sub = np.concatenate([[0], np.cumsum(lens.numpy())]).astype(np.int64)
    hi = torch.tensor(h_idx)

    def sel(x):
        return x.detach().cpu()[0][tok][:, hi]

    S0 = None
    if case.S0 is not None:
        S0 = case.S0.detach().cpu()[torch.tensor(seq_idx)][:, hi]
    out, S = oracle.forward(sel(case.q), sel(case.k), sel(case.v), sel(case.alpha),
                            sel(case.beta), S0=S0, cu_seqlens=cu_sub)
    return out, S, tok, hi
