"""Seeded synthetic inputs for the CKDA workloads.

This module only draws random numbers; it holds none of the recurrence's
arithmetic, and both the CUDA path's tests and the fp64 oracle consume the
tensors it returns (the oracle through exact fp64 upcasts of host copies).

Workloads (all synthetic; the pages publish no dataset for this path):

* ``tiny``      B=1, H=2, T=64, d=16, C=16, fp32.  q, k ~ N(0,1) then
                L2-normalised per token; v ~ N(0,1); alpha ~ U[-1,1] per
                channel; beta ~ U[0,2]; zero initial state.
* ``kda_prefill`` B=4, H=16, T=4096, d=128, C=64; q, k, v bf16 (q, k
                normalised in fp32, then cast); alpha = s * exp(-softplus(x))
                = s * sigmoid(-x), x ~ N(0,1), s = -1 with probability 0.25;
                beta = 2 * sigmoid(N(0,1)); alpha and beta fp32; zero state.
* ``long_prefill`` B=1, H=32, T=65536, d=128, C=64, gates as kda_prefill,
                S0 ~ N(0, 0.02^2).
* ``decode``    B=256, H=32, d=128, S0 ~ N(0, 0.02^2), 1024 steps of bf16
                q, k, v (q, k normalised), alpha ~ U[-1,1], beta ~ U[0,2].
* ``varlen``    64 packed sequences, lengths ~ U[128, 4096], H=16, d=128,
                fp32; in each sequence the first floor(L/2) tokens use
                near-zero gates (alpha ~ U[-0.05, 0.05], beta ~ U[0,2],
                v ~ N(0,1)) and the rest are orthogonal transitions
                (alpha_i = +-1 uniformly, beta = 2, v = 0).

Draw order is fixed (lengths, q, k, v, gate logits, signs, beta logits, S0),
so a (workload, seed, device) triple always gives the same tensors.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Optional

import math

import torch

F32 = torch.float32
BF16 = torch.bfloat16


@dataclass
class PrefillCase:
    name: str
    q: torch.Tensor          # [B, T, H, dk]  (packed: [1, T_total, H, dk])
    k: torch.Tensor
    v: torch.Tensor          # [B, T, H, dv]
    alpha: torch.Tensor      # [B, T, H, dk] fp32
    beta: torch.Tensor       # [B, T, H]     fp32
    S0: Optional[torch.Tensor]          # [N, H, dk, dv] fp32 or None
    cu_seqlens: Optional[torch.Tensor]  # int32 [N + 1] or None
    chunk: int
    extra: dict = field(default_factory=dict)

    @property
    def n_seqs(self) -> int:
        return self.q.shape[0] if self.cu_seqlens is None else self.cu_seqlens.numel() - 1

    @property
    def tokens(self) -> int:
        return self.q.shape[0] * self.q.shape[1]

    @property
    def H(self) -> int:
        return self.q.shape[2]

    @property
    def dk(self) -> int:
        return self.q.shape[3]

    @property
    def dv(self) -> int:
        return self.v.shape[3]


@dataclass
class DecodeCase:
    name: str
    S0: torch.Tensor     # [B, H, dk, dv] fp32
    q: torch.Tensor      # [steps, B, H, dk]
    k: torch.Tensor
    v: torch.Tensor      # [steps, B, H, dv]
    alpha: torch.Tensor  # [steps, B, H, dk] fp32
    beta: torch.Tensor   # [steps, B, H] fp32


def _gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _normal(shape, g, device):
    return torch.randn(shape, generator=g, device=device, dtype=F32)


def _uniform(shape, lo, hi, g, device):
    return torch.rand(shape, generator=g, device=device, dtype=F32) * (hi - lo) + lo


def _l2n(x: torch.Tensor) -> torch.Tensor:
    """L2-normalise along the last dimension in fp32 (workload recipe)."""
    return x / x.norm(dim=-1, keepdim=True).clamp_min(1e-12)


def _kda_gates(shape_k, shape_b, g, device):
    """alpha = s * sigmoid(-x), P(s = -1) = 0.25; beta = 2 * sigmoid(z)."""
    x = _normal(shape_k, g, device)
    sgn = torch.where(torch.rand(shape_k, generator=g, device=device) < 0.25, -1.0, 1.0)
    alpha = (sgn * torch.sigmoid(-x)).to(F32)
    beta = (2.0 * torch.sigmoid(_normal(shape_b, g, device))).to(F32)
    return alpha, beta


def random_prefill(B, T, H, dk, dv, *, dtype=F32, gates="uniform", s0_std=0.0,
                   chunk=64, seed=0, device="cpu", name="random") -> PrefillCase:
    """Fixed-length batch with q, k normalised, v ~ N(0,1).

    gates="uniform": alpha ~ U[-1,1], beta ~ U[0,2]  (tiny / decode recipe)
    gates="kda":     alpha = s*sigmoid(-x), beta = 2*sigmoid(z) (prefill recipe)
    """
    g = _gen(device, seed)
    q = _l2n(_normal((B, T, H, dk), g, device)).to(dtype)
    k = _l2n(_normal((B, T, H, dk), g, device)).to(dtype)
    v = _normal((B, T, H, dv), g, device).to(dtype)
    if gates == "kda":
        alpha, beta = _kda_gates((B, T, H, dk), (B, T, H), g, device)
    elif gates == "uniform":
        alpha = _uniform((B, T, H, dk), -1.0, 1.0, g, device)
        beta = _uniform((B, T, H), 0.0, 2.0, g, device)
    else:
        raise ValueError(gates)
    S0 = None
    if s0_std > 0:
        S0 = (_normal((B, H, dk, dv), g, device) * s0_std).contiguous()
    return PrefillCase(name, q, k, v, alpha.contiguous(), beta.contiguous(), S0, None, chunk)


def gdn2_prefill(B, T, H, dk, dv, *, dtype=F32, s0_std=0.0, chunk=64, seed=0, device="cpu",
                 name="gdn2") -> PrefillCase:
    """Gated DeltaNet-2 batch: q, k normalised, v ~ N(0,1), alpha as the KDA
    prefill recipe, erase gate b = sigmoid(x) per key channel and write gate
    w = sigmoid(y) per value channel (both in [0, 1]), x, y ~ N(0,1).  The
    gates go to ``extra["b"]`` and ``extra["w"]``; ``beta`` is unused (None)."""
    g = _gen(device, seed)
    q = _l2n(_normal((B, T, H, dk), g, device)).to(dtype)
    k = _l2n(_normal((B, T, H, dk), g, device)).to(dtype)
    v = _normal((B, T, H, dv), g, device).to(dtype)
    alpha, _ = _kda_gates((B, T, H, dk), (B, T, H), g, device)
    b = torch.sigmoid(_normal((B, T, H, dk), g, device)).to(F32).contiguous()
    w = torch.sigmoid(_normal((B, T, H, dv), g, device)).to(F32).contiguous()
    S0 = None
    if s0_std > 0:
        S0 = (_normal((B, H, dk, dv), g, device) * s0_std).contiguous()
    case = PrefillCase(name, q, k, v, alpha.contiguous(), None, S0, None, chunk)
    case.extra["b"] = b
    case.extra["w"] = w
    return case


def sfda_prefill(B, T, H, dk, dv, *, dtype=F32, s0_std=0.0, chunk=64, seed=0, device="cpu",
                 name="sfda") -> PrefillCase:
    """SFDA batch: q, k normalised, v ~ N(0,1), beta = 2 sigmoid(z) as the KDA
    prefill recipe; per channel pair a decay alpha = sigmoid(-x) in (0, 1) and
    a phase theta ~ U[-pi, pi) (the phase carries the sign), x, z ~ N(0,1).
    ``alpha`` is [B, T, H, dk / 2]; the phases go to ``extra["theta"]``."""
    g = _gen(device, seed)
    q = _l2n(_normal((B, T, H, dk), g, device)).to(dtype)
    k = _l2n(_normal((B, T, H, dk), g, device)).to(dtype)
    v = _normal((B, T, H, dv), g, device).to(dtype)
    alpha = torch.sigmoid(-_normal((B, T, H, dk // 2), g, device)).to(F32).contiguous()
    theta = _uniform((B, T, H, dk // 2), -math.pi, math.pi, g, device).contiguous()
    beta = (2.0 * torch.sigmoid(_normal((B, T, H), g, device))).to(F32).contiguous()
    S0 = None
    if s0_std > 0:
        S0 = (_normal((B, H, dk, dv), g, device) * s0_std).contiguous()
    case = PrefillCase(name, q, k, v, alpha, beta, S0, None, chunk)
    case.extra["theta"] = theta
    return case


def tiny(seed=0, device="cpu") -> PrefillCase:
    return random_prefill(1, 64, 2, 16, 16, dtype=F32, gates="uniform", chunk=16,
                          seed=seed, device=device, name="tiny B=1 H=2 T=64 d=16 C=16 fp32")


def kda_prefill(seed=0, device="cpu", B=4, T=4096, H=16, d=128) -> PrefillCase:
    return random_prefill(B, T, H, d, d, dtype=BF16, gates="kda", chunk=64, seed=seed,
                          device=device, name=f"kda_prefill B={B} H={H} T={T} d={d} C=64 bf16")


def long_prefill(seed=0, device="cpu", T=65536, H=32, d=128) -> PrefillCase:
    return random_prefill(1, T, H, d, d, dtype=BF16, gates="kda", s0_std=0.02, chunk=64,
                          seed=seed, device=device,
                          name=f"long_prefill B=1 H={H} T={T} d={d} C=64 bf16")


def decode(seed=0, device="cpu", B=256, H=32, d=128, steps=1024) -> DecodeCase:
    g = _gen(device, seed)
    q = _l2n(_normal((steps, B, H, d), g, device)).to(BF16)
    k = _l2n(_normal((steps, B, H, d), g, device)).to(BF16)
    v = _normal((steps, B, H, d), g, device).to(BF16)
    alpha = _uniform((steps, B, H, d), -1.0, 1.0, g, device)
    beta = _uniform((steps, B, H), 0.0, 2.0, g, device)
    S0 = (_normal((B, H, d, d), g, device) * 0.02).contiguous()
    return DecodeCase(f"decode B={B} H={H} d={d} steps={steps} bf16", S0, q, k, v, alpha, beta)


def varlen(seed=0, device="cpu", n_seqs=64, lmin=128, lmax=4096, H=16, d=128,
           dtype=F32, chunk=64) -> PrefillCase:
    """Gate-extreme packed batch: near-zero gates, then orthogonal transitions."""
    g = _gen(device, seed)
    lens = torch.randint(lmin, lmax + 1, (n_seqs,), generator=g, device=device)
    lens_cpu = lens.cpu().to(torch.int64)
    cu = torch.zeros(n_seqs + 1, dtype=torch.int64)
    cu[1:] = torch.cumsum(lens_cpu, 0)
    Tt = int(cu[-1])
    q = _l2n(_normal((1, Tt, H, d), g, device)).to(dtype)
    k = _l2n(_normal((1, Tt, H, d), g, device)).to(dtype)
    v_draw = _normal((1, Tt, H, d), g, device)
    a_small = _uniform((1, Tt, H, d), -0.05, 0.05, g, device)
    a_sign = torch.where(torch.rand((1, Tt, H, d), generator=g, device=device) < 0.5, -1.0, 1.0)
    b_draw = _uniform((1, Tt, H), 0.0, 2.0, g, device)
    # position of each token inside its own sequence
    seq_id = torch.repeat_interleave(torch.arange(n_seqs), lens_cpu)
    pos = torch.arange(Tt) - cu[:-1][seq_id]
    first_half = (pos < (lens_cpu[seq_id] // 2)).to(device)
    fh = first_half.view(1, Tt, 1)
    alpha = torch.where(fh.unsqueeze(-1), a_small, a_sign).to(F32).contiguous()
    beta = torch.where(fh, b_draw, torch.full_like(b_draw, 2.0)).to(F32).contiguous()
    v = torch.where(fh.unsqueeze(-1), v_draw, torch.zeros_like(v_draw)).to(dtype).contiguous()
    case = PrefillCase(f"varlen N={n_seqs} L~U[{lmin},{lmax}] H={H} d={d} C={chunk} "
                       f"{'fp32' if dtype == F32 else 'bf16'}",
                       q.contiguous(), k.contiguous(), v, alpha, beta, None,
                       cu.to(torch.int32).to(device), chunk)
    case.extra["lengths"] = lens_cpu
    return case


def first_halves(case: PrefillCase) -> PrefillCase:
    """The same packed batch cut to the first floor(L/2) tokens of each sequence
    (the near-zero-gate part of the ``varlen`` workload)."""
    lens = case.extra["lengths"]
    cu = torch.zeros(lens.numel() + 1, dtype=torch.int64)
    cu[1:] = torch.cumsum(lens, 0)
    halves = lens // 2
    idx = torch.cat([torch.arange(int(cu[i]), int(cu[i]) + int(halves[i])) for i in range(lens.numel())])
    idx = idx.to(case.q.device)
    cu_h = torch.zeros(lens.numel() + 1, dtype=torch.int64)
    cu_h[1:] = torch.cumsum(halves, 0)
    sub = PrefillCase(case.name + " (first halves)",
                      case.q[:, idx].contiguous(), case.k[:, idx].contiguous(),
                      case.v[:, idx].contiguous(), case.alpha[:, idx].contiguous(),
                      case.beta[:, idx].contiguous(), None,
                      cu_h.to(torch.int32).to(case.q.device), case.chunk)
    sub.extra["lengths"] = halves
    return sub


def gate_extremes(B, T, H, d, *, kind, dtype=BF16, s0_std=0.0, chunk=64, seed=0,
                  device="cpu") -> PrefillCase:
    """Fixed-length batch whose gates sit at the ends of the CKDA ranges
    (alpha in [-1, 1], beta in [0, 2]); q, k ~ N(0,1) normalised, v ~ N(0,1).

    kind="zero":       alpha = 0 everywhere, beta ~ U[0, 2]
    kind="orthogonal": alpha_i = +-1 uniformly, beta = 2, v = 0
    kind="reflect":    alpha_i = +-1 uniformly, beta = 2, v ~ N(0,1)
    kind="uniform":    alpha ~ U[-1, 1], beta ~ U[0, 2]
    kind="tiny":       alpha ~ U[-0.05, 0.05], beta ~ U[0, 2]
    kind="underflow":  per (token, head) with probability 0.15 alpha ~ U[-1e-3, 1e-3]
                       per channel, else alpha = +-U[0.9, 1]; beta ~ U[0, 2]
    kind="halves":     the first floor(T/2) tokens as "tiny", the rest as "orthogonal"

    Draw order: q, k, v, a uniform tensor, a sign tensor, a selector, beta, S0.
    """
    g = _gen(device, seed)
    q = _l2n(_normal((B, T, H, d), g, device)).to(dtype)
    k = _l2n(_normal((B, T, H, d), g, device)).to(dtype)
    v = _normal((B, T, H, d), g, device)
    u = _uniform((B, T, H, d), 0.0, 1.0, g, device)
    sgn = torch.where(torch.rand((B, T, H, d), generator=g, device=device) < 0.5, -1.0, 1.0)
    sel = torch.rand((B, T, H, 1), generator=g, device=device)
    bu = _uniform((B, T, H), 0.0, 2.0, g, device)
    two = torch.full_like(bu, 2.0)
    if kind == "zero":
        alpha, beta = torch.zeros_like(u), bu
    elif kind in ("orthogonal", "reflect"):
        alpha, beta = sgn, two
        if kind == "orthogonal":
            v = torch.zeros_like(v)
    elif kind == "uniform":
        alpha, beta = 2.0 * u - 1.0, bu
    elif kind == "tiny":
        alpha, beta = 0.1 * u - 0.05, bu
    elif kind == "underflow":
        alpha = torch.where(sel < 0.15, 2e-3 * u - 1e-3, sgn * (0.9 + 0.1 * u))
        beta = bu
    elif kind == "halves":
        first = (torch.arange(T, device=device) < T // 2).view(1, T, 1)
        alpha = torch.where(first.unsqueeze(-1), 0.1 * u - 0.05, sgn)
        beta = torch.where(first, bu, two)
        v = torch.where(first.unsqueeze(-1), v, torch.zeros_like(v))
    else:
        raise ValueError(kind)
    S0 = None
    if s0_std > 0:
        S0 = (_normal((B, H, d, d), g, device) * s0_std).contiguous()
    return PrefillCase(f"gate_extremes[{kind}] B={B} T={T} H={H} d={d} C={chunk}",
                       q.contiguous(), k.contiguous(), v.to(dtype).contiguous(),
                       alpha.to(F32).contiguous(), beta.to(F32).contiguous(), S0, None, chunk)
