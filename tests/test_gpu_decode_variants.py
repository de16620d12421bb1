"""Decode steps of the two gate variants on the GPU against the fp64 oracle
(needs a B200).

``ckda_gdn2_decode_step`` (erase gate b, write gate w: "Gated DeltaNet-2"
summary, Methodology section 1) and ``ckda_sfda_decode_step`` (phase-decay
gates on channel pairs: "Semidirect Fourier Delta Attention (SFDA)" summary,
"Arquitectura Central") run one token per (sequence, head) in place on the
state.  They are compared step by step with the pinned fp64 oracles
(``forward_gdn2`` / ``forward_sfda`` on one token per sequence), with their
reductions to the CKDA step (b = w = beta; theta = 0), and with the chunked
forward over the same tokens; at the decode workload's size on sampled
(sequence, head) units.
"""
import math

import pytest
import torch

import oracle
from gpu_util import TOL_BF16, TOL_F32, rel_max_err

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module")
def ck():
    import delta_rule_linear_ckda_b200 as ck

    return ck


def _inputs(B, H, dk, dv, steps, dtype, seed, kind):
    g = torch.Generator(device=DEV).manual_seed(seed)
    n = lambda *s: torch.randn(*s, generator=g, device=DEV)  # noqa: E731
    u = lambda *s: torch.rand(*s, generator=g, device=DEV)   # noqa: E731
    q = torch.nn.functional.normalize(n(steps, B, H, dk), dim=-1).to(dtype)
    k = torch.nn.functional.normalize(n(steps, B, H, dk), dim=-1).to(dtype)
    v = n(steps, B, H, dv).to(dtype)
    S0 = 0.3 * n(B, H, dk, dv)
    if kind == "gdn2":
        gates = (2 * u(steps, B, H, dk) - 1, u(steps, B, H, dk), u(steps, B, H, dv))
    else:
        gates = (u(steps, B, H, dk // 2), (2 * u(steps, B, H, dk // 2) - 1) * math.pi,
                 2 * u(steps, B, H))
    return q, k, v, gates, S0


def _run(ck, kind, q, k, v, gates, S, t):
    # fresh copies: a step's slice of a [steps, B, H] tensor need not be 16-byte aligned
    g = [x[t].clone() for x in gates]
    if kind == "gdn2":
        return ck.gdn2_decode_step(q[t].clone(), k[t].clone(), v[t].clone(), g[0], g[1], g[2], S,
                                   out_dtype=torch.float32)
    return ck.sfda_decode_step(q[t].clone(), k[t].clone(), v[t].clone(), g[0], g[1], g[2], S,
                               out_dtype=torch.float32)


def _ref(kind, q, k, v, gates, S, t):
    f = oracle.decode_step_gdn2 if kind == "gdn2" else oracle.decode_step_sfda
    return f(q[t], k[t], v[t], gates[0][t], gates[1][t], gates[2][t], S)


@pytest.mark.parametrize("kind", ["gdn2", "sfda"])
@pytest.mark.parametrize("dk,dv", [(16, 16), (32, 64), (64, 32), (128, 128), (16, 128)])
def test_fp32_steps_match_oracle(ck, kind, dk, dv):
    q, k, v, gates, S0 = _inputs(3, 2, dk, dv, 6, torch.float32, dk + dv, kind)
    S = S0.clone()
    Sref = S0.cpu().double().numpy()
    for t in range(6):
        o = _run(ck, kind, q, k, v, gates, S, t)
        ro, Sref = _ref(kind, q, k, v, gates, Sref, t)
        assert ck.device_status() == 0
        assert rel_max_err(o, ro) <= TOL_F32, t
    assert rel_max_err(S, Sref) <= TOL_F32


@pytest.mark.parametrize("kind", ["gdn2", "sfda"])
def test_bf16_steps_match_oracle(ck, kind):
    q, k, v, gates, S0 = _inputs(8, 4, 128, 128, 8, torch.bfloat16, 7, kind)
    S = S0.clone()
    Sref = S0.cpu().double().numpy()
    for t in range(8):
        o = _run(ck, kind, q, k, v, gates, S, t)
        ro, Sref = _ref(kind, q, k, v, gates, Sref, t)
        assert rel_max_err(o, ro) <= TOL_BF16, t
    assert ck.device_status() == 0
    assert rel_max_err(S, Sref) <= TOL_BF16


def test_reductions_to_the_ckda_step(ck):
    q, k, v, gates, S0 = _inputs(4, 2, 64, 64, 1, torch.float32, 11, "sfda")
    a_pair, _, beta = gates
    a_full = a_pair[0].repeat_interleave(2, dim=-1).contiguous()
    S1, S2, S3 = S0.clone(), S0.clone(), S0.clone()
    b0 = beta[0].clone()
    o1 = ck.decode_step(q[0], k[0], v[0], a_full, b0, S1, out_dtype=torch.float32)
    o2 = ck.sfda_decode_step(q[0], k[0], v[0], a_pair[0].contiguous(),
                             torch.zeros_like(a_pair[0]), b0, S2, out_dtype=torch.float32)
    bb = beta[0][..., None].expand(4, 2, 64).contiguous()
    o3 = ck.gdn2_decode_step(q[0], k[0], v[0], a_full, bb, bb, S3, out_dtype=torch.float32)
    assert ck.device_status() == 0
    ref = o1.double().cpu().numpy()
    assert rel_max_err(o2, ref) <= 1e-5 and rel_max_err(o3, ref) <= 1e-5
    assert rel_max_err(S2, S1.double().cpu().numpy()) <= 1e-5
    assert rel_max_err(S3, S1.double().cpu().numpy()) <= 1e-5


@pytest.mark.parametrize("kind", ["gdn2", "sfda"])
def test_steps_equal_the_chunked_forward(ck, kind):
    """Eight decode steps give what the chunked forward gives over the same
    eight tokens (fp32 kernel)."""
    T, B, H, d = 8, 2, 2, 64
    q, k, v, gates, S0 = _inputs(B, H, d, d, T, torch.float32, 21, kind)
    S = S0.clone()
    outs = [_run(ck, kind, q, k, v, gates, S, t) for t in range(T)]
    o_dec = torch.stack(outs, dim=1)  # [B, T, H, d]
    seq = lambda x: x.transpose(0, 1).contiguous()  # noqa: E731  [T, B, ...] -> [B, T, ...]
    if kind == "gdn2":
        o_fwd, S_fwd = ck.gdn2_fwd_chunked(seq(q), seq(k), seq(v), seq(gates[0]), seq(gates[1]),
                                           seq(gates[2]), S0=S0, chunk=16, out_dtype=torch.float32)
    else:
        o_fwd, S_fwd = ck.sfda_fwd_chunked(seq(q), seq(k), seq(v), seq(gates[0]), seq(gates[1]),
                                           seq(gates[2]), S0=S0, chunk=16, out_dtype=torch.float32)
    assert ck.device_status() == 0
    assert rel_max_err(o_dec, o_fwd.double().cpu().numpy()) <= 1e-5
    assert rel_max_err(S, S_fwd.double().cpu().numpy()) <= 1e-5


@pytest.mark.parametrize("kind", ["gdn2", "sfda"])
def test_bench_size_steps_sampled(ck, kind):
    """The decode workload's size (B=256, H=32, d=128, bf16 q/k/v, fp32 out):
    64 steps of every head, checked on sampled (sequence, head) units against
    the oracle run over the same 64 tokens."""
    steps, B, H, d = 64, 256, 32, 128
    q, k, v, gates, S0 = _inputs(B, H, d, d, steps, torch.bfloat16, 77, kind)
    S = S0.clone()
    outs = torch.stack([_run(ck, kind, q, k, v, gates, S, t) for t in range(steps)])
    assert ck.device_status() == 0
    b_idx = torch.tensor([0, 17, 128, 255], device=DEV)
    h_idx = torch.tensor([0, 9, 31], device=DEV)

    def sel(x):  # [steps, B, H, ...] -> [B', steps, H', ...] on the host
        return x[:, b_idx][:, :, h_idx].transpose(0, 1).cpu()

    f = oracle.forward_gdn2 if kind == "gdn2" else oracle.forward_sfda
    ro, rS = f(sel(q), sel(k), sel(v), *(sel(g) for g in gates), S0=S0[b_idx][:, h_idx].cpu())
    eo = rel_max_err(sel(outs), ro)
    es = rel_max_err(S[b_idx][:, h_idx], rS)
    assert eo <= TOL_BF16 and es <= TOL_BF16, (eo, es)
