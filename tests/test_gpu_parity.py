"""CUDA path vs the fp64 oracle on the seeded workloads (needs a B200).

Every call goes through the C ABI (``libckda.so``) via the thin torch
binding.  Tolerances: max|o - o_ref| / rms(o_ref) <= 1e-4 for fp32 inputs
and <= 2e-2 for bf16 inputs, the same bounds for the final state, and the
norm ratio of the orthogonal halves within 1e-4.  Outputs are requested in
fp32 (the accumulator type): rounding o to bf16 alone moves this metric by
up to 2^-9 * max|o| / rms(o), about 3e-2 on these workloads, so the bf16
output is checked separately as the exact rounding of the fp32 output.  Full-size workloads are
checked on sampled (sequence, head) units, each of which the oracle computes
over its whole length.
"""
import numpy as np
import pytest
import torch

from delta_rule_linear_ckda_b200 import inputs
from gpu_util import TOL_BF16, TOL_F32, oracle_fixed, oracle_packed, rel_max_err

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module")
def ck():
    import delta_rule_linear_ckda_b200 as ck

    return ck


def _check_fixed(ck, case, tol, fp32core=False, b_idx=None, h_idx=None):
    out, S = ck.fwd_chunked(case.q, case.k, case.v, case.alpha, case.beta, S0=case.S0,
                            chunk=case.chunk, fp32core=fp32core, out_dtype=torch.float32)
    assert ck.device_status() == 0
    ro, rS, bi, hi = oracle_fixed(case, b_idx, h_idx)
    got_o = out.cpu()[bi][:, :, hi]
    got_S = S.cpu()[bi][:, hi]
    eo, es = rel_max_err(got_o, ro), rel_max_err(got_S, rS)
    assert torch.isfinite(out).all() and torch.isfinite(S).all()
    assert eo <= tol and es <= tol, (case.name, eo, es)
    return eo, es


@pytest.mark.parametrize("fp32core", [False, True])
def test_tiny_fp32(ck, fp32core):
    case = inputs.tiny(seed=0, device=DEV)
    _check_fixed(ck, case, TOL_F32, fp32core=fp32core)


@pytest.mark.parametrize("fp32core", [False, True])
def test_kda_prefill_small_ragged(ck, fp32core):
    # several chunks and a ragged last chunk (T = 4*64 + 37)
    case = inputs.kda_prefill(seed=1, device=DEV, B=2, T=293, H=4, d=128)
    _check_fixed(ck, case, TOL_BF16, fp32core=fp32core)


def test_prefill_workloads_run_on_tensor_cores(ck):
    assert ck.fwd_path(4, 4096, 16, 128, 128, 64, torch.bfloat16, torch.float32) == "tcgen05"
    assert ck.fwd_path(1, 65536, 32, 128, 128, 64, torch.bfloat16, torch.float32) == "tcgen05"
    assert ck.fwd_path(64, 135000, 16, 128, 128, 64, torch.float32, torch.float32,
                       varlen=True) == "fp32core"


def test_kda_prefill_full_size_sampled(ck):
    case = inputs.kda_prefill(seed=0, device=DEV)  # B=4, H=16, T=4096, d=128
    _check_fixed(ck, case, TOL_BF16, b_idx=[0, 3], h_idx=[0, 5, 15])


def test_long_prefill_sampled(ck):
    case = inputs.long_prefill(seed=0, device=DEV)  # B=1, H=32, T=65536, S0 ~ N(0, 0.02^2)
    _check_fixed(ck, case, TOL_BF16, b_idx=[0], h_idx=[0, 31])


def test_decode_1024_steps_sampled(ck):
    case = inputs.decode(seed=0, device=DEV)  # B=256, H=32, d=128, 1024 steps
    S = case.S0.clone()
    steps = case.q.shape[0]
    outs = torch.empty(case.v.shape, dtype=torch.float32, device=DEV)
    for t in range(steps):
        ck.decode_step(case.q[t], case.k[t], case.v[t], case.alpha[t], case.beta[t], S, out=outs[t])
    torch.cuda.synchronize()
    b_idx = torch.tensor([0, 17, 128, 255])
    h_idx = torch.tensor([0, 9, 31])
    # oracle: the sampled units as fixed-length sequences of `steps` tokens
    import oracle

    def sel(x):
        return x.cpu()[:, b_idx][:, :, h_idx].transpose(0, 1)  # [B', steps, H', d]

    ro, rS = oracle.forward(sel(case.q), sel(case.k), sel(case.v), sel(case.alpha),
                            case.beta.cpu()[:, b_idx][:, :, h_idx].transpose(0, 1),
                            S0=case.S0.cpu()[b_idx][:, h_idx])
    got_o = outs.cpu()[:, b_idx][:, :, h_idx].transpose(0, 1)
    got_S = S.cpu()[b_idx][:, h_idx]
    eo, es = rel_max_err(got_o, ro), rel_max_err(got_S, rS)
    assert eo <= TOL_BF16 and es <= TOL_BF16, (eo, es)


def test_decode_fp32_matches_oracle_tightly(ck):
    g = torch.Generator(device=DEV).manual_seed(5)
    B, H, dk, dv = 3, 4, 64, 32
    q = torch.nn.functional.normalize(torch.randn(B, H, dk, device=DEV, generator=g), dim=-1)
    k = torch.nn.functional.normalize(torch.randn(B, H, dk, device=DEV, generator=g), dim=-1)
    v = torch.randn(B, H, dv, device=DEV, generator=g)
    a = torch.rand(B, H, dk, device=DEV, generator=g) * 2 - 1
    b = torch.rand(B, H, device=DEV, generator=g) * 2
    S = torch.randn(B, H, dk, dv, device=DEV, generator=g)
    import oracle

    ro, rS = oracle.decode_step(q, k, v, a, b, S)
    o = ck.decode_step(q, k, v, a, b, S)
    assert rel_max_err(o, ro) <= TOL_F32 and rel_max_err(S, rS) <= TOL_F32


def test_varlen_gate_extreme_sampled(ck):
    case = inputs.varlen(seed=0, device=DEV)  # 64 packed seqs, L ~ U[128, 4096], fp32
    out, S = ck.fwd_chunked(case.q, case.k, case.v, case.alpha, case.beta,
                            cu_seqlens=case.cu_seqlens, chunk=case.chunk)
    assert ck.device_status() == 0
    assert out.dtype == torch.float32
    assert torch.isfinite(out).all() and torch.isfinite(S).all()
    seqs = [0, 7, 31, 63]
    ro, rS, tok, hi = oracle_packed(case, seqs, [0, 15])
    got_o = out.cpu()[0][tok][:, hi]
    got_S = S.cpu()[torch.tensor(seqs)][:, hi]
    eo, es = rel_max_err(got_o, ro), rel_max_err(got_S, rS)
    assert eo <= TOL_F32 and es <= TOL_F32, (eo, es)

    # norm preservation over the orthogonal second halves: compare with a
    # second call on the first halves only
    half = inputs.first_halves(case)
    _, S_half = ck.fwd_chunked(half.q, half.k, half.v, half.alpha, half.beta,
                               cu_seqlens=half.cu_seqlens, chunk=half.chunk)
    nf = S.double().flatten(2).norm(dim=-1)
    nh = S_half.double().flatten(2).norm(dim=-1)
    ratio = (nf / nh).cpu().numpy()
    assert np.all(np.abs(ratio - 1.0) <= 1e-4), float(np.max(np.abs(ratio - 1.0)))


@pytest.mark.parametrize("fp32core", [False, True])
def test_bf16_output_is_exact_rounding_of_fp32_output(ck, fp32core):
    """A bf16 output is the round-to-nearest-even of the same call's fp32 output,
    so its error vs the oracle is bounded by the fp32 error plus half a bf16 ulp."""
    case = inputs.kda_prefill(seed=3, device=DEV, B=2, T=200, H=4, d=128)
    o32, S32 = ck.fwd_chunked(case.q, case.k, case.v, case.alpha, case.beta, chunk=64,
                              fp32core=fp32core, out_dtype=torch.float32)
    o16, S16 = ck.fwd_chunked(case.q, case.k, case.v, case.alpha, case.beta, chunk=64,
                              fp32core=fp32core, out_dtype=torch.bfloat16)
    assert o16.dtype == torch.bfloat16
    assert torch.equal(o16, o32.to(torch.bfloat16)) and torch.equal(S16, S32)
    ro, rS, _, _ = oracle_fixed(case)
    rms = float(np.sqrt(np.mean(ro * ro)))
    bound = TOL_BF16 + 2.0 ** -9 * float(np.max(np.abs(ro))) / rms
    assert rel_max_err(o16, ro) <= bound


def test_decode_bf16_output_is_exact_rounding(ck):
    case = inputs.decode(seed=4, device=DEV, B=8, H=4, d=128, steps=3)
    S_a, S_b = case.S0.clone(), case.S0.clone()
    for t in range(3):
        o32 = ck.decode_step(case.q[t], case.k[t], case.v[t], case.alpha[t], case.beta[t], S_a,
                             out_dtype=torch.float32)
        o16 = ck.decode_step(case.q[t], case.k[t], case.v[t], case.alpha[t], case.beta[t], S_b,
                             out_dtype=torch.bfloat16)
        assert torch.equal(o16, o32.to(torch.bfloat16))
    assert torch.equal(S_a, S_b)
