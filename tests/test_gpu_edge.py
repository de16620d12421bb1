"""Edge cases and invariants of the CUDA path (needs a B200).

Shapes span several chunks with ragged tails, every supported head size,
d_k != d_v, each chunk size, empty and zero-length sequences, aliasing of
S0 and S_final, and a malformed offsets array (reported through the device
status word).  Invariants that hold at any size: sign symmetry (bit-exact),
chunk-size independence, split-call resumability (the affine block transfer
between calls), identity padding, and the alpha = 0 closed form.
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


def _run_vs_oracle(ck, case, tol, fp32core=False):
    out, S = ck.fwd_chunked(case.q, case.k, case.v, case.alpha, case.beta, S0=case.S0,
                            chunk=case.chunk, fp32core=fp32core, out_dtype=torch.float32)
    assert ck.device_status() == 0
    ro, rS, _, _ = oracle_fixed(case)
    eo, es = rel_max_err(out, ro), rel_max_err(S, rS)
    assert eo <= tol and es <= tol, (case.name, eo, es)


@pytest.mark.parametrize("dk,dv", [(16, 16), (32, 32), (64, 64), (128, 128), (64, 128),
                                   (128, 32), (16, 128)])
@pytest.mark.parametrize("chunk", [16, 32, 64])
def test_shapes_fp32(ck, dk, dv, chunk):
    case = inputs.random_prefill(2, 2 * chunk + 7, 2, dk, dv, dtype=torch.float32, gates="uniform",
                                 s0_std=0.5, chunk=chunk, seed=dk + dv + chunk, device=DEV)
    _run_vs_oracle(ck, case, TOL_F32)


@pytest.mark.parametrize("dk,dv", [(64, 64), (128, 128), (128, 64)])
@pytest.mark.parametrize("chunk", [16, 64])
@pytest.mark.parametrize("fp32core", [False, True])
def test_shapes_bf16(ck, dk, dv, chunk, fp32core):
    case = inputs.random_prefill(2, 3 * chunk + 5, 3, dk, dv, dtype=torch.bfloat16, gates="kda",
                                 s0_std=0.02, chunk=chunk, seed=7 * dk + dv, device=DEV)
    _run_vs_oracle(ck, case, TOL_BF16, fp32core)


@pytest.mark.parametrize("T", [1, 5, 63, 64, 65])
def test_short_sequences(ck, T):
    case = inputs.random_prefill(3, T, 2, 128, 128, dtype=torch.bfloat16, gates="kda",
                                 s0_std=0.02, chunk=64, seed=T, device=DEV)
    _run_vs_oracle(ck, case, TOL_BF16)


def test_empty_batch(ck):
    z = torch.zeros(0, 8, 2, 16, device=DEV)
    out, S = ck.fwd_chunked(z, z, z, z, torch.zeros(0, 8, 2, device=DEV), chunk=16)
    assert out.shape == (0, 8, 2, 16) and S.shape == (0, 2, 16, 16)


def test_zero_length_sequences_keep_S0(ck):
    lens = [0, 70, 0, 3, 129, 0]
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32, device=DEV)
    Tt = int(cu[-1])
    g = torch.Generator(device=DEV).manual_seed(3)
    H, d = 2, 64
    q = torch.nn.functional.normalize(torch.randn(1, Tt, H, d, device=DEV, generator=g), dim=-1)
    k = torch.nn.functional.normalize(torch.randn(1, Tt, H, d, device=DEV, generator=g), dim=-1)
    v = torch.randn(1, Tt, H, d, device=DEV, generator=g)
    a = torch.rand(1, Tt, H, d, device=DEV, generator=g) * 2 - 1
    b = torch.rand(1, Tt, H, device=DEV, generator=g) * 2
    S0 = torch.randn(len(lens), H, d, d, device=DEV, generator=g)
    case = inputs.PrefillCase("zero-length", q, k, v, a, b, S0, cu, 32)
    out, S = ck.fwd_chunked(q, k, v, a, b, S0=S0, cu_seqlens=cu, chunk=32)
    assert ck.device_status() == 0
    for n, L in enumerate(lens):
        if L == 0:
            assert torch.equal(S[n], S0[n])
    ro, rS, tok, hi = oracle_packed(case)
    assert rel_max_err(out.cpu()[0][tok], ro) <= TOL_F32
    assert rel_max_err(S.cpu(), rS) <= TOL_F32


def test_s_final_may_alias_s0(ck):
    case = inputs.random_prefill(2, 100, 2, 64, 64, dtype=torch.float32, gates="uniform",
                                 s0_std=1.0, chunk=32, seed=11, device=DEV)
    ro, rS, _, _ = oracle_fixed(case)
    S = case.S0.clone()
    out, S_ret = ck.fwd_chunked(case.q, case.k, case.v, case.alpha, case.beta, S0=S, S_final=S,
                                chunk=32)
    assert S_ret.data_ptr() == S.data_ptr()
    assert rel_max_err(S, rS) <= TOL_F32 and rel_max_err(out, ro) <= TOL_F32
    out2, none = ck.fwd_chunked(case.q, case.k, case.v, case.alpha, case.beta, S0=case.S0,
                                chunk=32, return_final=False)
    assert none is None and rel_max_err(out2, ro) <= TOL_F32


def test_bad_cu_seqlens_reported_on_device(ck):
    H, d = 1, 16
    q = torch.zeros(1, 10, H, d, device=DEV)
    b = torch.zeros(1, 10, H, device=DEV)
    cu = torch.tensor([0, 6, 4, 10], dtype=torch.int32, device=DEV)  # decreasing
    ck.fwd_chunked(q, q, q, q, b, cu_seqlens=cu, chunk=16)
    assert ck.device_status() == -6
    assert ck.device_status() == 0  # the word is cleared by reading it
    cu = torch.tensor([0, 4, 11], dtype=torch.int32, device=DEV)  # past the end
    ck.fwd_chunked(q, q, q, q, b, cu_seqlens=cu, chunk=16)
    assert ck.device_status() == -6


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_sign_symmetry_bit_exact(ck, dtype):
    case = inputs.random_prefill(2, 200, 4, 128, 128, dtype=dtype, gates="kda", s0_std=0.02,
                                 chunk=64, seed=21, device=DEV)
    o1, S1 = ck.fwd_chunked(case.q, case.k, case.v, case.alpha, case.beta, S0=case.S0)
    o2, S2 = ck.fwd_chunked(case.q, -case.k, -case.v, case.alpha, case.beta, S0=case.S0)
    assert torch.equal(o1, o2) and torch.equal(S1, S2)


@pytest.mark.parametrize("dtype,tol", [(torch.float32, TOL_F32), (torch.bfloat16, TOL_BF16)])
def test_chunk_size_independence_and_resume(ck, dtype, tol):
    case = inputs.random_prefill(2, 300, 4, 128, 128, dtype=dtype, gates="kda", s0_std=0.02,
                                 chunk=64, seed=22, device=DEV)
    ref, Sref = ck.fwd_chunked(case.q, case.k, case.v, case.alpha, case.beta, S0=case.S0,
                               chunk=64, fp32core=True, out_dtype=torch.float32)
    for C in (16, 32, 64):
        o, S = ck.fwd_chunked(case.q, case.k, case.v, case.alpha, case.beta, S0=case.S0, chunk=C,
                              out_dtype=torch.float32)
        assert rel_max_err(o, ref.double().cpu().numpy()) <= tol
        assert rel_max_err(S, Sref.double().cpu().numpy()) <= tol
    # split call at T1 = 100 (not a chunk multiple) and resume from S_final
    T1 = 100
    parts = [x[:, :T1].contiguous() for x in (case.q, case.k, case.v, case.alpha, case.beta)]
    rest = [x[:, T1:].contiguous() for x in (case.q, case.k, case.v, case.alpha, case.beta)]
    o_a, S_mid = ck.fwd_chunked(*parts, S0=case.S0, out_dtype=torch.float32)
    o_b, S_end = ck.fwd_chunked(*rest, S0=S_mid, out_dtype=torch.float32)
    assert rel_max_err(torch.cat([o_a, o_b], 1), ref.double().cpu().numpy()) <= tol
    assert rel_max_err(S_end, Sref.double().cpu().numpy()) <= tol


def test_identity_padding_changes_nothing(ck):
    case = inputs.random_prefill(1, 90, 2, 64, 64, dtype=torch.float32, gates="uniform",
                                 s0_std=0.3, chunk=32, seed=23, device=DEV)
    o1, S1 = ck.fwd_chunked(case.q, case.k, case.v, case.alpha, case.beta, S0=case.S0, chunk=32)
    pad = 20

    def ext(x, fill):
        shape = list(x.shape)
        shape[1] = pad
        return torch.cat([x, torch.full(shape, fill, dtype=x.dtype, device=DEV)], 1).contiguous()

    o2, S2 = ck.fwd_chunked(ext(case.q, 0.0), ext(case.k, 0.0), ext(case.v, 0.0),
                            ext(case.alpha, 1.0), ext(case.beta, 0.0), S0=case.S0, chunk=32)
    assert torch.equal(S1, S2)
    assert torch.allclose(o2[:, :90], o1, rtol=0, atol=1e-6)


def test_alpha_zero_closed_form(ck):
    case = inputs.random_prefill(2, 130, 2, 128, 128, dtype=torch.float32, gates="uniform",
                                 s0_std=1.0, chunk=64, seed=24, device=DEV)
    a0 = torch.zeros_like(case.alpha)
    o, S = ck.fwd_chunked(case.q, case.k, case.v, a0, case.beta, S0=case.S0)
    kq = (case.k * case.q).sum(-1, keepdim=True)
    expect = case.beta.unsqueeze(-1) * kq * case.v
    assert torch.allclose(o, expect, rtol=1e-5, atol=1e-5)
    expect_S = case.beta[:, -1, :, None, None] * case.k[:, -1, :, :, None] * case.v[:, -1, :, None, :]
    assert torch.allclose(S, expect_S, rtol=1e-5, atol=1e-6)
