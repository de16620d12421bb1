"""The tensor-core forward as two phases, and its packed-batch path (needs a B200).

``ckda_fwd_factors`` writes the S0-independent WY factors of every chunk to a
workspace and ``ckda_fwd_carry`` applies them from S0 ("Semidirect Fourier
Delta Attention", "Principales Contribuciones" item 3: each chunk is an affine
map of the state).  The one-call forward is those two kernels in order, so
the checks here are bit-exact: two phases equal one call, one factor pass
serves several initial states, and nothing depends on what the workspace
held before.  Packed batches (ragged, empty and chunk-aligned sequences) are
checked against the fp64 oracle.
"""
import numpy as np
import pytest
import torch

from delta_rule_linear_ckda_b200 import inputs
from gpu_util import TOL_BF16, oracle_fixed, oracle_packed, rel_max_err

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module")
def ck():
    import delta_rule_linear_ckda_b200 as ck

    return ck


def _packed(lens, H=3, seed=0, with_s0=True):
    """Packed bf16 batch (d = 128, C = 64) with the given sequence lengths."""
    total = int(sum(lens))
    base = inputs.random_prefill(1, max(total, 1), H, 128, 128, dtype=torch.bfloat16, gates="kda",
                                 chunk=64, seed=seed, device=DEV)
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32, device=DEV)
    S0 = None
    if with_s0:
        g = torch.Generator(device=DEV).manual_seed(seed + 1)
        S0 = 0.02 * torch.randn(len(lens), H, 128, 128, generator=g, device=DEV)
    cut = lambda x: x[:, :total].contiguous()  # noqa: E731
    return inputs.PrefillCase("packed", cut(base.q), cut(base.k), cut(base.v), cut(base.alpha),
                              cut(base.beta), S0, cu, 64)


def _fixed(B=2, T=200, H=3, seed=0):
    return inputs.random_prefill(B, T, H, 128, 128, dtype=torch.bfloat16, gates="kda", s0_std=0.02,
                                 chunk=64, seed=seed, device=DEV)


@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("packed", [False, True])
def test_two_phases_equal_one_call(ck, out_dtype, packed):
    case = _packed([70, 0, 129, 64, 5]) if packed else _fixed()
    cu = case.cu_seqlens
    out1, S1 = ck.fwd_chunked(case.q, case.k, case.v, case.alpha, case.beta, S0=case.S0,
                              cu_seqlens=cu, out_dtype=out_dtype)
    ws = ck.fwd_factors(case.q, case.k, case.v, case.alpha, case.beta, cu_seqlens=cu)
    B = case.n_seqs
    T = case.q.shape[1]
    out2, S2 = ck.fwd_carry(ws, case.v, B, T, case.H, 128, 128, S0=case.S0, cu_seqlens=cu,
                            out_dtype=out_dtype)
    assert ck.device_status() == 0
    assert torch.equal(out1.view(-1), out2.view(-1))
    assert torch.equal(S1, S2)


def test_one_factor_pass_serves_several_initial_states(ck):
    case = _fixed(seed=3)
    ws = ck.fwd_factors(case.q, case.k, case.v, case.alpha, case.beta)
    B, T, H = case.q.shape[:3]
    for scale in (0.0, 1.0, -3.0):
        S0 = scale * case.S0
        ref_o, ref_S = ck.fwd_chunked(case.q, case.k, case.v, case.alpha, case.beta, S0=S0,
                                      out_dtype=torch.float32)
        o, S = ck.fwd_carry(ws, case.v, B, T, H, 128, 128, S0=S0)
        assert torch.equal(o, ref_o) and torch.equal(S, ref_S), scale
    assert ck.device_status() == 0


def test_workspace_contents_do_not_matter(ck):
    case = _fixed(seed=5)
    B, T, H = case.q.shape[:3]
    need = ck.workspace_bytes(B, T, H, 128, 128)
    results = []
    for fill in (0, 0xFF, 0x7C):  # zeros, NaN patterns, +inf halves
        ws = torch.full((need + 4096,), fill, dtype=torch.uint8, device=DEV)
        results.append(ck.fwd_chunked(case.q, case.k, case.v, case.alpha, case.beta, S0=case.S0,
                                      out_dtype=torch.float32, workspace=ws))
    assert ck.device_status() == 0
    for o, S in results[1:]:
        assert torch.equal(o, results[0][0]) and torch.equal(S, results[0][1])


def test_fixed_batch_matches_oracle(ck):
    case = _fixed(B=3, T=300, H=2, seed=9)
    out, S = ck.fwd_chunked(case.q, case.k, case.v, case.alpha, case.beta, S0=case.S0,
                            out_dtype=torch.float32)
    assert ck.device_status() == 0
    ro, rS, _, _ = oracle_fixed(case)
    assert rel_max_err(out, ro) <= TOL_BF16 and rel_max_err(S, rS) <= TOL_BF16


@pytest.mark.parametrize("lens", [[1], [64], [65, 0, 63], [0, 0, 130, 1, 191, 64, 0],
                                  [17] * 9])
def test_packed_tensor_core_path_matches_oracle(ck, lens):
    case = _packed(lens, seed=len(lens))
    cu = case.cu_seqlens
    assert ck.fwd_path(len(lens), int(sum(lens)), case.H, 128, 128, varlen=True) == "tcgen05"
    out, S = ck.fwd_chunked(case.q, case.k, case.v, case.alpha, case.beta, S0=case.S0,
                            cu_seqlens=cu, out_dtype=torch.float32)
    assert ck.device_status() == 0
    ro, rS, _, _ = oracle_packed(case)
    got = out.view(-1, case.H, 128)
    assert rel_max_err(got, ro) <= TOL_BF16
    assert rel_max_err(S, rS) <= TOL_BF16
    # zero-length sequences keep their initial state exactly
    for n, L in enumerate(lens):
        if L == 0:
            assert torch.equal(S[n], case.S0[n])


def test_packed_equals_separate_fixed_calls(ck):
    """Each sequence of a packed batch gives, bit for bit, what a fixed-length call
    on that sequence alone gives (the state restarts at every sequence start)."""
    lens = [130, 64, 7]
    case = _packed(lens, seed=11)
    out, S = ck.fwd_chunked(case.q, case.k, case.v, case.alpha, case.beta, S0=case.S0,
                            cu_seqlens=case.cu_seqlens, out_dtype=torch.float32)
    cu = [0] + list(np.cumsum(lens))
    for n, L in enumerate(lens):
        sl = slice(cu[n], cu[n + 1])
        # fresh copies: a slice of the packed tensors need not be 16-byte aligned
        o1, S1 = ck.fwd_chunked(case.q[:, sl].clone(), case.k[:, sl].clone(),
                                case.v[:, sl].clone(), case.alpha[:, sl].clone(),
                                case.beta[:, sl].clone(), S0=case.S0[n:n + 1].clone(),
                                out_dtype=torch.float32)
        assert torch.equal(out[:, sl], o1), n
        assert torch.equal(S[n], S1[0]), n
    assert ck.device_status() == 0
