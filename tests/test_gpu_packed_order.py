"""Packed batches walked longest first (needs a B200).

The fp32 CUDA-core forward and the tensor-core carry give the CTAs of
grid index z the sequence of rank z in decreasing length (ties by index),
so that the longest sequences start first.  These cases check that every
sequence is still computed once, from its own start state, whatever the
mix: many equal lengths, empty sequences among them, and more sequences
than the ordering handles (launch order then).  Each is compared with the
fp64 oracle on every token and every final state.
"""
import numpy as np
import pytest
import torch

from delta_rule_linear_ckda_b200 import inputs
from gpu_util import TOL_BF16, TOL_F32, oracle_packed, rel_max_err

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module")
def ck():
    import delta_rule_linear_ckda_b200 as ck

    return ck


def _packed_case(name, lens, H, d, dtype, seed):
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32, device=DEV)
    Tt = int(cu[-1])
    g = torch.Generator(device=DEV).manual_seed(seed)
    q = torch.nn.functional.normalize(torch.randn(1, Tt, H, d, device=DEV, generator=g), dim=-1)
    k = torch.nn.functional.normalize(torch.randn(1, Tt, H, d, device=DEV, generator=g), dim=-1)
    v = torch.randn(1, Tt, H, d, device=DEV, generator=g)
    a = torch.rand(1, Tt, H, d, device=DEV, generator=g) * 2 - 1
    b = torch.rand(1, Tt, H, device=DEV, generator=g) * 2
    S0 = 0.5 * torch.randn(len(lens), H, d, d, device=DEV, generator=g)
    return inputs.PrefillCase(name, q.to(dtype), k.to(dtype), v.to(dtype), a, b, S0, cu, 64)


def _check(ck, case, lens, dtype, path):
    H, d = case.q.shape[2], case.q.shape[3]
    assert ck.fwd_path(len(lens), case.q.shape[1], H, d, d, case.chunk, dtype, torch.float32,
                       varlen=True) == path
    out, S = ck.fwd_chunked(case.q, case.k, case.v, case.alpha, case.beta, S0=case.S0,
                            cu_seqlens=case.cu_seqlens, chunk=case.chunk,
                            out_dtype=torch.float32)
    assert ck.device_status() == 0
    for n, L in enumerate(lens):
        if L == 0:
            assert torch.equal(S[n], case.S0[n])
    ro, rS, tok, _ = oracle_packed(case)
    tol = TOL_F32 if dtype == torch.float32 else TOL_BF16
    eo = rel_max_err(out.cpu()[0][tok], ro)
    es = rel_max_err(S.cpu(), rS)
    assert eo <= tol and es <= tol, (case.name, eo, es)


@pytest.mark.parametrize("dtype,path", [(torch.float32, "fp32core"), (torch.bfloat16, "tcgen05")])
def test_ties_and_empty_sequences(ck, dtype, path):
    # 295 sequences: long runs of equal lengths, empty ones in between
    lens = np.array([40] * 200 + [0] * 5 + [17] * 50 + [64] * 30 + [1] * 10)
    lens = lens[np.random.default_rng(21).permutation(lens.size)]
    case = _packed_case("ties", lens, 2, 128, dtype, seed=22)
    _check(ck, case, lens, dtype, path)


@pytest.mark.parametrize("dtype,path", [(torch.float32, "fp32core"), (torch.bfloat16, "tcgen05")])
def test_more_sequences_than_the_ordering_handles(ck, dtype, path):
    # 1100 sequences (above the 1024 the CTAs rank among themselves)
    lens = np.random.default_rng(23).integers(0, 12, size=1100)
    case = _packed_case("many", lens, 1, 128, dtype, seed=24)
    _check(ck, case, lens, dtype, path)
