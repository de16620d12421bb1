"""Gated DeltaNet-2 forward on the GPU against the fp64 oracle (needs a B200).

``ckda_gdn2_fwd_chunked`` runs the chunk form of the Gated DeltaNet-2
recurrence ("Gated DeltaNet-2" summary, Methodology sections 1 and 3) on the
fp32 CUDA-core kernel.  The oracle it is compared with is pinned by
``pinlib_gdn2`` (G-1..G-7).  Shapes span several chunks with ragged tails,
every supported head size and chunk size, packed batches with empty
sequences, the full-size workload on sampled units, and the reduction
b = w = beta, which must reproduce the CKDA path.
"""
import numpy as np
import pytest
import torch

import oracle
from delta_rule_linear_ckda_b200 import inputs
from gpu_util import TOL_BF16, TOL_F32, rel_max_err

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module")
def ck():
    import delta_rule_linear_ckda_b200 as ck

    return ck


def _run(ck, c, cu=None, out_dtype=torch.float32):
    out, S = ck.gdn2_fwd_chunked(c.q, c.k, c.v, c.alpha, c.extra["b"], c.extra["w"], S0=c.S0,
                                 cu_seqlens=cu, chunk=c.chunk, out_dtype=out_dtype)
    assert ck.device_status() == 0
    return out, S


@pytest.mark.parametrize("dk,dv", [(16, 16), (64, 64), (128, 128), (64, 128), (128, 32)])
@pytest.mark.parametrize("chunk", [16, 32, 64])
def test_fp32_matches_oracle(ck, dk, dv, chunk):
    c = inputs.gdn2_prefill(2, 2 * chunk + 11, 2, dk, dv, dtype=torch.float32, s0_std=0.5,
                            chunk=chunk, seed=dk + 3 * dv + chunk, device=DEV)
    out, S = _run(ck, c)
    ro, rS = oracle.forward_gdn2(c.q, c.k, c.v, c.alpha, c.extra["b"], c.extra["w"], S0=c.S0)
    assert rel_max_err(out, ro) <= TOL_F32 and rel_max_err(S, rS) <= TOL_F32


def test_bf16_inputs_match_oracle(ck):
    c = inputs.gdn2_prefill(2, 300, 3, 128, 128, dtype=torch.bfloat16, s0_std=0.02, chunk=64,
                            seed=5, device=DEV)
    out, S = _run(ck, c, out_dtype=torch.float32)
    ro, rS = oracle.forward_gdn2(c.q, c.k, c.v, c.alpha, c.extra["b"], c.extra["w"], S0=c.S0)
    assert rel_max_err(out, ro) <= TOL_BF16 and rel_max_err(S, rS) <= TOL_BF16
    # a bf16 output is exactly the bf16 rounding of the fp32 result (parity is
    # checked on the fp32 output: the rounding alone can exceed the tolerance)
    o16, _ = _run(ck, c, out_dtype=torch.bfloat16)
    assert torch.equal(o16, out.to(torch.bfloat16))


def test_packed_batch_with_empty_sequences(ck):
    lens = [70, 0, 129, 1, 64]
    total = int(sum(lens))
    c = inputs.gdn2_prefill(1, total, 2, 64, 64, dtype=torch.float32, chunk=32, seed=9, device=DEV)
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32, device=DEV)
    g = torch.Generator(device=DEV).manual_seed(10)
    S0 = 0.3 * torch.randn(len(lens), 2, 64, 64, generator=g, device=DEV)
    out, S = ck.gdn2_fwd_chunked(c.q, c.k, c.v, c.alpha, c.extra["b"], c.extra["w"], S0=S0,
                                 cu_seqlens=cu, chunk=32, out_dtype=torch.float32)
    assert ck.device_status() == 0
    ro, rS = oracle.forward_gdn2(c.q, c.k, c.v, c.alpha, c.extra["b"], c.extra["w"], S0=S0,
                                 cu_seqlens=cu)
    assert rel_max_err(out, ro) <= TOL_F32 and rel_max_err(S, rS) <= TOL_F32
    assert torch.equal(S[1], S0[1])  # the empty sequence keeps its state


def test_tied_gates_reproduce_the_ckda_path(ck):
    c = inputs.random_prefill(2, 150, 2, 128, 128, dtype=torch.float32, gates="kda", s0_std=0.5,
                              chunk=64, seed=12, device=DEV)
    b = c.beta[..., None].expand(*c.k.shape).contiguous()
    w = c.beta[..., None].expand(*c.v.shape).contiguous()
    o1, S1 = ck.gdn2_fwd_chunked(c.q, c.k, c.v, c.alpha, b, w, S0=c.S0, out_dtype=torch.float32)
    o2, S2 = ck.fwd_chunked(c.q, c.k, c.v, c.alpha, c.beta, S0=c.S0, fp32core=True,
                            out_dtype=torch.float32)
    assert ck.device_status() == 0
    assert rel_max_err(o1, o2.double().cpu().numpy()) <= 1e-5
    assert rel_max_err(S1, S2.double().cpu().numpy()) <= 1e-5


@pytest.mark.parametrize("dv", [64, 128])
@pytest.mark.parametrize("T", [64, 200])
def test_tensor_core_path_matches_oracle(ck, dv, T):
    assert ck.fwd_path(2, T, 3, 128, dv, 64, torch.bfloat16, torch.float32) == "tcgen05"
    c = inputs.gdn2_prefill(2, T, 3, 128, dv, dtype=torch.bfloat16, s0_std=0.02, chunk=64,
                            seed=T + dv, device=DEV)
    out, S = _run(ck, c)
    ro, rS = oracle.forward_gdn2(c.q, c.k, c.v, c.alpha, c.extra["b"], c.extra["w"], S0=c.S0)
    assert rel_max_err(out, ro) <= TOL_BF16 and rel_max_err(S, rS) <= TOL_BF16


def test_tensor_core_packed_batch(ck):
    lens = [70, 0, 129, 1, 64]
    total = int(sum(lens))
    c = inputs.gdn2_prefill(1, total, 2, 128, 128, dtype=torch.bfloat16, chunk=64, seed=19,
                            device=DEV)
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32, device=DEV)
    g = torch.Generator(device=DEV).manual_seed(20)
    S0 = 0.02 * torch.randn(len(lens), 2, 128, 128, generator=g, device=DEV)
    out, S = ck.gdn2_fwd_chunked(c.q, c.k, c.v, c.alpha, c.extra["b"], c.extra["w"], S0=S0,
                                 cu_seqlens=cu, chunk=64, out_dtype=torch.float32)
    assert ck.device_status() == 0
    ro, rS = oracle.forward_gdn2(c.q, c.k, c.v, c.alpha, c.extra["b"], c.extra["w"], S0=S0,
                                 cu_seqlens=cu)
    assert rel_max_err(out, ro) <= TOL_BF16 and rel_max_err(S, rS) <= TOL_BF16
    assert torch.equal(S[1], S0[1])


def test_tensor_core_agrees_with_the_fp32_kernel(ck):
    """Same bf16 inputs through the tcgen05 pair and the fp32 CUDA-core kernel
    (chunk 32 forces the latter)."""
    c = inputs.gdn2_prefill(1, 256, 4, 128, 128, dtype=torch.bfloat16, s0_std=0.02, chunk=64,
                            seed=21, device=DEV)
    o_tc, S_tc = _run(ck, c)
    o_32, S_32 = ck.gdn2_fwd_chunked(c.q, c.k, c.v, c.alpha, c.extra["b"], c.extra["w"], S0=c.S0,
                                     chunk=32, out_dtype=torch.float32)
    assert ck.device_status() == 0
    assert rel_max_err(o_tc, o_32.double().cpu().numpy()) <= TOL_BF16
    assert rel_max_err(S_tc, S_32.double().cpu().numpy()) <= TOL_BF16


def test_full_size_workload_on_sampled_units(ck):
    """The bench workload (B=4, T=4096, H=16, d=128, bf16, tensor-core pair),
    checked on four sampled (sequence, head) units against the oracle."""
    assert ck.fwd_path(4, 4096, 16, 128, 128, 64, torch.bfloat16, torch.float32) == "tcgen05"
    c = inputs.gdn2_prefill(4, 4096, 16, 128, 128, dtype=torch.bfloat16, chunk=64, seed=0,
                            device=DEV)
    out, S = _run(ck, c)
    for b, h in [(0, 0), (1, 7), (2, 15), (3, 3)]:
        sel = lambda x: x[b:b + 1, :, h:h + 1].cpu()  # noqa: E731
        ro, rS = oracle.forward_gdn2(sel(c.q), sel(c.k), sel(c.v), sel(c.alpha),
                                     sel(c.extra["b"]), sel(c.extra["w"]))
        assert rel_max_err(out[b:b + 1, :, h:h + 1], ro) <= TOL_BF16, (b, h)
        assert rel_max_err(S[b:b + 1, h:h + 1], rS) <= TOL_BF16, (b, h)
