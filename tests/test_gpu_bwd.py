"""Backward of the CKDA forward on the GPU against the fp64 backward oracle
(needs a B200).

``ckda_bwd_chunked`` computes dq, dk, dv, dalpha, dbeta and dS0 of a scalar
loss from dL/dout and dL/dS_final: the adjoint of the recurrence, token by
token in reverse, with the states recomputed from checkpoints (every 64th
token, then every 4th).  The oracle it is compared with is pinned by
``pinlib_bwd`` (B-1..B-6: finite differences of the pinned forward, closed
forms, symmetries).  Shapes span several 64-token chunks and 4-token
segments with ragged tails, every supported head size (d_v = 16 runs one
CTA per (sequence, head); larger d_v a cluster of d_v / 32 CTAs that add up
their partial sums in distributed shared memory), packed batches with empty
sequences, missing S0 / dS_final, and the full-size workload on sampled
units.  Tolerances: max|g - g_ref| / rms(g_ref) per gradient tensor, 1e-4
for fp32 inputs and 2e-2 for bf16 inputs (the forward's bars).
"""
import numpy as np
import pytest
import torch

import oracle
from delta_rule_linear_ckda_b200 import inputs
from gpu_util import TOL_BF16, TOL_F32, rel_max_err

pytestmark = pytest.mark.gpu
DEV = "cuda"
NAMES = ("dq", "dk", "dv", "dalpha", "dbeta", "dS0")


@pytest.fixture(scope="module")
def ck():
    import delta_rule_linear_ckda_b200 as ck

    return ck


def _upstream(shape_o, shape_s, seed, dtype=torch.float32, with_dsf=True):
    g = torch.Generator(device=DEV).manual_seed(seed)
    dO = torch.randn(shape_o, generator=g, device=DEV).to(dtype)
    dSf = torch.randn(shape_s, generator=g, device=DEV) if with_dsf else None
    return dO, dSf


def _check(got, ref, tol, names=NAMES):
    for n in names:
        err = rel_max_err(got[n], ref[n])
        assert err <= tol, f"{n}: {err}"


@pytest.mark.parametrize("dk,dv", [(16, 16), (32, 32), (64, 64), (128, 128), (64, 128), (128, 32),
                                   (16, 64)])
def test_fp32_matches_oracle(ck, dk, dv):
    c = inputs.random_prefill(2, 150, 2, dk, dv, dtype=torch.float32, gates="uniform", s0_std=0.5,
                              chunk=64, seed=dk + 7 * dv, device=DEV)
    dO, dSf = _upstream(c.v.shape, (2, 2, dk, dv), seed=dk + dv)
    g = ck.bwd_chunked(c.q, c.k, c.v, c.alpha, c.beta, dO, S0=c.S0, dS_final=dSf)
    assert ck.device_status() == 0
    ref = oracle.backward(c.q, c.k, c.v, c.alpha, c.beta, dO, S0=c.S0, dS_final=dSf)
    _check(g, ref, TOL_F32)


def test_bf16_inputs_and_gradient_match_oracle(ck):
    c = inputs.random_prefill(2, 300, 3, 128, 128, dtype=torch.bfloat16, gates="kda", s0_std=0.02,
                              chunk=64, seed=5, device=DEV)
    dO, dSf = _upstream(c.v.shape, (2, 3, 128, 128), seed=6, dtype=torch.bfloat16)
    g = ck.bwd_chunked(c.q, c.k, c.v, c.alpha, c.beta, dO, S0=c.S0, dS_final=dSf)
    assert ck.device_status() == 0
    ref = oracle.backward(c.q, c.k, c.v, c.alpha, c.beta, dO, S0=c.S0, dS_final=dSf)
    _check(g, ref, TOL_BF16)


def test_packed_batch_with_empty_sequences(ck):
    lens = [70, 0, 129, 1, 64, 5, 0]
    total = int(sum(lens))
    H, d = 2, 64
    base = inputs.random_prefill(1, total, H, d, d, dtype=torch.float32, gates="kda", chunk=64,
                                 seed=9, device=DEV)
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32, device=DEV)
    gen = torch.Generator(device=DEV).manual_seed(10)
    S0 = 0.3 * torch.randn(len(lens), H, d, d, generator=gen, device=DEV)
    dO, dSf = _upstream(base.v.shape, (len(lens), H, d, d), seed=11)
    g = ck.bwd_chunked(base.q, base.k, base.v, base.alpha, base.beta, dO, S0=S0, dS_final=dSf,
                       cu_seqlens=cu)
    assert ck.device_status() == 0
    ref = oracle.backward(base.q, base.k, base.v, base.alpha, base.beta, dO, S0=S0,
                          dS_final=dSf, cu_seqlens=cu)
    _check(g, ref, TOL_F32)
    for n, L in enumerate(lens):
        if L == 0:  # nothing runs: the gradient of S0 is the upstream one
            assert torch.equal(g["dS0"][n], dSf[n])


def test_without_S0_and_final_state_gradient(ck):
    c = inputs.random_prefill(3, 97, 2, 32, 64, dtype=torch.float32, gates="uniform", chunk=64,
                              seed=13, device=DEV)
    dO, _ = _upstream(c.v.shape, None, seed=14, with_dsf=False)
    g = ck.bwd_chunked(c.q, c.k, c.v, c.alpha, c.beta, dO)
    assert ck.device_status() == 0
    ref = oracle.backward(c.q, c.k, c.v, c.alpha, c.beta, dO)
    _check(g, ref, TOL_F32)


def test_outputs_are_overwritten_and_calls_deterministic(ck):
    c = inputs.random_prefill(2, 200, 2, 128, 128, dtype=torch.float32, gates="kda", s0_std=0.5,
                              chunk=64, seed=15, device=DEV)
    dO, dSf = _upstream(c.v.shape, (2, 2, 128, 128), seed=16)
    g1 = ck.bwd_chunked(c.q, c.k, c.v, c.alpha, c.beta, dO, S0=c.S0, dS_final=dSf)
    pre = {"dq": torch.full_like(c.q, float("nan")), "dk": torch.full_like(c.k, 7.0),
           "dv": torch.full_like(c.v, -1.0), "dalpha": torch.full_like(c.alpha, float("inf")),
           "dbeta": torch.full_like(c.beta, 3.0), "dS0": torch.full_like(c.S0, 5.0)}
    ws = torch.full((ck.bwd_workspace_bytes(2, 200, 2, 128, 128),), 0xFF, dtype=torch.uint8,
                    device=DEV)
    g2 = ck.bwd_chunked(c.q, c.k, c.v, c.alpha, c.beta, dO, S0=c.S0, dS_final=dSf, grads=pre,
                        workspace=ws)
    assert ck.device_status() == 0
    for n in NAMES:
        assert torch.equal(g1[n], g2[n]), n


def test_full_size_workload_on_sampled_units(ck):
    """The bench workload (B=4, T=4096, H=16, d=128, bf16 q/k/v and dO),
    checked on three sampled (sequence, head) units against the oracle."""
    c = inputs.kda_prefill(seed=0, device=DEV)
    dO, _ = _upstream(c.v.shape, None, seed=17, dtype=torch.bfloat16, with_dsf=False)
    g = ck.bwd_chunked(c.q, c.k, c.v, c.alpha, c.beta, dO)
    assert ck.device_status() == 0
    for b, h in [(0, 0), (2, 9), (3, 15)]:
        sel = lambda x: x[b:b + 1, :, h:h + 1].cpu()  # noqa: E731
        ref = oracle.backward(sel(c.q), sel(c.k), sel(c.v), sel(c.alpha), sel(c.beta), sel(dO))
        got = {n: sel(g[n]) for n in ("dq", "dk", "dv", "dalpha", "dbeta")}
        got["dS0"] = g["dS0"][b:b + 1, h:h + 1].cpu()
        _check(got, ref, TOL_BF16)
