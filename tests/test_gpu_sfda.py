"""SFDA forward on the GPU against the fp64 oracle (needs a B200).

``ckda_sfda_fwd_chunked`` runs the chunk form of the SFDA recurrence
("Semidirect Fourier Delta Attention (SFDA)" summary, "Arquitectura Central"
and "El Teorema de Chunk-WY Constructivo"), the gate products being products
of the complex phase-decay scalars: on the tcgen05 pair for bf16 inputs with
d_k = 128, d_v in {64, 128}, chunk 64, on the fp32 CUDA-core kernel
otherwise.  The oracle it is compared with is pinned by ``pinlib_sfda``
(S-1..S-8).  Shapes span several chunks with ragged tails, every supported
head size (16 and 32 put one channel per lane, so the two halves of a pair
sit in neighbouring lanes) and chunk size, packed batches with empty
sequences, the full-size workload on sampled units, zero phases
(bit-identical to the CKDA kernel on the fp32 path; on the tensor-core path
equal up to the order of fp32 sums) and the constructed mod-5 counter.
"""
import math

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


def _run(ck, c, cu=None, out_dtype=torch.float32, S0="case", fp32core=False):
    S0 = c.S0 if isinstance(S0, str) else S0
    out, S = ck.sfda_fwd_chunked(c.q, c.k, c.v, c.alpha, c.extra["theta"], c.beta, S0=S0,
                                 cu_seqlens=cu, chunk=c.chunk, out_dtype=out_dtype,
                                 fp32core=fp32core)
    assert ck.device_status() == 0
    return out, S


def _oracle(c, S0="case", cu=None):
    S0 = c.S0 if isinstance(S0, str) else S0
    return oracle.forward_sfda(c.q, c.k, c.v, c.alpha, c.extra["theta"], c.beta, S0=S0,
                               cu_seqlens=cu)


@pytest.mark.parametrize("dk,dv", [(16, 16), (32, 32), (64, 64), (128, 128), (64, 128), (128, 32),
                                   (16, 64)])
@pytest.mark.parametrize("chunk", [16, 32, 64])
def test_fp32_matches_oracle(ck, dk, dv, chunk):
    c = inputs.sfda_prefill(2, 2 * chunk + 11, 2, dk, dv, dtype=torch.float32, s0_std=0.5,
                            chunk=chunk, seed=dk + 3 * dv + chunk, device=DEV)
    out, S = _run(ck, c)
    ro, rS = _oracle(c)
    assert rel_max_err(out, ro) <= TOL_F32 and rel_max_err(S, rS) <= TOL_F32


def test_bf16_inputs_match_oracle(ck):
    c = inputs.sfda_prefill(2, 300, 3, 128, 128, dtype=torch.bfloat16, s0_std=0.02, chunk=64,
                            seed=5, device=DEV)
    out, S = _run(ck, c, out_dtype=torch.float32)
    ro, rS = _oracle(c)
    assert rel_max_err(out, ro) <= TOL_BF16 and rel_max_err(S, rS) <= TOL_BF16
    # a bf16 output is exactly the bf16 rounding of the fp32 result
    o16, _ = _run(ck, c, out_dtype=torch.bfloat16)
    assert torch.equal(o16, out.to(torch.bfloat16))


def test_packed_batch_with_empty_sequences(ck):
    lens = [70, 0, 129, 1, 64, 0]
    total = int(sum(lens))
    c = inputs.sfda_prefill(1, total, 2, 64, 64, dtype=torch.float32, chunk=32, seed=9, device=DEV)
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32, device=DEV)
    g = torch.Generator(device=DEV).manual_seed(10)
    S0 = 0.3 * torch.randn(len(lens), 2, 64, 64, generator=g, device=DEV)
    out, S = _run(ck, c, cu=cu, S0=S0)
    ro, rS = _oracle(c, S0=S0, cu=cu)
    assert rel_max_err(out, ro) <= TOL_F32 and rel_max_err(S, rS) <= TOL_F32
    assert torch.equal(S[1], S0[1]) and torch.equal(S[5], S0[5])  # empty sequences


@pytest.mark.parametrize("dk", [16, 32, 64, 128])
def test_zero_phase_is_the_ckda_kernel_bit_for_bit(ck, dk):
    """theta = 0: every complex product has a zero imaginary part, and the
    kernel then performs the CKDA kernel's operations in the same order, with
    each decay on both rows of its pair."""
    c = inputs.sfda_prefill(2, 150, 2, dk, 64, dtype=torch.float32, s0_std=0.5, chunk=32,
                            seed=12 + dk, device=DEV)
    zero = torch.zeros_like(c.extra["theta"])
    o1, S1 = ck.sfda_fwd_chunked(c.q, c.k, c.v, c.alpha, zero, c.beta, S0=c.S0, chunk=32,
                                 out_dtype=torch.float32)
    a2 = c.alpha.repeat_interleave(2, dim=-1).contiguous()
    o2, S2 = ck.fwd_chunked(c.q, c.k, c.v, a2, c.beta, S0=c.S0, chunk=32, fp32core=True,
                            out_dtype=torch.float32)
    assert ck.device_status() == 0
    assert torch.equal(o1, o2) and torch.equal(S1, S2)


def test_phase_pi_is_a_negative_gate(ck):
    c = inputs.sfda_prefill(1, 200, 2, 64, 64, dtype=torch.float32, s0_std=0.5, chunk=64,
                            seed=21, device=DEV)
    pi = torch.full_like(c.extra["theta"], math.pi)
    o1, S1 = ck.sfda_fwd_chunked(c.q, c.k, c.v, c.alpha, pi, c.beta, S0=c.S0,
                                 out_dtype=torch.float32)
    ro, rS = oracle.forward(c.q, c.k, c.v, -c.alpha.repeat_interleave(2, dim=-1), c.beta, S0=c.S0)
    assert ck.device_status() == 0
    assert rel_max_err(o1, ro) <= TOL_F32 and rel_max_err(S1, rS) <= TOL_F32


@pytest.mark.parametrize("dt,d,tol", [(torch.float32, 16, 1e-4), (torch.bfloat16, 128, 2e-2)])
def test_constructed_mod5_counter(ck, dt, d, tol):
    """Phase-only counter in the first channel pair ("Resultados", constructed
    mod-5 counter): alpha = 1, beta = 0, theta = 2 pi x_t / 5 for input bits
    x_t; the read-out along e_0 is cos(2 pi count_t / 5) and the final state
    decodes count mod 5 exactly for lengths 27 to 213 (fp32 kernel at d = 16,
    tensor-core kernels at d = 128)."""
    dk = dv = d
    gen = torch.Generator().manual_seed(34)
    for L in (27, 100, 213):
        x = torch.randint(0, 2, (L,), generator=gen)
        theta = torch.zeros(1, L, 1, dk // 2)
        theta[0, :, 0, 0] = 2 * math.pi / 5 * x.float()
        alpha = torch.ones(1, L, 1, dk // 2)
        k = torch.zeros(1, L, 1, dk)
        k[..., 0] = 1.0
        S0 = torch.zeros(1, 1, dk, dv)
        S0[0, 0, 0, 0] = 1.0
        args = [t.to(DEV).contiguous() for t in (k.to(dt), k.to(dt), torch.zeros(1, L, 1, dv).to(dt),
                                                  alpha, theta, torch.zeros(1, L, 1), S0)]
        out, S = ck.sfda_fwd_chunked(*args[:6], S0=args[6], chunk=64, out_dtype=torch.float32)
        assert ck.device_status() == 0
        count = torch.cumsum(x, 0).double()
        o = out[0, :, 0, 0].double().cpu()
        assert float((o - torch.cos(2 * math.pi / 5 * count)).abs().max()) < tol
        ang = math.atan2(float(S[0, 0, 1, 0]), float(S[0, 0, 0, 0]))
        assert round(ang / (2 * math.pi / 5)) % 5 == int(count[-1]) % 5


def test_full_size_workload_on_sampled_units(ck):
    """The bench workload (B=4, T=4096, H=16, d=128, bf16), checked on four
    sampled (sequence, head) units against the oracle."""
    c = inputs.sfda_prefill(4, 4096, 16, 128, 128, dtype=torch.bfloat16, chunk=64, seed=0,
                            device=DEV)
    out, S = _run(ck, c)
    units = [(0, 0), (1, 7), (2, 15), (3, 3)]
    for b, h in units:
        sel = lambda x: x[b:b + 1, :, h:h + 1].cpu()  # noqa: E731
        ro, rS = oracle.forward_sfda(sel(c.q), sel(c.k), sel(c.v), sel(c.alpha),
                                     sel(c.extra["theta"]), sel(c.beta))
        assert rel_max_err(out[b:b + 1, :, h:h + 1], ro) <= TOL_BF16, (b, h)
        assert rel_max_err(S[b:b + 1, h:h + 1], rS) <= TOL_BF16, (b, h)


@pytest.mark.parametrize("dv", [64, 128])
@pytest.mark.parametrize("T", [64, 200])
def test_tensor_core_path_matches_oracle(ck, dv, T):
    assert ck.fwd_path(2, T, 3, 128, dv, 64, torch.bfloat16, torch.float32) == "tcgen05"
    c = inputs.sfda_prefill(2, T, 3, 128, dv, dtype=torch.bfloat16, s0_std=0.02, chunk=64,
                            seed=30 + T + dv, device=DEV)
    out, S = _run(ck, c)
    ro, rS = _oracle(c)
    assert rel_max_err(out, ro) <= TOL_BF16 and rel_max_err(S, rS) <= TOL_BF16
    o16, _ = _run(ck, c, out_dtype=torch.bfloat16)
    assert torch.equal(o16, out.to(torch.bfloat16))


def test_tensor_core_packed_batch(ck):
    lens = [65, 0, 130, 1, 191, 64, 0]
    total = int(sum(lens))
    c = inputs.sfda_prefill(1, total, 3, 128, 128, dtype=torch.bfloat16, chunk=64, seed=41,
                            device=DEV)
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32, device=DEV)
    assert ck.fwd_path(len(lens), total, 3, 128, 128, varlen=True) == "tcgen05"
    g = torch.Generator(device=DEV).manual_seed(42)
    S0 = 0.02 * torch.randn(len(lens), 3, 128, 128, generator=g, device=DEV)
    out, S = _run(ck, c, cu=cu, S0=S0)
    ro, rS = _oracle(c, S0=S0, cu=cu)
    assert rel_max_err(out, ro) <= TOL_BF16 and rel_max_err(S, rS) <= TOL_BF16
    assert torch.equal(S[1], S0[1]) and torch.equal(S[6], S0[6])  # empty sequences


@pytest.mark.parametrize("dv", [64, 128])
def test_tensor_core_zero_phase_matches_the_ckda_kernels(ck, dv):
    """theta = 0 on the tcgen05 pair: the complex gate products have zero
    imaginary parts and reduce to CKDA's real products, with each decay on
    both rows of its pair.  The SFDA factor kernel and the CKDA one sum their
    fp32 partial products in different orders, so the two results agree to
    the rounding of those sums (a few fp16 ulps of an operand), and each meets
    the oracle's bound."""
    c = inputs.sfda_prefill(2, 200, 3, 128, dv, dtype=torch.bfloat16, s0_std=0.02, chunk=64,
                            seed=50 + dv, device=DEV)
    zero = torch.zeros_like(c.extra["theta"])
    o1, S1 = ck.sfda_fwd_chunked(c.q, c.k, c.v, c.alpha, zero, c.beta, S0=c.S0,
                                 out_dtype=torch.float32)
    a2 = c.alpha.repeat_interleave(2, dim=-1).contiguous()
    o2, S2 = ck.fwd_chunked(c.q, c.k, c.v, a2, c.beta, S0=c.S0, out_dtype=torch.float32)
    assert ck.device_status() == 0
    assert rel_max_err(o1, o2.double().cpu().numpy()) <= 2e-3
    assert rel_max_err(S1, S2.double().cpu().numpy()) <= 2e-3
    c.extra["theta"] = zero
    ro, rS = _oracle(c)
    for o, S in ((o1, S1), (o2, S2)):
        assert rel_max_err(o, ro) <= TOL_BF16 and rel_max_err(S, rS) <= TOL_BF16


def test_tensor_core_agrees_with_the_fp32_kernel(ck):
    c = inputs.sfda_prefill(2, 300, 3, 128, 128, dtype=torch.bfloat16, s0_std=0.02, chunk=64,
                            seed=61, device=DEV)
    o1, S1 = _run(ck, c)
    o2, S2 = _run(ck, c, fp32core=True)
    ro, rS = _oracle(c)
    # the fp32 kernel is the closer of the two to the oracle; both pass the bar
    assert rel_max_err(o2, ro) <= TOL_F32 * 10 and rel_max_err(S2, rS) <= TOL_F32 * 10
    assert rel_max_err(o1, ro) <= TOL_BF16 and rel_max_err(S1, rS) <= TOL_BF16
    assert rel_max_err(o1, o2.double().cpu().numpy()) <= TOL_BF16


def test_tensor_core_large_phases(ck):
    """Phases far outside [-pi, pi]: |theta| up to about 5e3, and a quarter of
    the channel pairs beyond 1e5.  The factor kernel reduces each phase to
    [-pi, pi] before taking its sine and cosine (beyond 1e5 it uses the
    accurate library routine); the oracle evaluates cos and sin of the same
    fp32 phases in fp64."""
    c = inputs.sfda_prefill(2, 200, 3, 128, 128, dtype=torch.bfloat16, s0_std=0.02, chunk=64,
                            seed=71, device=DEV)
    g = torch.Generator(device=DEV).manual_seed(72)
    th = c.extra["theta"]
    turns = torch.randint(-800, 800, th.shape, generator=g, device=DEV).float()
    far = torch.randint(16000, 40000, th.shape, generator=g, device=DEV).float()
    beyond = torch.rand(th.shape, generator=g, device=DEV) < 0.25
    c.extra["theta"] = torch.where(beyond, th + 2 * math.pi * far,
                                   th + 2 * math.pi * turns).contiguous()
    assert float(c.extra["theta"].abs().max()) > 1e5
    out, S = _run(ck, c)
    ro, rS = _oracle(c)
    assert rel_max_err(out, ro) <= TOL_BF16 and rel_max_err(S, rS) <= TOL_BF16
