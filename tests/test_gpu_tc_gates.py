"""Gate extremes on the tensor-core forward (bf16 inputs, d = 128, C = 64).

The CKDA gates range over alpha in [-1, 1] per channel and beta in [0, 2]
("Complex KDA: Kimi Delta Attention ..." page, section "Complex KDA (CKDA)
Mimarisi ve Parametre Genişlemesi"), so gate products can be zero, negative
or far below fp16's smallest normal number (6.1e-5).  The tcgen05 kernels
keep the anchored gate products, the WY factors and the state operand in
fp16, which is where such gates could go wrong.  Every case here runs on
that path (asserted through ``fwd_path``) and is compared element by element
with the fp64 oracle at the bf16-input bound (2e-2 of max|err| / rms, on o
and on S_final):

* alpha = 0 everywhere: every product that spans a position is zero; the
  result also has a closed form, o_t = beta_t (k_t . q_t) v_t;
* alpha_i = +-1 with beta = 2 (orthogonal transitions), with v = 0 (the
  state's norm moves only through ||k|| != 1 in bf16, exactly as in the
  oracle) and with v != 0;
* alpha ~ U[-1, 1], beta ~ U[0, 2];
* alpha ~ U[-0.05, 0.05]: products fall below fp16's range within a few
  positions;
* occasional alpha ~ U[-1e-3, 1e-3] among |alpha| in [0.9, 1]: chunks whose
  products are normal, subnormal or zero in fp16 side by side;
* the gate-extreme workload (near-zero gates in the first half of each
  sequence, orthogonal transitions in the second) cast to bf16, fixed-length
  and packed: 64 packed sequences of 128 to 1024 tokens on sampled units.

Orthogonal transitions never damp an error, so the fp16 rounding of the WY
factors, the state operand and U adds up as a random walk over a run of
them: up to runs of about 1000 orthogonal tokens the error stays near
1.5e-2, and the full gate-extreme lengths (runs of up to 2048 such tokens
in sequences of up to 4096) reach 2.9e-2 on o.  The fp32-input form of that
workload runs on the fp32 kernel and meets 1e-4.
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


def _on_tensor_cores(ck, case, varlen=False):
    B, T, H, dk = case.q.shape
    n = case.n_seqs if varlen else B
    return ck.fwd_path(n, T, H, dk, case.dv, case.chunk, case.q.dtype, torch.float32,
                       varlen=varlen) == "tcgen05"


def _check(ck, case):
    assert _on_tensor_cores(ck, case)
    out, S = ck.fwd_chunked(case.q, case.k, case.v, case.alpha, case.beta, S0=case.S0,
                            chunk=case.chunk, out_dtype=torch.float32)
    assert ck.device_status() == 0
    assert torch.isfinite(out).all() and torch.isfinite(S).all()
    ro, rS, _, _ = oracle_fixed(case)
    eo, es = rel_max_err(out, ro), rel_max_err(S, rS)
    print(f"{case.name}: err o {eo:.2e}  S {es:.2e}")
    assert eo <= TOL_BF16 and es <= TOL_BF16, (case.name, eo, es)
    return out, S, rS


@pytest.mark.parametrize("kind", ["zero", "reflect", "uniform", "tiny", "underflow"])
@pytest.mark.parametrize("s0_std", [0.0, 0.5])
def test_gate_extremes_vs_oracle(ck, kind, s0_std):
    # 5 chunks and a ragged tail of 13 tokens, three sequences, four heads
    case = inputs.gate_extremes(3, 5 * 64 + 13, 4, 128, kind=kind, s0_std=s0_std,
                                seed=100 + len(kind), device=DEV)
    _check(ck, case)


def test_alpha_zero_closed_form_tensor_cores(ck):
    case = inputs.gate_extremes(2, 200, 4, 128, kind="zero", s0_std=1.0, seed=7, device=DEV)
    out, S, _ = _check(ck, case)
    q, k, v = (x.double() for x in (case.q, case.k, case.v))
    b = case.beta.double()
    expect = b.unsqueeze(-1) * (k * q).sum(-1, keepdim=True) * v
    assert rel_max_err(out, expect.cpu().numpy()) <= TOL_BF16
    expect_S = b[:, -1, :, None, None] * k[:, -1, :, :, None] * v[:, -1, :, None, :]
    assert rel_max_err(S, expect_S.cpu().numpy()) <= TOL_BF16


def test_orthogonal_transitions_keep_the_state_norm(ck):
    # v = 0 and beta = 2, alpha_i = +-1: each transition is orthogonal up to
    # ||k||^2 - 1 (k is rounded to bf16), so ||S_T|| / ||S_0|| is what the
    # oracle gives on the same inputs
    case = inputs.gate_extremes(2, 8 * 64 + 29, 4, 128, kind="orthogonal", s0_std=1.0, seed=8,
                                device=DEV)
    _, S, rS = _check(ck, case)
    n0 = case.S0.double().flatten(2).norm(dim=-1).cpu().numpy()
    got = S.double().flatten(2).norm(dim=-1).cpu().numpy() / n0
    ref = np.linalg.norm(rS.reshape(rS.shape[0], rS.shape[1], -1), axis=-1) / n0
    print("norm ratio: gpu - 1 in", float(np.min(got - 1)), float(np.max(got - 1)),
          "| gpu - oracle max", float(np.max(np.abs(got - ref))))
    assert np.all(np.abs(got - ref) <= TOL_BF16 * ref), float(np.max(np.abs(got - ref)))


def test_halves_fixed_length(ck):
    case = inputs.gate_extremes(4, 3 * 64 + 40, 4, 128, kind="halves", seed=9, device=DEV)
    _, S, rS = _check(ck, case)
    # the orthogonal second halves keep the norm reached after the first halves
    Th = case.q.shape[1] // 2
    first = [x[:, :Th].contiguous() for x in (case.q, case.k, case.v, case.alpha, case.beta)]
    _, S_half = ck.fwd_chunked(*first, chunk=case.chunk, out_dtype=torch.float32)
    ratio = (S.double().flatten(2).norm(dim=-1) / S_half.double().flatten(2).norm(dim=-1))
    ratio = ratio.cpu().numpy()
    print("halves norm ratio - 1 in", float(ratio.min() - 1), float(ratio.max() - 1))
    ref_ratio = np.linalg.norm(rS.reshape(rS.shape[0], rS.shape[1], -1), axis=-1) / \
        S_half.double().flatten(2).norm(dim=-1).cpu().numpy()
    assert np.all(np.abs(ratio - ref_ratio) <= TOL_BF16 * ref_ratio)


def test_gate_extreme_varlen_bf16_packed_small(ck):
    case = inputs.varlen(seed=1, device=DEV, n_seqs=6, lmin=1, lmax=700, H=4, dtype=torch.bfloat16)
    assert _on_tensor_cores(ck, case, varlen=True)
    out, S = ck.fwd_chunked(case.q, case.k, case.v, case.alpha, case.beta,
                            cu_seqlens=case.cu_seqlens, chunk=case.chunk, out_dtype=torch.float32)
    assert ck.device_status() == 0
    assert torch.isfinite(out).all() and torch.isfinite(S).all()
    ro, rS, tok, _ = oracle_packed(case)
    eo, es = rel_max_err(out.cpu()[0][tok], ro), rel_max_err(S, rS)
    print(f"{case.name}: err o {eo:.2e}  S {es:.2e}")
    assert eo <= TOL_BF16 and es <= TOL_BF16, (eo, es)


def test_gate_extreme_varlen_bf16_sampled(ck):
    # 64 packed sequences, L ~ U[128, 1024]: orthogonal runs of up to 512 tokens
    case = inputs.varlen(seed=0, device=DEV, lmax=1024, dtype=torch.bfloat16)
    assert _on_tensor_cores(ck, case, varlen=True)
    out, S = ck.fwd_chunked(case.q, case.k, case.v, case.alpha, case.beta,
                            cu_seqlens=case.cu_seqlens, chunk=case.chunk, out_dtype=torch.float32)
    assert ck.device_status() == 0
    assert torch.isfinite(out).all() and torch.isfinite(S).all()
    seqs = [0, 7, 31, 63]
    ro, rS, tok, hi = oracle_packed(case, seqs, [0, 15])
    got_o = out.cpu()[0][tok][:, hi]
    got_S = S.cpu()[torch.tensor(seqs)][:, hi]
    eo, es = rel_max_err(got_o, ro), rel_max_err(got_S, rS)
    print(f"{case.name}: err o {eo:.2e}  S {es:.2e}")
    assert eo <= TOL_BF16 and es <= TOL_BF16, (eo, es)
    half = inputs.first_halves(case)
    _, S_half = ck.fwd_chunked(half.q, half.k, half.v, half.alpha, half.beta,
                               cu_seqlens=half.cu_seqlens, chunk=half.chunk)
    ratio = (S.double().flatten(2).norm(dim=-1) / S_half.double().flatten(2).norm(dim=-1))
    ratio = ratio.cpu().numpy()
    print("orthogonal halves: norm ratio - 1 in", float(ratio.min() - 1), float(ratio.max() - 1))
    assert np.all(np.isfinite(ratio))
