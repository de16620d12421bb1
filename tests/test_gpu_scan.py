"""The chunk-parallel scan forward on the GPU (needs a B200).

``ckda_fwd_chunked_scan`` splits each sequence's chunks into segments,
forms every segment's affine summary [M | B] in parallel, scans the segment
start states (S_start(g + 1) = M_g S_start(g) + B_g, "Semidirect Fourier
Delta Attention" page, "Principales Contribuciones" item 3) and runs every
segment's carry in parallel.  Checked against the fp64 oracle (pinned by
``pinlib``) at the bf16 bar, against the plain forward, with one segment
(bit-identical to the plain forward), more segments than chunks (empty
segments), ragged last chunks, and the long-context size on sampled heads.
"""
import pytest
import torch

from delta_rule_linear_ckda_b200 import inputs
from gpu_util import TOL_BF16, oracle_fixed, rel_max_err

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module")
def ck():
    import delta_rule_linear_ckda_b200 as ck

    return ck


def _case(B, T, H, dv, seed):
    return inputs.random_prefill(B, T, H, 128, dv, dtype=torch.bfloat16, gates="kda", s0_std=0.02,
                                 chunk=64, seed=seed, device=DEV)


@pytest.mark.parametrize("dv", [64, 128])
@pytest.mark.parametrize("G", [2, 3, 5, 8])
def test_scan_matches_oracle_and_plain_forward(ck, dv, G):
    c = _case(2, 300, 3, dv, seed=G + dv)  # 5 chunks, the last one ragged
    out, S = ck.fwd_chunked_scan(c.q, c.k, c.v, c.alpha, c.beta, G, S0=c.S0,
                                 out_dtype=torch.float32)
    assert ck.device_status() == 0
    ro, rS, _, _ = oracle_fixed(c)
    assert rel_max_err(out, ro) <= TOL_BF16 and rel_max_err(S, rS) <= TOL_BF16
    o1, S1 = ck.fwd_chunked(c.q, c.k, c.v, c.alpha, c.beta, S0=c.S0, out_dtype=torch.float32)
    # the two orders of rounding agree far inside the bar
    assert rel_max_err(out, o1.double().cpu().numpy()) <= 5e-3
    assert rel_max_err(S, S1.double().cpu().numpy()) <= 5e-3


def test_one_segment_is_the_plain_forward(ck):
    c = _case(2, 200, 2, 128, seed=3)
    o1, S1 = ck.fwd_chunked(c.q, c.k, c.v, c.alpha, c.beta, S0=c.S0, out_dtype=torch.float32)
    o2, S2 = ck.fwd_chunked_scan(c.q, c.k, c.v, c.alpha, c.beta, 1, S0=c.S0,
                                 out_dtype=torch.float32)
    assert ck.device_status() == 0
    assert torch.equal(o1, o2) and torch.equal(S1, S2)


def test_bf16_output_and_no_initial_state(ck):
    c = _case(1, 640, 2, 128, seed=4)
    out, S = ck.fwd_chunked_scan(c.q, c.k, c.v, c.alpha, c.beta, 4, out_dtype=torch.float32)
    o16, _ = ck.fwd_chunked_scan(c.q, c.k, c.v, c.alpha, c.beta, 4, out_dtype=torch.bfloat16)
    assert ck.device_status() == 0
    assert torch.equal(o16, out.to(torch.bfloat16))
    case0 = inputs.PrefillCase("no S0", c.q, c.k, c.v, c.alpha, c.beta, None, None, 64)
    ro, rS, _, _ = oracle_fixed(case0)
    assert rel_max_err(out, ro) <= TOL_BF16 and rel_max_err(S, rS) <= TOL_BF16


def test_long_context_on_sampled_heads(ck):
    """The long-context size (B=1, T=65536, H=32) split in 4 segments, checked
    on two sampled heads against the oracle."""
    c = inputs.long_prefill(seed=0, device=DEV)
    out, S = ck.fwd_chunked_scan(c.q, c.k, c.v, c.alpha, c.beta, 4, S0=c.S0,
                                 out_dtype=torch.float32)
    assert ck.device_status() == 0
    ro, rS, bi, hi = oracle_fixed(c, b_idx=[0], h_idx=[0, 31])
    got = out.cpu()[bi][:, :, hi]
    assert rel_max_err(got, ro) <= TOL_BF16
    assert rel_max_err(S.cpu()[bi][:, hi], rS) <= TOL_BF16
