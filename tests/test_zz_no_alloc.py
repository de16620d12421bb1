"""ckda_fwd_chunked_static: the chunked forward on the library's fixed device
scratch instead of a caller workspace (needs a B200).

The file is collected last so that it also runs after every other GPU test
(the scratch then holds whatever earlier calls left; nothing in it has to
start at zero).  Each check compares against ckda_fwd_chunked with a
caller-owned workspace on the same inputs, bit for bit, over two calls in a
row with different inputs and sizes.
"""
import pytest
import torch

from delta_rule_linear_ckda_b200 import _lib, inputs

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module")
def ck():
    import delta_rule_linear_ckda_b200 as ck

    return ck


def _case(B, T, H, seed, dv=128):
    return inputs.random_prefill(B, T, H, 128, dv, dtype=torch.bfloat16, gates="kda", s0_std=0.02,
                                 chunk=64, seed=seed, device=DEV)


@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_two_calls_in_a_row_match_the_workspace_entry(ck, out_dtype):
    cases = [_case(2, 300, 4, seed=1), _case(1, 2048, 16, seed=2)]  # 40 and 512 units
    for c in cases:
        assert ck.workspace_bytes(*c.q.shape[:3], 128, 128) <= _lib.CKDA_STATIC_SCRATCH_BYTES
    got = [ck.fwd_chunked_static(c.q, c.k, c.v, c.alpha, c.beta, S0=c.S0, out_dtype=out_dtype)
           for c in cases]
    ref = [ck.fwd_chunked(c.q, c.k, c.v, c.alpha, c.beta, S0=c.S0, out_dtype=out_dtype)
           for c in cases]
    assert ck.device_status() == 0
    for (o, S), (ro, rS) in zip(got, ref):
        assert torch.equal(o, ro)
        assert torch.equal(S, rS)


def test_packed_batch_and_d_v_64(ck):
    c = _case(1, 400, 3, seed=3, dv=64)
    cu = torch.tensor([0, 130, 130, 400], dtype=torch.int32, device=DEV)
    S0 = torch.zeros(3, 3, 128, 64, device=DEV)
    for _ in range(2):
        o, S = ck.fwd_chunked_static(c.q, c.k, c.v, c.alpha, c.beta, S0=S0, cu_seqlens=cu,
                                     out_dtype=torch.float32)
        ro, rS = ck.fwd_chunked(c.q, c.k, c.v, c.alpha, c.beta, S0=S0, cu_seqlens=cu,
                                out_dtype=torch.float32)
        assert ck.device_status() == 0
        assert torch.equal(o, ro) and torch.equal(S, rS)


def test_sizes_beyond_the_scratch_are_rejected(ck):
    c = _case(1, 64, 1, seed=4)
    # 4 * 64 * 16 units need 271 MB: refused before any launch
    big_T = 4096
    assert ck.workspace_bytes(4, big_T, 16, 128, 128) > _lib.CKDA_STATIC_SCRATCH_BYTES
    rc = _lib.load().ckda_fwd_chunked_static(
        c.q.data_ptr(), c.k.data_ptr(), c.v.data_ptr(), c.alpha.data_ptr(), c.beta.data_ptr(),
        None, None, c.v.data_ptr() + 4096 * 1024, None, 4, big_T, 16, 128, 128, 64, 1, 0, None)
    assert rc == -2
