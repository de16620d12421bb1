"""Repeated calls give bit-identical results on the tensor-core path (needs a
B200).

The carry kernel's warps hand every chunk on through mbarriers (state
warps, an MMA thread, a copy thread, V-conversion warps); the kernels use
no atomics and fixed summation orders, so the same inputs must give the
same bits on every call.  A missing or misplaced handoff would show up as a
call that differs from the others.  Each case runs many chunks per
(sequence, head): fixed-length 64- and 32-column slices, a packed batch with
partial chunks, and the two gate variants.
"""
import numpy as np
import pytest
import torch

from delta_rule_linear_ckda_b200 import inputs

pytestmark = pytest.mark.gpu
DEV = "cuda"
CALLS = 4


@pytest.fixture(scope="module")
def ck():
    import delta_rule_linear_ckda_b200 as ck

    return ck


def _same_every_call(ck, fn):
    first = [t.clone() for t in fn()]
    assert ck.device_status() == 0
    for _ in range(CALLS - 1):
        again = fn()
        assert ck.device_status() == 0
        for a, b in zip(first, again):
            assert torch.equal(a, b)


@pytest.mark.parametrize("B,H", [(4, 16), (1, 8)])  # 64-column slices; 32-column slices
def test_fixed_length_forward_is_deterministic(ck, B, H):
    c = inputs.kda_prefill(seed=81, device=DEV, B=B, T=2048, H=H)
    assert ck.fwd_path(B, 2048, H, 128, 128, 64, torch.bfloat16, torch.float32) == "tcgen05"
    _same_every_call(ck, lambda: ck.fwd_chunked(c.q, c.k, c.v, c.alpha, c.beta, chunk=64,
                                                out_dtype=torch.float32))


def test_packed_forward_is_deterministic(ck):
    lens = np.random.default_rng(82).integers(1, 700, size=40)
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32, device=DEV)
    total = int(cu[-1])
    c = inputs.kda_prefill(seed=83, device=DEV, B=1, T=total, H=8)
    _same_every_call(ck, lambda: ck.fwd_chunked(c.q, c.k, c.v, c.alpha, c.beta, cu_seqlens=cu,
                                                chunk=64, out_dtype=torch.float32))


def test_gate_variants_are_deterministic(ck):
    g = inputs.gdn2_prefill(2, 1024, 8, 128, 128, dtype=torch.bfloat16, chunk=64, seed=84,
                            device=DEV)
    _same_every_call(ck, lambda: ck.gdn2_fwd_chunked(g.q, g.k, g.v, g.alpha, g.extra["b"],
                                                     g.extra["w"], chunk=64))
    s = inputs.sfda_prefill(2, 1024, 8, 128, 128, dtype=torch.bfloat16, chunk=64, seed=85,
                            device=DEV)
    _same_every_call(ck, lambda: ck.sfda_fwd_chunked(s.q, s.k, s.v, s.alpha, s.extra["theta"],
                                                     s.beta, chunk=64))
