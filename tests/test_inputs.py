"""The seeded input recipes on CPU.

Each workload's generator must give the stated shapes and dtypes, values in
the stated ranges with the stated distributions and structure, and the same
tensors for the same seed. Every parity test and bench line is built on
these inputs, so a drift here would change what all of them measure without
failing any of them.
"""
import math

import pytest
import torch

from delta_rule_linear_ckda_b200 import inputs


def _unit_norm(x, tol):
    n = x.float().norm(dim=-1)
    return bool(torch.all((n - 1).abs() <= tol))


def test_tiny_recipe():
    c = inputs.tiny(seed=0)
    assert c.q.shape == (1, 64, 2, 16) and c.v.shape == (1, 64, 2, 16)
    assert c.q.dtype == torch.float32 and c.chunk == 16 and c.S0 is None
    assert _unit_norm(c.q, 1e-5) and _unit_norm(c.k, 1e-5)
    assert c.alpha.min() >= -1 and c.alpha.max() <= 1
    assert c.beta.min() >= 0 and c.beta.max() <= 2


def test_kda_prefill_recipe_on_a_reduced_size():
    # the same draws as the full size, on a shape the CPU finishes at once
    c = inputs.kda_prefill(seed=0, B=2, T=2048, H=4, d=128)
    assert c.q.dtype == torch.bfloat16 and c.v.dtype == torch.bfloat16
    assert c.alpha.dtype == torch.float32 and c.beta.dtype == torch.float32
    assert c.alpha.shape == (2, 2048, 4, 128) and c.beta.shape == (2, 2048, 4)
    assert _unit_norm(c.q, 1e-2) and _unit_norm(c.k, 1e-2)  # normalised in fp32, then bf16
    a = c.alpha
    # alpha = s * sigmoid(-x): |alpha| in (0, 1), negative with probability 0.25
    assert a.abs().max() < 1 and a.abs().min() > 0
    neg = (a < 0).float().mean().item()
    assert abs(neg - 0.25) < 0.01, neg
    # |alpha| = sigmoid(-x), x ~ N(0, 1): median 1/2, mean 1/2 by symmetry
    assert abs(a.abs().median().item() - 0.5) < 0.01
    # beta = 2 sigmoid(z), z ~ N(0, 1): in (0, 2), median 1
    b = c.beta
    assert b.min() > 0 and b.max() < 2 and abs(b.median().item() - 1.0) < 0.02
    # v ~ N(0, 1)
    v = c.v.float()
    assert abs(v.mean().item()) < 0.01 and abs(v.std().item() - 1) < 0.01


def test_long_prefill_state_and_shape():
    c = inputs.long_prefill(seed=0, T=4096, H=2)
    assert c.q.shape == (1, 4096, 2, 128) and c.S0.shape == (1, 2, 128, 128)
    assert abs(c.S0.std().item() - 0.02) < 0.001 and abs(c.S0.mean().item()) < 0.001


def test_decode_recipe_on_a_reduced_size():
    c = inputs.decode(seed=0, B=16, H=4, d=128, steps=8)
    assert c.q.shape == (8, 16, 4, 128) and c.S0.shape == (16, 4, 128, 128)
    assert c.q.dtype == torch.bfloat16 and c.alpha.dtype == torch.float32
    assert _unit_norm(c.q, 1e-2) and _unit_norm(c.k, 1e-2)
    assert c.alpha.min() >= -1 and c.alpha.max() <= 1
    assert abs(c.alpha.mean().item()) < 0.02  # U[-1, 1]
    assert c.beta.min() >= 0 and c.beta.max() <= 2
    assert abs(c.S0.std().item() - 0.02) < 0.001


def test_varlen_structure():
    c = inputs.varlen(seed=0, n_seqs=6, lmin=128, lmax=512, H=2, d=32)
    lens = c.extra["lengths"]
    cu = c.cu_seqlens.to(torch.int64)
    assert cu[0] == 0 and torch.equal(cu[1:] - cu[:-1], lens)
    assert int(lens.min()) >= 128 and int(lens.max()) <= 512
    for i in range(lens.numel()):
        b, e = int(cu[i]), int(cu[i + 1])
        half = (e - b) // 2
        a0, a1 = c.alpha[0, b:b + half], c.alpha[0, b + half:e]
        # near-zero gates first, with beta ~ U[0, 2] and v ~ N(0, 1)
        assert a0.abs().max() <= 0.05
        assert c.beta[0, b:b + half].min() >= 0 and c.beta[0, b:b + half].max() <= 2
        assert c.v[0, b:b + half].abs().max() > 0
        # then orthogonal transitions: alpha_i = +-1, beta = 2, v = 0
        assert torch.all(a1.abs() == 1)
        assert torch.all(c.beta[0, b + half:e] == 2)
        assert torch.all(c.v[0, b + half:e] == 0)
    assert _unit_norm(c.k, 1e-5)
    sub = inputs.first_halves(c)
    assert torch.equal(sub.extra["lengths"], lens // 2)
    assert sub.alpha.abs().max() <= 0.05


@pytest.mark.parametrize("make", [
    lambda s: inputs.tiny(seed=s),
    lambda s: inputs.kda_prefill(seed=s, B=1, T=128, H=2, d=64),
    lambda s: inputs.decode(seed=s, B=2, H=2, d=32, steps=3),
    lambda s: inputs.varlen(seed=s, n_seqs=3, lmin=16, lmax=40, H=2, d=16),
    lambda s: inputs.gdn2_prefill(1, 70, 2, 32, 16, seed=s),
    lambda s: inputs.sfda_prefill(1, 70, 2, 32, 16, seed=s),
])
def test_same_seed_same_tensors_other_seed_other_tensors(make):
    a, b, c = make(3), make(3), make(4)
    assert torch.equal(a.q, b.q) and torch.equal(a.alpha, b.alpha)
    assert not torch.equal(a.q, c.q)


def test_variant_gate_recipes():
    g = inputs.gdn2_prefill(2, 300, 2, 64, 32, seed=1)
    assert g.beta is None
    assert g.extra["b"].shape == g.k.shape and g.extra["w"].shape == g.v.shape
    for t in (g.extra["b"], g.extra["w"]):
        assert t.min() > 0 and t.max() < 1 and abs(t.median().item() - 0.5) < 0.03
    s = inputs.sfda_prefill(2, 300, 2, 64, 32, seed=1)
    assert s.alpha.shape == (2, 300, 2, 32) and s.extra["theta"].shape == (2, 300, 2, 32)
    assert s.alpha.min() > 0 and s.alpha.max() < 1
    th = s.extra["theta"]
    assert th.min() >= -math.pi and th.max() < math.pi
    assert abs(th.mean().item()) < 0.1  # U[-pi, pi)
    assert s.beta.min() > 0 and s.beta.max() < 2
