"""The fp64 oracle against facts fixed by the pages and by the mathematics.

Runs on the CPU only.  Every oracle function is pinned here:
``oracle.forward`` by P-1..P-12 (through ``pinlib.oracle_unit`` and the
batched checks below), ``oracle.decode_step`` by its agreement with
``forward`` on one token per sequence, ``oracle.chunked`` by P-5/P-6.
"""
import numpy as np
import pytest

import oracle
from oracle import chunked
import pinlib


@pytest.mark.parametrize("check", pinlib.ALL_CHECKS, ids=lambda c: c.__name__)
def test_oracle_pin(check):
    check(pinlib.oracle_unit)


def test_batched_layout_and_threads():
    """Units are independent: a [B, T, H, d] call equals per-unit calls, for any thread count."""
    rng = np.random.default_rng(0)
    B, T, H, dk, dv = 2, 13, 3, 4, 5
    q = rng.standard_normal((B, T, H, dk))
    k = rng.standard_normal((B, T, H, dk))
    v = rng.standard_normal((B, T, H, dv))
    a = rng.uniform(-1, 1, (B, T, H, dk))
    b = rng.uniform(0, 2, (B, T, H))
    S0 = rng.standard_normal((B, H, dk, dv))
    o1, S1 = oracle.forward(q, k, v, a, b, S0=S0, n_threads=1)
    o4, S4 = oracle.forward(q, k, v, a, b, S0=S0, n_threads=4)
    assert np.array_equal(o1, o4) and np.array_equal(S1, S4)
    for bb in range(B):
        for h in range(H):
            o, S = pinlib.oracle_unit(q[bb, :, h], k[bb, :, h], v[bb, :, h], a[bb, :, h],
                                      b[bb, :, h], S0[bb, h])
            assert np.array_equal(o, o1[bb, :, h]) and np.array_equal(S, S1[bb, h])


def test_packed_equals_fixed_length():
    rng = np.random.default_rng(1)
    lens = [5, 0, 9, 1]
    Tt, H, dk, dv = sum(lens), 2, 3, 4
    q = rng.standard_normal((Tt, H, dk))
    k = rng.standard_normal((Tt, H, dk))
    v = rng.standard_normal((Tt, H, dv))
    a = rng.uniform(-1, 1, (Tt, H, dk))
    b = rng.uniform(0, 2, (Tt, H))
    S0 = rng.standard_normal((len(lens), H, dk, dv))
    cu = np.concatenate([[0], np.cumsum(lens)])
    o, S = oracle.forward(q, k, v, a, b, S0=S0, cu_seqlens=cu)
    for n, L in enumerate(lens):
        sl = slice(cu[n], cu[n + 1])
        for h in range(H):
            on, Sn = pinlib.oracle_unit(q[sl, h], k[sl, h], v[sl, h], a[sl, h], b[sl, h], S0[n, h])
            assert np.array_equal(on, o[sl, h]) and np.array_equal(Sn, S[n, h])
    # a zero-length sequence keeps its initial state
    assert np.array_equal(S[1], S0[1])


def test_decode_step_is_one_token_forward():
    rng = np.random.default_rng(2)
    B, H, dk, dv = 3, 2, 4, 6
    q = rng.standard_normal((B, H, dk))
    k = rng.standard_normal((B, H, dk))
    v = rng.standard_normal((B, H, dv))
    a = rng.uniform(-1, 1, (B, H, dk))
    b = rng.uniform(0, 2, (B, H))
    S = rng.standard_normal((B, H, dk, dv))
    o, S1 = oracle.decode_step(q, k, v, a, b, S)
    o2, S2 = oracle.forward(q[:, None], k[:, None], v[:, None], a[:, None], b[:, None], S0=S)
    assert np.array_equal(o, o2[:, 0]) and np.array_equal(S1, S2)


def test_chunked_full_batch_matches_sequential():
    rng = np.random.default_rng(3)
    B, T, H, d = 1, 45, 2, 6
    q = rng.standard_normal((B, T, H, d))
    k = rng.standard_normal((B, T, H, d)) / np.sqrt(d)
    v = rng.standard_normal((B, T, H, d))
    a = rng.uniform(-1, 1, (B, T, H, d))
    a[0, 17:19] = 0.0
    b = rng.uniform(0, 2, (B, T, H))
    S0 = rng.standard_normal((B, H, d, d))
    o1, S1 = oracle.forward(q, k, v, a, b, S0=S0)
    for C in (1, 4, 16, 64):
        o2, S2 = chunked.forward(q, k, v, a, b, S0=S0, chunk=C)
        assert np.max(np.abs(o2 - o1)) <= 1e-12 and np.max(np.abs(S2 - S1)) <= 1e-12


def test_argument_errors():
    with pytest.raises(ValueError):
        oracle.forward(np.zeros((2, 3, 1, 2)), np.zeros((2, 3, 1, 2)), np.zeros((2, 3, 1, 2)),
                       np.zeros((2, 3, 1, 2)), np.zeros((2, 3, 1)), cu_seqlens=[0, 4, 3])
