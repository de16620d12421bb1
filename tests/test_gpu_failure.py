"""Failure detection on the GPU without faulting it.

The bounded device-side wait gives up after its limit, records
CKDA_ERR_DEVICE_TIMEOUT in the status word and returns; the host reads the
status, the context stays usable and later work is unaffected.
"""
import time

import pytest
import torch

from delta_rule_linear_ckda_b200 import inputs

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_reports():
    import delta_rule_linear_ckda_b200 as ck
    from delta_rule_linear_ckda_b200 import _lib

    lib = _lib.load()
    assert ck.device_status() == 0
    t0 = time.perf_counter()
    assert lib.ckda_selftest_bounded_wait(50_000, None) == 0  # 50 ms
    assert ck.device_status() == -5  # CKDA_ERR_DEVICE_TIMEOUT, read and cleared
    elapsed = time.perf_counter() - t0
    assert 0.04 <= elapsed < 5.0
    assert ck.device_status() == 0
    # the context is still usable: a normal call afterwards succeeds
    case = inputs.tiny(seed=0, device="cuda")
    out, S = ck.fwd_chunked(case.q, case.k, case.v, case.alpha, case.beta, chunk=16)
    assert ck.device_status() == 0 and torch.isfinite(out).all()
