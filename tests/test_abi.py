"""The C-ABI library loads and exports every symbol its header declares.

CPU only: argument errors are rejected on the host before any CUDA call, so
these calls launch nothing and need no GPU.
"""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER_DIR = os.path.join(ROOT, "include")


@pytest.fixture(scope="module")
def lib():
    from delta_rule_linear_ckda_b200 import build as b

    b.build()
    from delta_rule_linear_ckda_b200 import _lib

    return _lib.load()


def declared_symbols():
    names = []
    for fn in sorted(os.listdir(HEADER_DIR)):
        if fn.endswith(".h"):
            text = open(os.path.join(HEADER_DIR, fn)).read()
            names += re.findall(r"CKDA_API\s+[\w\s\*]+?\b(ckda_\w+)\s*\(", text)
    return names


def test_header_declares_entry_points():
    names = declared_symbols()
    for required in ("ckda_fwd_chunked", "ckda_fwd_chunked_workspace_bytes", "ckda_fwd_factors",
                     "ckda_fwd_carry", "ckda_decode_step", "ckda_status_string",
                     "ckda_device_status"):
        assert required in names


def test_every_declared_symbol_is_exported(lib):
    from delta_rule_linear_ckda_b200._lib import LIB_PATH, SIGNATURES

    out = subprocess.run(["nm", "-D", "--defined-only", LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT\s+(ckda_\w+)", out))
    for name in declared_symbols():
        assert name in exported, name
        assert hasattr(lib, name)
        assert name in SIGNATURES, f"binding lacks a signature for {name}"


def test_library_has_no_runtime_dependency_on_libcudart():
    from delta_rule_linear_ckda_b200._lib import LIB_PATH

    out = subprocess.run(["ldd", LIB_PATH], capture_output=True, text=True).stdout
    assert "libcudart" not in out


def test_status_strings(lib):
    for code in (0, -1, -2, -3, -4, -5, -6, -7):
        s = lib.ckda_status_string(code)
        assert s and b"unknown" not in s
    assert lib.ckda_status_string(-99) == b"unknown status"
    assert lib.ckda_version() >= 100


# Fake, never-dereferenced "device" addresses: validation rejects the call
# before any CUDA call is made.
P = 1 << 20          # 16-byte aligned
MIS = (1 << 20) + 4  # misaligned


def fwd(lib, **kw):
    a = dict(q=P, k=P + 0x1000, v=P + 0x2000, alpha=P + 0x3000, beta=P + 0x4000, S0=None,
             cu=None, out=P + 0x5000, S_final=None, B=1, T=8, H=1, dk=16, dv=16, chunk=16,
             dtype=0, out_dtype=0, ws=None, ws_bytes=0, stream=None)
    a.update(kw)
    return lib.ckda_fwd_chunked(a["q"], a["k"], a["v"], a["alpha"], a["beta"], a["S0"], a["cu"],
                                a["out"], a["S_final"], a["B"], a["T"], a["H"], a["dk"], a["dv"],
                                a["chunk"], a["dtype"], a["out_dtype"], a["ws"], a["ws_bytes"],
                                a["stream"])


def test_fwd_argument_errors(lib):
    assert fwd(lib, q=None) == -1
    assert fwd(lib, beta=None) == -1
    assert fwd(lib, out=None) == -1
    assert fwd(lib, B=-1) == -1
    assert fwd(lib, H=0) == -1
    assert fwd(lib, T=-3) == -1
    assert fwd(lib, dk=48) == -2
    assert fwd(lib, dv=256) == -2
    assert fwd(lib, chunk=128) == -2
    assert fwd(lib, chunk=8) == -2
    assert fwd(lib, dtype=7) == -2
    assert fwd(lib, out_dtype=2) == -2
    assert fwd(lib, q=MIS) == -3
    assert fwd(lib, S_final=MIS) == -3
    assert fwd(lib, out=P) == -1        # out aliases q
    assert fwd(lib, cu=P + 0x9002) == -3  # cu_seqlens must be 4-byte aligned
    # packed batch with no sequences but tokens
    assert fwd(lib, cu=P + 0x9000, B=0, T=5) == -1


def test_fwd_fp32core_shares_validation(lib):
    r = lib.ckda_fwd_chunked_fp32core(None, P, P, P, P, None, None, P + 16, None, 1, 8, 1, 16, 16,
                                      16, 0, 0, None)
    assert r == -1


def test_decode_argument_errors(lib):
    def dec(**kw):
        a = dict(q=P, k=P + 0x1000, v=P + 0x2000, alpha=P + 0x3000, beta=P + 0x4000,
                 S=P + 0x5000, out=P + 0x6000, B=2, H=2, dk=16, dv=16, dtype=1, out_dtype=0)
        a.update(kw)
        return lib.ckda_decode_step(a["q"], a["k"], a["v"], a["alpha"], a["beta"], a["S"], a["out"],
                                    a["B"], a["H"], a["dk"], a["dv"], a["dtype"], a["out_dtype"],
                                    None)

    assert dec(S=None) == -1
    assert dec(H=0) == -1
    assert dec(dk=24) == -2
    assert dec(dtype=3) == -2
    assert dec(out_dtype=-1) == -2
    assert dec(alpha=MIS) == -3
    assert dec(out=P + 0x5000) == -1   # out aliases the state
    assert dec(B=0) == 0               # nothing to do, nothing launched


def test_zero_sequences_is_a_no_op(lib):
    assert fwd(lib, B=0) == 0


def test_path_query_needs_no_gpu(lib):
    F32, BF16 = 0, 1
    assert lib.ckda_fwd_chunked_path(4, 4096, 16, 128, 128, 64, BF16, F32, 0) == 1
    assert lib.ckda_fwd_chunked_path(1, 65536, 32, 128, 128, 0, BF16, BF16, 0) == 1
    assert lib.ckda_fwd_chunked_path(64, 135000, 16, 128, 128, 64, BF16, F32, 1) == 1
    assert lib.ckda_fwd_chunked_path(4, 4096, 16, 128, 64, 64, BF16, F32, 0) == 1
    assert lib.ckda_fwd_chunked_path(4, 4096, 16, 128, 128, 64, F32, F32, 0) == 0   # fp32 inputs
    assert lib.ckda_fwd_chunked_path(4, 4096, 16, 128, 128, 32, BF16, F32, 0) == 0  # chunk 32
    assert lib.ckda_fwd_chunked_path(4, 4096, 16, 64, 64, 64, BF16, F32, 0) == 0    # d_k 64
    assert lib.ckda_fwd_chunked_path(4, 0, 16, 128, 128, 64, BF16, F32, 0) == 0     # no tokens
    assert lib.ckda_fwd_chunked_path(4, 4096, 16, 128, 128, 48, BF16, F32, 0) == -2
    assert lib.ckda_fwd_chunked_path(4, 4096, 0, 128, 128, 64, BF16, F32, 0) == -1


def test_selftest_rejects_bad_limits(lib):
    assert lib.ckda_selftest_bounded_wait(0, None) == -1
    assert lib.ckda_selftest_bounded_wait(20000000, None) == -1


# per (chunk, head) unit: [-W; Q'] and K*rho (fp16), [Inv diag(beta); P] (fp16), gamma (fp32);
# the same for every d_v (V is read from the input by the carry kernel)
UNIT_BYTES = 2 * 64 * 128 * 2 + 64 * 128 * 2 + 2 * 64 * 64 * 2 + 128 * 4


def test_workspace_size_query_needs_no_gpu(lib):
    F32, BF16 = 0, 1
    q = lib.ckda_fwd_chunked_workspace_bytes
    # fixed-length: B * ceil(T / 64) * H units
    assert q(4, 4096, 16, 128, 128, 64, BF16, F32, 0) == 4 * 64 * 16 * UNIT_BYTES
    assert q(2, 100, 3, 128, 128, 64, BF16, F32, 0) == 2 * 2 * 3 * UNIT_BYTES
    assert q(1, 64, 1, 128, 64, 0, BF16, BF16, 0) == UNIT_BYTES
    # packed: (floor(T / 64) + N) * H units
    assert q(5, 1000, 2, 128, 128, 64, BF16, F32, 1) == (1000 // 64 + 5) * 2 * UNIT_BYTES
    # the CUDA-core path needs none
    assert q(4, 4096, 16, 128, 128, 64, F32, F32, 0) == 0
    assert q(4, 4096, 16, 64, 64, 64, BF16, F32, 0) == 0
    assert q(4, 4096, 16, 128, 128, 32, BF16, F32, 0) == 0
    # and argument errors come back as the call's status
    assert q(4, 4096, 0, 128, 128, 64, BF16, F32, 0) == -1
    assert q(4, 4096, 16, 128, 256, 64, BF16, F32, 0) == -2


def test_workspace_errors_launch_nothing(lib):
    tc = dict(dtype=1, out_dtype=0, dk=128, dv=128, chunk=64, T=128, B=1, H=1)
    need = lib.ckda_fwd_chunked_workspace_bytes(1, 128, 1, 128, 128, 64, 1, 0, 0)
    assert need == 2 * UNIT_BYTES
    WS = 1 << 32  # 256-byte aligned, never dereferenced
    assert fwd(lib, **tc) == -7                                   # missing
    assert fwd(lib, ws=WS, ws_bytes=need - 1, **tc) == -7         # too small
    assert fwd(lib, ws=WS + 16, ws_bytes=need, **tc) == -7        # not 256-byte aligned
    assert fwd(lib, ws=P, ws_bytes=need, **tc) == -7              # overlaps q
    # argument errors are reported before the workspace
    assert fwd(lib, q=None, **tc) == -1


def test_two_phase_calls_validate_without_a_gpu(lib):
    F32, BF16 = 0, 1
    WS = 1 << 32
    need = lib.ckda_fwd_chunked_workspace_bytes(1, 128, 1, 128, 128, 64, BF16, F32, 0)

    def factors(**kw):
        a = dict(q=P, k=P + 0x1000, v=P + 0x2000, alpha=P + 0x3000, beta=P + 0x4000, cu=None,
                 B=1, T=128, H=1, dk=128, dv=128, chunk=64, dtype=BF16, ws=None, ws_bytes=0)
        a.update(kw)
        return lib.ckda_fwd_factors(a["q"], a["k"], a["v"], a["alpha"], a["beta"], a["cu"], a["B"],
                                    a["T"], a["H"], a["dk"], a["dv"], a["chunk"], a["dtype"],
                                    a["ws"], a["ws_bytes"], None)

    def carry(**kw):
        a = dict(v=P + 0x2000, S0=None, cu=None, out=P + 0x5000, S_final=None, B=1, T=128, H=1,
                 dk=128, dv=128,
                 chunk=64, dtype=BF16, out_dtype=F32, ws=None, ws_bytes=0)
        a.update(kw)
        return lib.ckda_fwd_carry(a["v"], a["S0"], a["cu"], a["out"], a["S_final"], a["B"], a["T"], a["H"],
                                  a["dk"], a["dv"], a["chunk"], a["dtype"], a["out_dtype"], a["ws"],
                                  a["ws_bytes"], None)

    # the two phases exist only on the tensor-core path
    assert factors(dtype=F32) == -2
    assert factors(dk=64) == -2
    assert carry(chunk=32) == -2
    # each phase needs only its own tensors, and the workspace
    assert factors(q=None) == -1
    assert carry(out=None) == -1
    assert carry(v=None) == -1
    assert factors() == -7
    assert carry() == -7
    assert factors(ws=WS, ws_bytes=need - 256) == -7
    assert carry(ws=WS + 64, ws_bytes=need) == -7
    # nothing to do for an empty batch
    assert factors(B=0) == 0
    assert carry(B=0) == 0


def test_static_scratch_entry_rejects_oversized_calls_without_a_gpu(lib):
    from delta_rule_linear_ckda_b200._lib import CKDA_STATIC_SCRATCH_BYTES

    F32, BF16 = 0, 1
    # 4 x 64 x 16 units need 271 MB > the 64 MiB scratch
    assert lib.ckda_fwd_chunked_workspace_bytes(4, 4096, 16, 128, 128, 64, BF16, F32, 0) > \
        CKDA_STATIC_SCRATCH_BYTES
    r = lib.ckda_fwd_chunked_static(P, P + 0x1000, P + 0x2000, P + 0x3000, P + 0x4000, None, None,
                                    P + 0x5000, None, 4, 4096, 16, 128, 128, 64, BF16, F32, None)
    assert r == -2
    # argument errors come first, as in ckda_fwd_chunked
    r = lib.ckda_fwd_chunked_static(None, P, P, P, P, None, None, P + 0x5000, None, 1, 64, 1, 128,
                                    128, 64, BF16, F32, None)
    assert r == -1
    assert lib.ckda_fwd_chunked_static(P, P, P, P, P, None, None, P + 0x5000, None, 0, 64, 1, 128,
                                       128, 64, BF16, F32, None) == 0


def test_gdn2_entry_validates_its_gates(lib):
    def g2(**kw):
        a = dict(q=P, k=P + 0x1000, v=P + 0x2000, alpha=P + 0x3000, b=P + 0x4000, w=P + 0x6000,
                 S0=None, cu=None, out=P + 0x5000, S_final=None, B=1, T=8, H=1, dk=16, dv=16,
                 chunk=16, dtype=0, out_dtype=0)
        a.update(kw)
        return lib.ckda_gdn2_fwd_chunked(a["q"], a["k"], a["v"], a["alpha"], a["b"], a["w"], a["S0"],
                                         a["cu"], a["out"], a["S_final"], a["B"], a["T"], a["H"],
                                         a["dk"], a["dv"], a["chunk"], a["dtype"], a["out_dtype"],
                                         None, 0, None)

    assert g2(b=None) == -1
    assert g2(w=None) == -1
    assert g2(w=MIS) == -3
    assert g2(out=P + 0x6000) == -1   # out aliases w
    assert g2(dk=48) == -2
    assert g2(B=0) == 0
    # the tensor-core shapes need the same workspace as ckda_fwd_chunked
    assert g2(dtype=1, dk=128, dv=128, chunk=64, T=128) == -7


def test_sfda_entry_validates_its_gates(lib):
    def sf(**kw):
        a = dict(q=P, k=P + 0x1000, v=P + 0x2000, alpha=P + 0x3000, theta=P + 0x4000,
                 beta=P + 0x6000, S0=None, cu=None, out=P + 0x5000, S_final=None, B=1, T=8, H=1,
                 dk=16, dv=16, chunk=16, dtype=0, out_dtype=0)
        a.update(kw)
        return lib.ckda_sfda_fwd_chunked(a["q"], a["k"], a["v"], a["alpha"], a["theta"],
                                         a["beta"], a["S0"], a["cu"], a["out"], a["S_final"],
                                         a["B"], a["T"], a["H"], a["dk"], a["dv"], a["chunk"],
                                         a["dtype"], a["out_dtype"], None, 0, None)

    assert sf(theta=None) == -1
    assert sf(alpha=None) == -1
    assert sf(beta=None) == -1
    assert sf(theta=MIS) == -3
    assert sf(out=P + 0x4000) == -1   # out aliases theta
    assert sf(dk=48) == -2
    assert sf(chunk=128) == -2
    assert sf(B=0) == 0
    # the tensor-core shapes need the same workspace as ckda_fwd_chunked
    assert sf(dtype=1, dk=128, dv=128, chunk=64, T=128) == -7
    r = lib.ckda_sfda_fwd_chunked_fp32core(P, P + 0x1000, P + 0x2000, P + 0x3000, None,
                                           P + 0x6000, None, None, P + 0x5000, None, 1, 8, 1, 16,
                                           16, 16, 0, 0, None)
    assert r == -1  # theta missing


def test_bwd_entry_validates_without_a_gpu(lib):
    def bw(**kw):
        a = dict(q=P, k=P + 0x1000, v=P + 0x2000, alpha=P + 0x3000, beta=P + 0x4000, S0=None,
                 cu=None, dO=P + 0x5000, dSf=None, dq=P + 0x6000, dk=P + 0x7000, dv=P + 0x8000,
                 da=P + 0x9000, db=P + 0xA000, dS0=None, B=1, T=8, H=1, dk_=16, dv_=16, dtype=0,
                 gdt=0, ws=None, ws_bytes=0)
        a.update(kw)
        return lib.ckda_bwd_chunked(a["q"], a["k"], a["v"], a["alpha"], a["beta"], a["S0"],
                                    a["cu"], a["dO"], a["dSf"], a["dq"], a["dk"], a["dv"],
                                    a["da"], a["db"], a["dS0"], a["B"], a["T"], a["H"], a["dk_"],
                                    a["dv_"], a["dtype"], a["gdt"], a["ws"], a["ws_bytes"], None)

    assert bw(dO=None) == -1
    assert bw(dq=None) == -1
    assert bw(db=None) == -1
    assert bw(dk_=48) == -2
    assert bw(gdt=3) == -2
    assert bw(dv=MIS) == -3
    assert bw(dq=P) == -1          # an output aliases q
    assert bw() == -7              # no workspace
    assert bw(B=0) == 0
    need = lib.ckda_bwd_chunked_workspace_bytes(1, 8, 1, 16, 16, 0)
    assert need == (1 + 17) * 32 * 16 * 4       # d_k < 32 stores 32 rows per state
    assert lib.ckda_bwd_chunked_workspace_bytes(2, 130, 3, 128, 64, 0) == \
        (2 * 9 * 3 + 2 * 3 * 17) * 128 * 64 * 4     # 9 16-token slots per sequence
    assert lib.ckda_bwd_chunked_workspace_bytes(2, 130, 3, 128, 48, 0) == -2
    # a workspace that overlaps an input
    assert bw(ws=P, ws_bytes=need) == -7


def test_scan_entry_validates_without_a_gpu(lib):
    def sc(**kw):
        a = dict(q=P, k=P + 0x100000, v=P + 0x200000, alpha=P + 0x300000, beta=P + 0x400000,
                 S0=None, out=P + 0x500000, S_final=None, B=1, T=128, H=1, dk_=128, dv_=128,
                 chunk=64, dtype=1, odt=0, G=2, ws=None, ws_bytes=0)
        a.update(kw)
        return lib.ckda_fwd_chunked_scan(a["q"], a["k"], a["v"], a["alpha"], a["beta"], a["S0"],
                                         a["out"], a["S_final"], a["B"], a["T"], a["H"], a["dk_"],
                                         a["dv_"], a["chunk"], a["dtype"], a["odt"], a["G"],
                                         a["ws"], a["ws_bytes"], None)

    assert sc(G=0) == -1
    assert sc(dtype=0) == -2              # fp32 inputs: not a tensor-core shape
    assert sc(dk_=64) == -2
    assert sc() == -7                     # no workspace
    assert sc(B=0) == 0
    need1 = lib.ckda_fwd_chunked_workspace_bytes(2, 300, 3, 128, 128, 64, 1, 0, 0)
    need = lib.ckda_fwd_chunked_scan_workspace_bytes(2, 300, 3, 128, 128, 4)
    assert need == need1 + 2 * 3 * 3 * 128 * 256 * 4 + 2 * 4 * 3 * 128 * 128 * 4
    assert lib.ckda_fwd_chunked_scan_workspace_bytes(2, 300, 3, 128, 128, 0) == -1


def test_variant_decode_entries_validate_without_a_gpu(lib):
    args = (P, P + 0x1000, P + 0x2000, P + 0x3000)
    # Gated DeltaNet-2: b, w required
    assert lib.ckda_gdn2_decode_step(*args, None, P + 0x5000, P + 0x6000, P + 0x7000, 1, 1, 16,
                                     16, 0, 0, None) == -1
    assert lib.ckda_gdn2_decode_step(*args, P + 0x4000, MIS, P + 0x6000, P + 0x7000, 1, 1, 16,
                                     16, 0, 0, None) == -3
    assert lib.ckda_gdn2_decode_step(*args, P + 0x4000, P + 0x5000, P + 0x6000, P + 0x7000, 0, 1,
                                     16, 16, 0, 0, None) == 0
    # SFDA: theta required
    assert lib.ckda_sfda_decode_step(*args, None, P + 0x5000, P + 0x6000, P + 0x7000, 1, 1, 16,
                                     16, 0, 0, None) == -1
    assert lib.ckda_sfda_decode_step(*args, P + 0x4000, P + 0x5000, P + 0x6000, P + 0x7000, 1, 1,
                                     48, 16, 0, 0, None) == -2
    assert lib.ckda_sfda_decode_step(*args, P + 0x4000, P + 0x5000, P + 0x6000, P + 0x6000, 1, 1,
                                     16, 16, 0, 0, None) == -1   # out aliases the state
