"""ctypes loader for libckda.so (the C ABI declared in include/ckda.h).

The library is built in-tree by ``delta_rule_linear_ckda_b200.build``.  There
is no fallback: if the shared library is missing or lacks a symbol, loading
raises ``ImportError``.
"""
from __future__ import annotations

import ctypes
import os

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libckda.so")

CKDA_F32 = 0
CKDA_BF16 = 1
# capacity of the library's static device scratch (ckda_fwd_chunked_static)
CKDA_STATIC_SCRATCH_BYTES = 64 * 1024 * 1024

STATUS = {
    0: "CKDA_OK",
    -1: "CKDA_ERR_INVALID_ARG",
    -2: "CKDA_ERR_UNSUPPORTED",
    -3: "CKDA_ERR_MISALIGNED",
    -4: "CKDA_ERR_CUDA",
    -5: "CKDA_ERR_DEVICE_TIMEOUT",
    -6: "CKDA_ERR_BAD_SEQLENS",
    -7: "CKDA_ERR_WORKSPACE",
}

# name -> (restype, argtypes), mirroring include/ckda.h
_vp = ctypes.c_void_p
_i = ctypes.c_int
SIGNATURES = {
    "ckda_fwd_chunked": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _i,
                              _vp, ctypes.c_size_t, _vp]),
    "ckda_fwd_chunked_workspace_bytes": (ctypes.c_int64, [_i, _i, _i, _i, _i, _i, _i, _i, _i]),
    "ckda_fwd_chunked_static": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i,
                                     _i, _i, _i, _vp]),
    "ckda_gdn2_fwd_chunked": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i,
                                   _i, _i, _i, _i, _vp, ctypes.c_size_t, _vp]),
    "ckda_sfda_fwd_chunked": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i,
                                   _i, _i, _i, _i, _vp, ctypes.c_size_t, _vp]),
    "ckda_sfda_fwd_chunked_fp32core": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i,
                                            _i, _i, _i, _i, _i, _i, _vp]),
    "ckda_fwd_chunked_scan": (_i, [_vp] * 8 + [_i] * 9 + [_vp, ctypes.c_size_t, _vp]),
    "ckda_fwd_chunked_scan_workspace_bytes": (ctypes.c_int64, [_i] * 6),
    "ckda_bwd_chunked": (_i, [_vp] * 15 + [_i] * 7 + [_vp, ctypes.c_size_t, _vp]),
    "ckda_bwd_chunked_workspace_bytes": (ctypes.c_int64, [_i, _i, _i, _i, _i, _i]),
    "ckda_fwd_factors": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _vp,
                              ctypes.c_size_t, _vp]),
    "ckda_fwd_carry": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _i, _vp,
                            ctypes.c_size_t, _vp]),
    "ckda_fwd_chunked_fp32core": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _i, _vp]),
    "ckda_fwd_chunked_path": (_i, [_i, _i, _i, _i, _i, _i, _i, _i, _i]),
    "ckda_gdn2_decode_step": (_i, [_vp] * 8 + [_i] * 6 + [_vp]),
    "ckda_sfda_decode_step": (_i, [_vp] * 8 + [_i] * 6 + [_vp]),
    "ckda_decode_step": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _vp]),
    "ckda_status_string": (ctypes.c_char_p, [_i]),
    "ckda_device_status": (_i, [_vp]),
    "ckda_selftest_bounded_wait": (_i, [_i, _vp]),
    "ckda_version": (_i, []),
}

_lib = None


def load() -> ctypes.CDLL:
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python -m delta_rule_linear_ckda_b200.build` "
            "(there is no CPU fallback)")
    lib = ctypes.CDLL(LIB_PATH)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)  # AttributeError -> the build is broken
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


class CKDAError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        text = load().ckda_status_string(code).decode()
        super().__init__(f"{where}: {STATUS.get(code, code)} ({text})")
