"""CKDA (Complex Kimi Delta Attention) on NVIDIA B200: chunked WY prefill and
recurrent decode through the C ABI of ``libckda.so`` (include/ckda.h).

``fwd_chunked``, ``decode_step`` and ``device_status`` load the native
library on first use and raise if it is missing: there is no CPU fallback.
``delta_rule_linear_ckda_b200.inputs`` (seeded workload generators) imports
without the native library.
"""
from __future__ import annotations

_API = ("fwd_chunked", "fwd_chunked_static", "gdn2_fwd_chunked", "sfda_fwd_chunked", "fwd_factors",
        "fwd_carry", "fwd_path", "workspace_bytes", "bwd_chunked", "bwd_workspace_bytes",
        "fwd_chunked_scan", "scan_workspace_bytes",
        "decode_step", "gdn2_decode_step", "sfda_decode_step", "device_status")
__all__ = list(_API) + ["CKDAError", "lib_path"]


def __getattr__(name):
    if name in _API:
        from . import api

        api._lib.load()
        return getattr(api, name)
    if name == "CKDAError":
        from ._lib import CKDAError

        return CKDAError
    if name == "lib_path":
        from ._lib import LIB_PATH

        return LIB_PATH
    raise AttributeError(name)
