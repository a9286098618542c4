"""ctypes declarations of libstar's C ABI (include/star_attention.h).

Loading fails loudly: there is no CPU fallback anywhere in this package.
"""

from __future__ import annotations

import ctypes
import os

# STAR_LIB=checked selects the bounds-checked build (lib/libstar_checked.so)
LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "lib",
                        "libstar_checked.so" if os.environ.get("STAR_LIB") == "checked" else "libstar.so")

STAR_OK = 0
STAR_EINVAL = -1
STAR_ENOSPC = -2
STAR_ECUDA = -3
STAR_EUNSUPPORTED = -4
STAR_ENOMEM = -5

# Every symbol the header declares.
EXPORTS = (
    "star_cache_create", "star_cache_destroy", "star_cache_device_error", "star_cache_num_segments",
    "star_cache_segment", "star_cache_segment_fp8", "star_cache_reset_query", "star_ctx_encode",
    "star_query_prefill", "star_query_prefill_partials", "star_decode_step", "star_lse_merge",
    "star_decode_step_noalloc", "star_last_error", "star_version",
    "star_rope", "star_anchor_keys", "star_ctx_encode_anchored", "star_ctx_encode_after_anchor",
    "star_ctx_encode_host",
    "star_selftest_wait_timeout", "star_noalloc_device_error", "star_ctx_encode_fp32",
    "star_decode_step_partials", "star_partial_attend",
    "star_lse_merge_bf16", "star_cache_check_guards", "star_plan_prefill", "star_prefill_span_tiles",
)


class StarParams(ctypes.Structure):
    _fields_ = [
        ("B", ctypes.c_int), ("Hq", ctypes.c_int), ("Hkv", ctypes.c_int), ("D", ctypes.c_int),
        ("L", ctypes.c_longlong), ("block", ctypes.c_int), ("anchor", ctypes.c_int),
        ("q_cap", ctypes.c_int), ("scale", ctypes.c_float), ("kv_fp8", ctypes.c_int),
    ]


class StarError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"libstar error {code}: {msg}")
        self.code = code


_lib = None


def load(path: str = LIB_PATH):
    """Load libstar.so (built in-tree by ``block_sparse_long_phase_b200.build``)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise ImportError(f"libstar.so not found at {path}; run `python -m block_sparse_long_phase_b200.build`")
    lib = ctypes.CDLL(path)
    vp, i, ll = ctypes.c_void_p, ctypes.c_int, ctypes.c_longlong
    fp = ctypes.POINTER(ctypes.c_float)
    lib.star_cache_create.argtypes = [ctypes.POINTER(StarParams), ctypes.POINTER(vp)]
    lib.star_cache_destroy.argtypes = [vp]
    lib.star_cache_num_segments.argtypes = [vp]
    lib.star_cache_device_error.argtypes = [vp, ctypes.POINTER(i)]
    lib.star_cache_segment.argtypes = [vp, i, ctypes.POINTER(vp), ctypes.POINTER(vp),
                                       ctypes.POINTER(ll), ctypes.POINTER(ll), ctypes.POINTER(ll)]
    lib.star_cache_segment_fp8.argtypes = [vp, i, ctypes.POINTER(vp), ctypes.POINTER(vp),
                                           ctypes.POINTER(fp), ctypes.POINTER(fp)]
    lib.star_cache_reset_query.argtypes = [vp]
    lib.star_ctx_encode.argtypes = [vp, vp, vp, vp, vp, vp, vp]
    lib.star_query_prefill.argtypes = [vp, i, vp, vp, vp, vp, vp, vp]
    lib.star_selftest_wait_timeout.argtypes = [ctypes.c_uint, ctypes.POINTER(ctypes.c_int), vp]
    lib.star_ctx_encode_host.argtypes = [vp] + [vp] * 10 + [vp]
    lib.star_query_prefill_partials.argtypes = [vp, i, vp, vp, vp, vp, vp, vp, vp, vp, vp]
    lib.star_decode_step.argtypes = [vp, vp, vp, vp, vp, vp, vp]
    lib.star_lse_merge.argtypes = [i, ll, i, vp, vp, vp, vp, vp]
    lib.star_rope.argtypes = [i, i, ll, i, ctypes.c_double, vp, ll, vp, vp, vp]
    lib.star_anchor_keys.argtypes = [vp, i, vp, ctypes.c_double, vp, vp, vp]
    lib.star_ctx_encode_anchored.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp]
    lib.star_ctx_encode_after_anchor.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp]
    lib.star_decode_step_noalloc.argtypes = [ctypes.POINTER(StarParams), ll, vp, vp, vp, vp,
                                             vp, vp, vp, vp, vp, vp]
    lib.star_noalloc_device_error.argtypes = [ctypes.POINTER(i), vp]
    lib.star_ctx_encode_fp32.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp]
    lib.star_cache_check_guards.argtypes = [vp, ctypes.POINTER(i)]
    ip = ctypes.POINTER(i)
    lib.star_plan_prefill.argtypes = [ctypes.POINTER(StarParams), i, i, ll, i, i, i, i, i, ip, ip]
    lib.star_prefill_span_tiles.argtypes = [ctypes.POINTER(StarParams), ll, ll, i, i, ip, ip]
    lib.star_lse_merge_bf16.argtypes = [i, ll, i, vp, vp, vp, vp, vp]
    lib.star_partial_attend.argtypes = [vp, i, i, i, i, vp, vp, vp, vp, vp, vp]
    lib.star_decode_step_partials.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, ctypes.POINTER(ll), i,
                                              ctypes.POINTER(i), vp]
    for name in EXPORTS:
        getattr(lib, name).restype = i
    lib.star_last_error.restype = ctypes.c_char_p
    lib.star_version.restype = ctypes.c_char_p
    del fp
    _lib = lib
    return lib


def check(rc: int):
    if rc != STAR_OK:
        raise StarError(rc, load().star_last_error().decode())
    return rc
