"""Host-side checks of the C ABI: the library builds, loads and exports every
symbol include/star_attention.h declares.  No compute call (no GPU here)."""

import ctypes
import os
import re

import pytest

from block_sparse_long_phase_b200 import _abi, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def header_symbols():
    txt = open(os.path.join(ROOT, "include", "star_attention.h")).read()
    return sorted(set(re.findall(r"STAR_API\s+[\w\s\*]+?\b(star_\w+)\s*\(", txt)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return _abi.load()


def test_header_declares_the_four_entry_points():
    syms = header_symbols()
    for s in ("star_ctx_encode", "star_query_prefill", "star_decode_step", "star_lse_merge"):
        assert s in syms
    assert sorted(_abi.EXPORTS) == syms


def test_library_exports_every_declared_symbol(lib):
    for s in header_symbols():
        assert hasattr(lib, s), s
        assert ctypes.cast(getattr(lib, s), ctypes.c_void_p).value


def test_version_and_error_strings(lib):
    assert b"sm_100a" in lib.star_version()
    assert isinstance(lib.star_last_error(), bytes)


def test_argument_errors_are_caught_on_the_host(lib):
    """Shape errors never reach the device: these return before any CUDA call."""
    out = ctypes.c_void_p()
    bad = [
        _abi.StarParams(1, 4, 3, 64, 1024, 256, 256, 8, 0.0),    # Hq % Hkv
        _abi.StarParams(1, 4, 2, 64, 1024, 256, 300, 8, 0.0),    # b_a > b
        _abi.StarParams(1, 4, 2, 64, 0, 256, 256, 8, 0.0),       # L = 0
        _abi.StarParams(1, 4, 2, 64, 1024, 0, 0, 8, 0.0),        # b = 0
        _abi.StarParams(1, 4, 2, 64, 1024, 256, -1, 8, 0.0),     # b_a < 0
        _abi.StarParams(1, 4, 2, 64, 1024, 256, 256, 0, 0.0),    # q_cap = 0
        _abi.StarParams(1, 4, 2, 64, 1024, 256, 256, 8, 0.0, 2), # kv_fp8 not 0/1
    ]
    for p in bad:
        assert lib.star_cache_create(ctypes.byref(p), ctypes.byref(out)) == _abi.STAR_EINVAL
        assert out.value is None
        assert lib.star_last_error()
    p = _abi.StarParams(1, 4, 2, 96, 1024, 256, 256, 8, 0.0)     # D = 96
    assert lib.star_cache_create(ctypes.byref(p), ctypes.byref(out)) == _abi.STAR_EUNSUPPORTED
    p = _abi.StarParams(1, 4, 2, 64, 192 * 64, 64, 64, 8, 0.0)   # 192 blocks: beyond the chunk table
    assert lib.star_cache_create(ctypes.byref(p), ctypes.byref(out)) == _abi.STAR_EUNSUPPORTED
    assert b"192 blocks" in lib.star_last_error()
    p = _abi.StarParams(1, 4, 2, 64, 191 * 64 + 1, 64, 64, 8, 0.0)  # 192 blocks, the last one ragged
    assert lib.star_cache_create(ctypes.byref(p), ctypes.byref(out)) == _abi.STAR_EUNSUPPORTED
    p = _abi.StarParams(1024, 8, 8, 64, 1 << 18, 1 << 12, 1 << 12, 8, 0.0)  # 2^31 cached rows
    assert lib.star_cache_create(ctypes.byref(p), ctypes.byref(out)) == _abi.STAR_EUNSUPPORTED
    assert b"2^31" in lib.star_last_error()
    assert lib.star_cache_create(None, ctypes.byref(out)) == _abi.STAR_EINVAL
    assert lib.star_lse_merge(0, 4, 8, None, None, None, None, None) == _abi.STAR_EINVAL
    assert lib.star_lse_merge(1, 4, 2000, None, None, None, None, None) == _abi.STAR_EINVAL
    assert lib.star_lse_merge(1, 0, 8, None, None, None, None, None) == _abi.STAR_OK
    assert lib.star_lse_merge_bf16(0, 4, 8, None, None, None, None, None) == _abi.STAR_EINVAL
    assert lib.star_lse_merge_bf16(1, 4, 8, None, None, None, None, None) == _abi.STAR_EINVAL
    assert lib.star_ctx_encode(None, None, None, None, None, None, None) == _abi.STAR_EINVAL
    assert lib.star_ctx_encode_fp32(None, *([None] * 7)) == _abi.STAR_EINVAL
    assert lib.star_partial_attend(None, 0, 1, 0, 1, *([None] * 6)) == _abi.STAR_EINVAL
    n = ctypes.c_int(-1)
    assert lib.star_decode_step_partials(None, *([None] * 8), 0, ctypes.byref(n), None) == _abi.STAR_EINVAL
    assert lib.star_decode_step(None, None, None, None, None, None, None) == _abi.STAR_EINVAL
    assert lib.star_query_prefill(None, 4, None, None, None, None, None, None) == _abi.STAR_EINVAL
    assert lib.star_query_prefill_partials(None, 4, *([None] * 9)) == _abi.STAR_EINVAL
    assert lib.star_ctx_encode_host(*([None] * 12)) == _abi.STAR_EINVAL
    flag = ctypes.c_int(7)
    assert lib.star_selftest_wait_timeout(1000, None, None) == _abi.STAR_EINVAL
    assert lib.star_selftest_wait_timeout(0, ctypes.byref(flag), None) == _abi.STAR_EINVAL
    assert lib.star_selftest_wait_timeout((1 << 22) + 1, ctypes.byref(flag), None) == _abi.STAR_EINVAL
    assert flag.value == 7                                     # nothing launched
    assert lib.star_cache_segment_fp8(None, 0, None, None, None, None) == _abi.STAR_EINVAL
    p = _abi.StarParams(1, 4, 2, 64, 1024, 256, 256, 8, 0.0, 1)  # the no-alloc path is bf16 only
    assert lib.star_decode_step_noalloc(ctypes.byref(p), 0, *([None] * 10)) == _abi.STAR_EINVAL
    assert b"kv_fp8" in lib.star_last_error()
    # a full query region is refused before anything touches the device (any
    # non-null, 16-byte aligned pointers will do: none is dereferenced)
    p = _abi.StarParams(1, 4, 2, 64, 1024, 256, 256, 8, 0.0)
    fake = [ctypes.c_void_p(4096 * (i + 1)) for i in range(9)]
    assert lib.star_decode_step_noalloc(ctypes.byref(p), 8, *fake, None) == _abi.STAR_ENOSPC
    assert lib.star_decode_step_noalloc(ctypes.byref(p), -1, *fake, None) == _abi.STAR_EINVAL
    misaligned = fake[:4] + [ctypes.c_void_p(4096 + 8)] + fake[5:]
    assert lib.star_decode_step_noalloc(ctypes.byref(p), 0, *misaligned, None) == _abi.STAR_EINVAL
    assert lib.star_noalloc_device_error(None, None) == _abi.STAR_EINVAL
    assert lib.star_rope(1, 1, 8, 96, 500000.0, None, 0, None, None, None) == _abi.STAR_EUNSUPPORTED
    assert lib.star_rope(1, 1, 8, 64, 1.0, None, 0, None, None, None) == _abi.STAR_EINVAL     # theta <= 1
    assert lib.star_rope(1, 1, 8, 64, 500000.0, None, -1, None, None, None) == _abi.STAR_EINVAL
    assert lib.star_rope(1, 1, 8, 64, 500000.0, None, 0, None, None, None) == _abi.STAR_EINVAL  # NULL x
    assert lib.star_rope(1, 1, 0, 64, 500000.0, None, 0, None, None, None) == _abi.STAR_OK      # nothing to do
    assert lib.star_anchor_keys(None, 0, None, 500000.0, None, None, None) == _abi.STAR_EINVAL
    assert lib.star_ctx_encode_anchored(None, None, None, None, None, None, None, None) == _abi.STAR_EINVAL
    assert lib.star_cache_check_guards(None, None) == _abi.STAR_EINVAL
    assert lib.star_cache_destroy(None) == _abi.STAR_OK
    assert lib.star_cache_num_segments(None) == 0


def test_binding_refuses_to_run_without_cuda():
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    from block_sparse_long_phase_b200 import StarCache
    with pytest.raises(RuntimeError):
        StarCache(1, 4, 2, 64, 1024, 256, 256, 8)
