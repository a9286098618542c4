"""The query prefill's work split, checked on the host through libstar's
host-only introspection calls (star_plan_prefill, star_prefill_span_tiles):
no device is touched.

A wrong split is silent on the GPU as long as no tile goes missing, so the
invariants are checked over seeded random shapes: spans are non-empty and
cover exactly the rows the call attends to -- the context segments of the
range and, with the query, the query region -- with no row outside them
(a range that stops short of L must not pull in the rows before L); their
count fits the kernel's span table and the cache's scratch; and the tile walk
of a span covers it contiguously, never crosses a context segment's end, and
reads each row from the right place (context rows at their segment's layout
offset, query-region rows at bg * q_cap + r).
"""

import ctypes

import numpy as np
import pytest

from block_sparse_long_phase_b200 import _abi, build


@pytest.fixture(scope="module")
def lib():
    build.build()
    return _abi.load()


MAX_SPANS = 192


def plan(lib, p, sms, lq, len0, s0, ns, query, per_segment=False):
    n = ctypes.c_int(-1)
    buf = (ctypes.c_int * (2 * MAX_SPANS))()
    rc = lib.star_plan_prefill(ctypes.byref(p), sms, lq, len0, s0, ns, int(query), int(per_segment), MAX_SPANS,
                               ctypes.byref(n), buf)
    assert rc == _abi.STAR_OK, lib.star_last_error()
    return [(buf[2 * k], buf[2 * k + 1]) for k in range(n.value)]


def tiles(lib, p, x0, x1, bg):
    cap = (x1 - x0) // 128 + 400
    n = ctypes.c_int(-1)
    buf = (ctypes.c_int * (4 * cap))()
    rc = lib.star_prefill_span_tiles(ctypes.byref(p), x0, x1, bg, cap, ctypes.byref(n), buf)
    assert rc == _abi.STAR_OK, lib.star_last_error()
    return [tuple(buf[4 * t:4 * t + 4]) for t in range(n.value)]


def draw(r):
    B, Hkv, G = int(r.integers(1, 4)), int(r.choice([1, 2, 8])), int(r.choice([1, 4, 8, 16]))
    L = int(r.integers(1, 300000 if r.random() < 0.5 else 5000))
    b = int(r.integers(1, min(L, 70000) + 50))
    if -(-L // b) > 191:
        b = -(-L // 191)
    q_cap = int(r.integers(1, 800))
    return _abi.StarParams(B, G * Hkv, Hkv, 128, L, b, int(r.integers(0, b + 1)), q_cap, 0.0)


def test_spans_cover_exactly_the_attended_rows(lib):
    r = np.random.default_rng(5)
    for _ in range(3000):
        p = draw(r)
        n_seg = -(-p.L // p.block)
        lq = int(r.integers(1, p.q_cap + 1))
        len0 = int(r.integers(0, p.q_cap - lq + 1))
        s0 = int(r.integers(0, n_seg + 1))
        ns = int(r.integers(0, n_seg - s0 + 1))
        query = bool(r.integers(0, 2))
        if r.random() < 0.3:
            s0, ns, query = 0, n_seg, True
        sms = int(r.choice([1, 8, 148]))
        spans = plan(lib, p, sms, lq, len0, s0, ns, query)
        R0, R1 = s0 * p.block, min((s0 + ns) * p.block, p.L)
        want = []
        if R1 > R0:
            want.append([R0, R1])
        if query:
            if want and want[-1][1] == p.L:
                want[-1][1] = p.L + len0 + lq
            else:
                want.append([p.L, p.L + len0 + lq])
        got = []
        for x0, x1 in spans:
            assert x1 > x0, "empty span"
            if got and got[-1][1] == x0:
                got[-1][1] = x1
            else:
                got.append([x0, x1])
        assert got == want, (p.L, p.block, s0, ns, query, spans)
        # the span table and the cache's scratch hold every plan
        pairs = -(-(p.Hq // p.Hkv) * lq // 256)
        assert len(spans) <= min(MAX_SPANS, max(n_seg + 1, max(1, sms // (p.B * p.Hkv * pairs)) + 1))


def test_per_segment_plan_is_one_span_per_segment(lib):
    p = _abi.StarParams(1, 4, 2, 64, 1000, 256, 100, 20, 0.0)
    spans = plan(lib, p, 148, 5, 3, 0, 4, True, per_segment=True)
    assert spans == [(0, 256), (256, 512), (512, 768), (768, 1000), (1000, 1008)]


def test_tile_walk_stays_inside_segments_and_reads_the_right_rows(lib):
    r = np.random.default_rng(9)
    for _ in range(1500):
        p = draw(r)
        N = p.L + p.q_cap
        x0 = int(r.integers(0, N))
        x1 = int(r.integers(x0 + 1, min(N, x0 + 40000) + 1))
        bg = int(r.integers(0, p.B * p.Hkv))
        x = x0
        for row, region, k, r0 in tiles(lib, p, x0, x1, bg):
            assert 1 <= k <= 128
            if x < p.L:
                seg = x // p.block
                seg_len = min(p.block, p.L - seg * p.block)
                assert not region and x + k <= min((seg + 1) * p.block, p.L), "tile crosses a segment"
                assert row == seg * p.B * p.Hkv * p.block + bg * seg_len + (x - seg * p.block)
            else:
                assert region and r0 == x - p.L and row == bg * p.q_cap + r0
            x += k
        assert x == x1


def test_host_calls_reject_bad_arguments(lib):
    p = _abi.StarParams(1, 4, 2, 64, 1000, 256, 100, 20, 0.0)
    n = ctypes.c_int()
    buf = (ctypes.c_int * 8)()
    assert lib.star_plan_prefill(ctypes.byref(p), 148, 30, 0, 0, 4, 1, 0, 4, ctypes.byref(n), buf) == _abi.STAR_EINVAL
    assert lib.star_plan_prefill(ctypes.byref(p), 148, 5, 0, 2, 3, 1, 0, 4, ctypes.byref(n), buf) == _abi.STAR_EINVAL
    assert lib.star_prefill_span_tiles(ctypes.byref(p), 5, 5, 0, 2, ctypes.byref(n), buf) == _abi.STAR_EINVAL
    assert lib.star_prefill_span_tiles(ctypes.byref(p), 0, 100, 2, 2, ctypes.byref(n), buf) == _abi.STAR_EINVAL
    assert lib.star_plan_prefill(None, 148, 5, 0, 0, 4, 1, 0, 4, ctypes.byref(n), buf) == _abi.STAR_EINVAL
