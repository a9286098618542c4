"""The algorithmic work bench.py divides by, pinned on CPU.

Every roofline fraction the bench reports is (algorithmic flops or bytes) /
time / peak, so the counts are checked against independent forms: phase 1's
visible (query, key) pairs against the oracle's explicit Star mask, the query
prefill's pairs and a decode step's cached rows against a direct count of
what each row sees.
"""

import os
import sys

import numpy as np
import pytest

from block_sparse_long_phase_b200 import workloads as wl
from oracle import star_oracle as so

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


@pytest.mark.parametrize("L,b,b_a", [(64, 16, 16), (70, 16, 5), (50, 16, 0), (40, 64, 64), (33, 8, 8),
                                     (1, 1, 0), (100, 7, 3)])
def test_phase1_pairs_equal_the_star_mask(L, b, b_a):
    w = wl.get("tiny").with_(L=L, b=b, b_a=b_a)
    flops, pairs = bench.phase1_flops(w)
    assert pairs == int(so.star_mask(L, b, b_a).sum())
    assert flops == 4 * w.D * w.Hq * w.B * pairs


def test_phase1_flops_of_the_main_workload():
    # 8B-32K: 4 blocks of 8192, anchor 8192 -> 4 * 8192 * 8193 / 2 + 3 * 8192 * 8192 pairs
    w = wl.get("8b-32k")
    _, pairs = bench.phase1_flops(w)
    assert pairs == 4 * 8192 * 8193 // 2 + 3 * 8192 * 8192
    assert bench.phase1_flops(w)[0] == 5497826574336


@pytest.mark.parametrize("L,lq", [(1024, 16), (300, 1), (50, 13)])
def test_prefill_counts(L, lq):
    w = wl.get("tiny").with_(L=L, lq=lq)
    pk = {"bf16_tflops": 1000.0, "hbm_gbs": 1000.0}
    r = bench.prefill_roofline(w, 1.0, pk)
    # row r of the query sees every context key and query rows 0..r
    pairs = sum(L + (r + 1) for r in range(lq))
    assert r["flops"] == 4 * w.D * w.Hq * w.B * pairs
    kv = w.B * w.Hkv * (L + lq) * w.D * 2 * 2
    q_o = w.B * w.Hq * lq * w.D * 2 * 2 + w.B * w.Hq * lq * 4
    assert r["bytes"] == kv + q_o
    assert r["peak"] == min(1000.0, r["flops"] / r["bytes"] * 1000.0 / 1e3)


def test_decode_bytes_count_every_row_the_token_sees():
    w = wl.get("tiny")
    for t in (0, 1, w.T - 1):
        seen = w.L + (w.lq + t) + 1        # context, earlier query-region rows, the token itself
        assert bench.decode_bytes(w, t) == w.B * w.Hkv * seen * w.D * 2 * 2
        # FP8: codes + a float32 scale per row for K and V, the token's own row in bf16
        assert bench.decode_bytes_fp8(w, t) == w.B * w.Hkv * ((seen - 1) * (w.D + 4) * 2 + w.D * 4)


@pytest.mark.parametrize("L,b,b_a", [(1024, 256, 256), (1000, 256, 100), (300, 512, 512)])
def test_cpu_baseline_sample_pairs_equal_the_star_mask(L, b, b_a):
    """The CPU baseline extrapolates by visible pairs: the sampled rows' count
    must equal the explicit Star mask's row sums, and the sample must hold
    every block's first and last rows."""
    w = wl.get("tiny").with_(L=L, b=b, b_a=b_a)
    data = bench.oracle_sample_inputs(w)
    rows = np.concatenate(data["blocks"])
    assert bench.sample_pairs(w, data["blocks"]) == int(so.star_mask_rows(L, b, b_a, rows).sum()) * w.G
    for (s, n), blk in zip(so.block_table(L, b), data["blocks"]):
        assert blk[0] == s and blk[-1] == s + n - 1
    again = bench.oracle_sample_inputs(w)
    assert all(np.array_equal(x, y) for x, y in zip(data["blocks"], again["blocks"]))
    assert np.array_equal(data["K"], again["K"])
