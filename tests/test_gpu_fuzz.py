"""Seeded random shapes through the whole path, bf16 and FP8, against the oracle.

Each case draws batch, head counts (GQA group 1-16), head dim, context length,
block and anchor sizes over their whole legal range (blocks from 1 token up,
at most 191 of them, ragged last blocks included; anchors 0..b), query length
and decode steps from a fixed seed.  Phase 1 is checked through its float32
debug rows at the absolute bar (a row of a short block averages a few values,
whose bf16 rounding alone approaches the bar), with O equal to their bf16
rounding bit for bit; the cache bit-exact; prefill and decode at the bar.
"""

import numpy as np
import pytest

from block_sparse_long_phase_b200 import workloads as wl

from test_gpu_fp8 import check_fp8_case
from test_gpu_short_blocks import check_short_case

pytestmark = pytest.mark.gpu


def draw(seed):
    r = np.random.default_rng(seed)
    D = int(r.choice([64, 128]))
    Hkv = int(r.choice([1, 2, 4, 8]))
    G = int(r.choice([1, 2, 3, 4, 8, 16]))
    B = int(r.integers(1, 4))
    L = int(r.integers(1, 1600))
    # block sizes spread over orders of magnitude, at most 191 blocks
    b_min = -(-L // 191)
    b = int(max(b_min, round(np.exp(r.uniform(0.0, np.log(max(2, min(L + 200, 1024))))))))
    b_a = 0 if r.random() < 0.2 else int(r.integers(1, b + 1))
    lq = int(r.integers(1, 40))
    T = int(r.integers(0, 5))
    return dict(B=B, Hq=G * Hkv, Hkv=Hkv, D=D, L=L, b=b, b_a=b_a, lq=lq, T=T)


def test_draws_cover_the_legal_range():
    shapes = [draw(1000 + s) for s in range(16)] + [draw(2000 + s) for s in range(8)]
    assert all(-(-s["L"] // s["b"]) <= 191 and 0 <= s["b_a"] <= s["b"] for s in shapes)
    assert min(s["b"] for s in shapes) < 16
    assert any(0 < s["b_a"] < 32 for s in shapes)


@pytest.mark.parametrize("seed", range(16))
def test_random_shapes(seed):
    shape = draw(1000 + seed)
    check_short_case(wl.get("tiny").with_(**shape), f"random {seed} {shape}")


@pytest.mark.parametrize("seed", range(8))
def test_random_shapes_fp8(seed):
    shape = draw(2000 + seed)
    check_fp8_case(wl.get("tiny").with_(**shape), f"random fp8 {seed} {shape}")
