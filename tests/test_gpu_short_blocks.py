"""Short blocks and short anchors on the GPU, at the absolute bar.

The pages leave the block size free and let the last block be short ("Star
Attention" analysis page, section 3.4, Phase 1 Step 1).  With blocks of 1-33
tokens and anchors of 1-31, a phase-1 row averages only a handful of values;
the bf16 rounding of such an output (half an ulp is 7.8e-3 once |O| >= 2)
can then use up most of the 1e-2 max-abs bar by itself.  So phase 1 is checked
through the float32 debug rows of star_ctx_encode_fp32: mean-abs 1e-3 of the
fp64 oracle, O equal to the round-to-nearest-even bf16 of O32 bit for bit,
and O and LSE of the plain star_ctx_encode call identical to the debug
call's.  Each O32 element is held to max-abs 1e-2, or, where larger, to the
bound of the one rounding the kernel's arithmetic adds: the probabilities
enter the P.V contraction as bf16 (each within a relative 2^-8 of its exact
value), so an output element can move by up to 2^-8 times the softmax-
weighted mean of |v| over the row's visible keys.  A row of a 1-token block
with a 1-token anchor sees two keys, and there that bound reaches ~1e-2 by
itself (|v| near 5).  The cache is bit-exact,
and the query prefill and every decode step (which average the whole context)
meet the bar on their bf16 outputs.
"""

import numpy as np
import pytest
import torch

from block_sparse_long_phase_b200 import workloads as wl
from oracle import star_oracle as so

from test_gpu_parity import assert_close, bits, check_cache

pytestmark = pytest.mark.gpu

MAX_ABS = 1e-2
MEAN_ABS = 1e-3
LSE_ABS = 1e-3
P_ROUNDING = 2.0 ** -8      # relative error of one probability rounded to bf16 (nearest)

SHORT = {
    "b1-anchor1": dict(L=150, b=1, b_a=1),
    "b1-no-anchor": dict(L=120, b=1, b_a=0),
    "b2-anchor1-ragged": dict(L=301, b=2, b_a=1),            # 151 blocks, the last of 1 token
    "b2-anchor2": dict(L=256, b=2, b_a=2, D=128, Hq=8, Hkv=2),
    "b16-anchor9-ragged": dict(L=16 * 150 + 7, b=16, b_a=9),  # 151 blocks, the last of 7
    "b16-anchor16-gqa8": dict(L=800, b=16, b_a=16, Hq=16, Hkv=2, D=128),
    "b33-anchor31-ragged": dict(L=33 * 100 + 20, b=33, b_a=31),
    "b33-anchor1-batch2": dict(B=2, L=700, b=33, b_a=1, lq=5, T=3),
    "b16-anchor9-max-blocks": dict(L=191 * 16 - 3, b=16, b_a=9, lq=3, T=2),   # 191 blocks
}


def check_phase1_fp32(cache, w, x, cpu, what):
    """Phase 1 through the float32 debug rows, against the oracle."""
    O, LSE, O32 = cache.star_ctx_encode_fp32(x["Qc"], x["Kc"], x["Vc"])
    torch.cuda.synchronize()
    Oref, Lref = so.ctx_encode(cpu["Qc"], cpu["Kc"], cpu["Vc"], w.b, w.b_a, w.scale)
    g = O32.double().cpu().numpy()
    assert np.isfinite(g).all(), f"{what}: non-finite O32"
    err = np.abs(g - Oref)
    # softmax-weighted mean of |v| per output element: the same weights over |V|
    absv, _ = so.ctx_encode(cpu["Qc"], cpu["Kc"], cpu["Vc"].abs(), w.b, w.b_a, w.scale)
    bar = np.maximum(MAX_ABS, P_ROUNDING * absv + 1e-4)
    worst = np.unravel_index(np.argmax(err - bar), err.shape)
    assert (err <= bar).all(), f"{what}: O32 error {err[worst]:.3e} > bar {bar[worst]:.3e} at {worst}"
    assert err.mean() <= MEAN_ABS, f"{what}: O32 mean-abs {err.mean():.3e}"
    assert np.abs(LSE.double().cpu().numpy() - Lref).max() <= LSE_ABS, f"{what}: LSE"
    assert torch.equal(bits(O), bits(O32.to(torch.bfloat16))), f"{what}: O is not the bf16 rounding of O32"
    return O, LSE


def check_short_case(w, what):
    from block_sparse_long_phase_b200 import StarCache
    cpu = wl.make_inputs(w, "cpu")
    x = {k: v.cuda() for k, v in cpu.items()}
    cache = StarCache(w.B, w.Hq, w.Hkv, w.D, w.L, w.b, w.b_a, w.lq + w.T, w.scale)
    O, LSE = check_phase1_fp32(cache, w, x, cpu, what)
    # the plain entry point runs the same kernel without the debug rows
    O2, LSE2 = cache.star_ctx_encode(x["Qc"], x["Kc"], x["Vc"])
    torch.cuda.synchronize()
    assert torch.equal(bits(O), bits(O2)) and torch.equal(LSE, LSE2), f"{what}: debug form differs"
    Oq, LSEq = cache.star_query_prefill(x["Qq"], x["Kq"], x["Vq"])
    dec = [cache.star_decode_step(x["qd"][t], x["kd"][t], x["vd"][t]) for t in range(w.T)]
    torch.cuda.synchronize()
    assert cache.device_error() == 0
    check_cache(cache, w, x, w.T)
    segs = so.cache_segments(cpu["Kc"], cpu["Vc"], w.b)
    region = np.zeros((w.B, w.Hkv, w.lq + w.T, w.D))
    ref, lref, qk, qv = so.query_prefill(cpu["Qq"], cpu["Kq"], cpu["Vq"], segs, region, region, 0, w.scale)
    assert_close(Oq, ref, LSEq, lref, f"{what} prefill")
    for t in range(w.T):
        ref, lref, qk, qv = so.decode_step(cpu["qd"][t], cpu["kd"][t], cpu["vd"][t], segs, qk, qv,
                                           w.lq + t, w.scale)
        assert_close(dec[t][0], ref, dec[t][1], lref[:, :, 0], f"{what} decode {t}")
    cache.close()


@pytest.mark.parametrize("name", list(SHORT))
def test_short_blocks_and_anchors(name):
    check_short_case(wl.get("tiny").with_(lq=4, T=2).with_(**SHORT[name]), name)


def test_short_blocks_fp8_decode():
    """The FP8 cache on one-token segments: every decode stage holds one row."""
    from test_gpu_fp8 import check_fp8_case
    check_fp8_case(wl.get("tiny").with_(L=150, b=1, b_a=1, lq=3, T=2), "fp8 b1")
