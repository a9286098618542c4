"""GPU parity of the FP8 (E4M3) KV cache and the decode step that streams it.

What is compared, and against what:
  * the FP8 copy of every context segment and of the query region -- codes
    and per-row float32 scales -- bit-exact against the oracle's quantiser
    applied to the input K/V rows (cache contents are integer/byte work);
  * phase 1, the bf16 cache and the query prefill are unchanged by the
    option: bit-identical to a bf16-only cache;
  * each decode step against the fp64 oracle run on the DEQUANTISED cache
    (the oracle's own codes times its own scales) for every row cached
    before the step, and on the step's own new token exactly (the kernel
    folds it in from its bf16 input): max-abs 1e-2, mean-abs 1e-3, LSE 1e-3,
    as for the bf16 path.  The kernel multiplies in fp16 (E4M3 codes are
    exact in fp16; q is rounded from bf16 to fp16 -- exact for normal fp16
    magnitudes -- and p * s_v is rounded to fp16, a relative 2^-11 per term).
"""

import numpy as np
import pytest
import torch

from block_sparse_long_phase_b200 import workloads as wl
from oracle import star_oracle as so

pytestmark = pytest.mark.gpu

MAX_ABS = 1e-2
MEAN_ABS = 1e-3
LSE_ABS = 1e-3


def assert_close(got, ref, lse_got, lse_ref, what):
    g = got.detach().double().cpu().numpy()
    err = np.abs(g - ref)
    assert np.isfinite(g).all(), f"{what}: non-finite output"
    assert err.max() <= MAX_ABS, f"{what}: max-abs {err.max():.3e}"
    assert err.mean() <= MEAN_ABS, f"{what}: mean-abs {err.mean():.3e}"
    lerr = np.abs(lse_got.detach().double().cpu().numpy() - lse_ref)
    assert lerr.max() <= LSE_ABS, f"{what}: LSE max-abs {lerr.max():.3e}"


def bits(t):
    return t.contiguous().view(torch.int16)


def run(w, x, kv_fp8):
    from block_sparse_long_phase_b200 import StarCache
    cache = StarCache(w.B, w.Hq, w.Hkv, w.D, w.L, w.b, w.b_a, w.lq + w.T, w.scale, kv_fp8=kv_fp8)
    O, LSE = cache.star_ctx_encode(x["Qc"], x["Kc"], x["Vc"])
    Oq, LSEq = cache.star_query_prefill(x["Qq"], x["Kq"], x["Vq"])
    dec = [cache.star_decode_step(x["qd"][t], x["kd"][t], x["vd"][t]) for t in range(w.T)]
    torch.cuda.synchronize()
    assert cache.device_error() == 0, "a kernel gave up a bounded pipeline wait"
    return cache, O, LSE, Oq, LSEq, dec


def dequantised(Kc):
    codes, s = so.fp8_quantize_rows(Kc)
    return so.fp8_dequantize_rows(codes, s)


def check_fp8_copy(cache, w, Kc, Vc, rows_of_block=None):
    """Codes and scales of each context segment bit-exact against the oracle
    quantiser (every row, or the given rows of each block)."""
    for i, (s, n) in enumerate(so.block_table(w.L, w.b)):
        k8, v8, ks, vs = cache.segment_fp8_tensors(i)
        sel = np.arange(n) if rows_of_block is None else rows_of_block[i] - s
        for codes, scales, src in ((k8, ks, Kc), (v8, vs, Vc)):
            ref_c, ref_s = so.fp8_quantize_rows(src[:, :, s + sel])
            got_c = codes[:, :, sel].cpu().numpy()
            got_s = scales[:, :, sel].cpu().numpy()
            assert np.array_equal(got_c, ref_c), f"segment {i}: E4M3 codes differ"
            assert np.array_equal(got_s.view(np.uint32), ref_s.view(np.uint32)), f"segment {i}: scales differ"


def check_fp8_region(cache, qk, qv):
    """FP8 copy of the query region's rows in use bit-exact (qk, qv: the bf16
    rows appended so far, [B, Hkv, rows, D])."""
    n = qk.shape[2]
    k8, v8, ks, vs = cache.segment_fp8_tensors(cache.num_segments - 1)
    for codes, scales, src in ((k8, ks, qk), (v8, vs, qv)):
        ref_c, ref_s = so.fp8_quantize_rows(src)
        assert np.array_equal(codes[:, :, :n].cpu().numpy(), ref_c), "query region: E4M3 codes differ"
        assert np.array_equal(scales[:, :, :n].cpu().numpy().view(np.uint32), ref_s.view(np.uint32)), \
            "query region: scales differ"


def region_rows(x, t):
    """bf16 query-region K, V rows in use before decode step t (prefill rows,
    then the earlier decode tokens)."""
    qk = torch.cat([x["Kq"]] + [x["kd"][i] for i in range(t)], dim=2)
    qv = torch.cat([x["Vq"]] + [x["vd"][i] for i in range(t)], dim=2)
    return qk, qv


def decode_reference(x, segs_deq, t, lq, scale, bs=slice(None), gs=slice(None), hs=slice(None)):
    """Oracle of decode step t on an FP8 cache: earlier rows dequantised, the
    step's own token exact."""
    qk, qv = region_rows(x, t)
    qk, qv = qk[bs, gs].cpu(), qv[bs, gs].cpu()
    kd, vd = so._f64(x["kd"][t][bs, gs]), so._f64(x["vd"][t][bs, gs])
    rk = np.concatenate([dequantised(qk), kd], axis=2)
    rv = np.concatenate([dequantised(qv), vd], axis=2)
    return so.query_attend(x["qd"][t][bs, hs].cpu(), segs_deq, rk, rv, np.array([lq + t + 1]), scale)


VARIANTS = {
    "tiny": {},
    "ragged-last-block": dict(L=1000),
    "no-anchor": dict(b_a=0),
    "odd-sizes": dict(L=777, b=190, b_a=61, lq=13, T=5),
    "d128-gqa8": dict(Hq=16, Hkv=2, D=128, L=600, b=256, b_a=256, lq=7, T=3),
    "d128-long-ragged": dict(Hq=8, Hkv=2, D=128, L=3001, b=1024, b_a=512, lq=5, T=4),
    "batch2": dict(B=2, L=700, b=256, b_a=200, lq=9, T=4),
    "g16": dict(Hq=16, Hkv=1, L=400, b=128, b_a=128, lq=3, T=2),
    "tiny-blocks": dict(L=200, b=40, b_a=40, lq=70, T=3),
    # 32 (batch, kv head) pairs of about 100 rows on ~6 decode CTAs: every CTA streams
    # several short runs and flushes at each boundary
    "many-heads-short": dict(B=4, Hq=16, Hkv=8, D=64, L=96, b=32, b_a=32, lq=5, T=3),
}


@pytest.mark.parametrize("variant", list(VARIANTS))
def test_fp8_small_cases(variant):
    check_fp8_case(wl.get("tiny").with_(**VARIANTS[variant]), variant)


def check_fp8_case(w, variant):
    """The FP8 copy bit-exact, the bf16 side untouched, every decode step on
    the dequantised cache against the oracle."""
    x = {k: v.cuda() for k, v in wl.make_inputs(w, "cpu").items()}
    cache, O, LSE, Oq, LSEq, dec = run(w, x, kv_fp8=True)
    ref = run(w, x, kv_fp8=False)
    cpu = {k: v.cpu() for k, v in x.items()}
    check_fp8_copy(cache, w, cpu["Kc"], cpu["Vc"])
    # the bf16 side is untouched by the option
    assert torch.equal(bits(O), bits(ref[1])) and torch.equal(LSE, ref[2])
    assert torch.equal(bits(Oq), bits(ref[3])) and torch.equal(LSEq, ref[4])
    for i in range(cache.num_segments):
        k, v, _ = cache.segment_tensors(i)
        k2, v2, _ = ref[0].segment_tensors(i)
        assert torch.equal(bits(k), bits(k2)) and torch.equal(bits(v), bits(v2))
    # the query region's FP8 copy, and decode on the dequantised cache
    check_fp8_region(cache, *[t.cpu() for t in region_rows(cpu, w.T)])
    segs = so.cache_segments(dequantised(cpu["Kc"]), dequantised(cpu["Vc"]), w.b)
    for t in range(w.T):
        o_ref, l_ref = decode_reference(cpu, segs, t, w.lq, w.scale)
        assert_close(dec[t][0], o_ref, dec[t][1], l_ref[:, :, 0], f"{variant} fp8 decode {t}")
    cache.close()
    ref[0].close()


def test_fp8_zero_rows_and_wide_range():
    """All-zero rows take scale 1 and code 0; rows of very different
    magnitude each get their own scale."""
    w = wl.get("tiny").with_(L=513, b=256, b_a=256, lq=2, T=2)
    x = {k: v.cuda() for k, v in wl.make_inputs(w, "cpu").items()}
    x["Kc"][:, :, 5] = 0
    x["Vc"][:, :, 300] = 0
    x["Kc"][:, :, 7] *= 100.0
    x["Vc"][:, :, 9] *= 1e-3
    cache, O, LSE, Oq, LSEq, dec = run(w, x, kv_fp8=True)
    cpu = {k: v.cpu() for k, v in x.items()}
    check_fp8_copy(cache, w, cpu["Kc"], cpu["Vc"])
    _, _, ks, _ = cache.segment_fp8_tensors(0)
    _, _, _, vs = cache.segment_fp8_tensors(1)
    assert (ks[:, :, 5] == 1.0).all() and (vs[:, :, 300 - 256] == 1.0).all()
    segs = so.cache_segments(dequantised(cpu["Kc"]), dequantised(cpu["Vc"]), w.b)
    for t in range(w.T):
        o_ref, l_ref = decode_reference(cpu, segs, t, w.lq, w.scale)
        assert_close(dec[t][0], o_ref, dec[t][1], l_ref[:, :, 0], f"zero/wide rows decode {t}")
    cache.close()


@pytest.mark.parametrize("name", ["8b-128k-needle", "70b-128k-b4", "8b-1m"])
def test_fp8_full_size_sampled(name):
    """Full-size workload in the launch configuration the benchmark times:
    sampled FP8 rows bit-exact, sampled decode steps of two kv groups (first
    and last batch entry) against the oracle on the dequantised context."""
    w = wl.get(name)
    rng = np.random.default_rng(w.seed + 8)
    torch.cuda.empty_cache()
    x = wl.make_inputs(w, "cuda")
    cache, O, LSE, Oq, LSEq, dec = run(w, x, kv_fp8=True)
    rows = []
    for s, n in so.block_table(w.L, w.b):
        cand = {0, n - 1, 127, 128, n // 2} | set(rng.integers(0, n, 11).tolist())
        rows.append(np.array(sorted(s + c for c in cand if c < n)))
    check_fp8_copy(cache, w, x["Kc"].cpu(), x["Vc"].cpu(), rows_of_block=rows)
    for g in sorted({0, w.Hkv - 1}):
        hs, gs = slice(g * w.G, (g + 1) * w.G), slice(g, g + 1)
        for bi in sorted({0, w.B - 1}):
            bs = slice(bi, bi + 1)
            kc = dequantised(x["Kc"][bs, gs].cpu())
            vc = dequantised(x["Vc"][bs, gs].cpu())
            segs = so.cache_segments(kc, vc, w.b)
            for t in sorted({0, 1, w.T // 2, w.T - 1}):
                ref, lref = decode_reference(x, segs, t, w.lq, w.scale, bs, gs, hs)
                assert_close(dec[t][0][bs, hs], ref, dec[t][1][bs, hs], lref[:, :, 0],
                             f"{name} fp8 decode {t} kv{g} b{bi}")
    if w.needle:
        for t in (0, w.T - 1):
            assert (dec[t][1] > 10.0).all()
    cache.close()
    del x, O, LSE
    torch.cuda.empty_cache()
