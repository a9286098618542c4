"""The block-sharded layer's kernels on one GPU, its ranks run one after another.

Every run here gets one GPU, so the ranks of the multi-GPU layer
(block_sparse_long_phase_b200/sharded.py) are emulated in one process: each
rank's cache, its phase 1 on the local [anchor | zeros | own blocks] layout,
and its phase-2 partial (star_partial_attend) run on the GPU in turn; the
partials are stacked as all_gather would leave them and merged with
star_lse_merge_bf16.  No collective is issued and no kernel waits for
another.  Against the single-device fp64 oracle, at the parity bar.
"""

import numpy as np
import pytest
import torch

from block_sparse_long_phase_b200 import workloads as wl
from block_sparse_long_phase_b200.sharded import ShardedStarCache
from oracle import star_oracle as so

from test_gpu_parity import assert_close

pytestmark = pytest.mark.gpu

CASES = [
    (2, dict(L=1024, b=256, b_a=256, lq=5, T=2)),
    (3, dict(L=1000, b=256, b_a=100, lq=4, T=2)),
    (4, dict(L=700, b=128, b_a=64, B=2, Hq=8, Hkv=2, D=128, lq=3, T=2)),
    (3, dict(L=300, b=256, b_a=256, lq=3, T=1)),       # a rank without blocks
    (8, dict(L=4096, b=512, b_a=512, Hq=16, Hkv=4, D=128, lq=16, T=3)),
]


@pytest.mark.parametrize("world,shape", CASES)
def test_sharded_kernels_match_the_oracle(world, shape):
    w = wl.get("tiny").with_(**shape)
    cpu = wl.make_inputs(w, "cpu")
    x = {k: v.cuda() for k, v in cpu.items()}
    ranks = [ShardedStarCache(r, world, w.B, w.Hq, w.Hkv, w.D, w.L, w.b, w.b_a, w.lq + w.T, w.scale)
             for r in range(world)]
    # phase 1, rank by rank
    O = torch.empty_like(x["Qc"])
    LSE = torch.empty((w.B, w.Hq, w.L), dtype=torch.float32, device="cuda")
    for sc in ranks:
        lay = sc.layout
        r0, r1 = lay.rows0, lay.rows0 + lay.rows
        o, l = sc.encode(x["Qc"][:, :, r0:r1].contiguous(), x["Kc"][:, :, r0:r1].contiguous(),
                         x["Vc"][:, :, r0:r1].contiguous(), x["Kc"][:, :, :w.b_a].contiguous(),
                         x["Vc"][:, :, :w.b_a].contiguous())
        O[:, :, r0:r1] = o
        LSE[:, :, r0:r1] = l
    torch.cuda.synchronize()
    Oref, Lref = so.ctx_encode(cpu["Qc"], cpu["Kc"], cpu["Vc"], w.b, w.b_a, w.scale)
    assert_close(O, Oref, LSE, Lref, f"sharded x{world} phase 1")
    # each rank's cache holds exactly its own blocks' rows
    for sc in ranks:
        lay = sc.layout
        for j in range(lay.n_blocks):
            k, v, seg = sc.cache.segment_tensors(lay.first_seg + j)
            s0 = (lay.first_block + j) * w.b
            assert torch.equal(k.view(torch.int16), x["Kc"][:, :, s0:s0 + seg.len].contiguous().view(torch.int16))
            assert torch.equal(v.view(torch.int16), x["Vc"][:, :, s0:s0 + seg.len].contiguous().view(torch.int16))

    def step(Q, K, V):
        parts = [sc.local_partial(Q, K, V) for sc in ranks]
        A = torch.stack([p[0] for p in parts])
        s = torch.stack([p[1] for p in parts])
        return ranks[-1].merge(A, s)

    Oq, Lq = step(x["Qq"], x["Kq"], x["Vq"])
    dec = [step(x["qd"][t], x["kd"][t], x["vd"][t]) for t in range(w.T)]
    torch.cuda.synchronize()
    segs = so.cache_segments(cpu["Kc"], cpu["Vc"], w.b)
    region = np.zeros((w.B, w.Hkv, w.lq + w.T, w.D))
    ref, lref, qk, qv = so.query_prefill(cpu["Qq"], cpu["Kq"], cpu["Vq"], segs, region, region, 0, w.scale)
    assert_close(Oq, ref, Lq, lref, f"sharded x{world} prefill")
    for t in range(w.T):
        ref, lref, qk, qv = so.decode_step(cpu["qd"][t], cpu["kd"][t], cpu["vd"][t], segs, qk, qv, w.lq + t, w.scale)
        assert_close(dec[t][0], ref, dec[t][1], lref, f"sharded x{world} decode {t}")
    assert [sc.cache.q_len for sc in ranks] == [0] * (world - 1) + [w.lq + w.T]
    for sc in ranks:
        assert sc.cache.device_error() == 0
        sc.close()


def test_partial_attend_over_every_segment_equals_the_prefill():
    """star_partial_attend over all segments with the query region gives the
    prefill's rows (float32 before the rounding), and over no segment and no
    query region it gives empty rows (A = 0, s = -inf)."""
    from block_sparse_long_phase_b200 import StarCache
    w = wl.get("tiny").with_(L=1000, b=256, b_a=100, lq=6, T=0)
    x = {k: v.cuda() for k, v in wl.make_inputs(w, "cpu").items()}
    a = StarCache(w.B, w.Hq, w.Hkv, w.D, w.L, w.b, w.b_a, w.lq, w.scale)
    b = StarCache(w.B, w.Hq, w.Hkv, w.D, w.L, w.b, w.b_a, w.lq, w.scale)
    a.star_ctx_encode(x["Qc"], x["Kc"], x["Vc"])
    b.star_ctx_encode(x["Qc"], x["Kc"], x["Vc"])
    O, L = a.star_query_prefill(x["Qq"], x["Kq"], x["Vq"])
    A, s = b.star_partial_attend(x["Qq"], 0, b.num_segments - 1, x["Kq"], x["Vq"])
    A0, s0 = b.star_partial_attend(x["Qq"], 0, 0)
    torch.cuda.synchronize()
    assert (O.double() - A.double()).abs().max().item() <= 1e-2
    assert (L - s).abs().max().item() <= 1e-3
    assert (A0 == 0).all() and torch.isinf(s0).all() and (s0 < 0).all()
    a.close()
    b.close()


TAIL_SHAPES = {
    "tiny": dict(L=1000, b=256, b_a=100, lq=5, T=0),
    "d128-gqa8": dict(Hq=16, Hkv=2, D=128, L=700, b=128, b_a=128, lq=3, T=0),
    "g16-batch2": dict(B=2, Hq=16, Hkv=1, L=600, b=200, b_a=50, lq=4, T=0),
}


@pytest.mark.parametrize("name", list(TAIL_SHAPES))
def test_single_row_partials_over_tail_ranges(name):
    """One row over segments [first, n) -- the sharded layer's generation
    step, which runs on the split-KV decode kernel with the leading rows left
    out -- against the oracle's local partial over the same keys: every
    first segment (n: no context at all), without the query region, and with
    it after a prefill (the token appended and attended)."""
    from block_sparse_long_phase_b200 import StarCache
    w = wl.get("tiny").with_(**TAIL_SHAPES[name])
    cpu = wl.make_inputs(w, "cpu")
    x = {k: v.cuda() for k, v in cpu.items()}
    G = w.Hq // w.Hkv
    n = -(-w.L // w.b)
    Kc, Vc = so._f64(cpu["Kc"]), so._f64(cpu["Vc"])
    q1 = (torch.randn((w.B, w.Hq, 1, w.D), generator=torch.Generator().manual_seed(11))).to(torch.bfloat16)
    k1 = (torch.randn((w.B, w.Hkv, 1, w.D), generator=torch.Generator().manual_seed(12))).to(torch.bfloat16)
    v1 = (torch.randn((w.B, w.Hkv, 1, w.D), generator=torch.Generator().manual_seed(13))).to(torch.bfloat16)
    for first in range(n + 1):
        for with_query in (0, 1):
            c = StarCache(w.B, w.Hq, w.Hkv, w.D, w.L, w.b, w.b_a, w.lq + 1, w.scale)
            c.star_ctx_encode(x["Qc"], x["Kc"], x["Vc"])
            c.star_query_prefill(x["Qq"], x["Kq"], x["Vq"])
            if with_query:
                A, s = c.star_partial_attend(q1.cuda(), first, n - first, k1.cuda(), v1.cuda())
            else:
                A, s = c.star_partial_attend(q1.cuda(), first, n - first)
            torch.cuda.synchronize()
            assert c.device_error() == 0
            keys_k = [Kc[:, :, first * w.b:]]
            keys_v = [Vc[:, :, first * w.b:]]
            if with_query:
                keys_k += [so._f64(cpu["Kq"]), so._f64(k1)]
                keys_v += [so._f64(cpu["Vq"]), so._f64(v1)]
                assert c.q_len == w.lq + 1
            else:
                assert c.q_len == w.lq
            kk, vv = np.concatenate(keys_k, axis=2), np.concatenate(keys_v, axis=2)
            q = so._f64(q1)
            for bi in range(w.B):
                for h in range(w.Hq):
                    g = h // G
                    a_ref, s_ref = so.local_partial(q[bi, h], kk[bi, g], vv[bi, g], w.scale)
                    what = f"{name} first {first} query {with_query} b{bi} h{h}"
                    got_a = A[bi, h].double().cpu().numpy()
                    got_s = s[bi, h].double().cpu().numpy()
                    if kk.shape[2] == 0:
                        assert (got_a == 0).all() and np.isneginf(got_s).all(), what
                        continue
                    assert np.abs(got_a - a_ref).max() <= 1e-2, what
                    assert np.abs(got_a - a_ref).mean() <= 1e-3, what
                    assert np.abs(got_s - s_ref).max() <= 1e-3, what
            c.close()


AFTER_ANCHOR = {
    "tiny": dict(L=1024, b=256, b_a=256),
    "anchor-shorter-ragged": dict(L=1000, b=256, b_a=100),
    "d128-gqa4": dict(Hq=16, Hkv=4, D=128, L=777, b=128, b_a=128),
    "batch2-g1": dict(B=2, Hq=4, Hkv=4, L=600, b=200, b_a=37),
    "many-blocks": dict(L=48 * 20, b=48, b_a=48),
    "no-anchor": dict(L=500, b=128, b_a=0),
}


@pytest.mark.parametrize("name", list(AFTER_ANCHOR))
def test_ctx_encode_after_anchor_matches_the_oracle(name):
    """Blocks 1..n-1 of a context encoded as a context of their own behind the
    anchor rows (star_ctx_encode_after_anchor, every local block anchored)
    give the single-device rows of those blocks, and the cache holds each
    block's own K/V rows bit for bit."""
    from block_sparse_long_phase_b200 import StarCache
    w = wl.get("tiny").with_(**AFTER_ANCHOR[name])
    cpu = wl.make_inputs(w, "cpu")
    x = {k: v.cuda() for k, v in cpu.items()}
    r0 = w.b
    c = StarCache(w.B, w.Hq, w.Hkv, w.D, w.L - r0, w.b, w.b_a, 1, w.scale)
    Ka = x["Kc"][:, :, :w.b_a].contiguous() if w.b_a else None
    Va = x["Vc"][:, :, :w.b_a].contiguous() if w.b_a else None
    O, LSE = c.star_ctx_encode_after_anchor(
        x["Qc"][:, :, r0:].contiguous(), x["Kc"][:, :, r0:].contiguous(), x["Vc"][:, :, r0:].contiguous(), Ka, Va)
    torch.cuda.synchronize()
    assert c.device_error() == 0
    Oref, Lref = so.ctx_encode(cpu["Qc"], cpu["Kc"], cpu["Vc"], w.b, w.b_a, w.scale, rows=np.arange(r0, w.L))
    assert_close(O, Oref, LSE, Lref, f"{name}: after-anchor phase 1")
    for j in range(c.num_segments - 1):
        k, v, seg = c.segment_tensors(j)
        s0 = r0 + j * w.b
        assert torch.equal(k.view(torch.int16), x["Kc"][:, :, s0:s0 + seg.len].contiguous().view(torch.int16))
        assert torch.equal(v.view(torch.int16), x["Vc"][:, :, s0:s0 + seg.len].contiguous().view(torch.int16))
    c.close()


FP8_CASES = [
    (3, dict(L=1000, b=256, b_a=100, lq=4, T=3)),
    (4, dict(L=4096, b=512, b_a=512, Hq=16, Hkv=4, D=128, lq=8, T=3)),
]


@pytest.mark.parametrize("world,shape", FP8_CASES)
def test_sharded_fp8_decode_matches_the_dequantised_oracle(world, shape):
    """Ranks with FP8 caches: the query prefill reads the bf16 rows (exact
    oracle); each generation step's partials read the E4M3 copies, so the
    merged step equals the single-device FP8 decode: the oracle on the
    dequantised context and query region, the step's own token exact."""
    from test_gpu_fp8 import decode_reference, dequantised
    w = wl.get("tiny").with_(**shape)
    cpu = wl.make_inputs(w, "cpu")
    x = {k: v.cuda() for k, v in cpu.items()}
    ranks = [ShardedStarCache(r, world, w.B, w.Hq, w.Hkv, w.D, w.L, w.b, w.b_a, w.lq + w.T, w.scale,
                              kv_fp8=True) for r in range(world)]
    for sc in ranks:
        lay = sc.layout
        r0, r1 = lay.rows0, lay.rows0 + lay.rows
        sc.encode(x["Qc"][:, :, r0:r1].contiguous(), x["Kc"][:, :, r0:r1].contiguous(),
                  x["Vc"][:, :, r0:r1].contiguous(), x["Kc"][:, :, :w.b_a].contiguous(),
                  x["Vc"][:, :, :w.b_a].contiguous())

    def step(Q, K, V):
        parts = [sc.local_partial(Q, K, V) for sc in ranks]
        return ranks[-1].merge(torch.stack([p[0] for p in parts]), torch.stack([p[1] for p in parts]))

    Oq, Lq = step(x["Qq"], x["Kq"], x["Vq"])
    dec = [step(x["qd"][t], x["kd"][t], x["vd"][t]) for t in range(w.T)]
    torch.cuda.synchronize()
    segs = so.cache_segments(cpu["Kc"], cpu["Vc"], w.b)
    region = np.zeros((w.B, w.Hkv, w.lq + w.T, w.D))
    ref, lref, _, _ = so.query_prefill(cpu["Qq"], cpu["Kq"], cpu["Vq"], segs, region, region, 0, w.scale)
    assert_close(Oq, ref, Lq, lref, f"sharded fp8 x{world} prefill")
    segs_deq = so.cache_segments(dequantised(cpu["Kc"]), dequantised(cpu["Vc"]), w.b)
    for t in range(w.T):
        o_ref, l_ref = decode_reference(cpu, segs_deq, t, w.lq, w.scale)
        assert_close(dec[t][0], o_ref, dec[t][1][:, :, 0], l_ref[:, :, 0], f"sharded fp8 x{world} decode {t}")
    for sc in ranks:
        assert sc.cache.device_error() == 0
        sc.close()
