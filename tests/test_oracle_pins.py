"""Pins for the fp64 oracle, against things other than itself.

* library routines: torch scaled-dot-product attention in float64 (causal),
  ``scipy.special.logsumexp``;
* the pages' own construction of augmented blocks ``[anchor | block]`` with
  plain causal attention over them (Star Attention analysis page, section 3.4,
  "Phase 1" Steps 2 and 4), run through the library routine;
* a hand-computed example (``tests/golden/star_hand_example.json``);
* closed forms and brute force on tiny inputs;
* planted mistakes in the oracle that each pin must catch.
"""

import json
import math
import os

import numpy as np
import pytest
import scipy.special
import torch
import torch.nn.functional as F

from oracle import star_oracle as so

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "star_hand_example.json")


def sdpa_causal(q, k, v, scale):
    """torch SDPA (float64, causal, square) on [R, D] arrays."""
    q = torch.from_numpy(np.ascontiguousarray(q))[None, None]
    k = torch.from_numpy(np.ascontiguousarray(k))[None, None]
    v = torch.from_numpy(np.ascontiguousarray(v))[None, None]
    return F.scaled_dot_product_attention(q, k, v, is_causal=True, scale=scale)[0, 0].numpy()


def causal_lse(q, k, scale):
    x = scale * (torch.from_numpy(q) @ torch.from_numpy(k).T).numpy()
    x = np.where(np.tril(np.ones_like(x, dtype=bool)), x, -np.inf)
    return scipy.special.logsumexp(x, axis=1)


def rand_qkv(rng, B, Hq, Hkv, L, D):
    Q = rng.standard_normal((B, Hq, L, D))
    K = rng.standard_normal((B, Hkv, L, D))
    V = rng.standard_normal((B, Hkv, L, D))
    return Q, K, V


# ---------------------------------------------------------------------------
# Block table
# ---------------------------------------------------------------------------
def test_block_table_closed_forms():
    assert so.block_table(1024, 256) == [(0, 256), (256, 256), (512, 256), (768, 256)]
    assert so.block_table(1000, 256) == [(0, 256), (256, 256), (512, 256), (768, 232)]
    assert so.block_table(5, 8) == [(0, 5)]
    assert so.block_table(0, 4) == []
    for L in range(1, 40):
        for b in range(1, 12):
            t = so.block_table(L, b)
            assert len(t) == math.ceil(L / b)
            assert sum(n for _, n in t) == L
            assert all(n == b for _, n in t[:-1]) and 1 <= t[-1][1] <= b


# ---------------------------------------------------------------------------
# Mask
# ---------------------------------------------------------------------------
def augmented_visibility(L, b, b_a):
    """Brute force from the pages' construction: augmented block i >= 1 is the
    token list anchor + block i in that order; every token sees the tokens that
    precede it in its augmented block (causal self-attention over it).  Block 0
    is its own augmented block.  Only block tokens are outputs."""
    vis = np.zeros((L, L), dtype=bool)
    for i, (s, n) in enumerate(so.block_table(L, b)):
        seq = list(range(s, s + n)) if i == 0 else list(range(b_a)) + list(range(s, s + n))
        for pos, t in enumerate(seq):
            if t >= s:  # a block token (not an anchor copy)
                for j in seq[:pos + 1]:
                    vis[t, j] = True
    return vis


def test_mask_brute_force_all_small_cases():
    for L in range(1, 18):
        for b in range(1, L + 2):
            for b_a in range(0, b + 1):
                assert np.array_equal(so.star_mask(L, b, b_a), augmented_visibility(L, b, b_a)), (L, b, b_a)


def test_mask_single_block_is_causal():
    for L in (1, 7, 33):
        assert np.array_equal(so.star_mask(L, L, L), np.tril(np.ones((L, L), dtype=bool)))
        assert np.array_equal(so.star_mask(L, 4 * L, 0), np.tril(np.ones((L, L), dtype=bool)))


def test_mask_rejects_anchor_longer_than_block():
    with pytest.raises(ValueError):
        so.star_mask(8, 2, 3)


# ---------------------------------------------------------------------------
# Phase 1 against the library routine
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("L,D,Hq,Hkv", [(37, 8, 4, 2), (64, 16, 2, 2), (50, 4, 6, 3)])
def test_phase1_single_block_is_full_causal_attention(rng, L, D, Hq, Hkv):
    Q, K, V = rand_qkv(rng, 2, Hq, Hkv, L, D)
    scale = 1 / math.sqrt(D)
    for b in (L, L + 5):
        O, LSE = so.ctx_encode(Q, K, V, b, min(b, 3), scale)
        G = Hq // Hkv
        for bi in range(2):
            for h in range(Hq):
                ref = sdpa_causal(Q[bi, h], K[bi, h // G], V[bi, h // G], scale)
                np.testing.assert_allclose(O[bi, h], ref, rtol=0, atol=1e-12)
                np.testing.assert_allclose(LSE[bi, h], causal_lse(Q[bi, h], K[bi, h // G], scale),
                                           rtol=0, atol=1e-12)


@pytest.mark.parametrize("L,b,b_a", [(64, 16, 16), (64, 16, 5), (61, 16, 16), (61, 16, 0),
                                     (40, 7, 3), (33, 32, 32), (9, 1, 1), (9, 2, 0)])
def test_phase1_equals_causal_attention_over_augmented_blocks(rng, L, b, b_a):
    """Each block i >= 1 equals plain causal attention over [anchor | block i]
    (outputs of the block rows); block 0 equals causal attention over itself."""
    Hq, Hkv, D = 4, 2, 8
    Q, K, V = rand_qkv(rng, 1, Hq, Hkv, L, D)
    scale = 1 / math.sqrt(D)
    O, LSE = so.ctx_encode(Q, K, V, b, b_a, scale)
    for i, (s, n) in enumerate(so.block_table(L, b)):
        idx = np.arange(s, s + n) if i == 0 else np.concatenate([np.arange(b_a), np.arange(s, s + n)])
        for h in range(Hq):
            g = h // 2
            ref = sdpa_causal(Q[0, h, idx], K[0, g, idx], V[0, g, idx], scale)[-n:]
            np.testing.assert_allclose(O[0, h, s:s + n], ref, rtol=0, atol=1e-12)
            lse = causal_lse(Q[0, h, idx], K[0, g, idx], scale)[-n:]
            np.testing.assert_allclose(LSE[0, h, s:s + n], lse, rtol=0, atol=1e-12)


def test_phase1_row_subset_matches_full(rng):
    Q, K, V = rand_qkv(rng, 1, 2, 1, 48, 8)
    O, LSE = so.ctx_encode(Q, K, V, 16, 8, 0.3)
    rows = np.array([0, 15, 16, 31, 47])
    Os, LSEs = so.ctx_encode(Q, K, V, 16, 8, 0.3, rows=rows)
    assert Os.shape == (1, 2, len(rows), 8) and LSEs.shape == (1, 2, len(rows))
    np.testing.assert_array_equal(Os, O[:, :, rows])
    np.testing.assert_array_equal(LSEs, LSE[:, :, rows])
    # torch bf16 inputs give the same result as their exact float64 upcast
    Qt, Kt, Vt = (torch.from_numpy(x).to(torch.bfloat16) for x in (Q, K, V))
    Ob, Lb = so.ctx_encode(Qt, Kt, Vt, 16, 8, 0.3, rows=rows)
    Of, Lf = so.ctx_encode(Qt.double().numpy(), Kt.double().numpy(), Vt.double().numpy(),
                           16, 8, 0.3, rows=rows)
    np.testing.assert_array_equal(Ob, Of)
    np.testing.assert_array_equal(Lb, Lf)


def test_phase1_split_identity(rng):
    """Block rows of block i >= 1 equal the merge of (row vs anchor, unmasked)
    and (row vs own block, causal): phase 1 expressed through the merge."""
    L, b, b_a, D = 48, 16, 10, 8
    Q, K, V = rand_qkv(rng, 1, 1, 1, L, D)
    scale = 1 / math.sqrt(D)
    O, LSE = so.ctx_encode(Q, K, V, b, b_a, scale)
    for s in (16, 32):
        q = Q[0, 0, s:s + b]
        a1, s1 = so.local_partial(q, K[0, 0, :b_a], V[0, 0, :b_a], scale)
        a2, s2 = so.local_partial(q, K[0, 0, s:s + b], V[0, 0, s:s + b], scale,
                                  np.tril(np.ones((b, b), dtype=bool)))
        A, S = so.lse_merge(np.stack([a1, a2]), np.stack([s1, s2]))
        np.testing.assert_allclose(A, O[0, 0, s:s + b], atol=1e-12, rtol=0)
        np.testing.assert_allclose(S, LSE[0, 0, s:s + b], atol=1e-12, rtol=0)


# ---------------------------------------------------------------------------
# Golden, hand-computed example
# ---------------------------------------------------------------------------
def test_golden_hand_example():
    g = json.load(open(GOLDEN))
    L, b, b_a = g["L"], g["b"], g["b_a"]
    Q = np.array(g["q_ctx"], float).reshape(1, 1, L, 1)
    K = np.log(np.array(g["k_ctx_exp"], float)).reshape(1, 1, L, 1)
    V = np.array(g["v_ctx"], float).reshape(1, 1, L, 1)
    mask = so.star_mask(L, b, b_a)
    for t, vis in enumerate(g["phase1_visible"]):
        assert list(np.nonzero(mask[t])[0]) == vis
    O, LSE = so.ctx_encode(Q, K, V, b, b_a, g["scale"])
    np.testing.assert_allclose(O[0, 0, :, 0], g["phase1_out"], rtol=1e-13)
    np.testing.assert_allclose(np.exp(LSE[0, 0]), g["phase1_lse_exp"], rtol=1e-13)
    segs = so.cache_segments(K, V, b)
    qq = np.full((1, 1, 1, 1), float(g["query"]["q"]))
    kq = np.full((1, 1, 1, 1), math.log(g["query"]["k_exp"]))
    vq = np.full((1, 1, 1, 1), float(g["query"]["v"]))
    region = np.zeros((1, 1, 4, 1))
    O2, LSE2, qk, qv = so.query_prefill(qq, kq, vq, segs, region, region, 0, g["scale"])
    np.testing.assert_allclose(O2[0, 0, 0, 0], g["phase2_out_num"] / g["phase2_out_den"], rtol=1e-13)
    np.testing.assert_allclose(np.exp(LSE2[0, 0, 0]), g["phase2_lse_exp"], rtol=1e-13)
    O3, LSE3 = so.phase2_partials(qq, segs, qk, qv, np.array([1]), g["scale"])
    np.testing.assert_allclose(O3, O2, rtol=1e-13)
    parts = g["phase2_partials"]
    for name, (s, n) in zip(["segment0", "segment1"], so.block_table(L, b)):
        a, sh = so.local_partial(qq[0, 0], K[0, 0, s:s + n], V[0, 0, s:s + n], 1.0)
        np.testing.assert_allclose(a[0, 0], parts[name]["out"], rtol=1e-13)
        np.testing.assert_allclose(np.exp(sh[0]), parts[name]["lse_exp"], rtol=1e-13)


# ---------------------------------------------------------------------------
# Merge
# ---------------------------------------------------------------------------
def test_merge_closed_forms():
    A = np.array([[[1.0, 2.0]], [[5.0, -2.0]]])
    s = np.log(np.array([[1.0], [3.0]]))
    out, lse = so.lse_merge(A, s)
    np.testing.assert_allclose(out[0], [0.25 * 1 + 0.75 * 5, 0.25 * 2 - 0.75 * 2], rtol=1e-15)
    np.testing.assert_allclose(lse, [math.log(4.0)], rtol=1e-15)
    # one part is the identity
    out, lse = so.lse_merge(A[:1], s[:1])
    np.testing.assert_array_equal(out, A[0])
    # large values do not overflow
    out, lse = so.lse_merge(A, np.array([[1000.0], [1000.0]]))
    np.testing.assert_allclose(lse, [1000 + math.log(2)], rtol=1e-15)
    np.testing.assert_allclose(out[0], [3.0, 0.0], atol=1e-13)
    # empty parts contribute nothing; all-empty gives 0 / -inf
    out, lse = so.lse_merge(A, np.array([[-np.inf], [0.3]]))
    np.testing.assert_array_equal(out[0], A[1, 0])
    out, lse = so.lse_merge(A, np.array([[-np.inf], [-np.inf]]))
    assert lse[0] == -np.inf and (out == 0).all()


def test_merge_partition_identity(rng):
    """Merging partials over any partition of the keys (empty parts included)
    equals one softmax over all keys, and its LSE equals scipy's logsumexp."""
    R, N, D = 5, 57, 8
    q = rng.standard_normal((R, D))
    k = rng.standard_normal((N, D)) * 2
    v = rng.standard_normal((N, D))
    scale = 0.4
    full_o, full_lse = so.local_partial(q, k, v, scale)
    logits = scale * (torch.from_numpy(q) @ torch.from_numpy(k).T).numpy()
    np.testing.assert_allclose(full_lse, scipy.special.logsumexp(logits, axis=1), atol=1e-12)
    w = scipy.special.softmax(logits, axis=1)
    np.testing.assert_allclose(full_o, w @ v, atol=1e-12)
    for trial in range(20):
        cuts = np.sort(rng.integers(0, N + 1, size=rng.integers(1, 6)))
        bounds = [0, *cuts, N]
        As, ss = [], []
        for lo, hi in zip(bounds[:-1], bounds[1:]):
            a, s = so.local_partial(q, k[lo:hi], v[lo:hi], scale)
            As.append(a)
            ss.append(s)
        perm = rng.permutation(len(As))
        A, S = so.lse_merge(np.stack(As)[perm], np.stack(ss)[perm])
        np.testing.assert_allclose(A, full_o, atol=1e-12, rtol=0)
        np.testing.assert_allclose(S, full_lse, atol=1e-12, rtol=0)


# ---------------------------------------------------------------------------
# Cache
# ---------------------------------------------------------------------------
def test_cache_segments_cover_context_once():
    L, b = 1000, 256
    K = np.arange(2 * 3 * L * 4, dtype=np.uint16).reshape(2, 3, L, 4)
    V = K[..., ::-1].copy()
    segs = so.cache_segments(K, V, b)
    assert [(s, n) for s, n, _, _ in segs] == so.block_table(L, b)
    assert np.array_equal(np.concatenate([k for _, _, k, _ in segs], axis=2), K)
    assert np.array_equal(np.concatenate([v for _, _, _, v in segs], axis=2), V)
    # no segment i >= 1 holds an anchor row (rows 0..b_a-1, b_a <= b)
    for s, n, k, _ in segs[1:]:
        assert s >= b


# ---------------------------------------------------------------------------
# Phase 2 against global causal attention over [context | query region]
# ---------------------------------------------------------------------------
def _global_rows(Qc, Kc, Vc, Qn, Kn, Vn, scale):
    """Causal SDPA over the concatenation; returns the rows of the new tokens."""
    q = np.concatenate([Qc, Qn], axis=0)
    k = np.concatenate([Kc, Kn], axis=0)
    v = np.concatenate([Vc, Vn], axis=0)
    o = sdpa_causal(q, k, v, scale)[-Qn.shape[0]:]
    lse = causal_lse(q, k, scale)[-Qn.shape[0]:]
    return o, lse


def test_query_prefill_and_decode_are_global_attention(rng):
    B, Hq, Hkv, D, L, b, lq, T = 2, 4, 2, 8, 40, 16, 5, 4
    G = Hq // Hkv
    scale = 1 / math.sqrt(D)
    Qc, Kc, Vc = rand_qkv(rng, B, Hq, Hkv, L, D)
    Qq, Kq, Vq = rand_qkv(rng, B, Hq, Hkv, lq, D)
    segs = so.cache_segments(Kc, Vc, b)
    cap = lq + T
    qk = np.zeros((B, Hkv, cap, D))
    qv = np.zeros((B, Hkv, cap, D))
    O, LSE, qk, qv = so.query_prefill(Qq, Kq, Vq, segs, qk, qv, 0, scale)
    for bi in range(B):
        for h in range(Hq):
            o, lse = _global_rows(Qc[bi, h], Kc[bi, h // G], Vc[bi, h // G],
                                  Qq[bi, h], Kq[bi, h // G], Vq[bi, h // G], scale)
            np.testing.assert_allclose(O[bi, h], o, atol=1e-12, rtol=0)
            np.testing.assert_allclose(LSE[bi, h], lse, atol=1e-12, rtol=0)
    # the partials form agrees
    O2, LSE2 = so.phase2_partials(Qq, segs, qk, qv, np.arange(lq) + 1, scale)
    np.testing.assert_allclose(O2, O, atol=1e-12)
    np.testing.assert_allclose(LSE2, LSE, atol=1e-12)
    # decode steps: append then attend
    hist_q, hist_k, hist_v = Qq, Kq, Vq
    n = lq
    for t in range(T):
        q, k, v = rand_qkv(rng, B, Hq, Hkv, 1, D)
        o, lse, qk, qv = so.decode_step(q, k, v, segs, qk, qv, n, scale)
        hist_q = np.concatenate([hist_q, q], axis=2)
        hist_k = np.concatenate([hist_k, k], axis=2)
        hist_v = np.concatenate([hist_v, v], axis=2)
        n += 1
        assert np.array_equal(qk[:, :, :n], hist_k) and np.array_equal(qv[:, :, :n], hist_v)
        for bi in range(B):
            for h in range(Hq):
                ro, rl = _global_rows(Qc[bi, h], Kc[bi, h // G], Vc[bi, h // G],
                                      hist_q[bi, h], hist_k[bi, h // G], hist_v[bi, h // G], scale)
                np.testing.assert_allclose(o[bi, h, 0], ro[-1], atol=1e-12, rtol=0)
                np.testing.assert_allclose(lse[bi, h, 0], rl[-1], atol=1e-12, rtol=0)


def test_phase2_only_query_region_grows(rng):
    B, Hq, Hkv, D, L, b = 1, 2, 1, 4, 20, 8
    Qc, Kc, Vc = rand_qkv(rng, B, Hq, Hkv, L, D)
    segs = so.cache_segments(Kc, Vc, b)
    before = [(s, n, k.copy(), v.copy()) for s, n, k, v in segs]
    qk = np.zeros((B, Hkv, 3, D))
    q, k, v = rand_qkv(rng, B, Hq, Hkv, 1, D)
    _, _, qk2, _ = so.decode_step(q, k, v, segs, qk, qk, 0, 0.5)
    for (s0, n0, k0, v0), (s1, n1, k1, v1) in zip(before, segs):
        assert (s0, n0) == (s1, n1) and np.array_equal(k0, k1) and np.array_equal(v0, v1)
    assert np.array_equal(qk2[:, :, 0], k[:, :, 0]) and not qk2[:, :, 1:].any()


# ---------------------------------------------------------------------------
# Needle workload generator sanity (small context, same construction)
# ---------------------------------------------------------------------------
def test_needle_generator_peaks_the_merged_softmax():
    from block_sparse_long_phase_b200 import workloads as wl
    w = wl.get("8b-128k-needle").with_(L=4096, b=1024, b_a=1024, lq=4, T=1, Hq=8, Hkv=2)
    x = wl.make_inputs(w, "cpu")
    Kc = x["Kc"].double().numpy()
    Vc = x["Vc"].double().numpy()
    Qq = x["Qq"].double().numpy()
    segs = so.cache_segments(Kc, Vc, w.b)
    region = np.zeros((w.B, w.Hkv, w.lq, w.D))
    O, LSE, _, _ = so.query_prefill(Qq, x["Kq"].double().numpy(), x["Vq"].double().numpy(),
                                    segs, region, region, 0, w.scale)
    pos = x["needle_pos"].numpy()
    for h in range(w.Hq):
        g = h // w.G
        logits = w.scale * Qq[0, h] @ Kc[0, g].T
        lse_ctx = scipy.special.logsumexp(logits, axis=1)
        mass = np.exp(scipy.special.logsumexp(logits[:, pos[0, g]], axis=1) - lse_ctx)
        assert (mass >= 0.9).all(), mass
        assert (LSE[0, h] >= 12.0).all()


# ---------------------------------------------------------------------------
# Planted mistakes: each must be caught by a pin above.
# ---------------------------------------------------------------------------
def test_planted_mask_mistakes_are_caught(monkeypatch, rng):
    good = so.star_mask_rows

    def no_anchor(L, b, b_a, rows):
        return good(L, b, 0, rows)

    def whole_first_block_visible(L, b, b_a, rows):
        t = np.asarray(rows)[:, None]
        j = np.arange(L)[None, :]
        return good(L, b, b_a, rows) | (((t // b) >= 1) & (j // b == 0))

    for bad in (no_anchor, whole_first_block_visible):
        monkeypatch.setattr(so, "star_mask_rows", bad)
        with pytest.raises(AssertionError):
            test_phase1_equals_causal_attention_over_augmented_blocks(rng, 64, 16, 5)
    monkeypatch.setattr(so, "star_mask_rows", good)


def test_planted_merge_mistake_is_caught(monkeypatch, rng):
    good = so.lse_merge

    def sign_flip(A, s):  # exp(s - s_h) instead of exp(s_h - s)
        m = s.max(axis=0)
        sg = m + np.log(np.exp(s - m).sum(axis=0))
        return np.einsum("pr,prd->rd", np.exp(sg[None] - s), A), sg

    monkeypatch.setattr(so, "lse_merge", sign_flip)
    with pytest.raises(AssertionError):
        test_merge_partition_identity(rng)
    monkeypatch.setattr(so, "lse_merge", good)
