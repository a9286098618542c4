"""Plain, slow, fp64 CPU oracle for the Star Attention two-phase attention path.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path imports, calls or
links this module: only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` use it.  It shares
no code with the CUDA path; it takes plain NumPy arrays (the exact bf16 inputs
upcast to float64) and returns float64 results.

Sources (page title, then section / step / equation):

* [P2] "Star Attention: Efficient LLM Inference over Long Sequences"
  (paper-graph-ui analysis page), section 3.4 "Detailed, Sentence-Based
  Technical Breakdown":
    - "The Attention Decomposition" -- the causal softmax-attention equation
      with scale 1/sqrt(d);
    - "Phase 1: Context Encoding with Anchor Blocks", Steps 1-5 (partition,
      anchor augmentation with preserved positions, blockwise-local causal
      attention, anchor KV discard);
    - "Phase 2: Query Encoding and Token Generation with Distributed Softmax",
      Steps 3 (local A_h, s_h), the partition identity, Step 5 (log-sum-exp
      aggregation) and Step 7 (only the query region grows).
* [P3] "NVIDIA/Star-Attention" (README mirror), section "Two Phases of Star
  Attention": Phase 1 bullets (segmentation, anchor prefix, non-anchor KV kept)
  and Phase 2 bullets (A_h, s_h, s_global, A_global).

Readings where the pages are silent or garbled (the passage each one settles
is the [P2] Phase 1 / Phase 2 step named beside it):

* the anchor is the first ``b_a`` context tokens, ``0 <= b_a <= b`` ([P2]
  Phase 1 Step 2 names the first block as the anchor; its length is left open);
* block 0 is plain causal attention over its own rows, blocks i >= 1 see the
  whole anchor plus their own block causally; only block rows are outputs
  ([P2] Phase 1 Steps 2 and 4: causal attention over the augmented block,
  whose anchor KV Step 5 then discards);
* the last block may be short ([P2] Phase 1 Step 1);
* ``s_h`` is carried as a natural-log log-sum-exp over the *scaled* logits;
  the merge is ``s = log sum_h exp(s_h)``, ``A = sum_h exp(s_h - s) A_h``
  (algebraically the README's ``s_h / s_global`` weights); the garbled
  log-space update printed in [P2] Step 5 is not followed;
* grouped-query heads map contiguously: q head ``h`` reads kv head
  ``h // (Hq // Hkv)``;
* a query row ``r`` sees query-region rows ``0..r``; a decode token is
  appended to the query region first and then attends to it (itself included).

Every function here is pinned by ``tests/test_oracle_pins.py`` against
library routines (torch scaled-dot-product attention in float64,
``scipy.special.logsumexp``), closed forms and brute force.
"""

from __future__ import annotations

import numpy as np

NEG_INF = -np.inf


def _f64(x) -> np.ndarray:
    """Exact float64 copy on the host of a NumPy array or a torch tensor
    (bf16 and fp32 values are representable exactly in float64)."""
    if isinstance(x, np.ndarray):
        return x.astype(np.float64, copy=False)
    if hasattr(x, "detach"):
        return x.detach().double().cpu().numpy()
    return np.asarray(x, dtype=np.float64)


# ---------------------------------------------------------------------------
# Phase 1, Step 1: partition of the context into blocks.
# ---------------------------------------------------------------------------
def block_table(L: int, b: int) -> list[tuple[int, int]]:
    """Blocks ``c_1..c_n`` of a context of ``L`` tokens with block size ``b``.

    [P2] Phase 1 Step 1: ``n = ceil(L / b)`` contiguous blocks, the last one
    possibly shorter.  Returns ``[(start, length), ...]``.
    """
    if L < 0 or b < 1:
        raise ValueError("need L >= 0 and b >= 1")
    n = -(-L // b)
    return [(i * b, min((i + 1) * b, L) - i * b) for i in range(n)]


# ---------------------------------------------------------------------------
# Phase 1, Steps 2-4: the explicit Star mask.
# ---------------------------------------------------------------------------
def star_mask_rows(L: int, b: int, b_a: int, rows) -> np.ndarray:
    """Rows ``rows`` of the explicit Star-Attention context mask, bool [R, L].

    ``M[t, j]`` is True iff context token ``t`` attends to token ``j`` in
    phase 1 ([P2] Phase 1 Steps 2 and 4, [P3] Phase 1 bullets):

    * ``j <= t`` (causal), and
    * ``j`` lies in the same block as ``t``, or ``t`` lies in a block
      ``i >= 1`` and ``j`` is an anchor token (``j < b_a``).

    The anchor keeps its original positions (Step 2), so with pre-rotated
    inputs its keys are literally rows ``0..b_a-1`` of the context K/V.
    """
    if not (0 <= b_a <= b):
        raise ValueError("need 0 <= b_a <= b")
    t = np.asarray(rows, dtype=np.int64)[:, None]
    j = np.arange(L, dtype=np.int64)[None, :]
    causal = j <= t
    same_block = (j // b) == (t // b)
    anchor = ((t // b) >= 1) & (j < b_a)
    return causal & (same_block | anchor)


def star_mask(L: int, b: int, b_a: int) -> np.ndarray:
    """The full ``L x L`` Star mask (small ``L`` only)."""
    return star_mask_rows(L, b, b_a, np.arange(L))


# ---------------------------------------------------------------------------
# The attention equation ([P2] "The Attention Decomposition").
# ---------------------------------------------------------------------------
def masked_attention(q: np.ndarray, k: np.ndarray, v: np.ndarray,
                     mask: np.ndarray, scale: float):
    """Softmax attention of rows ``q`` [R, D] over keys ``k``/``v`` [N, D].

    Only keys with ``mask[r, j]`` True take part.  Returns ``(O [R, D],
    LSE [R])`` in float64, where ``LSE = log sum_j exp(scale * q.k_j)`` over
    the visible keys (natural log of the scaled logits) and ``O`` is the
    softmax-weighted mean of the visible values.  A row with no visible key
    gets ``O = 0`` and ``LSE = -inf``.
    """
    q = _f64(q)
    k = _f64(k)
    v = _f64(v)
    x = scale * (q @ k.T)
    x = np.where(mask, x, NEG_INF)
    m = x.max(axis=1, initial=NEG_INF)
    empty = ~np.isfinite(m)
    m_safe = np.where(empty, 0.0, m)
    e = np.exp(x - m_safe[:, None])
    ssum = e.sum(axis=1)
    with np.errstate(divide="ignore", invalid="ignore"):
        lse = np.where(empty, NEG_INF, m_safe + np.log(ssum))
        o = np.where(empty[:, None], 0.0, (e @ v) / ssum[:, None])
    return o, lse


# ---------------------------------------------------------------------------
# Phase 1: context encoding.
# ---------------------------------------------------------------------------
def ctx_encode(Q, K, V, b: int, b_a: int, scale: float, rows=None):
    """Phase-1 outputs for Q [B, Hq, L, D], K/V [B, Hkv, L, D].

    For every context token ``t`` and q head ``h`` (kv head ``h // G``), the
    output is softmax attention over the tokens the Star mask lets ``t`` see
    ([P2] Phase 1 Step 4).  ``rows`` (default: all) selects the token indices
    to compute; the result for a row does not depend on which other rows are
    computed.  Inputs may be NumPy arrays or torch tensors (only the rows and
    keys used are copied to float64).

    Returns ``(O [B, Hq, R, D], LSE [B, Hq, R])`` float64 for the R rows.
    """
    Bn, Hq, L, D = Q.shape
    Hkv = K.shape[1]
    if Hq % Hkv:
        raise ValueError("Hq must be a multiple of Hkv")
    G = Hq // Hkv
    rows = np.arange(L) if rows is None else np.asarray(rows, np.int64)
    O = np.zeros((Bn, Hq, len(rows), D))
    LSE = np.zeros((Bn, Hq, len(rows)))
    if len(rows) == 0:
        return O, LSE
    mask = star_mask_rows(L, b, b_a, rows)
    # Only the union of visible columns is needed; gather them once.
    cols = np.nonzero(mask.any(axis=0))[0]
    sub = mask[:, cols]
    for bi in range(Bn):
        for g in range(Hkv):
            k = _f64(K[bi, g][cols])
            v = _f64(V[bi, g][cols])
            for h in range(g * G, (g + 1) * G):
                o, lse = masked_attention(_f64(Q[bi, h][rows]), k, v, sub, scale)
                O[bi, h] = o
                LSE[bi, h] = lse
    return O, LSE


def cache_segments(K: np.ndarray, V: np.ndarray, b: int):
    """Per-block KV-cache segments kept after phase 1.

    [P2] Phase 1 Step 5 / [P3] Phase 1 last bullet: block ``i`` keeps only
    the K/V of its own tokens; the anchor's K/V is discarded, so every
    context token is cached exactly once.  Returns a list of
    ``(start, length, K_seg [B, Hkv, len, D], V_seg [B, Hkv, len, D])``.
    Works on any dtype (bit-exact comparisons use the raw bf16 bits).
    """
    L = K.shape[2]
    return [(s, n, K[:, :, s:s + n], V[:, :, s:s + n])
            for (s, n) in block_table(L, b)]


# ---------------------------------------------------------------------------
# Phase 2: local partials, their merge, query prefill and decode.
# ---------------------------------------------------------------------------
def local_partial(q: np.ndarray, k: np.ndarray, v: np.ndarray, scale: float,
                  mask: np.ndarray | None = None):
    """One partition's local attention ``A_h`` and its log-sum-exp ``s_h``.

    [P2] Phase 2 Step 3 / [P3] Phase 2: ``A_h`` is the softmax attention of
    ``q`` [R, D] over this partition's keys only; ``s_h`` (carried here in
    log space) is ``log sum_k exp(q.k / sqrt(d))`` over the same keys.  An
    empty partition gives ``A_h = 0``, ``s_h = -inf``.
    """
    if mask is None:
        mask = np.ones((q.shape[0], k.shape[0]), dtype=bool)
    return masked_attention(q, k, v, mask, scale)


def lse_merge(A: np.ndarray, s: np.ndarray):
    """Merge partials ``A [P, R, D]``, ``s [P, R]`` into ``(A [R, D], s [R])``.

    [P3] Phase 2: ``s_global = sum_h s_h`` and ``A_global = sum_h (s_h /
    s_global) A_h`` with raw exponent sums; written here in log space as
    [P2] Step 5 intends: ``s = log sum_h exp(s_h)`` and
    ``A = sum_h exp(s_h - s) A_h``.  The maximum is subtracted before
    exponentiating; partitions with ``s_h = -inf`` contribute nothing.
    """
    A = _f64(A)
    s = _f64(s)
    m = s.max(axis=0)
    empty = ~np.isfinite(m)
    m_safe = np.where(empty, 0.0, m)
    w = np.exp(s - m_safe[None])                  # exp(s_h - m), 0 for -inf
    tot = w.sum(axis=0)
    with np.errstate(divide="ignore", invalid="ignore"):
        s_glob = np.where(empty, NEG_INF, m_safe + np.log(tot))
        coef = np.where(empty[None], 0.0, np.exp(s - np.where(empty, 0.0, s_glob)[None]))
    A_glob = np.einsum("pr,prd->rd", coef, A)
    return A_glob, s_glob


def _context_keys(segments, bi, g):
    """Concatenation of every context segment's cache for (batch, kv head)."""
    ks = [_f64(seg[2][bi, g]) for seg in segments]
    vs = [_f64(seg[3][bi, g]) for seg in segments]
    return np.concatenate(ks, axis=0), np.concatenate(vs, axis=0)


def query_attend(q_rows: np.ndarray, segments, qk_region: np.ndarray,
                 qv_region: np.ndarray, visible_q: np.ndarray, scale: float):
    """Exact global attention of phase-2 rows over the whole cache.

    ``q_rows`` [B, Hq, R, D]; ``segments`` from :func:`cache_segments`;
    ``qk_region``/``qv_region`` [B, Hkv, Nq, D] is the query region's cache
    (query and generated tokens, [P2] Phase 2 Step 7); row ``r`` sees every
    context token and the first ``visible_q[r]`` query-region rows.

    This is the definition the distributed softmax reproduces exactly
    ([P2] Phase 2, the partition identity): one softmax over
    ``[context cache || query region]``.  Returns ``(O, LSE)`` float64.
    """
    Bn, Hq, R, D = q_rows.shape
    Hkv = qk_region.shape[1]
    G = Hq // Hkv
    Nq = qk_region.shape[2]
    O = np.zeros((Bn, Hq, R, D))
    LSE = np.zeros((Bn, Hq, R))
    for bi in range(Bn):
        for g in range(Hkv):
            kc, vc = _context_keys(segments, bi, g)
            k_all = np.concatenate([kc, _f64(qk_region[bi, g])], axis=0)
            v_all = np.concatenate([vc, _f64(qv_region[bi, g])], axis=0)
            Lc = kc.shape[0]
            mask = np.ones((R, Lc + Nq), dtype=bool)
            mask[:, Lc:] = np.arange(Nq)[None, :] < np.asarray(visible_q)[:, None]
            for h in range(g * G, (g + 1) * G):
                o, lse = masked_attention(_f64(q_rows[bi, h]), k_all, v_all, mask, scale)
                O[bi, h] = o
                LSE[bi, h] = lse
    return O, LSE


def query_prefill(Qq, Kq, Vq, segments, qk_region, qv_region, q_len0: int,
                  scale: float):
    """Phase-2 query prefill.

    Appends ``Kq``/``Vq`` [B, Hkv, lq, D] to the query region (which held
    ``q_len0`` rows) and attends each query row ``r`` to all context segments
    plus query-region rows ``0..q_len0 + r``.  Returns ``(O, LSE, qk_region,
    qv_region)`` with the regions updated (copies).
    """
    lq = Qq.shape[2]
    qk = _f64(qk_region).copy()
    qv = _f64(qv_region).copy()
    qk[:, :, q_len0:q_len0 + lq] = _f64(Kq)
    qv[:, :, q_len0:q_len0 + lq] = _f64(Vq)
    vis = q_len0 + np.arange(lq) + 1
    O, LSE = query_attend(Qq, segments, qk, qv, vis, scale)
    return O, LSE, qk, qv


def decode_step(q, k, v, segments, qk_region, qv_region, q_len: int,
                scale: float):
    """One phase-2 generation step for q [B, Hq, 1, D], k/v [B, Hkv, 1, D].

    [P2] Phase 2 Step 7: the new token's K/V is appended to the query region
    only (at row ``q_len``), then the token attends to every context token
    and query-region rows ``0..q_len`` (itself included).
    """
    qk = _f64(qk_region).copy()
    qv = _f64(qv_region).copy()
    qk[:, :, q_len] = _f64(k)[:, :, 0]
    qv[:, :, q_len] = _f64(v)[:, :, 0]
    O, LSE = query_attend(q, segments, qk, qv, np.array([q_len + 1]), scale)
    return O, LSE, qk, qv


def phase2_partials(q_rows, segments, qk_region, qv_region, visible_q, scale):
    """Second, independent form of phase 2: per-segment partials + merge.

    Each context segment ``h`` gives ``(A_h, s_h)`` ([P2] Phase 2 Step 3); the
    query region is one more partition with its causal visibility; the
    partials are merged with :func:`lse_merge` ([P2] Step 5).  Used only to
    check the partition identity against :func:`query_attend`.
    """
    Bn, Hq, R, D = q_rows.shape
    Hkv = qk_region.shape[1]
    G = Hq // Hkv
    Nq = qk_region.shape[2]
    O = np.zeros((Bn, Hq, R, D))
    LSE = np.zeros((Bn, Hq, R))
    qmask = np.arange(Nq)[None, :] < np.asarray(visible_q)[:, None]
    for bi in range(Bn):
        for h in range(Hq):
            g = h // G
            As, ss = [], []
            for seg in segments:
                a, s = local_partial(q_rows[bi, h], seg[2][bi, g], seg[3][bi, g], scale)
                As.append(a)
                ss.append(s)
            a, s = local_partial(q_rows[bi, h], qk_region[bi, g], qv_region[bi, g],
                                 scale, qmask)
            As.append(a)
            ss.append(s)
            o, lse = lse_merge(np.stack(As), np.stack(ss))
            O[bi, h] = o
            LSE[bi, h] = lse
    return O, LSE


# ---------------------------------------------------------------------------
# FP8 (E4M3) context cache for decode.
#
# The pages call KV-cache quantisation orthogonal to the method and fix no
# scheme, so this is the build's own definition, stated once here and in the
# C header: every cached K or V row (one token of one kv head) is scaled by
# s = max|x| / 448 (s = 1 when max|x| <= 1e-30), each value x * (1/s) (float32,
# round to nearest) is rounded to E4M3 (round to nearest even; |x/s| <= 448
# so nothing saturates), and the dequantised value is e4m3 * s.  Attention
# then runs on the dequantised rows exactly as before.
# ---------------------------------------------------------------------------
E4M3_MAX = 448.0


def fp8_quantize_rows(x):
    """Per-row E4M3 codes (uint8) and float32 scales of ``x`` [..., D]."""
    import torch
    x32 = _f64(x).astype(np.float32)
    amax = np.abs(x32).max(axis=-1)
    s = np.where(amax > np.float32(1e-30), amax / np.float32(E4M3_MAX), np.float32(1.0)).astype(np.float32)
    inv = (np.float32(1.0) / s).astype(np.float32)
    y = (x32 * inv[..., None]).astype(np.float32)
    codes = torch.from_numpy(np.ascontiguousarray(y)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    return codes, s


def e4m3_value(codes):
    """float64 value of E4M3 codes (no NaN codes are produced by the quantiser)."""
    c = np.asarray(codes, np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    normal = sign * (1.0 + m / 8.0) * np.exp2(e - 7.0)
    sub = sign * (m / 8.0) * np.exp2(-6.0)
    return np.where(e == 0, sub, normal)


def fp8_dequantize_rows(codes, s):
    return e4m3_value(codes) * np.asarray(s, np.float64)[..., None]


# ---------------------------------------------------------------------------
# RoPE front end and anchor position IDs (NEXT-1).
#
# [P2] "Phase 1: Context Encoding with Anchor Blocks", Step 2: the anchor
# tokens prepended to block i keep their original position IDs 0..b-1 while
# the block's own tokens keep theirs; [P2] ablation of section 4.1 (Table 4):
# anchor position IDs taken from the first block (proposed), from the block
# just before block i, or sampled at random from [0, start of block i).
# Readings (the pages name Llama 3.1 models but give no rotary details):
# rotary embedding in the RoFormer form on
# adjacent pairs (2k, 2k+1) with inverse frequencies base^(-2k/D), base
# 500000 (Llama 3) and no frequency rescaling; "previous" = the b_a positions
# right before block i; random positions are drawn by the caller; query-region
# row r sits at position L + r.  Pinned by tests/test_oracle_rope.py.
# ---------------------------------------------------------------------------
ROPE_BASE = 500000.0


def rope_inv_freq(D: int, base: float = ROPE_BASE) -> np.ndarray:
    """Inverse frequencies base^(-2k/D), k = 0..D/2-1 (float64)."""
    k = np.arange(D // 2, dtype=np.float64)
    return np.power(float(base), -2.0 * k / D)


def rope(x, pos, base: float = ROPE_BASE) -> np.ndarray:
    """Rotary embedding of x [..., n, D] at integer positions pos [n]:
    each pair (x_2k, x_2k+1) is rotated by the angle pos * base^(-2k/D)."""
    x = _f64(x)
    D = x.shape[-1]
    ang = np.asarray(pos, np.float64)[:, None] * rope_inv_freq(D, base)[None, :]
    c, s = np.cos(ang), np.sin(ang)
    x0, x1 = x[..., 0::2], x[..., 1::2]
    y = np.empty_like(x)
    y[..., 0::2] = x0 * c - x1 * s
    y[..., 1::2] = x0 * s + x1 * c
    return y


def anchor_positions(mode: str, n_blocks: int, b: int, b_a: int, given=None) -> np.ndarray:
    """Position IDs [n_blocks - 1, b_a] of the anchor keys prepended to blocks
    1..n-1: "first" -> 0..b_a-1 (the proposed method); "previous" -> the b_a
    positions right before block i, i*b - b_a .. i*b - 1; "given" -> the
    caller's array (e.g. random draws from [0, i*b))."""
    i = np.arange(1, n_blocks, dtype=np.int64)[:, None]
    j = np.arange(b_a, dtype=np.int64)[None, :]
    if mode == "first":
        return np.broadcast_to(j, (n_blocks - 1, b_a)).copy()
    if mode == "previous":
        return i * b - b_a + j
    if mode == "given":
        return np.asarray(given, np.int64).reshape(n_blocks - 1, b_a)
    raise ValueError(mode)


def round_bf16(x) -> np.ndarray:
    """Round float64 values to the nearest bfloat16 (ties to even), as float64."""
    import torch
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float64)).to(torch.bfloat16).double().numpy()


def ctx_encode_rope(Q, K, V, b: int, b_a: int, scale: float, anchor_pos, base: float = ROPE_BASE,
                    rows=None, rotated_bf16: bool = False):
    """Phase 1 on un-rotated Q, K [B, H, L, D] with rotary positions.

    Token t of block i is at position t (positions preserved, [P2] Phase 1
    Step 2).  Block 0 attends causally to itself; block i >= 1 attends to the
    whole anchor -- K rows 0..b_a-1 rotated at anchor_pos[i-1] -- and causally
    to its own block.  V is not rotated.  ``rotated_bf16`` rounds the rotated
    q and k to bf16 before the attention (the precision of a path whose
    attention operands are bf16).  Returns (O, LSE) for ``rows`` (default
    all), like ``ctx_encode``.
    """
    rnd = round_bf16 if rotated_bf16 else (lambda a: a)
    Bn, Hq, L, D = Q.shape
    Hkv = K.shape[1]
    G = Hq // Hkv
    rows = np.arange(L) if rows is None else np.asarray(rows, np.int64)
    O = np.zeros((Bn, Hq, len(rows), D))
    LSE = np.zeros((Bn, Hq, len(rows)))
    for i, (s, n) in enumerate(block_table(L, b)):
        sel = np.nonzero((rows >= s) & (rows < s + n))[0]
        if len(sel) == 0:
            continue
        t = rows[sel]
        own = np.arange(s, s + n)
        if i == 0:
            kpos = own
            mask = own[None, :] <= t[:, None]
        else:
            kpos = np.concatenate([np.asarray(anchor_pos[i - 1], np.int64), own])
            mask = np.concatenate([np.ones((len(t), b_a), bool), own[None, :] <= t[:, None]], axis=1)
        for bi in range(Bn):
            for g in range(Hkv):
                kraw = _f64(K[bi, g])
                kk = np.concatenate([rope(kraw[:b_a], kpos[:b_a], base), rope(kraw[s:s + n], own, base)]) \
                    if i > 0 else rope(kraw[s:s + n], own, base)
                kk = rnd(kk)
                vv = _f64(V[bi, g])
                vv = np.concatenate([vv[:b_a], vv[s:s + n]]) if i > 0 else vv[s:s + n]
                for h in range(g * G, (g + 1) * G):
                    q = rnd(rope(_f64(Q[bi, h])[t], t, base))
                    o, lse = masked_attention(q, kk, vv, mask, scale)
                    O[bi, h, sel] = o
                    LSE[bi, h, sel] = lse
    return O, LSE
