"""The oracle standing in for libstar's kernels behind a ShardedStarCache, so
the sharded layer's host logic (partition, local layouts, segment ranges,
gather, merge) runs on CPU ranks.  Test infrastructure only."""

import numpy as np
import torch

from oracle import star_oracle as so


class OracleCache:
    def __init__(self, B, Hq, Hkv, D, L, block, anchor, q_cap, scale):
        self.B, self.Hq, self.Hkv, self.D, self.L = B, Hq, Hkv, D, L
        self.b, self.b_a, self.q_cap = block, anchor, q_cap
        self.scale = scale if scale > 0 else 1.0 / np.sqrt(D)
        self.segs = None
        self.qk = np.zeros((B, Hkv, q_cap, D))
        self.qv = np.zeros((B, Hkv, q_cap, D))
        self.q_len = 0


class OracleOps:
    def create(self, B, Hq, Hkv, D, L, block, anchor, q_cap, scale):
        return OracleCache(B, Hq, Hkv, D, L, block, anchor, q_cap, scale)

    def ctx_encode(self, c, Q, K, V):
        O, LSE = so.ctx_encode(Q, K, V, c.b, c.b_a, c.scale)
        c.segs = so.cache_segments(so._f64(K), so._f64(V), c.b)
        c.q_len = 0
        return torch.from_numpy(O), torch.from_numpy(LSE)

    def ctx_encode_after_anchor(self, c, Q, K, V, Ka, Va):
        """Every block behind the anchor rows Ka, Va: the anchor with no mask,
        then the block's own rows causally (the single-GPU mask of a block
        i >= 1, written out block by block)."""
        q, k, v, ka, va = (so._f64(t) for t in (Q, K, V, Ka, Va))
        B, Hq, L, D = q.shape
        G = Hq // c.Hkv
        O = np.zeros((B, Hq, L, D))
        LSE = np.zeros((B, Hq, L))
        for s0, n in so.block_table(L, c.b):
            mask = np.concatenate([np.ones((n, c.b_a), dtype=bool), np.tril(np.ones((n, n), dtype=bool))], axis=1)
            for bi in range(B):
                for h in range(Hq):
                    g = h // G
                    keys = np.concatenate([ka[bi, g], k[bi, g, s0:s0 + n]], axis=0)
                    vals = np.concatenate([va[bi, g], v[bi, g, s0:s0 + n]], axis=0)
                    O[bi, h, s0:s0 + n], LSE[bi, h, s0:s0 + n] = so.masked_attention(
                        q[bi, h, s0:s0 + n], keys, vals, mask, c.scale)
        c.segs = so.cache_segments(k, v, c.b)
        c.q_len = 0
        return torch.from_numpy(O), torch.from_numpy(LSE)

    def partial_attend(self, c, Q, first_seg, n_seg, K=None, V=None):
        q = so._f64(Q)
        B, Hq, lq, D = q.shape
        G = Hq // c.Hkv
        if K is not None:
            c.qk[:, :, c.q_len:c.q_len + lq] = so._f64(K)
            c.qv[:, :, c.q_len:c.q_len + lq] = so._f64(V)
        A = np.zeros((B, Hq, lq, D))
        s = np.full((B, Hq, lq), -np.inf)
        for bi in range(B):
            for g in range(c.Hkv):
                segs = (c.segs or [])[first_seg:first_seg + n_seg]   # a rank without blocks encodes none
                ks = [seg[2][bi, g] for seg in segs]
                vs = [seg[3][bi, g] for seg in segs]
                n_ctx = sum(len(k) for k in ks)
                nq = c.q_len + lq if K is not None else 0
                ks.append(c.qk[bi, g, :nq])
                vs.append(c.qv[bi, g, :nq])
                k = np.concatenate(ks, axis=0)
                v = np.concatenate(vs, axis=0)
                mask = np.ones((lq, len(k)), dtype=bool)
                mask[:, n_ctx:] = np.arange(nq)[None, :] <= (c.q_len + np.arange(lq))[:, None]
                for h in range(g * G, (g + 1) * G):
                    A[bi, h], s[bi, h] = so.masked_attention(q[bi, h], k, v, mask, c.scale)
        if K is not None:
            c.q_len += lq
        return torch.from_numpy(A), torch.from_numpy(s)

    def lse_merge(self, A, s):
        O, L = so.lse_merge(A.numpy(), s.numpy())
        return torch.from_numpy(O), torch.from_numpy(L)
