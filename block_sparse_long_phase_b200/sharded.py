"""Star Attention with the context blocks spread over several GPUs.

"Star Attention: Efficient LLM Inference over Long Sequences" (analysis page),
section 3.4.  Phase 1: the context blocks are distributed over the hosts and
every block after the first is encoded with the anchor block in front of it
(Steps 3-4); each host keeps only its own blocks' KV (Step 5).  Phase 2: the
query is broadcast to every host (Step 2), each host computes the local
attention A_h of the query over its own blocks and the log of its exponent
sum s_h (Step 3), the partials travel to the query host (Step 4), which
merges them with the log-sum-exp rule (Step 5); only the query host caches
the query and generated tokens (Step 7).

A host here is one process per GPU in a torch.distributed group.  Rank r
holds the contiguous blocks ``block_ranges(n, world)[r]``; the last rank is
the query host.  A rank's local context is its own rows, cut into blocks of
the same size: the rank holding block 0 encodes them as a context of its own
(star_ctx_encode), every other rank encodes each of its blocks behind the
anchor rows it receives (star_ctx_encode_after_anchor), so local block j is
global block first + j with exactly the single-GPU mask: the whole anchor,
then itself causally.  A rank without blocks keeps a one-row placeholder
context that is never encoded or attended.

Everything arithmetic runs in libstar's kernels (star_ctx_encode,
star_ctx_encode_after_anchor, star_partial_attend, star_lse_merge_bf16); this
module partitions, slices inputs and moves the partials (one ``all_gather`` per call: B*Hq*lq*(D+1)
floats per rank, a few KB per decode step, after one broadcast of the query
rows).  No remote memory is ever read by
a kernel or a TMA copy: the partials land in each rank's own buffers first.

The kernel calls go through an ``ops`` object (``LibstarOps`` by default) so
that the host logic can be checked on CPU ranks with the oracle standing in
for the kernels; the product path has no CPU implementation.
"""

from __future__ import annotations

from dataclasses import dataclass

import torch


def block_ranges(n_blocks: int, world: int):
    """Contiguous block ranges [first, end) per rank, as equal as possible."""
    if world < 1 or n_blocks < 0:
        raise ValueError("need world >= 1 and n_blocks >= 0")
    return [(r * n_blocks // world, (r + 1) * n_blocks // world) for r in range(world)]


@dataclass(frozen=True)
class LocalLayout:
    """Where rank r's blocks sit in its local context."""
    first_block: int     # first global block of the rank
    n_blocks: int        # how many (may be 0)
    rows0: int           # first global context row of the rank
    rows: int            # its context rows
    L_local: int         # local context length: its rows (a one-row placeholder when none)
    first_seg: int       # local segment of the first own block (1, past the placeholder, when none)
    after_anchor: bool   # its blocks follow an anchor it does not hold (the first block is not 0)


def local_layout(rank: int, world: int, L: int, b: int) -> LocalLayout:
    n = -(-L // b)
    i0, i1 = block_ranges(n, world)[rank]
    if i1 == i0:
        return LocalLayout(i0, 0, min(i0 * b, L), 0, 1, 1, False)
    rows0 = i0 * b
    rows = min(i1 * b, L) - rows0
    return LocalLayout(i0, i1 - i0, rows0, rows, rows, 0, i0 > 0)


class LibstarOps:
    """The kernels behind a shard: libstar's C ABI on the rank's GPU."""

    def create(self, B, Hq, Hkv, D, L, block, anchor, q_cap, scale, kv_fp8=False):
        from .api import StarCache
        return StarCache(B, Hq, Hkv, D, L, block, anchor, q_cap, scale, kv_fp8=kv_fp8)

    def ctx_encode(self, cache, Q, K, V):
        return cache.star_ctx_encode(Q, K, V)

    def ctx_encode_after_anchor(self, cache, Q, K, V, Ka, Va):
        return cache.star_ctx_encode_after_anchor(Q, K, V, Ka, Va)

    def partial_attend(self, cache, Q, first_seg, n_seg, K=None, V=None):
        return cache.star_partial_attend(Q, first_seg, n_seg, K, V)

    def lse_merge(self, A, s):
        from .api import star_lse_merge_bf16
        return star_lse_merge_bf16(A, s)


class ShardedStarCache:
    """One rank's share of a Star Attention layer whose context blocks are
    spread over ``world`` GPUs (see the module docstring).

    ``group`` is a torch.distributed process group (None: the default one);
    with ``world = 1`` no collective is issued.  ``query_rank`` defaults to the
    last rank.  Outputs of phase 2 are the merged rows on every rank.  With
    ``kv_fp8`` every rank's cache keeps the FP8 copy and the generation steps
    read it (as star_decode_step on such a cache); phase 1 and the query
    prefill read the bf16 rows.
    """

    def __init__(self, rank, world, B, Hq, Hkv, D, L, block, anchor, q_cap, scale=0.0,
                 query_rank=None, group=None, ops=None, device=None, kv_fp8=False):
        if not (0 <= anchor <= block):
            raise ValueError("need 0 <= anchor <= block")
        self.rank, self.world = rank, world
        self.B, self.Hq, self.Hkv, self.D, self.L = B, Hq, Hkv, D, L
        self.block, self.anchor, self.q_cap = block, anchor, q_cap
        self.scale = scale
        self.query_rank = world - 1 if query_rank is None else query_rank
        self.group = group
        self.ops = LibstarOps() if ops is None else ops
        self.device = device if device is not None else (
            torch.device("cuda", torch.cuda.current_device()) if torch.cuda.is_available() else torch.device("cpu"))
        self.layout = local_layout(rank, world, L, block)
        if kv_fp8:
            self.cache = self.ops.create(B, Hq, Hkv, D, self.layout.L_local, block, anchor, q_cap, scale,
                                         kv_fp8=True)
        else:
            self.cache = self.ops.create(B, Hq, Hkv, D, self.layout.L_local, block, anchor, q_cap, scale)

    @property
    def is_query_rank(self) -> bool:
        return self.rank == self.query_rank

    # -- phase 1 ---------------------------------------------------------------
    def encode(self, Q_own, K_own, V_own, K_anchor, V_anchor):
        """Phase 1 of this rank's blocks.  ``*_own``: the rank's context rows
        [B, H, rows, D] bf16; ``K_anchor``, ``V_anchor``: context rows 0..b_a-1
        [B, Hkv, b_a, D] (the anchor block, copied to every rank once).
        Returns (O, LSE) of the rank's own rows."""
        lay = self.layout
        if lay.n_blocks == 0:
            return (Q_own.new_empty((self.B, self.Hq, 0, self.D)),
                    Q_own.new_empty((self.B, self.Hq, 0), dtype=torch.float32))
        if not lay.after_anchor:
            return self.ops.ctx_encode(self.cache, Q_own, K_own, V_own)
        return self.ops.ctx_encode_after_anchor(self.cache, Q_own, K_own, V_own, K_anchor, V_anchor)

    # -- phase 2 ---------------------------------------------------------------
    def local_partial(self, Q, K=None, V=None):
        """(A_h, s_h) of rows Q over this rank's blocks, and, on the query
        rank, over the query region after appending K, V ([P2] Phase 2 Step 3)."""
        lay = self.layout
        if self.is_query_rank:
            return self.ops.partial_attend(self.cache, Q, lay.first_seg, lay.n_blocks, K, V)
        return self.ops.partial_attend(self.cache, Q, lay.first_seg, lay.n_blocks)

    def merge(self, A_all, s_all):
        """Log-sum-exp merge of every rank's partial ([P2] Phase 2 Step 5):
        A_all [R, B, Hq, lq, D], s_all [R, B, Hq, lq] -> (O bf16, LSE)."""
        R, B, Hq, lq, D = A_all.shape
        O, LSE = self.ops.lse_merge(A_all.reshape(R, B * Hq * lq, D).contiguous(),
                                    s_all.reshape(R, B * Hq * lq).contiguous())
        return O.view(B, Hq, lq, D), LSE.view(B, Hq, lq)

    def _gather(self, A, s):
        """Every rank's (A, s), stacked in rank order: one all_gather of the
        partials packed as [A | s] float32 rows (the collective is
        latency-bound at these sizes, so one call rather than two)."""
        if self.world == 1:
            return A[None], s[None]
        import torch.distributed as dist
        B, Hq, lq, D = A.shape
        packed = torch.cat([A.reshape(B * Hq * lq, D), s.reshape(B * Hq * lq, 1)], dim=1).contiguous()
        out = torch.empty((self.world * packed.shape[0], D + 1), dtype=packed.dtype, device=packed.device)
        dist.all_gather_into_tensor(out, packed, group=self.group)
        out = out.view(self.world, B * Hq * lq, D + 1)
        return (out[:, :, :D].reshape(self.world, B, Hq, lq, D),
                out[:, :, D].reshape(self.world, B, Hq, lq))

    def _broadcast(self, *xs):
        """The query rank's tensors to every rank, in one broadcast of their
        concatenated bytes."""
        if self.world == 1:
            return xs
        import torch.distributed as dist
        flat = torch.cat([x.reshape(-1) for x in xs]).contiguous()
        dist.broadcast(flat, src=self.query_rank, group=self.group)
        out, o = [], 0
        for x in xs:
            out.append(flat[o:o + x.numel()].view(x.shape))
            o += x.numel()
        return tuple(out)

    def query_prefill(self, Q, K, V):
        """Phase 2 for the query rows: Q [B, Hq, lq, D], K, V [B, Hkv, lq, D]
        bf16, taken from the query rank (broadcast to the others).  Returns
        (O [B, Hq, lq, D] bf16, LSE [B, Hq, lq]) on every rank."""
        Q, K, V = self._broadcast(Q, K, V)
        A, s = self.local_partial(Q, K, V)
        return self.merge(*self._gather(A, s))

    def decode_step(self, q, k, v):
        """One generation step (lq = 1): the query rank appends (k, v)."""
        return self.query_prefill(q, k, v)

    def close(self):
        if hasattr(self.cache, "close"):
            self.cache.close()
