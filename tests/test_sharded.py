"""Host logic of the multi-GPU block-sharded layer, on CPU ranks (gloo).

"Star Attention" analysis page, section 3.4: Phase 1 Steps 3-5 (blocks spread
over hosts, each encoded behind the anchor, only its own KV kept) and Phase 2
Steps 2-5 (query broadcast, local A_h / s_h per host, gathered and merged with
the log-sum-exp rule on the query host).  The oracle stands in for libstar's
kernels (tests/sharded_oracle_ops.py), so every rank's phase-1 rows and the
merged phase-2 rows must equal the single-device oracle to float64 rounding;
this pins the partition, the local [anchor | zeros | own blocks] layout, the
segment ranges each rank attends to, the query rank's region, the gather and
the merge.  Ranks with no block at all are covered.
"""

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from block_sparse_long_phase_b200 import workloads as wl
from block_sparse_long_phase_b200.sharded import ShardedStarCache, block_ranges, local_layout
from oracle import star_oracle as so


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def test_block_ranges_and_layouts():
    for n in range(0, 12):
        for world in range(1, 6):
            r = block_ranges(n, world)
            assert r[0][0] == 0 and r[-1][1] == n
            assert all(a[1] == b_[0] for a, b_ in zip(r, r[1:]))
            assert max(e - s for s, e in r) - min(e - s for s, e in r) <= 1
    lay = local_layout(0, 3, 1000, 256)            # 4 blocks over 3 ranks: [0,1) [1,2) [2,4)
    assert (lay.after_anchor, lay.L_local, lay.first_seg, lay.n_blocks) == (False, 256, 0, 1)
    lay = local_layout(2, 3, 1000, 256)
    assert (lay.after_anchor, lay.rows0, lay.rows, lay.L_local, lay.first_seg) == (True, 512, 488, 488, 0)
    lay = local_layout(2, 3, 300, 256)             # 2 blocks over 3 ranks: rank 0 holds none
    empty = local_layout(0, 3, 300, 256)
    assert (empty.n_blocks, empty.rows, empty.L_local, empty.first_seg) == (0, 0, 1, 1)
    assert (lay.n_blocks, lay.rows0, lay.rows, lay.after_anchor) == (1, 256, 44, True)
    # every row of the context is held by exactly one rank
    for L, b, world in ((1000, 256, 3), (300, 256, 3), (4096, 512, 8), (777, 100, 5)):
        lays = [local_layout(r, world, L, b) for r in range(world)]
        assert sum(x.rows for x in lays) == L
        assert all(x.rows0 + x.rows == y.rows0 for x, y in zip(lays, lays[1:]) if x.n_blocks and y.n_blocks)


def _worker(rank, world, port, shape, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from sharded_oracle_ops import OracleOps
        w = wl.get("tiny").with_(**shape)
        x = wl.make_inputs(w, "cpu")
        sc = ShardedStarCache(rank, world, w.B, w.Hq, w.Hkv, w.D, w.L, w.b, w.b_a, w.lq + w.T, w.scale,
                              ops=OracleOps(), device=torch.device("cpu"))
        lay = sc.layout
        r0, r1 = lay.rows0, lay.rows0 + lay.rows
        O, LSE = sc.encode(x["Qc"][:, :, r0:r1], x["Kc"][:, :, r0:r1], x["Vc"][:, :, r0:r1],
                           x["Kc"][:, :, :w.b_a], x["Vc"][:, :, :w.b_a])
        Oref, Lref = so.ctx_encode(x["Qc"], x["Kc"], x["Vc"], w.b, w.b_a, w.scale, rows=np.arange(r0, r1))
        e1 = float(np.abs(O.numpy() - Oref).max()) if lay.rows else 0.0
        e2 = float(np.abs(LSE.numpy() - Lref).max()) if lay.rows else 0.0
        # phase 2: the query rank's inputs, broadcast to the others
        blank = lambda t: t if rank == sc.query_rank else torch.zeros_like(t)
        Oq, Lq = sc.query_prefill(blank(x["Qq"]), blank(x["Kq"]), blank(x["Vq"]))
        segs = so.cache_segments(x["Kc"], x["Vc"], w.b)
        region = np.zeros((w.B, w.Hkv, w.lq + w.T, w.D))
        ref, lref, qk, qv = so.query_prefill(x["Qq"], x["Kq"], x["Vq"], segs, region, region, 0, w.scale)
        e3 = float(np.abs(Oq.numpy() - ref).max())
        e4 = float(np.abs(Lq.numpy() - lref).max())
        for t in range(w.T):
            o, l = sc.decode_step(blank(x["qd"][t]), blank(x["kd"][t]), blank(x["vd"][t]))
            ref, lref, qk, qv = so.decode_step(x["qd"][t], x["kd"][t], x["vd"][t], segs, qk, qv, w.lq + t, w.scale)
            e3 = max(e3, float(np.abs(o.numpy() - ref).max()))
            e4 = max(e4, float(np.abs(l.numpy() - lref).max()))
        q.put((rank, e1, e2, e3, e4, lay.n_blocks, sc.cache.q_len))
    finally:
        dist.destroy_process_group()


SHAPES = [
    (2, dict(L=1024, b=256, b_a=256, lq=5, T=2)),
    (3, dict(L=1000, b=256, b_a=100, lq=4, T=2)),            # ragged last block, anchor shorter
    (4, dict(L=700, b=128, b_a=64, B=2, Hq=8, Hkv=2, lq=3, T=2)),
    (3, dict(L=300, b=256, b_a=256, lq=3, T=1)),             # 2 blocks on 3 ranks: rank 0 has none
    (2, dict(L=90, b=16, b_a=0, lq=2, T=2)),                 # no anchor
]


@pytest.mark.parametrize("world,shape", SHAPES)
def test_sharded_layer_matches_the_single_device_oracle(world, shape):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, shape, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=180) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    res.sort()
    w = wl.get("tiny").with_(**shape)
    assert sum(r[5] for r in res) == -(-w.L // w.b)           # every block on exactly one rank
    for rank, e1, e2, e3, e4, nb, qlen in res:
        assert e1 < 1e-10 and e2 < 1e-10, (rank, e1, e2)       # phase-1 rows of the rank
        assert e3 < 1e-10 and e4 < 1e-10, (rank, e3, e4)       # merged phase-2 rows
        assert qlen == (w.lq + w.T if rank == world - 1 else 0)  # only the query rank caches the query
