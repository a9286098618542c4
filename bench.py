"""Benchmark of the Star Attention two-phase hot path on B200.

One step = the whole path over one synthetic batch of the Llama-3.1-8B
attention shape at 1M-token context (H_q=32, H_kv=8, D=128, b = b_a = 65536,
16 blocks; 64 query tokens, 64 decode steps): phase-1 context encoding,
phase-2 query prefill, and every decode step.  This is the largest of the
metric's configurations and the pages' headline context length; the 32K,
128K and 70B configurations are reported in sub-sections.

Reported (one JSON line from rank 0):
  value      -- phase-1 context-encode tokens/s (B*L / encode time), all ranks
  decode     -- phase-2 decode tokens/s over all 64 steps and their HBM roofline
  roofline   -- phase-1 kernel against the measured bf16 dense peak (the
                sustained one: a 1.5 s launch runs under the power cap)
  e2e        -- the same metric through the public API star_ctx_encode_host:
                page-locked host Q, K, V in and O, LSE out, copies inside the
                timed region
  cpu_baseline -- the fp64 oracle on a fixed row sample, extrapolated

L2 is flushed before every timed kernel region, outside the CUDA-event
brackets: a 512 MB write, then a 512 MB read.  The read evicts the dirty
lines the write leaves behind; otherwise their write-back (up to the 126 MB
of L2) would run inside the next timed kernel and be charged to it.
Multi-GPU runs are independent replicas (the single-GPU path has no exchange
step): value = all ranks' tokens / the slowest rank's time.

``--impl reference`` times the fp64 CPU oracle (the only reference this path
has) on the same fixed sample of the same workload, with the same code as the
GPU arm's cpu_baseline, and prints the same line with "impl": "reference".
"""

from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

WORKLOAD = "8b-1m"
METRIC = "ctx-encode tok/s & decode tok/s per attn layer; % of bf16 TC / HBM roofline"


# DRAM traffic per launch (dram__bytes_read.sum + dram__bytes_write.sum) from the
# ncu captures summarised under profiles/, valid only for the kernel source they
# were taken on (first 16 hex digits of its sha256); null otherwise.
TRAFFIC = {
    # the 1M launch scaled from captures at L = b and L = 3b (block 0, then two
    # anchored blocks: each anchored 64K-row block is an L2 group of its own)
    "phase1 8b-1m": ("block_sparse_long_phase_b200/csrc/attn_tc.cu", "3da1c828dfe05ede", 55308552448),
    "phase1 8b-32k": ("block_sparse_long_phase_b200/csrc/attn_tc.cu", "3da1c828dfe05ede", 1448725248),
    "decode 8b-128k": ("block_sparse_long_phase_b200/csrc/decode_splitkv.cu", "0bfa638da1bfd739", 543287808),
    "decode fp8 8b-128k": ("block_sparse_long_phase_b200/csrc/decode_splitkv.cu", "0bfa638da1bfd739", 286823680),
}


def traffic(key):
    import hashlib
    if key not in TRAFFIC:
        return None
    path, sha, nbytes = TRAFFIC[key]
    with open(os.path.join(ROOT, path), "rb") as f:
        return nbytes if hashlib.sha256(f.read()).hexdigest()[:16] == sha else None


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


def phase1_flops(w):
    """Algorithmic flops of phase 1: 4*D per visible (query, key) pair of block rows."""
    pairs = 0
    for i in range(w.n_blocks):
        n = min(w.b, w.L - i * w.b)
        pairs += n * (n + 1) // 2 + (w.b_a * n if i > 0 else 0)
    return 4 * w.D * w.Hq * w.B * pairs, pairs


def prefill_roofline(w, ms, pk):
    """Query prefill against min(bf16 peak, intensity x HBM): flops 4*D per
    (query row, visible key) pair -- row r sees the L context keys and query
    rows 0..r -- and bytes of the cache read once plus the query rows in and
    the outputs out."""
    pairs = w.lq * w.L + w.lq * (w.lq + 1) // 2
    flops = 4 * w.D * w.Hq * w.B * pairs
    nbytes = (w.B * w.Hkv * (w.L + w.lq) * w.D * 2 * 2            # K, V of the cache
              + w.B * w.Hq * w.lq * w.D * 2 * 2 + w.B * w.Hq * w.lq * 4)   # Q in, O out, LSE out
    peak_tf = min(pk["bf16_tflops"], flops / nbytes * pk["hbm_gbs"] / 1e3)
    tf = flops / (ms / 1e3) / 1e12
    return {"bound": "tensor" if peak_tf == pk["bf16_tflops"] else "hbm", "achieved": tf, "peak": peak_tf,
            "unit": "TFLOP/s", "frac": tf / peak_tf, "flops": flops, "bytes": nbytes,
            "intensity_flops_per_byte": flops / nbytes}


def decode_bytes(w, t):
    """Algorithmic bytes of decode step t: the K and V of every cached row."""
    return w.B * w.Hkv * (w.L + w.lq + t + 1) * w.D * 2 * 2


def decode_bytes_fp8(w, t):
    """Same, FP8 cache: one byte per element plus a float32 scale per row, for K
    and for V, of every row cached before the step; the step's own token is
    read in bf16."""
    return w.B * w.Hkv * ((w.L + w.lq + t) * (w.D + 4) * 2 + w.D * 2 * 2)


class Clocks:
    """nvidia-smi sampling of SM clocks and throttle reasons during timing."""

    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.path = os.path.join("/tmp", f"star_clocks_{os.getpid()}.csv")

    def start(self):
        """Start sampling (call before warm-up: nvidia-smi takes a moment to start)."""
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"], stdout=self.f,
                stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        self.t0 = self.t1 = None

    def mark(self, begin: bool):
        """Wall-clock bounds of the timed region; samples outside it are ignored."""
        import datetime
        now = datetime.datetime.now()
        if begin:
            self.t0 = now
        else:
            self.t1 = now

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        self.proc.wait()
        self.f.close()
        import datetime
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 10:
                continue
            try:
                ts = datetime.datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f")
                rows.append((ts, float(parts[2]), float(parts[3]), parts[6:10]))
            except ValueError:
                continue
        inside = [r for r in rows if self.t0 and self.t1 and
                  self.t0 - datetime.timedelta(milliseconds=150) <= r[0] <= self.t1]
        if not inside and rows and self.t1:
            inside = [min(rows, key=lambda r: abs((r[0] - self.t1).total_seconds()))]
        for ts, clk, cmax, rs in inside:
            sm.append(clk)
            mx = cmax
            for n, v in zip(names, rs):
                if v.lower() == "active":
                    reasons.add(n)
        os.unlink(self.path)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


class L2Flush:
    """Empties L2 of inputs and dirty lines: a 512 MB write, then a 512 MB read."""

    def __init__(self, dev):
        import torch
        n = 512 * 1024 * 1024 // 4
        self.w = torch.empty(n, dtype=torch.float32, device=dev)
        self.r = torch.ones(n, dtype=torch.float32, device=dev)
        self.acc = torch.zeros((), dtype=torch.float32, device=dev)

    def flush(self, value):
        import torch
        self.w.fill_(value)
        torch.sum(self.r, dim=0, out=self.acc)


ORACLE_SEED = 977
ORACLE_ROWS_PER_BLOCK = 5


def oracle_sample_inputs(w):
    """Host inputs of the CPU baseline: kv group 0 of batch entry 0 of workload
    ``w`` -- K and V over the whole context as float64 arrays, and the G query
    heads of that group as a bf16 tensor holding values only at a fixed row
    sample (every block's first and last rows, its row 127 and a multiple of 128
    near its middle -- the tile edges -- and one seeded row).  Drawn once, outside
    every timed region, with a CPU generator, so both bench arms time the same
    bytes with the same code (same shapes and N(0, 1) bf16 distribution as the
    workload)."""
    import numpy as np
    import torch
    from oracle import star_oracle as so
    g = torch.Generator().manual_seed(ORACLE_SEED)
    K = torch.randn(w.L, w.D, generator=g).to(torch.bfloat16).double().numpy()[None, None]
    V = torch.randn(w.L, w.D, generator=g).to(torch.bfloat16).double().numpy()[None, None]
    rng = np.random.default_rng(ORACLE_SEED)
    blocks = []
    for s, n in so.block_table(w.L, w.b):
        r = {0, n - 1, min(127, n - 1), (n // 2) // 128 * 128, int(rng.integers(0, n))}
        blocks.append(np.array(sorted(s + x for x in r), dtype=np.int64))
    Q = torch.zeros((1, w.G, w.L, w.D), dtype=torch.bfloat16)
    allrows = np.concatenate(blocks)
    Q[:, :, torch.from_numpy(allrows)] = torch.randn(1, w.G, len(allrows), w.D, generator=g).to(torch.bfloat16)
    qd = torch.randn(1, w.G, 1, w.D, generator=g).to(torch.bfloat16)
    kq = torch.randn(1, 1, w.lq + 1, w.D, generator=g).to(torch.bfloat16).double().numpy()
    vq = torch.randn(1, 1, w.lq + 1, w.D, generator=g).to(torch.bfloat16).double().numpy()
    return {"K": K, "V": V, "Q": Q, "blocks": blocks, "qd": qd, "kq": kq, "vq": vq}


def sample_pairs(w, blocks):
    """Visible (query, key) pairs of the sampled rows over the G heads of one
    kv group: row t of block i sees t - i*b + 1 keys of its block and, for
    i >= 1, the b_a anchor keys."""
    pairs = 0
    for i, rows in enumerate(blocks):
        pairs += int(((rows - i * w.b + 1) + (w.b_a if i > 0 else 0)).sum()) * w.G
    return pairs


def oracle_baseline(w, data, warmup, reps):
    """The fp64 oracle as it stands, timed on the host cores.

    One pass = phase 1 of the sampled rows (``ctx_encode`` called block by
    block on that block's rows, all G heads of kv group 0), extrapolated to
    the whole layer by visible (query, key) pairs.  ``warmup`` untimed passes,
    then ``reps`` timed ones; afterwards one decode step of kv group 0 against
    the full context (``query_attend``), extrapolated to all B x H_kv groups.
    Returns a dict with the per-pass ctx tok/s, the decode tok/s, the sample
    description and the thread count."""
    import numpy as np
    from oracle import star_oracle as so
    _, total_pairs = phase1_flops(w)
    total_pairs *= w.Hq * w.B
    pairs = sample_pairs(w, data["blocks"])

    def one_pass():
        t = time.perf_counter()
        for rows in data["blocks"]:
            so.ctx_encode(data["Q"], data["K"], data["V"], w.b, w.b_a, w.scale, rows=rows)
        return time.perf_counter() - t

    for _ in range(warmup):
        one_pass()
    ctx = [w.B * w.L / (one_pass() * total_pairs / pairs) for _ in range(reps)]
    segs = so.cache_segments(data["K"], data["V"], w.b)
    t = time.perf_counter()
    so.query_attend(data["qd"], segs, data["kq"], data["vq"], np.array([w.lq + 1]), w.scale)
    t_dec = (time.perf_counter() - t) * w.B * w.Hkv
    nrows = sum(len(r) for r in data["blocks"])
    sample = (f"phase 1: {nrows} fixed rows (first, last, row 127 and a mid multiple of 128 of each of the "
              f"{len(data['blocks'])} blocks, plus one seeded row each) x {w.G} heads of kv group 0, "
              f"ctx_encode block by block, extrapolated by visible (q,k) pairs to {w.B}x{w.Hq} heads x "
              f"{w.L} rows; host float64 inputs drawn once (seed {ORACLE_SEED}); decode: one step of kv "
              f"group 0 against the {w.L}-token cache, x{w.B * w.Hkv} kv groups")
    return {"ctx": ctx, "decode": 1.0 / t_dec, "sample": sample, "threads": _blas_threads()}


def baseline_summary(r):
    v = statistics.median(r["ctx"])
    spread = (max(r["ctx"]) - min(r["ctx"])) / v if v > 0 else None
    return v, spread


def _blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return max(n)
    except Exception:
        pass
    return os.cpu_count()


def max_over_ranks(values, device, world):
    """Element-wise maximum over ranks of per-rank timings: the slowest rank
    decides a replica run's time (NCCL on GPUs; any backend works)."""
    import torch
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    if world > 1:
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return t.tolist()


def measure_long_decode(dev, flush, warmup, steps, world, kv_fp8=False, name="8b-128k-needle"):
    """Decode steps of a long-context workload (8B-128K unless named), L2 flushed
    before each; with ``kv_fp8`` the context is streamed from the cache's FP8 copy."""
    import torch
    from block_sparse_long_phase_b200 import StarCache, workloads as wl
    w = wl.get(name)
    x = wl.make_inputs(w, dev)
    cache = StarCache(w.B, w.Hq, w.Hkv, w.D, w.L, w.b, w.b_a, w.lq + w.T, w.scale, kv_fp8=kv_fp8)
    cache.star_ctx_encode(x["Qc"], x["Kc"], x["Vc"])
    cache.star_query_prefill(x["Qq"], x["Kq"], x["Vq"])
    del x["Qc"]
    stream = torch.cuda.current_stream(dev)
    o = torch.empty((w.B, w.Hq, 1, w.D), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((w.B, w.Hq), dtype=torch.float32, device=dev)
    n = min(w.T, warmup + steps)
    ms = []
    for t in range(n):
        flush.flush(5.0)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        cache.star_decode_step(x["qd"][t], x["kd"][t], x["vd"][t], o, lse)
        b.record(stream)
        ms.append((a, b))
    torch.cuda.synchronize(dev)
    times = [a.elapsed_time(b) for a, b in ms[warmup:]]
    (t_ms,) = max_over_ranks([sum(times) / len(times)], dev, world)
    cache.close()
    del x
    torch.cuda.empty_cache()
    return w, t_ms * 1e3


def measure_sharded(dev, flush, w, ranks=8, steps=8):
    """The block-sharded layer's per-rank work on one GPU, its ranks run one
    after another: each rank's phase 1 on its own blocks behind the anchor rows
    (input slicing included), its phase-2 partial of the query rows and of
    ``steps`` decode tokens (star_partial_attend), each timed alone after an L2
    flush, and the merge of the gathered partials; then the decode partials
    again with FP8 rank caches.  The all_gather between ranks is not run (one
    GPU); its bytes are reported."""
    import torch
    from block_sparse_long_phase_b200 import workloads as wl
    from block_sparse_long_phase_b200.api import star_lse_merge_bf16
    from block_sparse_long_phase_b200.sharded import ShardedStarCache
    stream = torch.cuda.current_stream(dev)
    ev = lambda: torch.cuda.Event(enable_timing=True)
    n = -(-w.L // w.b)
    R = max(1, min(ranks, n))
    T = min(w.T, steps + 1)
    x = wl.make_inputs(w, dev)
    Ka, Va = x["Kc"][:, :, :w.b_a].contiguous(), x["Vc"][:, :, :w.b_a].contiguous()

    def ranks_pass(kv_fp8):
        enc, pre, dec, dec_bytes, parts = [], [], [], [], []
        for r in range(R):
            sc = ShardedStarCache(r, R, w.B, w.Hq, w.Hkv, w.D, w.L, w.b, w.b_a, w.lq + w.T, w.scale,
                                  device=dev, kv_fp8=kv_fp8)
            lay = sc.layout
            r0, r1 = lay.rows0, lay.rows0 + lay.rows
            own = [x[k][:, :, r0:r1].contiguous() for k in ("Qc", "Kc", "Vc")]
            flush.flush(11.0)
            a, b = ev(), ev()
            a.record(stream)
            sc.encode(*own, Ka, Va)
            b.record(stream)
            del own
            qkv = (x["Qq"], x["Kq"], x["Vq"]) if sc.is_query_rank else (x["Qq"],)
            flush.flush(12.0)
            c, d = ev(), ev()
            c.record(stream)
            sc.local_partial(*qkv)
            d.record(stream)
            steps_ev = []
            for t in range(T):
                qkv = (x["qd"][t], x["kd"][t], x["vd"][t]) if sc.is_query_rank else (x["qd"][t],)
                flush.flush(13.0)
                e0, e1 = ev(), ev()
                e0.record(stream)
                A, s_ = sc.local_partial(*qkv)
                e1.record(stream)
                steps_ev.append((e0, e1))
            torch.cuda.synchronize(dev)
            assert sc.cache.device_error() == 0, "a kernel gave up a bounded pipeline wait"
            enc.append(a.elapsed_time(b))
            pre.append(c.elapsed_time(d))
            dec.append(sum(e0.elapsed_time(e1) for e0, e1 in steps_ev[1:]) / max(1, len(steps_ev) - 1) * 1e3)
            rows = lay.rows + ((w.lq + T) if sc.is_query_rank else 0)
            row_bytes = (w.D + 4) * 2 if kv_fp8 else w.D * 2 * 2   # K and V of one cached row
            dec_bytes.append(w.B * w.Hkv * rows * row_bytes)
            parts.append((A, s_))
            sc.close()
        return enc, pre, dec, dec_bytes, parts

    enc, pre, dec, dec_bytes, parts = ranks_pass(False)
    A = torch.stack([p_[0] for p_ in parts]).reshape(R, w.B * w.Hq, w.D).contiguous()
    S = torch.stack([p_[1] for p_ in parts]).reshape(R, w.B * w.Hq).contiguous()
    del parts
    m = []
    for _ in range(5):
        flush.flush(14.0)
        a, b = ev(), ev()
        a.record(stream)
        star_lse_merge_bf16(A, S)
        b.record(stream)
        m.append((a, b))
    torch.cuda.synchronize(dev)
    merge_us = sum(a.elapsed_time(b) for a, b in m[1:]) / (len(m) - 1) * 1e3
    del A, S
    _, _, dec8, dec8_bytes, parts8 = ranks_pass(True)
    del x, Ka, Va, parts8
    torch.cuda.empty_cache()
    pk = peaks()
    gbs = [by / (us * 1e-6) / 1e9 for by, us in zip(dec_bytes, dec)]
    gbs8 = [by / (us * 1e-6) / 1e9 for by, us in zip(dec8_bytes, dec8)]
    return {
        "workload": w.name, "ranks": R, "how": "ranks run one after another on one GPU; the all_gather "
        "of the partials between them is not run",
        "phase1_ms_per_rank": enc, "phase1_ms_max": max(enc),
        "ctx_tok_s_if_ranks_run_at_once": w.B * w.L / (max(enc) / 1e3),
        "prefill_partial_ms_per_rank": pre,
        "decode_partial_us_per_rank": dec, "decode_partial_us_max": max(dec),
        "decode_partial_frac_per_rank": [g / pk["hbm_gbs"] for g in gbs],
        "decode_partial_fp8_us_per_rank": dec8, "decode_partial_fp8_us_max": max(dec8),
        "decode_partial_fp8_frac_per_rank": [g / pk["hbm_gbs"] for g in gbs8],
        "merge_us": merge_us,
        "gather_bytes_per_rank_per_step": w.B * w.Hq * (w.D + 1) * 4}


CONFIGS = ["tiny", "8b-32k", "8b-128k-needle", "70b-128k", "70b-128k-b4"]
DATASHEET_HBM_GBS = 7700.0   # B200 HBM3e, HGX figure: context for the decode fractions


def measure_configs(dev, flush, warmup, steps, world, dec_steps=8):
    """Every other configuration of the metric (8B-1M is the main line): phase 1,
    the query prefill and the first ``dec_steps`` decode steps, each timed on its
    own with L2 flushed before it; phase-1 launches are ``steps`` per config after
    ``warmup`` (the 1M-token launch takes seconds)."""
    import torch
    from block_sparse_long_phase_b200 import StarCache, workloads as wl
    pk = peaks()
    stream = torch.cuda.current_stream(dev)
    ev = lambda: torch.cuda.Event(enable_timing=True)
    out = {}
    for name in CONFIGS:
        w = wl.get(name)
        x = wl.make_inputs(w, dev)
        cache = StarCache(w.B, w.Hq, w.Hkv, w.D, w.L, w.b, w.b_a, w.lq + w.T, w.scale)
        O = torch.empty_like(x["Qc"])
        LSE = torch.empty((w.B, w.Hq, w.L), dtype=torch.float32, device=dev)
        Oq = torch.empty_like(x["Qq"])
        LSEq = torch.empty((w.B, w.Hq, w.lq), dtype=torch.float32, device=dev)
        od = torch.empty((w.B, w.Hq, 1, w.D), dtype=torch.bfloat16, device=dev)
        lsed = torch.empty((w.B, w.Hq), dtype=torch.float32, device=dev)
        T = min(w.T, dec_steps)
        enc, pre, dec = [], [], []
        for it in range(warmup + steps):
            flush.flush(8.0)
            a, b = ev(), ev()
            a.record(stream)
            cache.star_ctx_encode(x["Qc"], x["Kc"], x["Vc"], O, LSE)
            b.record(stream)
            flush.flush(9.0)
            c, d = ev(), ev()
            c.record(stream)
            cache.star_query_prefill(x["Qq"], x["Kq"], x["Vq"], Oq, LSEq)
            d.record(stream)
            steps_ev = []
            for t in range(T):
                flush.flush(10.0)
                e0, e1 = ev(), ev()
                e0.record(stream)
                cache.star_decode_step(x["qd"][t], x["kd"][t], x["vd"][t], od, lsed)
                e1.record(stream)
                steps_ev.append((e0, e1))
            if it >= warmup:
                enc.append((a, b))
                pre.append((c, d))
                dec.extend(steps_ev)
        torch.cuda.synchronize(dev)
        t_enc = sum(a.elapsed_time(b) for a, b in enc) / len(enc)
        t_pre = sum(a.elapsed_time(b) for a, b in pre) / len(pre)
        t_dec = sum(a.elapsed_time(b) for a, b in dec) / len(dec)
        t_enc, t_pre, t_dec = max_over_ranks([t_enc, t_pre, t_dec], dev, world)
        flops, _ = phase1_flops(w)
        dbytes = sum(decode_bytes(w, t) for t in range(T)) / T
        tf = flops / (t_enc / 1e3) / 1e12
        gbs = dbytes / (t_dec / 1e3) / 1e9
        out[name] = {
            "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "D": w.D, "L": w.L, "block": w.b, "anchor": w.b_a, "lq": w.lq,
            "phase1_ms": t_enc, "ctx_tok_s": world * w.B * w.L / (t_enc / 1e3), "tflops": tf,
            "frac": tf / pk["bf16_tflops"],
            "frac_sustained": tf / pk["bf16_tflops_sustained"] if pk["bf16_tflops_sustained"] else None,
            "prefill_ms": t_pre, "prefill_frac": prefill_roofline(w, t_pre, pk)["frac"],
            "decode_steps_timed": T * steps, "decode_us": t_dec * 1e3,
            "decode_tok_s": world * w.B / (t_dec / 1e3), "decode_gbs": gbs, "decode_frac": gbs / pk["hbm_gbs"],
            "decode_frac_datasheet": gbs / DATASHEET_HBM_GBS}
        cache.close()
        del x, O, LSE, Oq, LSEq
        torch.cuda.empty_cache()
    return out


PHASE1_VARIANTS = {
    # anchor shorter than the block (the pages' anchor-size sweep), ragged last block, batch 4
    "8b-32k-anchor2k": dict(b_a=2048),
    "8b-30000-ragged": dict(L=30000, b=8000, b_a=8000),
    "8b-32k-batch4": dict(B=4),
}


def measure_phase1_variants(dev, flush, warmup, steps, world):
    """Phase-1 TFLOP/s on the variant shapes (same kernel, same timing rules)."""
    import torch
    from block_sparse_long_phase_b200 import StarCache, workloads as wl
    out = {}
    stream = torch.cuda.current_stream(dev)
    for name, over in PHASE1_VARIANTS.items():
        w = wl.get("8b-32k").with_(name=name, **over)
        g = torch.Generator(device=dev).manual_seed(w.seed + 7)
        Q = torch.randn((w.B, w.Hq, w.L, w.D), generator=g, device=dev).to(torch.bfloat16)
        K = torch.randn((w.B, w.Hkv, w.L, w.D), generator=g, device=dev).to(torch.bfloat16)
        V = torch.randn((w.B, w.Hkv, w.L, w.D), generator=g, device=dev).to(torch.bfloat16)
        cache = StarCache(w.B, w.Hq, w.Hkv, w.D, w.L, w.b, w.b_a, 1, w.scale)
        O = torch.empty_like(Q)
        LSE = torch.empty((w.B, w.Hq, w.L), dtype=torch.float32, device=dev)
        evs = []
        for it in range(warmup + steps):
            flush.flush(6.0)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            cache.star_ctx_encode(Q, K, V, O, LSE)
            b.record(stream)
            if it >= warmup:
                evs.append((a, b))
        torch.cuda.synchronize(dev)
        ms = sum(a.elapsed_time(b) for a, b in evs) / len(evs)
        (ms,) = max_over_ranks([ms], dev, world)
        flops, _ = phase1_flops(w)
        out[name] = {"B": w.B, "L": w.L, "block": w.b, "anchor": w.b_a, "ms": ms,
                     "ctx_tok_s": world * w.B * w.L / (ms / 1e3), "tflops": flops / (ms / 1e3) / 1e12}
        cache.close()
        del Q, K, V, O, LSE
        torch.cuda.empty_cache()
    return out


def measure_rope(dev, flush, warmup, steps, world):
    """RoPE front end on the 8B-32K shape: the rotation of Q and K (HBM-bound),
    and phase 1 on un-rotated inputs with the previous-block anchor IDs
    (rotation + anchor keys + phase 1 on per-block anchor keys)."""
    import torch
    from block_sparse_long_phase_b200 import StarCache, star_rope, workloads as wl
    w = wl.get("8b-32k")
    g = torch.Generator(device=dev).manual_seed(w.seed + 11)
    Q = torch.randn((w.B, w.Hq, w.L, w.D), generator=g, device=dev).to(torch.bfloat16)
    K = torch.randn((w.B, w.Hkv, w.L, w.D), generator=g, device=dev).to(torch.bfloat16)
    V = torch.randn((w.B, w.Hkv, w.L, w.D), generator=g, device=dev).to(torch.bfloat16)
    Qr, Kr = torch.empty_like(Q), torch.empty_like(K)
    cache = StarCache(w.B, w.Hq, w.Hkv, w.D, w.L, w.b, w.b_a, 1, w.scale)
    nb = cache.num_segments - 1
    Ka = torch.empty((nb - 1, w.B, w.Hkv, w.b_a, w.D), dtype=torch.bfloat16, device=dev)
    O = torch.empty_like(Q)
    LSE = torch.empty((w.B, w.Hq, w.L), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    ev = lambda: torch.cuda.Event(enable_timing=True)
    rope_ms, all_ms = [], []
    for it in range(warmup + steps):
        flush.flush(7.0)
        a, b, c = ev(), ev(), ev()
        a.record(stream)
        star_rope(Q, out=Qr)
        star_rope(K, out=Kr)
        b.record(stream)
        cache.star_anchor_keys(K, "previous", Ka=Ka)
        cache.star_ctx_encode(Qr, Kr, V, O, LSE, Ka=Ka)
        c.record(stream)
        if it >= warmup:
            rope_ms.append((a, b))
            all_ms.append((a, c))
    torch.cuda.synchronize(dev)
    t_rope = sum(x.elapsed_time(y) for x, y in rope_ms) / steps
    t_all = sum(x.elapsed_time(y) for x, y in all_ms) / steps
    t_rope, t_all = max_over_ranks([t_rope, t_all], dev, world)
    nbytes = 2 * 2 * (Q.numel() + K.numel())          # read + write, bf16
    flops, _ = phase1_flops(w)
    cache.close()
    del Q, K, V, Qr, Kr, Ka, O, LSE
    torch.cuda.empty_cache()
    return {"workload": w.name, "rotation_us": t_rope * 1e3, "rotation_bytes": nbytes,
            "rotation_gbs": nbytes / (t_rope / 1e3) / 1e9,
            "phase1_previous_ids_ms": t_all, "ctx_tok_s": world * w.B * w.L / (t_all / 1e3),
            "phase1_tflops_incl_rope": flops / (t_all / 1e3) / 1e12}


def dist_setup(args):
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    return world, rank, local


def config_of(w, world):
    return {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "D": w.D, "L": w.L,
            "block": w.b, "anchor": w.b_a, "lq": w.lq, "decode_steps": w.T,
            "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
            "l2": "flushed before every timed kernel region (512 MB write, then 512 MB read: "
                  "no inputs, no dirty lines left in L2)"}


def run_reference(args):
    """The reference arm: the fp64 oracle on the host cores, each step one pass
    over the same fixed sample the GPU arm's cpu_baseline times, same code."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    from block_sparse_long_phase_b200 import workloads as wl
    w = wl.get(args.workload)
    data = oracle_sample_inputs(w)
    t0 = time.perf_counter()
    r = oracle_baseline(w, data, args.warmup, args.steps)
    el = time.perf_counter() - t0
    v, spread = baseline_summary(r)
    line = {
        "impl": "reference", "metric": METRIC, "value": v, "unit": "ctx tok/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": el / (args.steps + args.warmup) * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_of(w, world),
        "decode": {"value": r["decode"], "unit": "decode tok/s"},
        "cpu_baseline": {"value": v, "unit": "ctx tok/s", "cores": r["threads"], "kind": "oracle",
                         "sample": r["sample"], "spread": spread, "passes": len(r["ctx"])},
        "e2e": {"value": v, "unit": "ctx tok/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def profile_case(args):
    """Launches of one kernel for an ncu capture (no bench line): ``phase1``
    runs star_ctx_encode ``steps`` times; ``prefill`` runs phase 1 once and the
    query prefill ``steps`` times; ``decode`` runs phase 1 and the query
    prefill once and then ``steps`` decode steps.  ``--blocks N`` keeps the
    first N blocks of the workload (a capture small enough to replay)."""
    import torch
    from block_sparse_long_phase_b200 import StarCache, workloads as wl
    torch.cuda.set_device(0)
    w = wl.get(args.workload)
    if args.blocks:
        w = w.with_(L=min(w.L, args.blocks * w.b))
    if args.profile == "decode":
        w = w.with_(T=max(w.T, args.steps))
    x = wl.make_inputs(w, "cuda")
    cache = StarCache(w.B, w.Hq, w.Hkv, w.D, w.L, w.b, w.b_a, w.lq + w.T, w.scale, kv_fp8=args.kv_fp8)
    O = torch.empty_like(x["Qc"])
    LSE = torch.empty((w.B, w.Hq, w.L), dtype=torch.float32, device="cuda")
    n = args.steps if args.profile == "phase1" else 1
    for _ in range(n):
        cache.star_ctx_encode(x["Qc"], x["Kc"], x["Vc"], O, LSE)
    if args.profile == "prefill":
        for _ in range(args.steps):
            cache.reset_query()
            cache.star_query_prefill(x["Qq"], x["Kq"], x["Vq"])
    if args.profile == "decode":
        cache.star_query_prefill(x["Qq"], x["Kq"], x["Vq"])
        for t in range(args.steps):
            cache.star_decode_step(x["qd"][t], x["kd"][t], x["vd"][t])
    torch.cuda.synchronize()
    if cache.device_error():
        raise SystemExit("a kernel gave up a bounded wait")
    cache.close()
    print(f"profile case {args.profile}: {w.name} L={w.L} kv_fp8={args.kv_fp8} launches={args.steps}")


def measure_e2e(args, w, x, O, LSE, cache, flush, dev, world):
    """Phase 1 through star_ctx_encode_host with page-locked host Q, K, V in and
    O, LSE out, copies inside the timed region.  Every rank of a node holds its
    own host copies; if they would take more than half of the host memory
    available, the leg runs on the 8B-128K workload instead (named in the
    result)."""
    import torch
    from block_sparse_long_phase_b200 import StarCache, workloads as wl
    need = sum(t.numel() * t.element_size() for t in (x["Qc"], x["Kc"], x["Vc"], O, LSE))
    local_world = int(os.environ.get("LOCAL_WORLD_SIZE", str(world)))
    try:
        import psutil
        avail = psutil.virtual_memory().available
    except Exception:
        avail = None
    own = None
    small = avail is not None and need * local_world > avail // 2
    # every rank takes the same workload: the smaller one if any rank's node is short
    (small_any,) = max_over_ranks([1.0 if small else 0.0], dev, world)
    if small_any > 0:
        w = wl.get("8b-128k-needle")
        x = wl.make_inputs(w, dev, with_decode=False)
        own = StarCache(w.B, w.Hq, w.Hkv, w.D, w.L, w.b, w.b_a, w.lq + w.T, w.scale)
        cache = own
        O = torch.empty_like(x["Qc"])
        LSE = torch.empty((w.B, w.Hq, w.L), dtype=torch.float32, device=dev)
    h, locked = host_buffers(x, O, LSE)
    # the device tensors double as the call's staging buffers (same shapes)
    staging = {"Q": x["Qc"], "K": x["Kc"], "V": x["Vc"], "O": O, "LSE": LSE}
    stream = torch.cuda.current_stream(dev)
    e2e_ms = []
    for it in range(args.warmup + args.steps):
        flush.flush(4.0)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        cache.star_ctx_encode_host(h["Q"], h["K"], h["V"], h["O"], h["LSE"], staging)
        b.record(stream)
        torch.cuda.synchronize(dev)
        if it >= args.warmup:
            e2e_ms.append(a.elapsed_time(b))
    (e2e_total,) = max_over_ranks([sum(e2e_ms)], dev, world)
    h2d = sum(h[k].numel() * h[k].element_size() for k in ("Q", "K", "V"))
    d2h = h["O"].numel() * 2 + h["LSE"].numel() * 4
    out = {"value": world * w.B * w.L * args.steps / (e2e_total / 1e3), "unit": "ctx tok/s",
           "ms_per_step": e2e_total / args.steps, "workload": w.name,
           "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
           "host_memory": "page-locked (cudaHostRegister)" if locked else "pageable (page-locking refused)",
           "what": "star_ctx_encode_host: host Q,K,V in, O,LSE out, copies overlapped with the "
                   "encoding block by block, all inside the timed region"}
    cudart = torch.cuda.cudart()
    for t in locked:
        cudart.cudaHostUnregister(t.data_ptr())
    if own is not None:
        own.close()
    return out


def host_buffers(x, O, LSE):
    """Host copies of the phase-1 inputs and room for its outputs, page-locked
    in place (cudaHostRegister of exactly their bytes); pageable if the host
    refuses to lock that much."""
    import torch
    h = {"Q": torch.empty(x["Qc"].shape, dtype=torch.bfloat16),
         "K": torch.empty(x["Kc"].shape, dtype=torch.bfloat16),
         "V": torch.empty(x["Vc"].shape, dtype=torch.bfloat16),
         "O": torch.empty(O.shape, dtype=torch.bfloat16),
         "LSE": torch.empty(LSE.shape, dtype=torch.float32)}
    cudart = torch.cuda.cudart()
    locked = []
    for t in h.values():
        rc = cudart.cudaHostRegister(t.data_ptr(), t.numel() * t.element_size(), 0)
        if int(rc) != 0:
            break
        locked.append(t)
    if len(locked) < len(h):
        for t in locked:
            cudart.cudaHostUnregister(t.data_ptr())
        locked = []
    h["Q"].copy_(x["Qc"])
    h["K"].copy_(x["Kc"])
    h["V"].copy_(x["Vc"])
    return h, locked


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="star", choices=["star", "reference"])
    ap.add_argument("--workload", default=WORKLOAD)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-long-decode", action="store_true",
                    help="skip the decode measurement at 128K context")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip phase 1 / prefill / decode on the other configurations")
    ap.add_argument("--no-variants", action="store_true",
                    help="skip the phase-1 variants (anchor shorter than the block, ragged context, batch 4)")
    ap.add_argument("--no-sharded", action="store_true",
                    help="skip the block-sharded layer's per-rank kernels (ranks emulated on one GPU)")
    ap.add_argument("--profile", choices=["phase1", "prefill", "decode"],
                    help="only launch this kernel `steps` times for an ncu capture (no bench line)")
    ap.add_argument("--blocks", type=int, default=0, help="--profile: keep the first N blocks")
    ap.add_argument("--kv-fp8", action="store_true", help="--profile decode: stream the FP8 cache")
    args = ap.parse_args()
    if args.impl == "reference":
        return run_reference(args)
    if args.profile:
        return profile_case(args)

    import torch
    from block_sparse_long_phase_b200 import StarCache, workloads as wl

    world, rank, local = dist_setup(args)
    dev = torch.device("cuda", local)
    w = wl.get(args.workload)
    x = wl.make_inputs(w, dev)
    cache = StarCache(w.B, w.Hq, w.Hkv, w.D, w.L, w.b, w.b_a, w.lq + w.T, w.scale)
    O = torch.empty((w.B, w.Hq, w.L, w.D), dtype=torch.bfloat16, device=dev)
    LSE = torch.empty((w.B, w.Hq, w.L), dtype=torch.float32, device=dev)
    Oq = torch.empty((w.B, w.Hq, w.lq, w.D), dtype=torch.bfloat16, device=dev)
    LSEq = torch.empty((w.B, w.Hq, w.lq), dtype=torch.float32, device=dev)
    od = torch.empty((w.T, w.B, w.Hq, 1, w.D), dtype=torch.bfloat16, device=dev)
    lsed = torch.empty((w.T, w.B, w.Hq), dtype=torch.float32, device=dev)
    # 2 x 512 MB: larger than L2, and long enough (~160 us) for the host to queue
    # the timed launch behind it, so the start event is not recorded on an idle GPU
    flush = L2Flush(dev)
    stream = torch.cuda.current_stream(dev)

    def ev():
        return torch.cuda.Event(enable_timing=True)

    def step(times):
        flush.flush(1.0)
        e0, e1 = ev(), ev()
        e0.record(stream)
        cache.star_ctx_encode(x["Qc"], x["Kc"], x["Vc"], O, LSE)
        e1.record(stream)
        flush.flush(2.0)
        e2, e3 = ev(), ev()
        e2.record(stream)
        cache.star_query_prefill(x["Qq"], x["Kq"], x["Vq"], Oq, LSEq)
        e3.record(stream)
        dec = []
        for t in range(w.T):
            flush.flush(3.0)
            a, b = ev(), ev()
            a.record(stream)
            cache.star_decode_step(x["qd"][t], x["kd"][t], x["vd"][t], od[t], lsed[t])
            b.record(stream)
            dec.append((a, b))
        times.append(((e0, e1), (e2, e3), dec))

    clocks = Clocks(local)
    clocks.start()
    for _ in range(args.warmup):
        step([])
    torch.cuda.synchronize(dev)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    clocks.mark(True)
    t_wall = time.perf_counter()
    times = []
    for _ in range(args.steps):
        step(times)
    torch.cuda.synchronize(dev)
    wall = time.perf_counter() - t_wall
    clocks.mark(False)
    if world > 1:
        torch.distributed.barrier()
    clk = clocks.stop()
    enc_ms = [a.elapsed_time(b) for (a, b), _, _ in times]
    pre_ms = [a.elapsed_time(b) for _, (a, b), _ in times]
    dec_ms = [[a.elapsed_time(b) for a, b in d] for _, _, d in times]
    step_ms = [e + p + sum(d) for e, p, d in zip(enc_ms, pre_ms, dec_ms)]
    enc_total = sum(enc_ms)
    dec_total = sum(sum(d) for d in dec_ms)
    pre_total = sum(pre_ms)
    enc_total, dec_total, pre_total, step_total = max_over_ranks(
        [enc_total, dec_total, pre_total, sum(step_ms)], dev, world)

    # ---- end to end through the public API (page-locked host buffers) ----------
    e2e = None
    if not args.no_e2e:
        torch.cuda.synchronize(dev)
        e2e = measure_e2e(args, w, x, O, LSE, cache, flush, dev, world)

    # the main workload's buffers are no longer needed
    cache.close()
    del x, O, LSE, Oq, LSEq, od, lsed, cache
    torch.cuda.empty_cache()

    def settle(seconds=1.0):
        # each further section starts from an idle GPU rather than under the
        # power and thermal state the section before it left behind
        torch.cuda.synchronize(dev)
        time.sleep(seconds)

    long_dec = long_dec_fp8_main = None
    if not args.no_long_decode:
        # the short FP8 steps are clock-sensitive (their consumers convert and
        # multiply): the GPU cools down from the seconds-long phase-1 section first
        settle(5.0)
        long_dec = measure_long_decode(dev, flush, args.warmup, args.steps, world)
        settle()
        long_dec_fp8 = measure_long_decode(dev, flush, args.warmup, args.steps, world, kv_fp8=True)
        if w.name != "8b-128k-needle":
            # the FP8 stream on the main workload's context too, where it dominates the step
            settle()
            long_dec_fp8_main = measure_long_decode(dev, flush, args.warmup, args.steps, world, kv_fp8=True,
                                                    name=w.name)
    sharded = None
    if not args.no_sharded and world == 1:
        settle()
        sharded = measure_sharded(dev, flush, w)
    rope = variants = None
    if not args.no_variants:
        settle()
        rope = measure_rope(dev, flush, args.warmup, min(args.steps, 10), world)
        settle()
        variants = measure_phase1_variants(dev, flush, args.warmup, min(args.steps, 10), world)
    configs = None
    if not args.no_configs:
        settle()
        configs = measure_configs(dev, flush, args.warmup, min(args.steps, 3), world)

    pk = peaks()
    flops, _ = phase1_flops(w)
    enc_avg_s = enc_total / args.steps / 1e3
    achieved_tf = flops / enc_avg_s / 1e12
    dbytes = sum(decode_bytes(w, t) for t in range(w.T))
    dec_avg_s = dec_total / args.steps / 1e3
    achieved_gbs = dbytes / dec_avg_s / 1e9
    value = world * w.B * w.L / enc_avg_s
    # a launch of a second or more runs under the power cap: the sustained peak
    # is its denominator; a launch of a few ms is timed against the burst peak
    long_launch = enc_avg_s > 0.1 and pk["bf16_tflops_sustained"]
    peak_tf = pk["bf16_tflops_sustained"] if long_launch else pk["bf16_tflops"]
    line = {
        "metric": METRIC, "value": value, "unit": "ctx tok/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_total / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": config_of(w, world),
        "decode": {"value": world * w.B * w.T / dec_avg_s, "unit": "decode tok/s",
                   "us_per_step": dec_avg_s / w.T * 1e6, "steps_per_iteration": w.T,
                   "roofline": {"bound": "hbm", "achieved": achieved_gbs, "peak": pk["hbm_gbs"],
                                "unit": "GB/s", "frac": achieved_gbs / pk["hbm_gbs"],
                                "frac_datasheet": achieved_gbs / DATASHEET_HBM_GBS,
                                "traffic": traffic(f"decode {w.name}"),
                                "bytes_per_iteration": dbytes,
                                "peak_source": pk["source"] + " copy bandwidth (datasheet 7.7 TB/s in frac_datasheet)"}},
        "prefill_ms": pre_total / args.steps,
        "prefill_roofline": prefill_roofline(w, pre_total / args.steps, pk),
        "roofline": {"bound": "tensor", "achieved": achieved_tf, "peak": peak_tf,
                     "unit": "TFLOP/s", "frac": achieved_tf / peak_tf,
                     "frac_burst": achieved_tf / pk["bf16_tflops"],
                     "traffic": traffic(f"phase1 {w.name}"),
                     "kernel": "phase-1 context encode", "flops_per_launch": flops,
                     "ms_per_launch": enc_avg_s * 1e3,
                     "peak_source": pk["source"] + (" sustained bf16 dense (the launch lasts over 0.1 s, under the power cap)"
                                                    if long_launch else " burst bf16 dense")},
        "clocks": clk,
        # per step: phase 1 (1 launch), prefill (append, tile kernel, merge: 3), one per decode step
        "gpu_launches": args.steps * (1 + 3 + w.T),
        "wall_s_timed_region": wall,
    }
    if e2e:
        line["e2e"] = e2e
    if rope:
        rope["rotation_frac"] = rope["rotation_gbs"] / pk["hbm_gbs"]
        line["rope"] = rope
    if configs:
        line["configs"] = configs
    if sharded:
        line["sharded_emulated"] = sharded
    if variants:
        for v in variants.values():
            # burst peak for a launch of a few ms; a launch of 10+ ms runs under
            # the power cap, where the sustained peak is the fair denominator
            v["frac"] = v["tflops"] / pk["bf16_tflops"]
            v["frac_sustained"] = v["tflops"] / pk["bf16_tflops_sustained"]
        line["phase1_variants"] = variants
    if long_dec:
        wl2, t_us = long_dec
        gbs = decode_bytes(wl2, 0) / (t_us * 1e-6) / 1e9
        line["decode_long"] = {
            "workload": wl2.name, "value": world * wl2.B / (t_us * 1e-6), "unit": "decode tok/s",
            "us_per_step": t_us,
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": pk["hbm_gbs"], "unit": "GB/s",
                         "frac": gbs / pk["hbm_gbs"], "frac_datasheet": gbs / DATASHEET_HBM_GBS,
                         "traffic": traffic("decode 8b-128k"), "bytes_per_step": decode_bytes(wl2, 0)}}
        wl3, t3 = long_dec_fp8
        gbs = decode_bytes_fp8(wl3, 0) / (t3 * 1e-6) / 1e9
        line["decode_long_fp8"] = {
            "workload": wl3.name, "kv_cache": "K/V rows in E4M3 with a float32 scale per row",
            "value": world * wl3.B / (t3 * 1e-6), "unit": "decode tok/s", "us_per_step": t3,
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": pk["hbm_gbs"], "unit": "GB/s",
                         "frac": gbs / pk["hbm_gbs"], "frac_datasheet": gbs / DATASHEET_HBM_GBS,
                         "traffic": traffic("decode fp8 8b-128k"), "bytes_per_step": decode_bytes_fp8(wl3, 0)}}
    if long_dec_fp8_main:
        wl4, t4 = long_dec_fp8_main
        gbs = decode_bytes_fp8(wl4, 0) / (t4 * 1e-6) / 1e9
        line["decode_fp8"] = {
            "workload": wl4.name, "kv_cache": "K/V rows in E4M3 with a float32 scale per row",
            "value": world * wl4.B / (t4 * 1e-6), "unit": "decode tok/s", "us_per_step": t4,
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": pk["hbm_gbs"], "unit": "GB/s",
                         "frac": gbs / pk["hbm_gbs"], "frac_datasheet": gbs / DATASHEET_HBM_GBS,
                         "traffic": None, "bytes_per_step": decode_bytes_fp8(wl4, 0)}}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        data = oracle_sample_inputs(w)
        r = oracle_baseline(w, data, 1, 5)
        v, spread = baseline_summary(r)
        line["cpu_baseline"] = {"value": v, "unit": "ctx tok/s", "cores": r["threads"], "kind": "oracle",
                                "sample": r["sample"], "spread": spread, "passes": len(r["ctx"]),
                                "decode_value": r["decode"]}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
