"""Seeded synthetic inputs shaped like the Star Attention long-context workloads.

This module only draws random numbers and plants the needle keys; it holds
none of the attention arithmetic.  The same tensors feed the CUDA path and the
fp64 oracle (upcast exactly from bf16).

Shapes follow the Llama-3.1-8B and Llama-3.1-70B attention layers the
"Star Attention: Efficient LLM Inference over Long Sequences" analysis page
evaluates ("Hyperparameters and Configuration Choices", models tested: 32/8
and 64/8 heads, head dim 128; block size one quarter of the context up to
128K, anchor size equal to the block size).  No dataset is used: RULER,
BABILong and InfiniteBench are replaced by i.i.d. N(0, 1) bf16 Q/K/V.

Draw order (one generator per workload, ``seed = 20241126 + index``):
context Q, K, V; query Q, K, V; then (q, k, v) for every decode step; for
the needle workload the needle directions and positions come last.  Each
tensor is drawn one (batch, head) slice at a time as float32 N(0, 1) and
rounded to bf16 (round to nearest even).  Small workloads draw on the CPU;
large ones draw on the device that will use them (same order, the device's
own Philox stream), which keeps a 1M-token workload to seconds.
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field, replace

import torch

BASE_SEED = 20241126


@dataclass(frozen=True)
class Workload:
    name: str
    B: int          # batch
    Hq: int         # query heads
    Hkv: int        # key/value heads (GQA)
    D: int          # head dim
    L: int          # context length
    b: int          # block size
    b_a: int        # anchor size
    lq: int         # query tokens (phase-2 prefill)
    T: int          # decode steps
    needle: bool = False
    index: int = 0
    notes: str = field(default="", compare=False)

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    @property
    def n_blocks(self) -> int:
        return -(-self.L // self.b)

    @property
    def scale(self) -> float:
        # 1/sqrt(d) rounded to fp32, the value the C ABI receives.
        return float(torch.tensor(1.0 / math.sqrt(self.D), dtype=torch.float32))

    @property
    def seed(self) -> int:
        return BASE_SEED + self.index

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


WORKLOADS = {
    "tiny": Workload("tiny", 1, 4, 2, 64, 1024, 256, 256, 16, 8, index=0),
    "8b-32k": Workload("8b-32k", 1, 32, 8, 128, 32768, 8192, 8192, 64, 32, index=1),
    "8b-128k-needle": Workload("8b-128k-needle", 1, 32, 8, 128, 131072, 32768, 32768,
                               128, 256, needle=True, index=2),
    "70b-128k": Workload("70b-128k", 1, 64, 8, 128, 131072, 16384, 16384, 64, 128, index=3),
    "70b-128k-b4": Workload("70b-128k-b4", 4, 64, 8, 128, 131072, 16384, 16384, 64, 128,
                            index=3, notes="batch-4 decode variant"),
    "8b-1m": Workload("8b-1m", 1, 32, 8, 128, 1048576, 65536, 65536, 64, 64, index=4),
}

# Needle construction for the 8B-128K workload: every query / decode q row of
# kv group g has component NEEDLE_ALPHA along a seeded unit direction u_g, and
# NEEDLE_COUNT seeded context keys per (batch, kv head) have component
# NEEDLE_BETA along u_g, so a needle's scaled logit is about 14 while the
# largest noise logit over 128K keys is about 5-6 (a gap of about +8).
NEEDLE_COUNT = 8
NEEDLE_ALPHA = 4.0
NEEDLE_LOGIT = 14.0


def needle_beta(D: int) -> float:
    return NEEDLE_LOGIT * math.sqrt(D) / NEEDLE_ALPHA


def _randn_bf16(gen, shape, device):
    """float32 N(0,1) drawn one leading-dims slice at a time, rounded to bf16."""
    out = torch.empty(shape, dtype=torch.bfloat16, device=device)
    lead = shape[:-2]
    flat = out.view(-1, shape[-2], shape[-1])
    for i in range(flat.shape[0]):
        flat[i] = torch.randn(shape[-2], shape[-1], generator=gen, device=device,
                              dtype=torch.float32).to(torch.bfloat16)
    del lead
    return out


def _set_component(x_bf16, u, value):
    """x <- x + (value - x.u) u along the last dim, in fp32, then back to bf16."""
    x = x_bf16.float()
    c = (x * u).sum(-1, keepdim=True)
    return (x + (value - c) * u).to(torch.bfloat16)


def make_inputs(w: Workload, device="cpu", with_decode=True):
    """All inputs of one workload as bf16 tensors on ``device``.

    Returns a dict with ``Qc [B,Hq,L,D]``, ``Kc``/``Vc [B,Hkv,L,D]``,
    ``Qq [B,Hq,lq,D]``, ``Kq``/``Vq [B,Hkv,lq,D]`` and, if ``with_decode``,
    ``qd [T,B,Hq,1,D]``, ``kd``/``vd [T,B,Hkv,1,D]``; for the needle workload
    also ``needle_dir [B,Hkv,D]`` (float32) and ``needle_pos [B,Hkv,8]``.
    """
    device = torch.device(device)
    gen = torch.Generator(device=device)
    gen.manual_seed(w.seed)
    B, Hq, Hkv, D, L, lq, T = w.B, w.Hq, w.Hkv, w.D, w.L, w.lq, w.T
    r = {}
    r["Qc"] = _randn_bf16(gen, (B, Hq, L, D), device)
    r["Kc"] = _randn_bf16(gen, (B, Hkv, L, D), device)
    r["Vc"] = _randn_bf16(gen, (B, Hkv, L, D), device)
    r["Qq"] = _randn_bf16(gen, (B, Hq, lq, D), device)
    r["Kq"] = _randn_bf16(gen, (B, Hkv, lq, D), device)
    r["Vq"] = _randn_bf16(gen, (B, Hkv, lq, D), device)
    if with_decode:
        steps = [(_randn_bf16(gen, (B, Hq, 1, D), device),
                  _randn_bf16(gen, (B, Hkv, 1, D), device),
                  _randn_bf16(gen, (B, Hkv, 1, D), device)) for _ in range(T)]
        r["qd"] = torch.stack([s[0] for s in steps]) if T else torch.empty(
            (0, B, Hq, 1, D), dtype=torch.bfloat16, device=device)
        r["kd"] = torch.stack([s[1] for s in steps]) if T else torch.empty(
            (0, B, Hkv, 1, D), dtype=torch.bfloat16, device=device)
        r["vd"] = torch.stack([s[2] for s in steps]) if T else torch.empty(
            (0, B, Hkv, 1, D), dtype=torch.bfloat16, device=device)
    if w.needle:
        u = torch.randn(B, Hkv, D, generator=gen, device=device, dtype=torch.float32)
        u = u / u.norm(dim=-1, keepdim=True)
        pos = torch.stack([torch.stack([
            torch.randperm(L, generator=gen, device=device)[:NEEDLE_COUNT].sort().values
            for _ in range(Hkv)]) for _ in range(B)])
        G = w.G
        uq = u.repeat_interleave(G, dim=1)                 # [B, Hq, D]
        r["Qq"] = _set_component(r["Qq"], uq[:, :, None, :], NEEDLE_ALPHA)
        if with_decode and T:
            r["qd"] = _set_component(r["qd"], uq[None, :, :, None, :], NEEDLE_ALPHA)
        beta = needle_beta(D)
        Kc = r["Kc"]
        for bi in range(B):
            for g in range(Hkv):
                p = pos[bi, g]
                Kc[bi, g, p] = _set_component(Kc[bi, g, p], u[bi, g][None, :], beta)
        r["needle_dir"] = u
        r["needle_pos"] = pos
    return r


def get(name: str) -> Workload:
    return WORKLOADS[name]
