"""The allocation-free decode entry point, against the regular one and the oracle.

star_decode_step_noalloc serves callers that may not call cudaMalloc while
they serve (a runtime that owns all device memory through its own pool, or
one that forbids the CUDA allocator on its serving path): the KV cache is the
caller's memory and the split-KV scratch is a static array of the library.
Here the caller's buffers are either copies of a regular cache's segments and
query region, or built directly from the inputs in the segmented layout; two
decode steps in a row must agree with the regular entry point and with the
fp64 oracle within the tolerance of the parity tests.  This file is collected
last so a failure here leaves every other test already run.
"""

import ctypes

import numpy as np
import pytest
import torch

from block_sparse_long_phase_b200 import workloads as wl
from oracle import star_oracle as so

pytestmark = pytest.mark.gpu

MAX_ABS = 1e-2
MEAN_ABS = 1e-3
LSE_ABS = 1e-3

# size of the static scratch's partial-output area, in floats (header limit)
SCRATCH_FLOATS = 1 << 20


def scratch_floats(B, Hkv, G, D, L, len0, sms):
    """Partial-output floats one no-alloc step needs: the decode plan's part
    slots per (batch, kv head) times G rows of D floats (the header's limit)."""
    bgs = B * Hkv
    n = max(1, min(sms, bgs * (L + len0) // 512))
    aligned = n // bgs * bgs
    if n == sms and aligned > 0 and aligned * 25 >= n * 24:
        n = aligned
    maxp = -(-n // bgs) + 3
    return bgs * maxp * G * D


def close(got, ref, lg, lr, what):
    g = got.double().cpu().numpy()
    err = np.abs(g - ref)
    assert np.isfinite(g).all(), what
    assert err.max() <= MAX_ABS and err.mean() <= MEAN_ABS, (what, err.max(), err.mean())
    assert np.abs(lg.double().cpu().numpy() - lr).max() <= LSE_ABS, what


def segmented(K, b):
    """K [B, Hkv, L, D] in the cache's context layout: segment i = rows
    [i*b, i*b + len_i) of every (batch, kv head), segments back to back."""
    L = K.shape[2]
    return torch.cat([K[:, :, s:s + n].contiguous().view(-1) for s, n in so.block_table(L, b)])


def run_against_oracle(w, steps=2):
    """Caller-owned buffers built from the inputs; `steps` decode steps in a
    row through the no-alloc entry point, each against the oracle."""
    from block_sparse_long_phase_b200 import _abi
    from block_sparse_long_phase_b200.api import star_decode_step_noalloc, star_noalloc_device_error
    cpu = wl.make_inputs(w, "cpu")
    x = {k: v.cuda() for k, v in cpu.items()}
    q_cap = w.lq + steps
    ctx_k, ctx_v = segmented(x["Kc"], w.b), segmented(x["Vc"], w.b)
    q_k = torch.zeros((w.B, w.Hkv, q_cap, w.D), dtype=torch.bfloat16, device="cuda")
    q_v = torch.zeros_like(q_k)
    q_k[:, :, :w.lq] = x["Kq"]
    q_v[:, :, :w.lq] = x["Vq"]
    params = _abi.StarParams(w.B, w.Hq, w.Hkv, w.D, w.L, w.b, w.b_a, q_cap, w.scale)
    segs = so.cache_segments(cpu["Kc"], cpu["Vc"], w.b)
    qk = np.zeros((w.B, w.Hkv, q_cap, w.D))
    qv = np.zeros_like(qk)
    qk[:, :, :w.lq] = cpu["Kq"].double().numpy()
    qv[:, :, :w.lq] = cpu["Vq"].double().numpy()
    for t in range(steps):
        o, l = star_decode_step_noalloc(params, w.lq + t, ctx_k, ctx_v, q_k, q_v,
                                        x["qd"][t], x["kd"][t], x["vd"][t])
        torch.cuda.synchronize()
        ref, lref, qk, qv = so.decode_step(cpu["qd"][t], cpu["kd"][t], cpu["vd"][t], segs, qk, qv,
                                           w.lq + t, w.scale)
        close(o, ref, l, lref[:, :, 0], f"no-alloc decode {t}")
    assert star_noalloc_device_error() == 0
    return params


@pytest.mark.parametrize("name,over", [("tiny", {}), ("8b-32k", dict(T=4))])
def test_noalloc_decode_matches_regular_entry_point(name, over):
    from block_sparse_long_phase_b200 import StarCache, _abi
    from block_sparse_long_phase_b200.api import (star_decode_step_noalloc, star_noalloc_device_error,
                                                  _tensor_from_ptr)
    w = wl.get(name).with_(**over)
    dev = "cpu" if name == "tiny" else "cuda"
    x = {k: v.cuda() for k, v in wl.make_inputs(w, dev).items()}
    cache = StarCache(w.B, w.Hq, w.Hkv, w.D, w.L, w.b, w.b_a, w.lq + w.T, w.scale)
    cache.star_ctx_encode(x["Qc"], x["Kc"], x["Vc"])
    cache.star_query_prefill(x["Qq"], x["Kq"], x["Vq"])
    torch.cuda.synchronize()
    # the caller's own buffers: copies of the cache's segments and query region
    n_ctx = w.B * w.Hkv * w.L * w.D
    ctx_k = torch.empty(n_ctx, dtype=torch.bfloat16, device="cuda")
    ctx_v = torch.empty(n_ctx, dtype=torch.bfloat16, device="cuda")
    ctx_k.copy_(_tensor_from_ptr(cache.segment(0).k, n_ctx, ctx_k.device))
    ctx_v.copy_(_tensor_from_ptr(cache.segment(0).v, n_ctx, ctx_v.device))
    qk_c, qv_c, qseg = cache.segment_tensors(cache.num_segments - 1)
    q_k = qk_c.clone()
    q_v = qv_c.clone()
    q_len = qseg.len
    params = _abi.StarParams(w.B, w.Hq, w.Hkv, w.D, w.L, w.b, w.b_a, w.lq + w.T, w.scale)
    for t in range(2):
        o_ref, l_ref = cache.star_decode_step(x["qd"][t], x["kd"][t], x["vd"][t])
        o, l = star_decode_step_noalloc(params, q_len + t, ctx_k, ctx_v, q_k, q_v,
                                        x["qd"][t], x["kd"][t], x["vd"][t])
        torch.cuda.synchronize()
        err = (o.double() - o_ref.double()).abs()
        assert torch.isfinite(o.float()).all()
        assert err.max().item() <= MAX_ABS and err.mean().item() <= MEAN_ABS, (t, err.max().item())
        assert (l.double() - l_ref.double()).abs().max().item() <= LSE_ABS
        # the query region of the caller's buffers received this step's k, v
        assert torch.equal(q_k[:, :, q_len + t].view(torch.int16), x["kd"][t][:, :, 0].view(torch.int16))
        assert torch.equal(q_v[:, :, q_len + t].view(torch.int16), x["vd"][t][:, :, 0].view(torch.int16))
    assert cache.device_error() == 0
    assert star_noalloc_device_error() == 0
    cache.close()


def test_noalloc_decode_matches_the_oracle_on_ragged_blocks():
    """Four blocks, the last one ragged, an anchor shorter than the block."""
    run_against_oracle(wl.get("tiny").with_(L=1000, b=256, b_a=100, lq=5, T=2))


def test_noalloc_just_under_and_just_over_the_static_scratch():
    """A shape whose partials fill the static array to within 3 % runs and
    matches the oracle; one a few (batch, kv head) pairs larger is refused."""
    from block_sparse_long_phase_b200 import _abi
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    under = wl.get("tiny").with_(B=25, Hq=64, Hkv=4, D=128, L=768, b=256, b_a=256, lq=4, T=2)
    need = scratch_floats(under.B, under.Hkv, under.G, under.D, under.L, under.lq, sms)
    if not (0.9 * SCRATCH_FLOATS < need <= SCRATCH_FLOATS):
        pytest.skip(f"shape is not near the limit on {sms} SMs ({need} floats)")
    run_against_oracle(under)
    over = under.with_(B=103, Hq=16, Hkv=1)
    assert scratch_floats(over.B, over.Hkv, over.G, over.D, over.L, over.lq, sms) > SCRATCH_FLOATS
    lib = _abi.load()
    p = _abi.StarParams(over.B, over.Hq, over.Hkv, over.D, over.L, over.b, over.b_a, over.lq + 2, 0.0)
    buf = torch.zeros(16, dtype=torch.bfloat16, device="cuda")
    ptr = buf.data_ptr()
    rc = lib.star_decode_step_noalloc(ctypes.byref(p), over.lq, ptr, ptr, ptr, ptr, ptr, ptr, ptr, ptr,
                                      ptr, None)
    assert rc == _abi.STAR_EINVAL
    assert b"static decode scratch" in lib.star_last_error()


def test_noalloc_rejects_oversized_problems():
    from block_sparse_long_phase_b200 import _abi
    lib = _abi.load()
    p = _abi.StarParams(64, 128, 64, 128, 1024, 256, 256, 8, 0.0)   # B*Hkv = 4096 > 1024
    buf = torch.zeros(16, dtype=torch.bfloat16, device="cuda")
    ptr = buf.data_ptr()
    rc = lib.star_decode_step_noalloc(ctypes.byref(p), 0, ptr, ptr, ptr, ptr, ptr, ptr, ptr, ptr,
                                      ptr, None)
    assert rc == _abi.STAR_EINVAL
    assert b"static decode scratch" in lib.star_last_error()
    # an FP8 cache is refused on this path, and so is a full query region
    p8 = _abi.StarParams(1, 4, 2, 64, 1024, 256, 256, 8, 0.0, 1)
    assert lib.star_decode_step_noalloc(ctypes.byref(p8), 0, *([ptr] * 9), None) == _abi.STAR_EINVAL
    p = _abi.StarParams(1, 4, 2, 64, 1024, 256, 256, 8, 0.0)
    assert lib.star_decode_step_noalloc(ctypes.byref(p), 8, *([ptr] * 9), None) == _abi.STAR_ENOSPC
