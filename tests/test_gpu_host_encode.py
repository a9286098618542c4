"""Phase 1 from host memory (star_ctx_encode_host) against the device entry.

The host form runs the same tiles in pipeline units with the copies
overlapped; every output tile is still computed by one CTA with the same
arithmetic, so O, LSE and the cache must equal star_ctx_encode's bit for bit.
The device call itself is checked against the oracle in the parity suite; one
small case here also goes to the oracle directly.
"""

import numpy as np
import pytest
import torch

from block_sparse_long_phase_b200 import workloads as wl
from oracle import star_oracle as so

pytestmark = pytest.mark.gpu

VARIANTS = {
    "tiny": {},
    "ragged-anchor-shorter": dict(L=1000, b_a=100),
    "batch2": dict(B=2, L=700, b=256, b_a=200),
    "d128-gqa8-batch3": dict(B=3, Hq=16, Hkv=2, D=128, L=600, b=256, b_a=256),
    "single-block": dict(b=1024, b_a=1024),
}


def bits(t):
    return t.contiguous().view(torch.int16)


def encode_both(w, x, pinned=True, kv_fp8=False):
    from block_sparse_long_phase_b200 import StarCache
    cap = w.lq + w.T
    ref = StarCache(w.B, w.Hq, w.Hkv, w.D, w.L, w.b, w.b_a, cap, w.scale, kv_fp8=kv_fp8)
    O, LSE = ref.star_ctx_encode(x["Qc"], x["Kc"], x["Vc"])
    host = StarCache(w.B, w.Hq, w.Hkv, w.D, w.L, w.b, w.b_a, cap, w.scale, kv_fp8=kv_fp8)
    h = {k: x[k].cpu() for k in ("Qc", "Kc", "Vc")}
    if pinned:
        h = {k: v.pin_memory() for k, v in h.items()}
    hO = torch.empty(O.shape, dtype=O.dtype)
    hL = torch.empty(LSE.shape, dtype=LSE.dtype)
    if pinned:
        hO, hL = hO.pin_memory(), hL.pin_memory()
    hO, hL, staging = host.star_ctx_encode_host(h["Qc"], h["Kc"], h["Vc"], hO, hL)
    torch.cuda.synchronize()
    assert host.device_error() == 0
    return ref, host, O, LSE, hO, hL, staging


def check_same(w, ref, host, O, LSE, hO, hL, staging):
    assert torch.equal(bits(O.cpu()), bits(hO)), "O differs"
    assert torch.equal(LSE.cpu(), hL), "LSE differs"
    assert torch.equal(bits(staging["O"]), bits(O))
    for i in range(ref.num_segments - 1):
        k1, v1, s1 = ref.segment_tensors(i)
        k2, v2, s2 = host.segment_tensors(i)
        assert (s1.start, s1.len) == (s2.start, s2.len)
        assert torch.equal(bits(k1), bits(k2)) and torch.equal(bits(v1), bits(v2)), f"segment {i}"


@pytest.mark.parametrize("variant", list(VARIANTS))
def test_host_encode_equals_device_encode(variant):
    w = wl.get("tiny").with_(**VARIANTS[variant])
    x = {k: v.cuda() for k, v in wl.make_inputs(w, "cpu", with_decode=False).items()}
    out = encode_both(w, x)
    check_same(w, *out)
    if variant == "tiny":
        cpu = {k: v.cpu() for k, v in x.items()}
        Oref, Lref = so.ctx_encode(cpu["Qc"], cpu["Kc"], cpu["Vc"], w.b, w.b_a, w.scale)
        err = np.abs(out[4].double().numpy() - Oref)
        assert err.max() <= 1e-2 and err.mean() <= 1e-3
        assert np.abs(out[5].double().numpy() - Lref).max() <= 1e-3
    out[0].close()
    out[1].close()


def test_pageable_host_memory_is_still_correct():
    w = wl.get("tiny").with_(**VARIANTS["batch2"])
    x = {k: v.cuda() for k, v in wl.make_inputs(w, "cpu", with_decode=False).items()}
    out = encode_both(w, x, pinned=False)
    check_same(w, *out)
    out[0].close()
    out[1].close()


def test_host_encode_fills_the_fp8_copy():
    """With an FP8 cache the copy is quantised once every unit is done: codes
    and scales equal the device entry's."""
    w = wl.get("tiny").with_(**VARIANTS["d128-gqa8-batch3"])
    x = {k: v.cuda() for k, v in wl.make_inputs(w, "cpu", with_decode=False).items()}
    out = encode_both(w, x, kv_fp8=True)
    check_same(w, *out)
    ref, host = out[0], out[1]
    for i in range(ref.num_segments - 1):
        for a, b in zip(ref.segment_fp8_tensors(i), host.segment_fp8_tensors(i)):
            assert torch.equal(a, b), f"FP8 segment {i}"
    ref.close()
    host.close()


def test_full_size_8b_32k_host_encode_is_bit_exact():
    """The bench's end-to-end call on its own workload: 16 pipeline units."""
    w = wl.get("8b-32k")
    x = wl.make_inputs(w, "cuda", with_decode=False)
    out = encode_both(w, x)
    check_same(w, *out)
    # then phase 2 runs on the cache the host form filled
    cache = out[1]
    Oq, LSEq = cache.star_query_prefill(x["Qq"], x["Kq"], x["Vq"])
    Oq2, LSEq2 = out[0].star_query_prefill(x["Qq"], x["Kq"], x["Vq"])
    assert torch.equal(bits(Oq), bits(Oq2)) and torch.equal(LSEq, LSEq2)
    out[0].close()
    out[1].close()
