"""The allocation-free decode entry point against the regular one.

star_decode_step_noalloc serves callers that may not call cudaMalloc while
they serve (a runtime that owns all device memory through its own pool): the
KV cache is the caller's memory and the split-KV scratch is a static array of
the library.  Here the caller's buffers are copies of a regular cache's
segments and query region; two decode steps in a row through each entry point
must agree within the tolerance of the parity tests.  This file is collected
last so a failure here leaves every other test already run.
"""

import numpy as np
import pytest
import torch

from block_sparse_long_phase_b200 import workloads as wl

pytestmark = pytest.mark.gpu

MAX_ABS = 1e-2
MEAN_ABS = 1e-3
LSE_ABS = 1e-3


@pytest.mark.parametrize("name,over", [("tiny", {}), ("8b-32k", dict(T=4))])
def test_noalloc_decode_matches_regular_entry_point(name, over):
    from block_sparse_long_phase_b200 import StarCache, _abi
    from block_sparse_long_phase_b200.api import star_decode_step_noalloc
    w = wl.get(name).with_(**over)
    dev = "cpu" if name == "tiny" else "cuda"
    x = {k: v.cuda() for k, v in wl.make_inputs(w, dev).items()}
    cache = StarCache(w.B, w.Hq, w.Hkv, w.D, w.L, w.b, w.b_a, w.lq + w.T, w.scale)
    cache.star_ctx_encode(x["Qc"], x["Kc"], x["Vc"])
    cache.star_query_prefill(x["Qq"], x["Kq"], x["Vq"])
    torch.cuda.synchronize()
    # the caller's own buffers: copies of the cache's segments and query region
    n_ctx = w.B * w.Hkv * w.L * w.D
    seg0k, seg0v, _ = cache.segment_tensors(0)
    ctx_k = torch.empty(n_ctx, dtype=torch.bfloat16, device="cuda")
    ctx_v = torch.empty(n_ctx, dtype=torch.bfloat16, device="cuda")
    from block_sparse_long_phase_b200.api import _tensor_from_ptr
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
    cache.close()


def test_noalloc_rejects_oversized_problems():
    from block_sparse_long_phase_b200 import _abi
    lib = _abi.load()
    p = _abi.StarParams(64, 128, 64, 128, 1024, 256, 256, 8, 0.0)   # B*Hkv = 4096 > 1024
    buf = torch.zeros(16, dtype=torch.bfloat16, device="cuda")
    ptr = buf.data_ptr()
    import ctypes
    rc = lib.star_decode_step_noalloc(ctypes.byref(p), 0, ptr, ptr, ptr, ptr, ptr, ptr, ptr, ptr,
                                      ptr, None)
    assert rc == _abi.STAR_EINVAL
    assert b"static decode scratch" in lib.star_last_error()
