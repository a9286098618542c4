"""GPU parity of the RoPE front end (NEXT-1): the rotation kernel, the anchor
keys of each position-ID variant, and phase 1 / prefill / decode on
un-rotated inputs, against the oracle.

Tolerances: a rotated element is rounded once to bf16, so the rotation is
checked at half a bf16 ulp of the result plus float32 evaluation error
(2^-8 relative, 1e-5 absolute per unit input).  Attention outputs use the
path's bar (max-abs 1e-2, mean-abs 1e-3, LSE 1e-3) against the oracle with
its rotated q, k rounded to bf16 -- the operands the attention kernels
take -- and against the unrounded oracle at three times that bar (LSE 1e-2:
rounding q and k moves a logit by about 2^-8 of its size).
"""

import numpy as np
import pytest
import torch

from block_sparse_long_phase_b200 import workloads as wl
from oracle import star_oracle as so

pytestmark = pytest.mark.gpu

THETA = 500000.0


def check_rotation(got, x, pos, theta=THETA):
    ref = so.rope(x.double().cpu().numpy(), pos, theta)
    g = got.double().cpu().numpy()
    bound = np.abs(ref) * 2 ** -8 + 1e-5 * (np.abs(x.double().cpu().numpy()).max() + 1)
    assert (np.abs(g - ref) <= bound).all(), f"max excess {(np.abs(g - ref) - bound).max():.3e}"


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("where", ["zero", "far", "given", "inplace"])
def test_rope_kernel(D, where):
    from block_sparse_long_phase_b200 import star_rope
    g = torch.Generator().manual_seed(D + len(where))
    B, H, L = 2, 3, 301
    x = (torch.randn(B, H, L, D, generator=g) * 3).to(torch.bfloat16).cuda()
    if where == "given":
        pos = torch.randint(0, 1 << 21, (L,), generator=g, dtype=torch.int32)
        y = star_rope(x, positions=pos.cuda())
        check_rotation(y, x, pos.numpy())
    elif where == "far":
        y = star_rope(x, pos0=1_048_000)
        check_rotation(y, x, 1_048_000 + np.arange(L))
    elif where == "inplace":
        x0 = x.clone()
        y = star_rope(x, pos0=17, out=x)
        assert y.data_ptr() == x.data_ptr()
        check_rotation(y, x0, 17 + np.arange(L))
    else:
        y = star_rope(x)
        check_rotation(y, x, np.arange(L))


def make_cache(w):
    from block_sparse_long_phase_b200 import StarCache
    return StarCache(w.B, w.Hq, w.Hkv, w.D, w.L, w.b, w.b_a, w.lq + w.T, w.scale)


def anchor_ids(mode, w, seed=7):
    n = len(so.block_table(w.L, w.b))
    if mode == "given":
        rng = np.random.default_rng(seed)
        given = np.stack([np.sort(rng.choice(i * w.b, size=w.b_a, replace=False)) for i in range(1, n)])
        return so.anchor_positions("given", n, w.b, w.b_a, given)
    return so.anchor_positions(mode, n, w.b, w.b_a)


@pytest.mark.parametrize("mode", ["first", "previous", "given"])
def test_anchor_keys(mode):
    w = wl.get("tiny").with_(D=128, Hq=8, Hkv=2, L=700, b=256, b_a=200)
    x = {k: v.cuda() for k, v in wl.make_inputs(w, "cpu").items()}
    cache = make_cache(w)
    ap = anchor_ids(mode, w)
    arg = mode if mode != "given" else torch.from_numpy(ap.astype(np.int32)).cuda()
    Ka = cache.star_anchor_keys(x["Kc"], arg, THETA)
    torch.cuda.synchronize()
    K = x["Kc"].cpu()
    for i in range(1, ap.shape[0] + 1):
        check_rotation(Ka[i - 1], K[:, :, :w.b_a], ap[i - 1])
    cache.close()


def assert_close(got, ref, lse_got, lse_ref, what, k=1.0, lse_tol=1e-3):
    g = got.detach().double().cpu().numpy()
    err = np.abs(g - ref)
    assert np.isfinite(g).all(), f"{what}: non-finite output"
    assert err.max() <= 1e-2 * k, f"{what}: max-abs {err.max():.3e}"
    assert err.mean() <= 1e-3 * k, f"{what}: mean-abs {err.mean():.3e}"
    lerr = np.abs(lse_got.detach().double().cpu().numpy() - lse_ref)
    assert lerr.max() <= lse_tol, f"{what}: LSE max-abs {lerr.max():.3e}"


VARIANTS = {
    "tiny": {},
    "ragged": dict(L=1000, b_a=100),
    "no-anchor": dict(b_a=0),
    "single-block": dict(b=1024, b_a=1024),
    "d128-gqa4": dict(Hq=8, Hkv=2, D=128, L=700, b=256, b_a=200),
}


@pytest.mark.parametrize("mode", ["first", "previous", "given"])
@pytest.mark.parametrize("variant", list(VARIANTS))
def test_phase1_with_rope(mode, variant):
    w = wl.get("tiny").with_(**VARIANTS[variant])
    x = {k: v.cuda() for k, v in wl.make_inputs(w, "cpu").items()}
    cache = make_cache(w)
    n = len(so.block_table(w.L, w.b))
    ap = anchor_ids(mode, w) if n > 1 and w.b_a > 0 else np.zeros((max(n - 1, 0), w.b_a), np.int64)
    arg = mode if mode != "given" else torch.from_numpy(ap.astype(np.int32)).cuda()
    O, LSE = cache.star_ctx_encode_rope(x["Qc"], x["Kc"], x["Vc"], anchor=arg, theta=THETA)
    torch.cuda.synchronize()
    assert cache.device_error() == 0
    cpu = {k: v.cpu() for k, v in x.items()}
    ref, lref = so.ctx_encode_rope(cpu["Qc"], cpu["Kc"], cpu["Vc"], w.b, w.b_a, w.scale, ap, THETA,
                                   rotated_bf16=True)
    assert_close(O, ref, LSE, lref, f"{variant} {mode}")
    ref, lref = so.ctx_encode_rope(cpu["Qc"], cpu["Kc"], cpu["Vc"], w.b, w.b_a, w.scale, ap, THETA)
    # against exact rotation: bf16 rounding of q and k (2^-9 relative each)
    # moves a logit by about 2^-8 of its size, the LSE as much
    assert_close(O, ref, LSE, lref, f"{variant} {mode} (unrounded oracle)", k=3.0, lse_tol=1e-2)
    # the cache holds each block's own K rotated at its own positions, once
    Kr = so.round_bf16(so.rope(cpu["Kc"], np.arange(w.L), THETA))
    for i, (s, m) in enumerate(so.block_table(w.L, w.b)):
        k, _, _ = cache.segment_tensors(i)
        assert np.abs(k.double().cpu().numpy() - Kr[:, :, s:s + m]).max() <= 2 ** -8 * np.abs(Kr).max()
    cache.close()


def test_prefill_and_decode_with_rope():
    """Query rows sit at positions L + r: rotate q, k there, attend to the
    rotated cache (rounded to bf16 as stored)."""
    w = wl.get("tiny").with_(D=128, Hq=8, Hkv=2, L=700, b=256, b_a=256, lq=9, T=4)
    x = {k: v.cuda() for k, v in wl.make_inputs(w, "cpu").items()}
    cache = make_cache(w)
    cache.star_ctx_encode_rope(x["Qc"], x["Kc"], x["Vc"], anchor="previous", theta=THETA)
    Oq, Lq = cache.star_query_prefill_rope(x["Qq"], x["Kq"], x["Vq"], theta=THETA)
    dec = [cache.star_decode_step_rope(x["qd"][t], x["kd"][t], x["vd"][t], theta=THETA) for t in range(w.T)]
    torch.cuda.synchronize()
    assert cache.device_error() == 0
    cpu = {k: v.cpu() for k, v in x.items()}
    rot = lambda a, p: so.round_bf16(so.rope(a, p, THETA))
    Kc = rot(cpu["Kc"], np.arange(w.L))
    segs = so.cache_segments(Kc, so._f64(cpu["Vc"]), w.b)
    qpos = w.L + np.arange(w.lq + w.T)
    Kreg = np.concatenate([cpu["Kq"].double().numpy()] + [cpu["kd"][t].double().numpy() for t in range(w.T)], axis=2)
    Vreg = np.concatenate([cpu["Vq"].double().numpy()] + [cpu["vd"][t].double().numpy() for t in range(w.T)], axis=2)
    Kreg = rot(Kreg, qpos)
    Qq = rot(cpu["Qq"], qpos[:w.lq])
    ref, lref = so.query_attend(Qq, segs, Kreg, Vreg, np.arange(1, w.lq + 1), w.scale)
    assert_close(Oq, ref, Lq, lref, "prefill")
    for t in range(w.T):
        q = rot(cpu["qd"][t], [w.L + w.lq + t])
        ref, lref = so.query_attend(q, segs, Kreg, Vreg, np.array([w.lq + t + 1]), w.scale)
        assert_close(dec[t][0], ref, dec[t][1], lref[:, :, 0], f"decode {t}")
    cache.close()


def test_phase1_with_rope_full_size_sampled():
    """8B-32K in the benchmark's launch configuration, previous-block anchor
    IDs: sampled rows of every block (first, last, tile edges) of two kv groups."""
    from block_sparse_long_phase_b200 import StarCache
    w = wl.get("8b-32k")
    rng = np.random.default_rng(w.seed + 3)
    x = wl.make_inputs(w, "cuda")
    cache = StarCache(w.B, w.Hq, w.Hkv, w.D, w.L, w.b, w.b_a, w.lq + w.T, w.scale)
    O, LSE = cache.star_ctx_encode_rope(x["Qc"], x["Kc"], x["Vc"], anchor="previous", theta=THETA)
    torch.cuda.synchronize()
    assert cache.device_error() == 0
    ap = anchor_ids("previous", w)
    rows = []
    for s, n in so.block_table(w.L, w.b):
        cand = {0, n - 1, 127, 128, n // 2} | set(rng.integers(0, n, 3).tolist())
        rows += [s + c for c in sorted(cand)]
    rows = np.array(rows)
    for g in (0, w.Hkv - 1):
        hs, gs = slice(g * w.G, (g + 1) * w.G), slice(g, g + 1)
        ref, lref = so.ctx_encode_rope(x["Qc"][:, hs].cpu(), x["Kc"][:, gs].cpu(), x["Vc"][:, gs].cpu(),
                                       w.b, w.b_a, w.scale, ap, THETA, rows=rows, rotated_bf16=True)
        assert_close(O[:, hs][:, :, rows], ref, LSE[:, hs][:, :, rows], lref, f"8b-32k previous kv{g}")
    cache.close()
