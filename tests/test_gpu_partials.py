"""GPU parity of the debug outputs: one partial per context segment and one
for the query region, and the fp32 merged rows.

Each (A_h, s_h) is compared with the oracle's local partial of that segment
alone ("Star Attention: Efficient LLM Inference over Long Sequences",
Phase 2 Step 3), the query region's with its causal visibility (Step 7);
the fp32 rows with the oracle's dense softmax, and their bf16 rounding with
the O the same call returns, bit for bit.  A generation step is the same
call with one row.
"""

import numpy as np
import pytest
import torch

from block_sparse_long_phase_b200 import workloads as wl
from oracle import star_oracle as so

pytestmark = pytest.mark.gpu

MAX_ABS, MEAN_ABS, LSE_ABS = 1e-2, 1e-3, 1e-3

VARIANTS = {
    "tiny": {},
    "ragged-last-block": dict(L=1000, lq=11, T=3),
    "d128-gqa8": dict(Hq=16, Hkv=2, D=128, L=600, b=256, b_a=256, lq=7, T=3),
    "batch2-many-blocks": dict(B=2, L=700, b=100, b_a=100, lq=9, T=2),
    "max-blocks": dict(L=191 * 16, b=16, b_a=16, lq=3, T=1),     # 191 segments: the chunk table is full
}


def close(got, ref, what, max_abs=MAX_ABS, mean_abs=MEAN_ABS):
    g = got.double().cpu().numpy()
    assert np.isfinite(g).all(), what
    err = np.abs(g - ref)
    assert err.max() <= max_abs, f"{what}: max-abs {err.max():.3e}"
    assert err.mean() <= mean_abs, f"{what}: mean-abs {err.mean():.3e}"


def oracle_partials(q_rows, segs, qk, qv, visible, scale, G):
    """[n+1, B, Hq, R, D] and [n+1, B, Hq, R] from the oracle's local partials."""
    Bn, Hq, R, D = q_rows.shape
    P = len(segs) + 1
    A = np.zeros((P, Bn, Hq, R, D))
    S = np.zeros((P, Bn, Hq, R))
    qmask = np.arange(qk.shape[2])[None, :] < np.asarray(visible)[:, None]
    for bi in range(Bn):
        for h in range(Hq):
            g = h // G
            for p, seg in enumerate(segs):
                A[p, bi, h], S[p, bi, h] = so.local_partial(q_rows[bi, h], seg[2][bi, g], seg[3][bi, g], scale)
            A[P - 1, bi, h], S[P - 1, bi, h] = so.local_partial(q_rows[bi, h], qk[bi, g], qv[bi, g], scale, qmask)
    return A, S


def check_call(got, q_rows, segs, qk, qv, visible, w, what):
    O, LSE, Ah, sh, O32 = got
    A_ref, S_ref = oracle_partials(q_rows, segs, qk, qv, visible, w.scale, w.Hq // w.Hkv)
    assert Ah.shape == A_ref.shape and sh.shape == S_ref.shape
    close(Ah, A_ref, f"{what}: A_h")
    lerr = np.abs(sh.double().cpu().numpy() - S_ref)
    assert lerr.max() <= LSE_ABS, f"{what}: s_h max-abs {lerr.max():.3e}"
    O_ref, L_ref = so.lse_merge(A_ref.reshape(A_ref.shape[0], -1, w.D), S_ref.reshape(S_ref.shape[0], -1))
    close(O32, O_ref.reshape(O32.shape), f"{what}: O32")
    close(O, O_ref.reshape(O.shape), f"{what}: O")
    assert np.abs(LSE.double().cpu().numpy() - L_ref.reshape(LSE.shape)).max() <= LSE_ABS
    # O is the bf16 rounding of the fp32 rows, bit for bit
    assert torch.equal(O32.to(torch.bfloat16).view(torch.int16), O.view(torch.int16)), f"{what}: O != bf16(O32)"


@pytest.mark.parametrize("variant", list(VARIANTS))
def test_per_segment_partials_match_the_oracle(variant):
    from block_sparse_long_phase_b200 import StarCache
    w = wl.get("tiny").with_(**VARIANTS[variant])
    cpu = wl.make_inputs(w, "cpu")
    x = {k: v.cuda() for k, v in cpu.items()}
    cache = StarCache(w.B, w.Hq, w.Hkv, w.D, w.L, w.b, w.b_a, w.lq + w.T, w.scale)
    cache.star_ctx_encode(x["Qc"], x["Kc"], x["Vc"])
    got = cache.star_query_prefill_partials(x["Qq"], x["Kq"], x["Vq"])
    steps = [cache.star_query_prefill_partials(x["qd"][t], x["kd"][t], x["vd"][t]) for t in range(w.T)]
    torch.cuda.synchronize()
    assert cache.device_error() == 0
    assert cache.q_len == w.lq + w.T
    segs = so.cache_segments(cpu["Kc"], cpu["Vc"], w.b)
    region = np.zeros((w.B, w.Hkv, w.lq + w.T, w.D))
    _, _, qk, qv = so.query_prefill(cpu["Qq"], cpu["Kq"], cpu["Vq"], segs, region, region, 0, w.scale)
    check_call(got, cpu["Qq"].double().numpy(), segs, qk, qv, np.arange(w.lq) + 1, w, f"{variant} prefill")
    for t in range(w.T):
        _, _, qk, qv = so.decode_step(cpu["qd"][t], cpu["kd"][t], cpu["vd"][t], segs, qk, qv, w.lq + t, w.scale)
        check_call(steps[t], cpu["qd"][t].double().numpy(), segs, qk, qv, np.array([w.lq + t + 1]), w,
                   f"{variant} step {t}")
    cache.close()


def test_partials_form_agrees_with_the_fast_path():
    """The per-segment form and the normal chunked prefill give the same rows
    within the output tolerance, and both append the same query region."""
    from block_sparse_long_phase_b200 import StarCache
    w = wl.get("tiny").with_(**VARIANTS["d128-gqa8"])
    x = wl.make_inputs(w, "cuda")
    out = []
    for debug in (False, True):
        cache = StarCache(w.B, w.Hq, w.Hkv, w.D, w.L, w.b, w.b_a, w.lq + w.T, w.scale)
        cache.star_ctx_encode(x["Qc"], x["Kc"], x["Vc"])
        if debug:
            O, LSE = cache.star_query_prefill_partials(x["Qq"], x["Kq"], x["Vq"])[:2]
        else:
            O, LSE = cache.star_query_prefill(x["Qq"], x["Kq"], x["Vq"])
        k, v, _ = cache.segment_tensors(cache.num_segments - 1)
        out.append((O.double(), LSE.double(), k[:, :, :w.lq].clone(), v[:, :, :w.lq].clone()))
        cache.close()
    (O1, L1, k1, v1), (O2, L2, k2, v2) = out
    assert (O1 - O2).abs().max().item() <= MAX_ABS and (L1 - L2).abs().max().item() <= LSE_ABS
    assert torch.equal(k1.view(torch.int16), k2.view(torch.int16))
    assert torch.equal(v1.view(torch.int16), v2.view(torch.int16))


# ---------------------------------------------------------------------------
# The decode kernel's own partials: one per piece of cached rows a CTA folds.
# ---------------------------------------------------------------------------
DECODE_VARIANTS = {
    "tiny": {},
    "ragged-anchor-shorter": dict(L=1000, b=256, b_a=100, lq=11, T=2),
    # 32 (batch, kv head) pairs of about 100 rows on a few CTAs: spans cross pairs
    "many-heads-short": dict(B=4, Hq=16, Hkv=8, D=64, L=96, b=32, b_a=32, lq=5, T=2),
    "8b-32k": None,
}


def check_decode_parts(parts, x_cpu, t, segs, qk, qv, w, what):
    """Every listed part against the oracle's local partial over its rows; the
    parts of each (batch, kv head) tile its cached rows exactly; their merge,
    with the step's own token as one more part, gives o and lse."""
    o, lse, Ah, sh, spans = parts
    G = w.Hq // w.Hkv
    rpb = w.L + w.lq + t                         # rows cached before the step
    A = Ah.double().cpu().numpy()
    S = sh.double().cpu().numpy()
    q = x_cpu["qd"][t].double().numpy()
    for bg in range(w.B * w.Hkv):
        bi, g = divmod(bg, w.Hkv)
        idx = np.nonzero(spans[:, 0] == bg)[0]
        assert len(idx) >= 1, f"{what}: no part for pair {bg}"
        rng_ = spans[idx, 1:]
        assert rng_[0, 0] == 0 and rng_[-1, 1] == rpb and np.all(rng_[1:, 0] == rng_[:-1, 1]), \
            f"{what}: parts of pair {bg} do not tile its {rpb} rows"
        kc = np.concatenate([so._f64(s[2][bi, g]) for s in segs] + [qk[bi, g, :w.lq + t]], axis=0)
        vc = np.concatenate([so._f64(s[3][bi, g]) for s in segs] + [qv[bi, g, :w.lq + t]], axis=0)
        qh = q[bi, g * G:(g + 1) * G, 0]
        parts_a, parts_s = [], []
        for p, (x0, x1) in zip(idx, rng_):
            a_ref, s_ref = so.local_partial(qh, kc[x0:x1], vc[x0:x1], w.scale)
            err = np.abs(A[p] - a_ref)
            assert err.max() <= MAX_ABS and err.mean() <= MEAN_ABS, f"{what}: part {p} A_h max {err.max():.3e}"
            assert np.abs(S[p] - s_ref).max() <= LSE_ABS, f"{what}: part {p} s_h"
            parts_a.append(A[p])
            parts_s.append(S[p])
        # the token itself: s = scale q.k_new, A = v_new
        kn, vn = qk[bi, g, w.lq + t], qv[bi, g, w.lq + t]
        parts_a.append(np.repeat(vn[None], G, axis=0))
        parts_s.append(w.scale * (qh @ kn))
        m_a, m_s = so.lse_merge(np.stack(parts_a), np.stack(parts_s))
        og = o[bi, g * G:(g + 1) * G, 0].double().cpu().numpy()
        assert np.abs(og - m_a).max() <= MAX_ABS, f"{what}: merge of the parts != o"
        assert np.abs(lse[bi, g * G:(g + 1) * G].double().cpu().numpy() - m_s).max() <= LSE_ABS


@pytest.mark.parametrize("variant", list(DECODE_VARIANTS))
def test_decode_kernel_partials_match_the_oracle(variant):
    from block_sparse_long_phase_b200 import StarCache
    if DECODE_VARIANTS[variant] is None:
        w = wl.get(variant).with_(T=2)
        x = wl.make_inputs(w, "cuda")
        cpu = {k: v.cpu() for k, v in x.items() if k != "Qc"}
    else:
        w = wl.get("tiny").with_(**DECODE_VARIANTS[variant])
        cpu = wl.make_inputs(w, "cpu")
        x = {k: v.cuda() for k, v in cpu.items()}
    cache = StarCache(w.B, w.Hq, w.Hkv, w.D, w.L, w.b, w.b_a, w.lq + w.T, w.scale)
    cache.star_ctx_encode(x["Qc"], x["Kc"], x["Vc"])
    cache.star_query_prefill(x["Qq"], x["Kq"], x["Vq"])
    got = []
    for t in range(w.T):
        got.append(cache.star_decode_step_partials(x["qd"][t], x["kd"][t], x["vd"][t]))
    torch.cuda.synchronize()
    assert cache.device_error() == 0
    segs = so.cache_segments(cpu["Kc"], cpu["Vc"], w.b)
    qk = np.zeros((w.B, w.Hkv, w.lq + w.T, w.D))
    qv = np.zeros_like(qk)
    qk[:, :, :w.lq] = cpu["Kq"].double().numpy()
    qv[:, :, :w.lq] = cpu["Vq"].double().numpy()
    for t in range(w.T):
        qk[:, :, w.lq + t] = cpu["kd"][t][:, :, 0].double().numpy()
        qv[:, :, w.lq + t] = cpu["vd"][t][:, :, 0].double().numpy()
        check_decode_parts(got[t], cpu, t, segs, qk, qv, w, f"{variant} step {t}")
        if variant == "8b-32k":
            assert len(got[t][4]) > 2 * w.B * w.Hkv          # several CTAs per (batch, kv head)
    cache.close()
