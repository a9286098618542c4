"""Thin PyTorch binding of libstar: argument marshalling only.

Every step of the path runs in libstar's kernels; this module checks tensor
shapes and dtypes, allocates outputs with torch (device memory is PyTorch's),
and passes raw pointers and torch's current CUDA stream through the C ABI.
The names follow the C entry points.
"""

from __future__ import annotations

import ctypes
from dataclasses import dataclass

import torch

from . import _abi


# Rotary base of the Llama 3 family (no frequency rescaling).
ROPE_THETA = 500000.0


def _ptr(t: torch.Tensor) -> ctypes.c_void_p:
    return ctypes.c_void_p(t.data_ptr())


def _stream(device) -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _need(t: torch.Tensor, shape, dtype, name):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (libstar has no CPU path)")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


@dataclass
class Segment:
    k: int          # device pointer
    v: int
    start: int
    len: int
    cap: int


class StarCache:
    """A Star Attention KV cache: per-block context segments + query region.

    Wraps ``star_cache_create``; the cache lives on the current CUDA device.
    """

    def __init__(self, B, Hq, Hkv, D, L, block, anchor, q_cap, scale=0.0, kv_fp8=False):
        if not torch.cuda.is_available():
            raise RuntimeError("libstar needs a CUDA device; there is no CPU fallback")
        self.lib = _abi.load()
        self.params = _abi.StarParams(B, Hq, Hkv, D, L, block, anchor, q_cap, float(scale),
                                      int(bool(kv_fp8)))
        self.device = torch.device("cuda", torch.cuda.current_device())
        h = ctypes.c_void_p()
        _abi.check(self.lib.star_cache_create(ctypes.byref(self.params), ctypes.byref(h)))
        self.handle = h
        self.B, self.Hq, self.Hkv, self.D, self.L = B, Hq, Hkv, D, L
        self.block, self.anchor, self.q_cap = block, anchor, q_cap
        self.kv_fp8 = bool(kv_fp8)

    # -- lifetime ------------------------------------------------------------
    def close(self):
        if getattr(self, "handle", None) is not None and self.handle.value:
            _abi.check(self.lib.star_cache_destroy(self.handle))
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.close()

    # -- introspection -------------------------------------------------------
    @property
    def num_segments(self) -> int:
        return self.lib.star_cache_num_segments(self.handle)

    def segment(self, i: int) -> Segment:
        k, v = ctypes.c_void_p(), ctypes.c_void_p()
        s, n, c = ctypes.c_longlong(), ctypes.c_longlong(), ctypes.c_longlong()
        _abi.check(self.lib.star_cache_segment(self.handle, i, ctypes.byref(k), ctypes.byref(v),
                                               ctypes.byref(s), ctypes.byref(n), ctypes.byref(c)))
        return Segment(k.value, v.value, s.value, n.value, c.value)

    def segment_tensors(self, i: int):
        """(K, V) views of segment ``i`` as bf16 tensors [B, Hkv, cap, D]."""
        seg = self.segment(i)
        n = self.B * self.Hkv * seg.cap * self.D
        out = []
        for p in (seg.k, seg.v):
            t = _tensor_from_ptr(p, n, self.device).view(self.B, self.Hkv, seg.cap, self.D)
            out.append(t)
        return out[0], out[1], seg

    def segment_fp8_tensors(self, i: int):
        """FP8 copy of segment ``i`` (``kv_fp8`` caches; ``i = num_segments - 1`` is
        the query region): E4M3 codes of K and V as uint8 [B, Hkv, cap, D] and
        their float32 row scales [B, Hkv, cap]."""
        k8, v8 = ctypes.c_void_p(), ctypes.c_void_p()
        ks, vs = ctypes.POINTER(ctypes.c_float)(), ctypes.POINTER(ctypes.c_float)()
        _abi.check(self.lib.star_cache_segment_fp8(self.handle, i, ctypes.byref(k8), ctypes.byref(v8),
                                                   ctypes.byref(ks), ctypes.byref(vs)))
        n = self.segment(i).cap
        shape = (self.B, self.Hkv, n)
        codes = [_view_from_ptr(p, self.B * self.Hkv * n * self.D, "|u1", self.device)
                 .view(*shape, self.D) for p in (k8.value, v8.value)]
        scales = [_view_from_ptr(ctypes.cast(p, ctypes.c_void_p).value, self.B * self.Hkv * n, "<f4",
                                 self.device).view(*shape) for p in (ks, vs)]
        return codes[0], codes[1], scales[0], scales[1]

    def device_error(self) -> int:
        """Reads and clears the device error word (non-zero: a bounded wait gave up)."""
        f = ctypes.c_int()
        _abi.check(self.lib.star_cache_device_error(self.handle, ctypes.byref(f)))
        return f.value

    def check_guards(self):
        """(-1, "") if every canary guard of the cache is intact, else (index of
        the first overwritten guard, which part it follows)."""
        f = ctypes.c_int()
        _abi.check(self.lib.star_cache_check_guards(self.handle, ctypes.byref(f)))
        return f.value, (self.lib.star_last_error().decode() if f.value >= 0 else "")

    @property
    def q_len(self) -> int:
        return self.segment(self.num_segments - 1).len

    def reset_query(self):
        _abi.check(self.lib.star_cache_reset_query(self.handle))

    # -- the hot path --------------------------------------------------------
    def star_ctx_encode(self, Q, K, V, O=None, LSE=None, Ka=None):
        """Phase 1.  ``Ka`` (optional, from ``star_anchor_keys``): per-block anchor keys."""
        B, Hq, Hkv, D, L = self.B, self.Hq, self.Hkv, self.D, self.L
        _need(Q, (B, Hq, L, D), torch.bfloat16, "Q")
        _need(K, (B, Hkv, L, D), torch.bfloat16, "K")
        _need(V, (B, Hkv, L, D), torch.bfloat16, "V")
        if Ka is not None:
            _need(Ka, (self.num_segments - 2, B, Hkv, self.anchor, D), torch.bfloat16, "Ka")
        if O is None:
            O = torch.empty((B, Hq, L, D), dtype=torch.bfloat16, device=Q.device)
        if LSE is None:
            LSE = torch.empty((B, Hq, L), dtype=torch.float32, device=Q.device)
        _need(O, (B, Hq, L, D), torch.bfloat16, "O")
        _need(LSE, (B, Hq, L), torch.float32, "LSE")
        _abi.check(self.lib.star_ctx_encode_anchored(self.handle, _ptr(Q), _ptr(K), _ptr(V),
                                                     _ptr(Ka) if Ka is not None else None, _ptr(O),
                                                     _ptr(LSE), _stream(Q.device)))
        return O, LSE

    def star_ctx_encode_after_anchor(self, Q, K, V, Ka, Va, O=None, LSE=None):
        """Phase 1 of blocks that all follow an anchor held outside this
        context: every block, block 0 included, attends to ``Ka``, ``Va``
        [B, Hkv, anchor, D] bf16 and causally to itself."""
        B, Hq, Hkv, D, L = self.B, self.Hq, self.Hkv, self.D, self.L
        _need(Q, (B, Hq, L, D), torch.bfloat16, "Q")
        _need(K, (B, Hkv, L, D), torch.bfloat16, "K")
        _need(V, (B, Hkv, L, D), torch.bfloat16, "V")
        if self.anchor > 0:
            _need(Ka, (B, Hkv, self.anchor, D), torch.bfloat16, "Ka")
            _need(Va, (B, Hkv, self.anchor, D), torch.bfloat16, "Va")
        if O is None:
            O = torch.empty((B, Hq, L, D), dtype=torch.bfloat16, device=Q.device)
        if LSE is None:
            LSE = torch.empty((B, Hq, L), dtype=torch.float32, device=Q.device)
        _need(O, (B, Hq, L, D), torch.bfloat16, "O")
        _need(LSE, (B, Hq, L), torch.float32, "LSE")
        _abi.check(self.lib.star_ctx_encode_after_anchor(
            self.handle, _ptr(Q), _ptr(K), _ptr(V), _ptr(Ka) if self.anchor > 0 else None,
            _ptr(Va) if self.anchor > 0 else None, _ptr(O), _ptr(LSE), _stream(Q.device)))
        return O, LSE

    def star_ctx_encode_fp32(self, Q, K, V, O=None, LSE=None, O32=None):
        """Debug form of phase 1: also returns O32 [B, Hq, L, D] float32, the
        rows before their bf16 rounding.  Returns (O, LSE, O32)."""
        B, Hq, Hkv, D, L = self.B, self.Hq, self.Hkv, self.D, self.L
        _need(Q, (B, Hq, L, D), torch.bfloat16, "Q")
        _need(K, (B, Hkv, L, D), torch.bfloat16, "K")
        _need(V, (B, Hkv, L, D), torch.bfloat16, "V")
        if O is None:
            O = torch.empty((B, Hq, L, D), dtype=torch.bfloat16, device=Q.device)
        if LSE is None:
            LSE = torch.empty((B, Hq, L), dtype=torch.float32, device=Q.device)
        if O32 is None:
            O32 = torch.empty((B, Hq, L, D), dtype=torch.float32, device=Q.device)
        _need(O, (B, Hq, L, D), torch.bfloat16, "O")
        _need(LSE, (B, Hq, L), torch.float32, "LSE")
        _need(O32, (B, Hq, L, D), torch.float32, "O32")
        _abi.check(self.lib.star_ctx_encode_fp32(self.handle, _ptr(Q), _ptr(K), _ptr(V), _ptr(O), _ptr(LSE),
                                                 _ptr(O32), _stream(Q.device)))
        return O, LSE, O32

    def star_ctx_encode_host(self, hQ, hK, hV, hO=None, hLSE=None, staging=None):
        """Phase 1 from host tensors: the copies in and out overlap the encoding.

        ``hQ``, ``hK``, ``hV``: CPU bf16 tensors (pinned for overlap) shaped as
        for :meth:`star_ctx_encode`; ``hO``, ``hLSE``: CPU outputs (pinned ones
        are allocated if None).  ``staging``: optional dict of device tensors
        ``Q, K, V, O, LSE`` reused between calls (allocated if None).
        Returns ``(hO, hLSE, staging)``; the host outputs are complete once the
        current stream reaches this point.
        """
        B, Hq, Hkv, D, L = self.B, self.Hq, self.Hkv, self.D, self.L
        shapes = {"Q": (B, Hq, L, D), "K": (B, Hkv, L, D), "V": (B, Hkv, L, D),
                  "O": (B, Hq, L, D), "LSE": (B, Hq, L)}
        for name, t in (("hQ", hQ), ("hK", hK), ("hV", hV)):
            if not isinstance(t, torch.Tensor) or t.is_cuda or t.dtype != torch.bfloat16 \
                    or tuple(t.shape) != shapes[name[1:]] or not t.is_contiguous():
                raise ValueError(f"{name} must be a contiguous CPU bf16 tensor of shape {shapes[name[1:]]}")
        if hO is None:
            hO = torch.empty(shapes["O"], dtype=torch.bfloat16).pin_memory()
        if hLSE is None:
            hLSE = torch.empty(shapes["LSE"], dtype=torch.float32).pin_memory()
        for name, t, dt in (("hO", hO, torch.bfloat16), ("hLSE", hLSE, torch.float32)):
            if t.is_cuda or t.dtype != dt or tuple(t.shape) != shapes[name[1:]] or not t.is_contiguous():
                raise ValueError(f"{name} must be a contiguous CPU {dt} tensor of shape {shapes[name[1:]]}")
        if staging is None:
            staging = {k: torch.empty(v, dtype=torch.float32 if k == "LSE" else torch.bfloat16,
                                      device=self.device) for k, v in shapes.items()}
        for k, v in shapes.items():
            _need(staging[k], v, torch.float32 if k == "LSE" else torch.bfloat16, k)
        _abi.check(self.lib.star_ctx_encode_host(
            self.handle, hQ.data_ptr(), hK.data_ptr(), hV.data_ptr(), hO.data_ptr(), hLSE.data_ptr(),
            *(_ptr(staging[k]) for k in ("Q", "K", "V", "O", "LSE")), _stream(self.device)))
        return hO, hLSE, staging

    def star_anchor_keys(self, K, anchor="first", theta=ROPE_THETA, Ka=None):
        """Anchor keys of blocks 1..n-1 from un-rotated K [B, Hkv, L, D]:
        ``anchor`` = "first" (IDs 0..b_a-1), "previous" (the b_a positions before
        each block) or an int32 CUDA tensor [n-1, b_a] of IDs.  Returns Ka
        [n-1, B, Hkv, b_a, D] bf16."""
        B, Hkv, D, L = self.B, self.Hkv, self.D, self.L
        _need(K, (B, Hkv, L, D), torch.bfloat16, "K")
        nb = self.num_segments - 1
        if Ka is None:
            Ka = torch.empty((max(nb - 1, 0), B, Hkv, self.anchor, D), dtype=torch.bfloat16, device=K.device)
        pos = None
        if isinstance(anchor, str):
            mode = {"first": 0, "previous": 1}[anchor]
        else:
            mode = 2
            pos = anchor
            _need(pos, (nb - 1, self.anchor), torch.int32, "anchor positions")
        _abi.check(self.lib.star_anchor_keys(self.handle, mode, _ptr(pos) if pos is not None else None,
                                             float(theta), _ptr(K), _ptr(Ka) if Ka.numel() else None,
                                             _stream(K.device)))
        return Ka

    def star_ctx_encode_rope(self, Q, K, V, anchor="first", theta=ROPE_THETA, O=None, LSE=None):
        """Phase 1 on un-rotated Q, K: rotates them at positions 0..L-1, builds the
        anchor keys of the chosen position-ID variant (none needed for "first"),
        encodes.  Returns (O, LSE)."""
        Qr = star_rope(Q, theta=theta)
        Kr = star_rope(K, theta=theta)
        Ka = None if (isinstance(anchor, str) and anchor == "first") else self.star_anchor_keys(K, anchor, theta)
        return self.star_ctx_encode(Qr, Kr, V, O, LSE, Ka=Ka)

    def star_query_prefill_rope(self, Q, K, V, theta=ROPE_THETA, O=None, LSE=None):
        """Query prefill on un-rotated Q, K: query row r sits at position L + q_len + r."""
        p0 = self.L + self.q_len
        return self.star_query_prefill(star_rope(Q, pos0=p0, theta=theta), star_rope(K, pos0=p0, theta=theta),
                                       V, O, LSE)

    def star_decode_step_rope(self, q, k, v, theta=ROPE_THETA, o=None, lse=None):
        """Decode step on un-rotated q, k: the token sits at position L + q_len."""
        p0 = self.L + self.q_len
        return self.star_decode_step(star_rope(q, pos0=p0, theta=theta), star_rope(k, pos0=p0, theta=theta),
                                     v, o, lse)

    def star_query_prefill(self, Q, K, V, O=None, LSE=None):
        B, Hq, Hkv, D = self.B, self.Hq, self.Hkv, self.D
        lq = Q.shape[2]
        _need(Q, (B, Hq, lq, D), torch.bfloat16, "Q")
        _need(K, (B, Hkv, lq, D), torch.bfloat16, "K")
        _need(V, (B, Hkv, lq, D), torch.bfloat16, "V")
        if O is None:
            O = torch.empty((B, Hq, lq, D), dtype=torch.bfloat16, device=Q.device)
        if LSE is None:
            LSE = torch.empty((B, Hq, lq), dtype=torch.float32, device=Q.device)
        _need(O, (B, Hq, lq, D), torch.bfloat16, "O")
        _need(LSE, (B, Hq, lq), torch.float32, "LSE")
        _abi.check(self.lib.star_query_prefill(self.handle, lq, _ptr(Q), _ptr(K), _ptr(V),
                                               _ptr(O), _ptr(LSE), _stream(Q.device)))
        return O, LSE

    def star_query_prefill_partials(self, Q, K, V, fp32_out=True):
        """Debug form of :meth:`star_query_prefill`: one partial per context
        segment plus one for the query region, returned with the outputs.

        Returns ``(O, LSE, Ah, sh, O32)``: Ah [n+1, B, Hq, lq, D] and sh
        [n+1, B, Hq, lq] float32 (part n is the query region), O32 the merged
        rows in float32 (None unless ``fp32_out``).  With lq = 1 it is a
        generation step on the bf16 cache.
        """
        B, Hq, Hkv, D = self.B, self.Hq, self.Hkv, self.D
        lq = Q.shape[2]
        _need(Q, (B, Hq, lq, D), torch.bfloat16, "Q")
        _need(K, (B, Hkv, lq, D), torch.bfloat16, "K")
        _need(V, (B, Hkv, lq, D), torch.bfloat16, "V")
        P = self.num_segments
        dev = Q.device
        O = torch.empty((B, Hq, lq, D), dtype=torch.bfloat16, device=dev)
        LSE = torch.empty((B, Hq, lq), dtype=torch.float32, device=dev)
        Ah = torch.empty((P, B, Hq, lq, D), dtype=torch.float32, device=dev)
        sh = torch.empty((P, B, Hq, lq), dtype=torch.float32, device=dev)
        O32 = torch.empty((B, Hq, lq, D), dtype=torch.float32, device=dev) if fp32_out else None
        _abi.check(self.lib.star_query_prefill_partials(
            self.handle, lq, _ptr(Q), _ptr(K), _ptr(V), _ptr(O), _ptr(LSE), _ptr(Ah), _ptr(sh),
            _ptr(O32) if O32 is not None else None, _stream(dev)))
        return O, LSE, Ah, sh, O32

    def star_decode_step(self, q, k, v, o=None, lse=None):
        B, Hq, Hkv, D = self.B, self.Hq, self.Hkv, self.D
        _need(q, (B, Hq, 1, D), torch.bfloat16, "q")
        _need(k, (B, Hkv, 1, D), torch.bfloat16, "k")
        _need(v, (B, Hkv, 1, D), torch.bfloat16, "v")
        if o is None:
            o = torch.empty((B, Hq, 1, D), dtype=torch.bfloat16, device=q.device)
        if lse is None:
            lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
        _need(o, (B, Hq, 1, D), torch.bfloat16, "o")
        _need(lse, (B, Hq), torch.float32, "lse")
        _abi.check(self.lib.star_decode_step(self.handle, _ptr(q), _ptr(k), _ptr(v), _ptr(o),
                                             _ptr(lse), _stream(q.device)))
        return o, lse


    def star_partial_attend(self, Q, first_seg, n_seg, K=None, V=None):
        """Phase-2 partial of rows Q [B, Hq, lq, D] over context segments
        [first_seg, first_seg + n_seg) and, when K and V are given, the query
        region after appending them.  Returns (A [B, Hq, lq, D], s [B, Hq, lq])
        float32."""
        B, Hq, Hkv, D = self.B, self.Hq, self.Hkv, self.D
        lq = Q.shape[2]
        _need(Q, (B, Hq, lq, D), torch.bfloat16, "Q")
        with_query = K is not None
        if with_query:
            _need(K, (B, Hkv, lq, D), torch.bfloat16, "K")
            _need(V, (B, Hkv, lq, D), torch.bfloat16, "V")
        A = torch.empty((B, Hq, lq, D), dtype=torch.float32, device=Q.device)
        s = torch.empty((B, Hq, lq), dtype=torch.float32, device=Q.device)
        _abi.check(self.lib.star_partial_attend(
            self.handle, int(first_seg), int(n_seg), int(with_query), lq, _ptr(Q),
            _ptr(K) if with_query else None, _ptr(V) if with_query else None, _ptr(A), _ptr(s),
            _stream(Q.device)))
        return A, s

    def star_decode_step_partials(self, q, k, v):
        """Debug form of :meth:`star_decode_step` that also returns the decode
        kernel's own partials: ``(o, lse, Ah [P, G, D], sh [P, G], spans)``,
        ``spans`` an int64 array [P, 3] of (b*Hkv + kv head, first row, end
        row) over that kv head's cached rows (context, then query region)."""
        import numpy as np
        B, Hq, Hkv, D = self.B, self.Hq, self.Hkv, self.D
        _need(q, (B, Hq, 1, D), torch.bfloat16, "q")
        _need(k, (B, Hkv, 1, D), torch.bfloat16, "k")
        _need(v, (B, Hkv, 1, D), torch.bfloat16, "v")
        G = Hq // Hkv
        o = torch.empty((B, Hq, 1, D), dtype=torch.bfloat16, device=q.device)
        lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
        n = ctypes.c_int(0)
        cap = 4 * B * Hkv + 4 * torch.cuda.get_device_properties(q.device).multi_processor_count
        Ah = torch.empty((cap, G, D), dtype=torch.float32, device=q.device)
        sh = torch.empty((cap, G), dtype=torch.float32, device=q.device)
        spans = np.zeros((cap, 3), dtype=np.int64)
        _abi.check(self.lib.star_decode_step_partials(
            self.handle, _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(Ah), _ptr(sh),
            spans.ctypes.data_as(ctypes.POINTER(ctypes.c_longlong)), cap, ctypes.byref(n), _stream(q.device)))
        P = n.value
        return o, lse, Ah[:P], sh[:P], spans[:P]


def star_rope(x: torch.Tensor, positions=None, pos0=0, theta=ROPE_THETA, out=None):
    """Rotary embedding of x [B, H, L, D] bf16 (CUDA) at positions
    ``positions`` (int32 CUDA tensor [L]) or pos0 + t; ``out`` may be ``x``."""
    lib = _abi.load()
    B, H, L, D = x.shape
    _need(x, (B, H, L, D), torch.bfloat16, "x")
    if out is None:
        out = torch.empty_like(x)
    _need(out, (B, H, L, D), torch.bfloat16, "out")
    if positions is not None:
        _need(positions, (L,), torch.int32, "positions")
    _abi.check(lib.star_rope(B, H, L, D, float(theta), _ptr(positions) if positions is not None else None,
                             int(pos0), _ptr(x), _ptr(out), _stream(x.device)))
    return out


def star_lse_merge(A: torch.Tensor, s: torch.Tensor, out_A=None, out_s=None):
    """Merge partials A [P, R, D], s [P, R] (float32, CUDA) -> ([R, D], [R])."""
    lib = _abi.load()
    P, R, D = A.shape
    _need(A, (P, R, D), torch.float32, "A")
    _need(s, (P, R), torch.float32, "s")
    if out_A is None:
        out_A = torch.empty((R, D), dtype=torch.float32, device=A.device)
    if out_s is None:
        out_s = torch.empty((R,), dtype=torch.float32, device=A.device)
    _need(out_A, (R, D), torch.float32, "out_A")
    _need(out_s, (R,), torch.float32, "out_s")
    _abi.check(lib.star_lse_merge(P, R, D, _ptr(A), _ptr(s), _ptr(out_A), _ptr(out_s),
                                  _stream(A.device)))
    return out_A, out_s


def star_decode_step_noalloc(params, q_len, ctx_k, ctx_v, q_k, q_v, q, k, v, o=None, lse=None):
    """Decode step that allocates no device memory in libstar.

    For callers that cannot call the CUDA allocator while serving (a runtime
    that hands out all device memory from its own pool): the KV cache is the
    caller's tensors -- ``ctx_k``/``ctx_v`` in the segmented layout of
    ``star_cache_create`` (flat bf16, B*Hkv*L*D elements), ``q_k``/``q_v`` as
    [B, Hkv, q_cap, D] -- and the split-KV scratch is a static device array of
    the library.  ``params`` is a ``_abi.StarParams``; row ``q_len`` of the
    query region receives ``k``/``v``.  Calls that overlap on the GPU race on
    the shared scratch.
    """
    lib = _abi.load()
    B, Hq, Hkv, D = params.B, params.Hq, params.Hkv, params.D
    n_ctx = B * Hkv * params.L * D
    _need(ctx_k, (n_ctx,), torch.bfloat16, "ctx_k")
    _need(ctx_v, (n_ctx,), torch.bfloat16, "ctx_v")
    _need(q_k, (B, Hkv, params.q_cap, D), torch.bfloat16, "q_k")
    _need(q_v, (B, Hkv, params.q_cap, D), torch.bfloat16, "q_v")
    _need(q, (B, Hq, 1, D), torch.bfloat16, "q")
    _need(k, (B, Hkv, 1, D), torch.bfloat16, "k")
    _need(v, (B, Hkv, 1, D), torch.bfloat16, "v")
    if o is None:
        o = torch.empty((B, Hq, 1, D), dtype=torch.bfloat16, device=q.device)
    if lse is None:
        lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
    _need(o, (B, Hq, 1, D), torch.bfloat16, "o")
    _need(lse, (B, Hq), torch.float32, "lse")
    _abi.check(lib.star_decode_step_noalloc(ctypes.byref(params), q_len, _ptr(ctx_k), _ptr(ctx_v),
                                            _ptr(q_k), _ptr(q_v), _ptr(q), _ptr(k), _ptr(v),
                                            _ptr(o), _ptr(lse), _stream(q.device)))
    return o, lse


def star_lse_merge_bf16(A: torch.Tensor, s: torch.Tensor, out_O=None, out_s=None):
    """Merge partials A [P, R, D], s [P, R] (float32, CUDA) -> (O [R, D] bf16, s [R])."""
    lib = _abi.load()
    P, R, D = A.shape
    _need(A, (P, R, D), torch.float32, "A")
    _need(s, (P, R), torch.float32, "s")
    if out_O is None:
        out_O = torch.empty((R, D), dtype=torch.bfloat16, device=A.device)
    if out_s is None:
        out_s = torch.empty((R,), dtype=torch.float32, device=A.device)
    _need(out_O, (R, D), torch.bfloat16, "out_O")
    _need(out_s, (R,), torch.float32, "out_s")
    _abi.check(lib.star_lse_merge_bf16(P, R, D, _ptr(A), _ptr(s), _ptr(out_O), _ptr(out_s), _stream(A.device)))
    return out_O, out_s


def star_noalloc_device_error(device=None) -> int:
    """Reads and clears the error word of the no-alloc decode scratch on the
    current device, after the work queued on the current stream: non-zero if
    a step since the last read gave up a bounded wait (its outputs are invalid)."""
    lib = _abi.load()
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else device
    f = ctypes.c_int()
    _abi.check(lib.star_noalloc_device_error(ctypes.byref(f), _stream(dev)))
    return f.value


def _view_from_ptr(ptr: int, n_elems: int, typestr: str, device) -> torch.Tensor:
    """A flat view of ``n_elems`` elements of device memory owned by libstar."""

    class _CudaArray:
        def __init__(self):
            self.__cuda_array_interface__ = {
                "shape": (n_elems,), "typestr": typestr, "data": (ptr, False), "version": 3,
                "strides": None,
            }

    return torch.as_tensor(_CudaArray(), device=device)


def _tensor_from_ptr(ptr: int, n_elems: int, device) -> torch.Tensor:
    """A bf16 view of ``n_elems`` elements of device memory owned by libstar."""
    return _view_from_ptr(ptr, n_elems, "<u2", device).view(torch.bfloat16)
