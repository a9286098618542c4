// C ABI of libstar: argument validation, the segmented KV cache, work plans
// and kernel launches.  Declarations and contracts: include/star_attention.h.
#include <cuda_runtime.h>
#include <math.h>
#include <stdarg.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <algorithm>
#include <vector>

#include "../../include/star_attention.h"
#include "star_internal.h"

using star::bf16;

struct star_cache {
  star_params p;
  star::CacheView view;
  star::Scratch scratch;
  long long q_len;          // query-region rows in use (host-side; calls are stream-ordered)
  int device;
  int num_sms;
  void* block;              // the one cudaMalloc holding everything below
  int4* ctx_work;           // phase-1 work list: L2-sized groups of blocks, longest tile first
  int n_ctx_work;
  star::DecodeMaps dmaps;   // TMA maps of the cache (built once)
  // star_ctx_encode_host: the same work cut into pipeline units, and the copy
  // streams and events, created on its first call
  std::vector<star::CtxUnit> units;
  int4* unit_work;
  cudaStream_t s_in = nullptr, s_out = nullptr, s_comp = nullptr;
  std::vector<cudaEvent_t> events;     // start, end, compute done, then (input ready, output ready) per unit
  // canary guard regions, one after each part of the allocation
  struct Guard {
    size_t off;
    const char* after;
  };
  std::vector<Guard> guards;
};

namespace {

thread_local char g_err[512] = "";

int fail(int code, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return code;
}

int cuda_fail(cudaError_t e, const char* what) {
  return fail(STAR_ECUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Canary guard after each part of a cache's allocation.
constexpr size_t kGuardBytes = 4096;
constexpr int kCanary = 0xA5;

// ---- phase-2 plans --------------------------------------------------------
// Prefill spans.  The call attends to the context rows [R0, R1) (R0 = s0 * b,
// R1 = min(s1 * b, L)) and, with the query, to the query region's len0 + lq
// rows, numbered from L on.  Those rows are cut into m spans of about equal
// length, boundaries at multiples of 128 rows from R0 (tiles stay full inside
// a segment), so that (batch x kv head) x (256-row pairs) x m is about one CTA
// per SM.  A span never holds rows the call does not attend to: when the
// context part stops short of L and the query region is attended, the region
// is a span of its own.
}  // namespace

star::PrefillPlan star::plan_prefill(const star::CacheView& v, int num_sms, int lq, long long len0, int s0, int s1,
                                     bool query) {
  if (s1 < 0) s1 = v.n_seg;
  star::PrefillPlan pl{};
  const long long R0 = (long long)s0 * v.b, R1 = std::min((long long)s1 * v.b, v.L);
  const long long ctx = std::max(0LL, R1 - R0), nq = query ? len0 + lq : 0;
  const long long bgp = (long long)v.B * v.Hkv * star::prefill_row_pairs(v, lq);
  long long m = std::max(1LL, (long long)num_sms / bgp);
  m = std::min<long long>(m, star::kMaxPrefillSpans);
  auto cut = [&](long long lo, long long n, long long parts) {   // rows [lo, lo + n) into parts spans
    parts = std::max(1LL, std::min(parts, n / 128));
    long long prev = 0;
    for (long long k = 1; k <= parts; ++k) {
      const long long e = k == parts ? n : (k * n / parts) / 128 * 128;
      pl.span[pl.n_spans++] = {(int)(lo + prev), (int)(lo + e)};
      prev = e;
    }
  };
  if (ctx > 0 && nq > 0 && R1 < v.L) {
    cut(R0, ctx, std::max(1LL, m - 1));
    cut(v.L, nq, 1);
  } else if (ctx > 0 && nq > 0) {
    // [R0, L) and the region are contiguous rows: one range
    const long long n = ctx + nq;
    long long parts = std::max(1LL, std::min(m, n / 128)), prev = 0;
    for (long long k = 1; k <= parts; ++k) {
      const long long e = k == parts ? n : (k * n / parts) / 128 * 128;
      pl.span[pl.n_spans++] = {(int)(R0 + prev), (int)(R0 + e)};
      prev = e;
    }
  } else if (ctx > 0) {
    cut(R0, ctx, m);
  } else if (nq > 0) {
    cut(v.L, nq, m);
  }
  return pl;
}

// One span per context segment and one for the query region: the partials
// are then exactly the per-segment (A_h, s_h) of the method.
star::PrefillPlan star::plan_prefill_per_segment(const star::CacheView& v, int lq, long long len0) {
  star::PrefillPlan pl{};
  for (int s = 0; s < v.n_seg; ++s) pl.span[s] = {(int)((long long)s * v.b), (int)((long long)s * v.b + star::seg_len(v, s))};
  pl.span[v.n_seg] = {(int)v.L, (int)(v.L + len0 + lq)};
  pl.n_spans = v.n_seg + 1;
  return pl;
}

namespace {

star::DecodePlan plan_decode(const star_cache* c, long long len0) {
  star::DecodePlan pl;
  pl = star::decode_plan(c->view, len0, c->num_sms);
  return pl;
}

int validate_params(const star_params* p) {
  if (!p) return fail(STAR_EINVAL, "params is NULL");
  if (p->B < 1 || p->Hq < 1 || p->Hkv < 1) return fail(STAR_EINVAL, "B, Hq, Hkv must be >= 1");
  if (p->Hq % p->Hkv) return fail(STAR_EINVAL, "Hq (%d) must be a multiple of Hkv (%d)", p->Hq, p->Hkv);
  if (p->D != 64 && p->D != 128) return fail(STAR_EUNSUPPORTED, "head dim %d not in {64, 128}", p->D);
  if (p->Hq / p->Hkv > 16) return fail(STAR_EUNSUPPORTED, "group size %d > 16", p->Hq / p->Hkv);
  if (p->L < 1) return fail(STAR_EINVAL, "context length must be >= 1");
  if (p->block < 1) return fail(STAR_EINVAL, "block size must be >= 1");
  if (p->anchor < 0 || p->anchor > p->block)
    return fail(STAR_EINVAL, "anchor %d must satisfy 0 <= b_a <= b (%d)", p->anchor, p->block);
  if (p->q_cap < 1) return fail(STAR_EINVAL, "q_cap must be >= 1");
  if (p->kv_fp8 != 0 && p->kv_fp8 != 1) return fail(STAR_EINVAL, "kv_fp8 must be 0 or 1");
  if (p->L + p->q_cap + 1 > 0x7fffffffLL) return fail(STAR_EINVAL, "L + q_cap too large");
  if ((long long)p->B * p->Hkv * (p->L + p->q_cap) >= 0x7fffffffLL)
    return fail(STAR_EUNSUPPORTED, "B * Hkv * (L + q_cap) cached rows must stay below 2^31");
  if ((p->L + p->block - 1) / p->block > star::kMaxPrefillSpans - 1)
    return fail(STAR_EUNSUPPORTED, "%lld blocks: at most %d", (p->L + p->block - 1) / p->block,
                star::kMaxPrefillSpans - 1);
  return STAR_OK;
}

// The cache geometry of `p` without device memory (host-side planning only).
star::CacheView host_view(const star_params* p) {
  star::CacheView v{};
  v.B = p->B; v.Hq = p->Hq; v.Hkv = p->Hkv; v.D = p->D; v.G = p->Hq / p->Hkv;
  v.L = p->L; v.b = p->block; v.b_a = p->anchor;
  v.n_seg = (int)((p->L + p->block - 1) / p->block);
  v.q_cap = p->q_cap;
  return v;
}

}  // namespace

namespace star {
int set_error(int code, const char* msg) {
  snprintf(g_err, sizeof(g_err), "%s", msg);
  return code;
}
int check_params(const star_params* p) { return validate_params(p); }
}  // namespace star

namespace {
// star_query_prefill and its debug form with per-segment partials.
int query_prefill(star_cache* c, int lq, const void* Q, const void* K, const void* V, void* O, float* LSE,
                  void* stream, bool per_segment, float* Ah, float* sh, float* O32) {
  if (!c) return fail(STAR_EINVAL, "cache is NULL");
  if (lq < 1) return fail(STAR_EINVAL, "lq must be >= 1");
  if (!Q || !K || !V || !O || !LSE) return fail(STAR_EINVAL, "NULL tensor pointer");
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O) || !aligned16(LSE))
    return fail(STAR_EINVAL, "tensor pointers must be 16-byte aligned");
  if (per_segment && (!Ah || !sh)) return fail(STAR_EINVAL, "NULL partials pointer");
  if (c->q_len + lq > c->view.q_cap)
    return fail(STAR_ENOSPC, "query region full: %lld + %d > q_cap %d", c->q_len, lq, c->view.q_cap);
  const star::PrefillPlan pl =
      per_segment ? star::plan_prefill_per_segment(c->view, lq, c->q_len)
                  : star::plan_prefill(c->view, c->num_sms, lq, c->q_len);
  cudaError_t e = star::launch_query_prefill_tc(
      c->view, c->dmaps, c->p.scale, lq, (int)c->q_len, static_cast<const bf16*>(Q),
      static_cast<const bf16*>(K), static_cast<const bf16*>(V), static_cast<bf16*>(O), LSE, pl,
      c->scratch, static_cast<cudaStream_t>(stream), O32, Ah, sh);
  if (e == cudaSuccess && c->view.qK8)
    e = star::launch_quantize_qregion_fp8(c->view, static_cast<const bf16*>(K), static_cast<const bf16*>(V),
                                          (int)c->q_len, lq, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "star_query_prefill launch");
  c->q_len += lq;
  return STAR_OK;
}
}  // namespace

extern "C" {

const char* star_last_error(void) { return g_err; }
const char* star_version(void) { return "libstar 0.2 (sm_100a)"; }

int star_cache_create(const star_params* p, star_cache** out) {
  if (!out) return fail(STAR_EINVAL, "out is NULL");
  *out = nullptr;
  int rc = validate_params(p);
  if (rc) return rc;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  cudaDeviceProp prop;
  e = cudaGetDeviceProperties(&prop, dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDeviceProperties");
  if (prop.major != 10) return fail(STAR_EUNSUPPORTED, "device is sm_%d%d, need sm_100", prop.major, prop.minor);

  star_cache* c = new star_cache();
  c->p = *p;
  if (c->p.scale <= 0.f) c->p.scale = 1.0f / sqrtf((float)p->D);
  c->device = dev;
  c->num_sms = prop.multiProcessorCount;
  star::CacheView& v = c->view;
  v.B = p->B; v.Hq = p->Hq; v.Hkv = p->Hkv; v.D = p->D; v.G = p->Hq / p->Hkv;
  v.L = p->L; v.b = p->block; v.b_a = p->anchor;
  v.n_seg = (int)((p->L + p->block - 1) / p->block);
  v.q_cap = p->q_cap;

  // Scratch sizing: the largest prefill plan over every lq the query region
  // admits, and the decode plan at the fullest query region.
  long long partA = 0, partS = 0;
  for (int lq = 1; lq <= p->q_cap; ++lq) {
    // every plan has at most max(n_seg + 1, SMs / (B*Hkv*pairs) + 1) spans
    // (per segment and region; or the balanced cut plus a region span)
    const long long bgp = (long long)v.B * v.Hkv * star::prefill_row_pairs(v, lq);
    const long long nmax = std::max<long long>(v.n_seg + 1, std::max(1LL, (long long)c->num_sms / bgp) + 1);
    const long long rows = (long long)v.B * v.Hkv * std::min<long long>(nmax, star::kMaxPrefillSpans) * v.G * lq;
    partA = std::max(partA, rows * v.D);
    partS = std::max(partS, rows);
  }
  {
    const long long rows = (long long)v.B * v.Hkv * star::decode_max_partials(v, c->num_sms) * v.G;
    partA = std::max(partA, rows * v.D);
    partS = std::max(partS, rows);
  }
  std::vector<int4> work(star::ctx_tc_work_count(v));
  star::ctx_tc_fill_work(v, work.data());
  c->n_ctx_work = (int)work.size();
  std::vector<int4> unit_work(work.size());
  star::ctx_tc_fill_units(v, c->num_sms, c->units, unit_work.data());

  const long long kv_ctx = (long long)p->B * p->Hkv * p->L * p->D;        // elements
  const long long kv_q = (long long)p->B * p->Hkv * p->q_cap * p->D;
  const long long n_tickets = (long long)p->B * p->Hkv;
  size_t off = 0;
  // every part is followed by a canary guard (star_cache_check_guards): a
  // kernel writing past the end of one part lands in its guard first
  auto take = [&](size_t bytes, const char* what) {
    size_t o = off;
    off = (off + bytes + 255) & ~size_t(255);
    c->guards.push_back({off, what});
    off += kGuardBytes;
    return o;
  };
  const size_t o_ck = take(kv_ctx * 2, "context K"), o_cv = take(kv_ctx * 2, "context V");
  const size_t o_qk = take(kv_q * 2, "query-region K"), o_qv = take(kv_q * 2, "query-region V");
  const size_t o_pa = take(partA * 4, "partials A"), o_ps = take(partS * 4, "partials s");
  const size_t o_t = take(n_tickets * 4, "merge tickets");
  const size_t o_e = take(sizeof(int), "error word");
  const size_t o_w = take(work.size() * sizeof(int4), "phase-1 work list");
  const size_t o_uw = take(unit_work.size() * sizeof(int4), "phase-1 units");
  const bool fp8 = p->kv_fp8 != 0;
  const long long ctx_rows = (long long)p->B * p->Hkv * p->L;
  const size_t o_k8 = fp8 ? take(kv_ctx, "FP8 context K") : 0, o_v8 = fp8 ? take(kv_ctx, "FP8 context V") : 0;
  // scales padded to whole groups of 4 rows (zeroed below): decode loads them 4 rows at a time
  const size_t scl_bytes = (size_t)((ctx_rows + 3) / 4) * 16;
  const size_t o_ks = fp8 ? take(scl_bytes, "FP8 context K scales") : 0;
  const size_t o_vs = fp8 ? take(scl_bytes, "FP8 context V scales") : 0;
  const long long q_rows = (long long)p->B * p->Hkv * p->q_cap;
  const size_t qscl_bytes = (size_t)((q_rows + 3) / 4) * 16;
  const size_t o_qk8 = fp8 ? take(kv_q, "FP8 query-region K") : 0, o_qv8 = fp8 ? take(kv_q, "FP8 query-region V") : 0;
  const size_t o_qks = fp8 ? take(qscl_bytes, "FP8 query-region K scales") : 0;
  const size_t o_qvs = fp8 ? take(qscl_bytes, "FP8 query-region V scales") : 0;
  // STAR_FAULT_INJECT=alloc makes this allocation fail (a test hook for the
  // STAR_ENOMEM path)
  const char* inject = getenv("STAR_FAULT_INJECT");
  e = inject && strcmp(inject, "alloc") == 0 ? cudaErrorMemoryAllocation : cudaMalloc(&c->block, off);
  if (e != cudaSuccess) {
    delete c;
    return fail(STAR_ENOMEM, "cudaMalloc(%zu bytes): %s", off, cudaGetErrorString(e));
  }
  char* base = static_cast<char*>(c->block);
  v.ctxK = reinterpret_cast<bf16*>(base + o_ck);
  v.ctxV = reinterpret_cast<bf16*>(base + o_cv);
  v.qK = reinterpret_cast<bf16*>(base + o_qk);
  v.qV = reinterpret_cast<bf16*>(base + o_qv);
  c->scratch.partA = reinterpret_cast<float*>(base + o_pa);
  c->scratch.partS = reinterpret_cast<float*>(base + o_ps);
  c->scratch.tickets = reinterpret_cast<unsigned*>(base + o_t);
  c->scratch.err = reinterpret_cast<int*>(base + o_e);
  v.err = c->scratch.err;
  c->scratch.partA_elems = partA;
  c->scratch.partS_elems = partS;
  c->scratch.n_tickets = (int)n_tickets;
  c->ctx_work = reinterpret_cast<int4*>(base + o_w);
  c->unit_work = reinterpret_cast<int4*>(base + o_uw);
  v.ctxK8 = fp8 ? reinterpret_cast<uint8_t*>(base + o_k8) : nullptr;
  v.ctxV8 = fp8 ? reinterpret_cast<uint8_t*>(base + o_v8) : nullptr;
  v.ctxKs = fp8 ? reinterpret_cast<float*>(base + o_ks) : nullptr;
  v.ctxVs = fp8 ? reinterpret_cast<float*>(base + o_vs) : nullptr;
  v.qK8 = fp8 ? reinterpret_cast<uint8_t*>(base + o_qk8) : nullptr;
  v.qV8 = fp8 ? reinterpret_cast<uint8_t*>(base + o_qv8) : nullptr;
  v.qKs = fp8 ? reinterpret_cast<float*>(base + o_qks) : nullptr;
  v.qVs = fp8 ? reinterpret_cast<float*>(base + o_qvs) : nullptr;
  // Zero everything once: decode streams whole 128-row boxes and masks the
  // rows past the end, which must hold finite values.
  e = cudaMemset(c->block, 0, off);
  for (size_t g = 0; e == cudaSuccess && g < c->guards.size(); ++g)
    e = cudaMemset(base + c->guards[g].off, kCanary, kGuardBytes);
  if (e == cudaSuccess) e = cudaMemset(c->scratch.tickets, 0, n_tickets * 4);
  if (e == cudaSuccess) e = cudaMemset(c->scratch.err, 0, sizeof(int));
  if (e == cudaSuccess)
    e = cudaMemcpy(c->ctx_work, work.data(), work.size() * sizeof(int4), cudaMemcpyHostToDevice);
  if (e == cudaSuccess)
    e = cudaMemcpy(c->unit_work, unit_work.data(), unit_work.size() * sizeof(int4), cudaMemcpyHostToDevice);
  if (e != cudaSuccess) {
    cudaFree(c->block);
    delete c;
    return cuda_fail(e, "cache initialisation");
  }
  if (const char* bad = star::decode_make_maps(v, &c->dmaps)) {
    cudaFree(c->block);
    delete c;
    return fail(STAR_EINVAL, "TMA tensor map of the cache rejected by the driver: %s", bad);
  }
  e = star::decode_prepare(v.D);
  if (e == cudaSuccess) e = star::attn_tc_prepare(v.D);
  if (e != cudaSuccess) {
    cudaFree(c->block);
    delete c;
    return cuda_fail(e, "decode kernel attributes");
  }
  c->q_len = 0;
  *out = c;
  g_err[0] = 0;
  return STAR_OK;
}

int star_cache_destroy(star_cache* c) {
  if (!c) return STAR_OK;
  cudaError_t e = cudaDeviceSynchronize();
  for (cudaEvent_t ev : c->events) cudaEventDestroy(ev);
  if (c->s_in) cudaStreamDestroy(c->s_in);
  if (c->s_out) cudaStreamDestroy(c->s_out);
  if (c->s_comp) cudaStreamDestroy(c->s_comp);
  cudaError_t f = cudaFree(c->block);
  delete c;
  if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceSynchronize");
  if (f != cudaSuccess) return cuda_fail(f, "cudaFree");
  return STAR_OK;
}

int star_cache_device_error(star_cache* c, int* flag) {
  if (!c || !flag) return fail(STAR_EINVAL, "NULL argument");
  int h = 0;
  cudaError_t e = cudaMemcpy(&h, c->scratch.err, sizeof(int), cudaMemcpyDeviceToHost);
  if (e == cudaSuccess && h) e = cudaMemset(c->scratch.err, 0, sizeof(int));
  // a step that gave up may have left its decode counters behind
  if (e == cudaSuccess && h) e = cudaMemset(c->scratch.tickets, 0, (size_t)c->scratch.n_tickets * 4);
  if (e != cudaSuccess) return cuda_fail(e, "reading the device error word");
  *flag = h;
  return STAR_OK;
}

int star_cache_check_guards(star_cache* c, int* first_bad) {
  if (!c || !first_bad) return fail(STAR_EINVAL, "NULL argument");
  std::vector<unsigned char> h(kGuardBytes);
  *first_bad = -1;
  // every stream's work first: a plain copy orders only after the legacy stream
  cudaError_t es = cudaDeviceSynchronize();
  if (es != cudaSuccess) return cuda_fail(es, "cudaDeviceSynchronize");
  for (size_t g = 0; g < c->guards.size(); ++g) {
    cudaError_t e = cudaMemcpy(h.data(), static_cast<char*>(c->block) + c->guards[g].off, kGuardBytes,
                               cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return cuda_fail(e, "reading the cache's guard regions");
    for (size_t i = 0; i < kGuardBytes; ++i)
      if (h[i] != (unsigned char)kCanary) {
        *first_bad = (int)g;
        return fail(STAR_OK, "guard %zu (after %s) overwritten at byte %zu", g, c->guards[g].after, i);
      }
  }
  return STAR_OK;
}

int star_cache_num_segments(const star_cache* c) { return c ? c->view.n_seg + 1 : 0; }

int star_cache_segment(const star_cache* c, int seg, void** k, void** v, long long* start,
                       long long* len, long long* cap) {
  if (!c) return fail(STAR_EINVAL, "cache is NULL");
  const star::CacheView& w = c->view;
  if (seg < 0 || seg > w.n_seg) return fail(STAR_EINVAL, "segment %d out of range", seg);
  if (seg == w.n_seg) {
    if (k) *k = w.qK;
    if (v) *v = w.qV;
    if (start) *start = w.L;
    if (len) *len = c->q_len;
    if (cap) *cap = w.q_cap;
    return STAR_OK;
  }
  const long long off = (long long)seg * w.B * w.Hkv * (long long)w.b * w.D;
  if (k) *k = w.ctxK + off;
  if (v) *v = w.ctxV + off;
  if (start) *start = (long long)seg * w.b;
  if (len) *len = star::seg_len(w, seg);
  if (cap) *cap = star::seg_len(w, seg);
  return STAR_OK;
}

int star_cache_segment_fp8(const star_cache* c, int seg, void** k8, void** v8, float** k_scale,
                           float** v_scale) {
  if (!c) return fail(STAR_EINVAL, "cache is NULL");
  const star::CacheView& w = c->view;
  if (!w.ctxK8) return fail(STAR_EINVAL, "cache has no FP8 copy (kv_fp8 = 0)");
  if (seg < 0 || seg > w.n_seg) return fail(STAR_EINVAL, "segment %d out of range", seg);
  if (seg == w.n_seg) {                     // the query region
    if (k8) *k8 = w.qK8;
    if (v8) *v8 = w.qV8;
    if (k_scale) *k_scale = w.qKs;
    if (v_scale) *v_scale = w.qVs;
    return STAR_OK;
  }
  const long long rows = (long long)seg * w.B * w.Hkv * (long long)w.b;
  if (k8) *k8 = w.ctxK8 + rows * w.D;
  if (v8) *v8 = w.ctxV8 + rows * w.D;
  if (k_scale) *k_scale = w.ctxKs + rows;
  if (v_scale) *v_scale = w.ctxVs + rows;
  return STAR_OK;
}

int star_cache_reset_query(star_cache* c) {
  if (!c) return fail(STAR_EINVAL, "cache is NULL");
  c->q_len = 0;
  return STAR_OK;
}

}  // extern "C"

namespace {
// star_ctx_encode and its forms: per-block anchor keys (Ka) and the float32
// debug rows (O32), either may be null.
int ctx_encode(star_cache* c, const void* Q, const void* K, const void* V, const void* Ka, void* O,
               float* LSE, float* O32, void* stream, const void* Va = nullptr) {
  if (!c) return fail(STAR_EINVAL, "cache is NULL");
  if (!Q || !K || !V || !O || !LSE) return fail(STAR_EINVAL, "NULL tensor pointer");
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O) || !aligned16(LSE) ||
      (Ka && !aligned16(Ka)) || (Va && !aligned16(Va)) || (O32 && !aligned16(O32)))
    return fail(STAR_EINVAL, "tensor pointers must be 16-byte aligned");
  cudaError_t e = star::launch_ctx_encode_tc(
      c->view, c->p.scale, static_cast<const bf16*>(Q), static_cast<const bf16*>(K),
      static_cast<const bf16*>(V), static_cast<bf16*>(O), LSE, c->ctx_work, c->n_ctx_work, c->scratch.err,
      static_cast<cudaStream_t>(stream), static_cast<const bf16*>(Ka), O32, static_cast<const bf16*>(Va));
  if (e == cudaErrorInvalidValue) return fail(STAR_EINVAL, "TMA tensor map rejected (alignment or size)");
  if (e == cudaSuccess && c->view.ctxK8) e = star::launch_quantize_ctx_fp8(c->view, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "star_ctx_encode launch");
  c->q_len = 0;
  return STAR_OK;
}
}  // namespace

extern "C" {

int star_ctx_encode_anchored(star_cache* c, const void* Q, const void* K, const void* V, const void* Ka,
                             void* O, float* LSE, void* stream) {
  return ctx_encode(c, Q, K, V, Ka, O, LSE, nullptr, stream);
}

int star_ctx_encode(star_cache* c, const void* Q, const void* K, const void* V, void* O,
                    float* LSE, void* stream) {
  return ctx_encode(c, Q, K, V, nullptr, O, LSE, nullptr, stream);
}

int star_ctx_encode_after_anchor(star_cache* c, const void* Q, const void* K, const void* V,
                                 const void* Ka, const void* Va, void* O, float* LSE, void* stream) {
  if (!c) return fail(STAR_EINVAL, "cache is NULL");
  if (c->view.b_a > 0 && (!Ka || !Va)) return fail(STAR_EINVAL, "NULL anchor pointer");
  if (c->view.b_a == 0) return ctx_encode(c, Q, K, V, nullptr, O, LSE, nullptr, stream);
  return ctx_encode(c, Q, K, V, Ka, O, LSE, nullptr, stream, Va);
}

int star_ctx_encode_fp32(star_cache* c, const void* Q, const void* K, const void* V, void* O, float* LSE,
                         float* O32, void* stream) {
  if (!O32) return fail(STAR_EINVAL, "O32 is NULL");
  return ctx_encode(c, Q, K, V, nullptr, O, LSE, O32, stream);
}

int star_ctx_encode_host(star_cache* c, const void* hQ, const void* hK, const void* hV, void* hO,
                         float* hLSE, void* Q, void* K, void* V, void* O, float* LSE, void* stream) {
  if (!c) return fail(STAR_EINVAL, "cache is NULL");
  if (!hQ || !hK || !hV || !hO || !hLSE || !Q || !K || !V || !O || !LSE)
    return fail(STAR_EINVAL, "NULL tensor pointer");
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O) || !aligned16(LSE))
    return fail(STAR_EINVAL, "device tensor pointers must be 16-byte aligned");
  const star::CacheView& w = c->view;
  cudaError_t e = cudaSuccess;
  if (!c->s_in) {
    // created once, all or nothing: a failure leaves the cache as it was
    cudaStream_t st3[3] = {nullptr, nullptr, nullptr};
    std::vector<cudaEvent_t> evs;
    for (int i = 0; e == cudaSuccess && i < 3; ++i) e = cudaStreamCreateWithFlags(&st3[i], cudaStreamNonBlocking);
    for (size_t i = 0; e == cudaSuccess && i < 3 + 2 * c->units.size(); ++i) {
      cudaEvent_t ev;
      e = cudaEventCreateWithFlags(&ev, cudaEventDisableTiming);
      if (e == cudaSuccess) evs.push_back(ev);
    }
    if (e != cudaSuccess) {
      for (cudaEvent_t ev : evs) cudaEventDestroy(ev);
      for (cudaStream_t x : st3)
        if (x) cudaStreamDestroy(x);
      return cuda_fail(e, "copy streams");
    }
    c->s_in = st3[0];
    c->s_out = st3[1];
    c->s_comp = st3[2];
    c->events = std::move(evs);
  }
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaEvent_t ev_start = c->events[0], ev_end = c->events[1], ev_comp = c->events[2];
  // the device buffers are free once the work before this call on `stream` is done
  e = cudaEventRecord(ev_start, st);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(c->s_in, ev_start, 0);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(c->s_out, ev_start, 0);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(c->s_comp, ev_start, 0);
  const size_t row_b = (size_t)w.D * sizeof(bf16), row_l = sizeof(float);
  // rows [start, start + len) of heads [h0, h1) of batch entry bb of a [B][H][L] tensor of rb-byte rows
  auto rows2d = [&](void* dst, const void* src, int H, int bb, int h0, int h1, long long start, long long len,
                    size_t rb, cudaMemcpyKind kind, cudaStream_t s) {
    const size_t pit = (size_t)w.L * rb;
    const size_t o = (((size_t)bb * H + h0) * w.L + start) * rb;
    return cudaMemcpy2DAsync(static_cast<char*>(dst) + o, pit, static_cast<const char*>(src) + o, pit,
                             (size_t)len * rb, (size_t)(h1 - h0), kind, s);
  };
  for (size_t u = 0; u < c->units.size() && e == cudaSuccess; ++u) {
    const star::CtxUnit& un = c->units[u];
    const long long start = (long long)un.blk * w.b, len = star::seg_len(w, un.blk);
    cudaEvent_t ev_in = c->events[3 + 2 * u], ev_out = c->events[4 + 2 * u];
    const cudaStream_t cs = (u & 1) ? c->s_comp : st;      // units alternate between two compute streams
    // inputs of the unit, one 2-D copy per batch entry it touches
    for (int bb = un.bg0 / w.Hkv; bb * w.Hkv < un.bg1 && e == cudaSuccess; ++bb) {
      const int g0 = std::max(un.bg0, bb * w.Hkv) - bb * w.Hkv, g1 = std::min(un.bg1, (bb + 1) * w.Hkv) - bb * w.Hkv;
      e = rows2d(Q, hQ, w.Hq, bb, g0 * w.G, g1 * w.G, start, len, row_b, cudaMemcpyHostToDevice, c->s_in);
      if (e == cudaSuccess) e = rows2d(K, hK, w.Hkv, bb, g0, g1, start, len, row_b, cudaMemcpyHostToDevice, c->s_in);
      if (e == cudaSuccess) e = rows2d(V, hV, w.Hkv, bb, g0, g1, start, len, row_b, cudaMemcpyHostToDevice, c->s_in);
    }
    if (e == cudaSuccess) e = cudaEventRecord(ev_in, c->s_in);
    // the unit's tiles (their anchor rows came with block 0's units, earlier on the same copy stream)
    if (e == cudaSuccess) e = cudaStreamWaitEvent(cs, ev_in, 0);
    if (e == cudaSuccess)
      e = star::launch_ctx_encode_tc(w, c->p.scale, static_cast<const bf16*>(Q), static_cast<const bf16*>(K),
                                     static_cast<const bf16*>(V), static_cast<bf16*>(O), LSE,
                                     c->unit_work + un.off, un.n, c->scratch.err, cs, nullptr);
    if (e == cudaSuccess) e = cudaEventRecord(ev_out, cs);
    // outputs of the unit
    if (e == cudaSuccess) e = cudaStreamWaitEvent(c->s_out, ev_out, 0);
    for (int bb = un.bg0 / w.Hkv; bb * w.Hkv < un.bg1 && e == cudaSuccess; ++bb) {
      const int g0 = std::max(un.bg0, bb * w.Hkv) - bb * w.Hkv, g1 = std::min(un.bg1, (bb + 1) * w.Hkv) - bb * w.Hkv;
      e = rows2d(hO, O, w.Hq, bb, g0 * w.G, g1 * w.G, start, len, row_b, cudaMemcpyDeviceToHost, c->s_out);
      if (e == cudaSuccess)
        e = rows2d(hLSE, LSE, w.Hq, bb, g0 * w.G, g1 * w.G, start, len, row_l, cudaMemcpyDeviceToHost, c->s_out);
    }
  }
  // the caller's stream takes over once every unit's tiles are done
  if (e == cudaSuccess) e = cudaEventRecord(ev_comp, c->s_comp);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(st, ev_comp, 0);
  if (e == cudaSuccess && w.ctxK8) e = star::launch_quantize_ctx_fp8(w, st);
  if (e == cudaSuccess) e = cudaEventRecord(ev_end, c->s_out);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(st, ev_end, 0);
  if (e != cudaSuccess) {
    // whatever was enqueued on the side streams still ends before `stream` goes on
    const cudaStream_t side[3] = {c->s_in, c->s_comp, c->s_out};
    for (cudaStream_t x : side)
      if (cudaEventRecord(ev_end, x) == cudaSuccess) cudaStreamWaitEvent(st, ev_end, 0);
    if (e == cudaErrorInvalidValue) return fail(STAR_EINVAL, "TMA tensor map rejected (alignment or size)");
    return cuda_fail(e, "star_ctx_encode_host");
  }
  c->q_len = 0;
  return STAR_OK;
}

int star_rope(int B, int H, long long L, int D, double theta, const int* pos, long long pos0, const void* x,
              void* y, void* stream) {
  if (B < 1 || H < 1 || L < 0) return fail(STAR_EINVAL, "need B, H >= 1 and L >= 0");
  if (D != 64 && D != 128) return fail(STAR_EUNSUPPORTED, "head dim %d: RoPE supports D = 64 or 128", D);
  if (!(theta > 1.0)) return fail(STAR_EINVAL, "theta must be > 1");
  if (B > 65535) return fail(STAR_EINVAL, "B must be <= 65535");
  if (pos0 < 0) return fail(STAR_EINVAL, "pos0 must be >= 0");
  if (L == 0) return STAR_OK;
  if (!x || !y) return fail(STAR_EINVAL, "NULL tensor pointer");
  if (!aligned16(x) || !aligned16(y)) return fail(STAR_EINVAL, "tensor pointers must be 16-byte aligned");
  star::RopeJob j;
  j.x = static_cast<const bf16*>(x);
  j.y = static_cast<bf16*>(y);
  j.x_seq = j.y_seq = L;
  j.x_grp = j.y_grp = 0;
  j.n = L;
  j.H = H;
  j.pos = pos;
  j.pos_grp = 0;
  j.pos0 = pos0;
  j.pos0_grp = 0;
  star::rope_inv_freq(D, theta, j.inv_freq);
  cudaError_t e = star::launch_rope(j, D, B, 1, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "star_rope launch");
  return STAR_OK;
}

int star_anchor_keys(const star_cache* c, int mode, const int* pos, double theta, const void* K, void* Ka,
                     void* stream) {
  if (!c) return fail(STAR_EINVAL, "cache is NULL");
  const star::CacheView& w = c->view;
  if (mode < 0 || mode > 2) return fail(STAR_EINVAL, "mode must be 0 (first), 1 (previous) or 2 (given)");
  if (!(theta > 1.0)) return fail(STAR_EINVAL, "theta must be > 1");
  if (w.n_seg < 2 || w.b_a == 0) return STAR_OK;          // no block has an anchor
  if (mode == 2 && !pos) return fail(STAR_EINVAL, "mode 2 needs the position array");
  if (!K || !Ka) return fail(STAR_EINVAL, "NULL tensor pointer");
  if (!aligned16(K) || !aligned16(Ka)) return fail(STAR_EINVAL, "tensor pointers must be 16-byte aligned");
  star::RopeJob j;
  j.x = static_cast<const bf16*>(K);
  j.y = static_cast<bf16*>(Ka);
  j.x_seq = w.L;                                      // K [B][Hkv][L][D]: rows 0..b_a-1 of each (b, g)
  j.x_grp = 0;                                        // every block reads the same anchor rows
  j.y_seq = w.b_a;                                    // Ka [n-1][B][Hkv][b_a][D]
  j.y_grp = (long long)w.B * w.Hkv * w.b_a;
  j.n = w.b_a;
  j.H = w.Hkv;
  j.pos = mode == 2 ? pos : nullptr;
  j.pos_grp = w.b_a;                                  // pos [n-1][b_a]
  j.pos0 = mode == 1 ? (long long)w.b - w.b_a : 0;    // block i = z + 1: positions i*b - b_a + t
  j.pos0_grp = mode == 1 ? w.b : 0;
  star::rope_inv_freq(w.D, theta, j.inv_freq);
  cudaError_t e = star::launch_rope(j, w.D, w.B, w.n_seg - 1, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "star_anchor_keys launch");
  return STAR_OK;
}

int star_query_prefill(star_cache* c, int lq, const void* Q, const void* K, const void* V,
                       void* O, float* LSE, void* stream) {
  return query_prefill(c, lq, Q, K, V, O, LSE, stream, false, nullptr, nullptr, nullptr);
}

int star_query_prefill_partials(star_cache* c, int lq, const void* Q, const void* K, const void* V,
                                void* O, float* LSE, float* Ah, float* sh, float* O32, void* stream) {
  return query_prefill(c, lq, Q, K, V, O, LSE, stream, true, Ah, sh, O32);
}

int star_decode_step(star_cache* c, const void* q, const void* k, const void* v, void* o,
                     float* lse, void* stream) {
  if (!c) return fail(STAR_EINVAL, "cache is NULL");
  if (!q || !k || !v || !o || !lse) return fail(STAR_EINVAL, "NULL tensor pointer");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse))
    return fail(STAR_EINVAL, "tensor pointers must be 16-byte aligned");
  if (c->q_len + 1 > c->view.q_cap)
    return fail(STAR_ENOSPC, "query region full: %lld rows, q_cap %d", c->q_len, c->view.q_cap);
  star::DecodePlan pl = plan_decode(c, c->q_len);
  cudaError_t e = star::launch_decode_step(
      c->view, c->dmaps, c->p.scale, (int)c->q_len, static_cast<const bf16*>(q),
      static_cast<const bf16*>(k), static_cast<const bf16*>(v), static_cast<bf16*>(o), lse, pl,
      c->scratch, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "star_decode_step launch");
  c->q_len += 1;
  return STAR_OK;
}

int star_partial_attend(star_cache* c, int first_seg, int n_seg, int with_query, int lq, const void* Q,
                        const void* K, const void* V, float* A, float* s, void* stream) {
  if (!c) return fail(STAR_EINVAL, "cache is NULL");
  const star::CacheView& w = c->view;
  if (lq < 1) return fail(STAR_EINVAL, "lq must be >= 1");
  if (first_seg < 0 || n_seg < 0 || first_seg + n_seg > w.n_seg)
    return fail(STAR_EINVAL, "segments [%d, %d) outside 0..%d", first_seg, first_seg + n_seg, w.n_seg);
  if (with_query != 0 && with_query != 1) return fail(STAR_EINVAL, "with_query must be 0 or 1");
  if (!Q || !A || !s || (with_query && (!K || !V))) return fail(STAR_EINVAL, "NULL tensor pointer");
  if (!aligned16(Q) || !aligned16(A) || !aligned16(s) || (with_query && (!aligned16(K) || !aligned16(V))))
    return fail(STAR_EINVAL, "tensor pointers must be 16-byte aligned");
  if (with_query && c->q_len + lq > w.q_cap)
    return fail(STAR_ENOSPC, "query region full: %lld + %d > q_cap %d", c->q_len, lq, w.q_cap);
  if (lq > w.q_cap) return fail(STAR_EINVAL, "lq %d beyond q_cap %d (the scratch is sized by it)", lq, w.q_cap);
  // One row over segments that run to the end of the context (a generation
  // step of the block-sharded layer): the split-KV decode kernel streams them
  // at the HBM rate, where the prefill tile kernel would fill 128-row tiles
  // from G rows.  On an FP8 cache it reads the E4M3 copy, as star_decode_step
  // does on that cache.
  const long long skip = std::min<long long>((long long)first_seg * w.b, w.L);   // rows before first_seg
  const long long len0 = with_query ? c->q_len : 0;
  if (lq == 1 && first_seg + n_seg == w.n_seg && w.L - skip + len0 >= 1) {
    const star::DecodePlan dp = star::decode_plan(w, len0, c->num_sms, skip);
    cudaError_t e = star::launch_decode_step(
        w, c->dmaps, c->p.scale, (int)len0, static_cast<const bf16*>(Q), static_cast<const bf16*>(K),
        static_cast<const bf16*>(V), nullptr, s, dp, c->scratch, static_cast<cudaStream_t>(stream), skip,
        with_query != 0, A);
    if (e != cudaSuccess) return cuda_fail(e, "star_partial_attend launch");
    if (with_query) c->q_len += 1;
    return STAR_OK;
  }
  const star::PrefillPlan pl =
      star::plan_prefill(w, c->num_sms, lq, c->q_len, first_seg, first_seg + n_seg, with_query != 0);
  cudaError_t e = star::launch_query_prefill_tc(
      w, c->dmaps, c->p.scale, lq, (int)c->q_len, static_cast<const bf16*>(Q), static_cast<const bf16*>(K),
      static_cast<const bf16*>(V), nullptr, s, pl, c->scratch, static_cast<cudaStream_t>(stream), A, nullptr,
      nullptr, with_query != 0);
  if (e == cudaSuccess && with_query && w.qK8)
    e = star::launch_quantize_qregion_fp8(w, static_cast<const bf16*>(K), static_cast<const bf16*>(V),
                                          (int)c->q_len, lq, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "star_partial_attend launch");
  if (with_query) c->q_len += lq;
  return STAR_OK;
}

int star_decode_step_partials(star_cache* c, const void* q, const void* k, const void* v, void* o, float* lse,
                              float* Ah, float* sh, long long* spans, int max_parts, int* n_parts, void* stream) {
  if (!c) return fail(STAR_EINVAL, "cache is NULL");
  if (!Ah || !sh || !spans || !n_parts) return fail(STAR_EINVAL, "NULL partials pointer");
  const star::CacheView& w = c->view;
  if (c->q_len + 1 > w.q_cap)
    return fail(STAR_ENOSPC, "query region full: %lld rows, q_cap %d", c->q_len, w.q_cap);
  const star::DecodePlan pl = plan_decode(c, c->q_len);
  std::vector<star::DecodePart> parts;
  star::decode_parts(w, c->q_len, pl, parts);
  *n_parts = (int)parts.size();
  if ((int)parts.size() > max_parts)
    return fail(STAR_EINVAL, "%d parts do not fit max_parts = %d", (int)parts.size(), max_parts);
  const int rc = star_decode_step(c, q, k, v, o, lse, stream);
  if (rc) return rc;
  // the step left every part in the cache's scratch: [B*Hkv][maxp][G][D] and [B*Hkv][maxp][G]
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t rowA = (size_t)w.G * w.D, rowS = (size_t)w.G;
  cudaError_t e = cudaSuccess;
  size_t i = 0;
  while (i < parts.size() && e == cudaSuccess) {
    size_t j = i;                                    // the parts of one bg are consecutive slots
    while (j < parts.size() && parts[j].bg == parts[i].bg) ++j;
    const size_t src = (size_t)parts[i].bg * pl.maxp;
    e = cudaMemcpyAsync(Ah + i * rowA, c->scratch.partA + src * rowA, (j - i) * rowA * sizeof(float),
                        cudaMemcpyDeviceToDevice, st);
    if (e == cudaSuccess)
      e = cudaMemcpyAsync(sh + i * rowS, c->scratch.partS + src * rowS, (j - i) * rowS * sizeof(float),
                          cudaMemcpyDeviceToDevice, st);
    i = j;
  }
  if (e != cudaSuccess) return cuda_fail(e, "star_decode_step_partials copies");
  for (size_t p = 0; p < parts.size(); ++p) {
    spans[3 * p] = parts[p].bg;
    spans[3 * p + 1] = parts[p].first;
    spans[3 * p + 2] = parts[p].end;
  }
  return STAR_OK;
}

int star_plan_prefill(const star_params* p, int num_sms, int lq, long long len0, int first_seg, int n_seg,
                      int with_query, int per_segment, int max_spans, int* n_spans, int* spans) {
  int rc = validate_params(p);
  if (rc) return rc;
  if (!n_spans || !spans) return fail(STAR_EINVAL, "NULL output pointer");
  if (num_sms < 1 || lq < 1 || len0 < 0 || len0 + lq > p->q_cap) return fail(STAR_EINVAL, "bad num_sms, lq or len0");
  const star::CacheView v = host_view(p);
  if (first_seg < 0 || n_seg < 0 || first_seg + n_seg > v.n_seg) return fail(STAR_EINVAL, "segment range");
  const star::PrefillPlan pl = per_segment ? star::plan_prefill_per_segment(v, lq, len0)
                                           : star::plan_prefill(v, num_sms, lq, len0, first_seg, first_seg + n_seg,
                                                                with_query != 0);
  *n_spans = pl.n_spans;
  if (pl.n_spans > max_spans) return fail(STAR_EINVAL, "%d spans do not fit max_spans = %d", pl.n_spans, max_spans);
  for (int k = 0; k < pl.n_spans; ++k) {
    spans[2 * k] = pl.span[k].x0;
    spans[2 * k + 1] = pl.span[k].x1;
  }
  return STAR_OK;
}

int star_prefill_span_tiles(const star_params* p, long long x0, long long x1, int bg, int max_tiles, int* n_tiles,
                            int* tiles) {
  int rc = validate_params(p);
  if (rc) return rc;
  if (!n_tiles || !tiles) return fail(STAR_EINVAL, "NULL output pointer");
  const star::CacheView v = host_view(p);
  if (x0 < 0 || x1 <= x0 || x1 > v.L + v.q_cap || bg < 0 || bg >= v.B * v.Hkv)
    return fail(STAR_EINVAL, "span or (batch, kv head) out of range");
  const int n = star::span_tiles(x0, x1, v);
  *n_tiles = n;
  if (n > max_tiles) return fail(STAR_EINVAL, "%d tiles do not fit max_tiles = %d", n, max_tiles);
  star::TileWalk walk;
  walk.start(x0, x1, v);
  for (int t = 0; t < n; ++t) {
    int row, r0;
    bool region;
    const int k = walk.next(v, bg, row, region, r0);
    tiles[4 * t] = row;
    tiles[4 * t + 1] = region ? 1 : 0;
    tiles[4 * t + 2] = k;
    tiles[4 * t + 3] = r0;
  }
  if (walk.x != x1) return fail(STAR_EINVAL, "the walk did not end at the span's end");
  return STAR_OK;
}

int star_selftest_wait_timeout(unsigned polls, int* gave_up, void* stream) {
  if (!gave_up) return fail(STAR_EINVAL, "gave_up is NULL");
  if (polls < 1 || polls > (1u << 22)) return fail(STAR_EINVAL, "polls must be in 1..2^22");
  *gave_up = 0;
  cudaError_t e = star::run_wait_timeout(polls, gave_up, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "star_selftest_wait_timeout");
  return STAR_OK;
}

int star_lse_merge_bf16(int P, long long R, int D, const float* A, const float* s, void* out_O,
                        float* out_s, void* stream) {
  if (P < 1 || R < 0 || D < 1 || D > 1024) return fail(STAR_EINVAL, "need P >= 1, R >= 0, 1 <= D <= 1024");
  if (R == 0) return STAR_OK;
  if (!A || !s || !out_O || !out_s) return fail(STAR_EINVAL, "NULL tensor pointer");
  cudaError_t e = star::launch_lse_merge(P, R, D, A, s, nullptr, out_s, static_cast<cudaStream_t>(stream),
                                         static_cast<bf16*>(out_O));
  if (e != cudaSuccess) return cuda_fail(e, "star_lse_merge_bf16 launch");
  return STAR_OK;
}

int star_lse_merge(int P, long long R, int D, const float* A, const float* s, float* out_A,
                   float* out_s, void* stream) {
  if (P < 1 || R < 0 || D < 1 || D > 1024) return fail(STAR_EINVAL, "need P >= 1, R >= 0, 1 <= D <= 1024");
  if (R == 0) return STAR_OK;
  if (!A || !s || !out_A || !out_s) return fail(STAR_EINVAL, "NULL tensor pointer");
  cudaError_t e = star::launch_lse_merge(P, R, D, A, s, out_A, out_s, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "star_lse_merge launch");
  return STAR_OK;
}

}  // extern "C"
