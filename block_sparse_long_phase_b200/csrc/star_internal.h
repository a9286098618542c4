// Host/device view of a star_cache shared by the libstar kernels.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include <vector>

namespace star {

typedef __nv_bfloat16 bf16;

// Error reporting shared by the C entry points (star_last_error()).
int set_error(int code, const char* msg);

// Geometry of the per-block KV cache.  Context segment i holds rows
// [i*b, i*b + len_i) of every (batch, kv head), laid out [B][Hkv][len_i][D];
// segments are back to back, so segment i starts i*B*Hkv*b*D elements in.
struct CacheView {
  int B, Hq, Hkv, D, G;
  long long L;
  int b, b_a, n_seg;
  int q_cap;
  bf16* ctxK;
  bf16* ctxV;
  bf16* qK;  // query region [B][Hkv][q_cap][D]
  bf16* qV;
  // optional FP8 (E4M3) copy of the context cache, same row order, and the
  // per-row scales (null when the cache keeps bf16 only)
  uint8_t* ctxK8;
  uint8_t* ctxV8;
  float* ctxKs;
  float* ctxVs;
  // ... and of the query region ([B][Hkv][q_cap] rows)
  uint8_t* qK8;
  uint8_t* qV8;
  float* qKs;
  float* qVs;
  int* err;      // the cache's device error word (bounds-checked builds report into it)
};

__host__ __device__ inline long long seg_len(const CacheView& c, int seg) {
  long long s = (long long)seg * c.b;
  long long r = c.L - s;
  return r < c.b ? r : c.b;
}

// Element offset of context row `row` (absolute token index) of (batch bb,
// kv head g) inside the segmented context cache.
__host__ __device__ inline long long ctx_row_offset(const CacheView& c, int bb, int g,
                                                    long long row) {
  int seg = (int)(row / c.b);
  long long off = row - (long long)seg * c.b;
  long long len = seg_len(c, seg);
  long long base = (long long)seg * c.B * c.Hkv * (long long)c.b * c.D;
  return base + (((long long)bb * c.Hkv + g) * len + off) * c.D;
}

// Element offset of query-region row `row` of (bb, g).
__host__ __device__ inline long long q_row_offset(const CacheView& c, int bb, int g,
                                                  long long row) {
  return (((long long)bb * c.Hkv + g) * c.q_cap + row) * c.D;
}

// Scratch owned by the cache for phase-2 partials.
struct Scratch {
  float* partA;        // partial outputs A_h
  float* partS;        // partial log-sum-exp s_h
  unsigned* tickets;   // per (batch, kv head) rows folded into parts, kept at 0 between calls
  int* err;            // device error word: set by a kernel whose bounded wait gave up
  long long partA_elems;
  long long partS_elems;
  int n_tickets;
};

// ---- launchers (defined in the .cu files) --------------------------------
size_t ctx_tc_work_count(const CacheView& c);
// phase-1 work list (b*Hkv + g, head pair, block, q tile), block by block
void ctx_tc_fill_work(const CacheView& c, int4* out);
// Phase-1 work cut into pipeline units for copies overlapped with compute: a
// unit is (block, batch x kv head range [bg0, bg1)), its items a contiguous
// run [off, off + n) of the list, longest tile first; units run block 0 first.
struct CtxUnit {
  int blk, bg0, bg1;
  int off, n;
};
void ctx_tc_fill_units(const CacheView& c, int num_sms, std::vector<CtxUnit>& units, int4* out);
// Ka (may be null): anchor keys of blocks 1..n-1 as [n-1][B][Hkv][b_a][D];
// block i >= 1 then reads its anchor keys from Ka[i-1] instead of K rows 0..b_a-1.
// With Va too, Ka and Va are one anchor [B][Hkv][b_a][D] held outside this
// context that every block, block 0 included, follows.
// O32 (may be null): the phase-1 rows in float32 before their bf16 rounding.
cudaError_t launch_ctx_encode_tc(const CacheView& c, float scale, const bf16* Q, const bf16* K,
                                 const bf16* V, bf16* O, float* LSE, const int4* work, int n_work,
                                 int* err, cudaStream_t st, const bf16* Ka = nullptr,
                                 float* O32 = nullptr, const bf16* Va = nullptr);

// Rotary embedding of rows: for group z < groups, batch b < B, head h < H and
// t < n, row (z*x_grp + (b*H + h)*x_seq + t) of x is rotated at position
// pos[z*pos_grp + t] (pos non-null) or pos0 + z*pos0_grp + t, and written to
// row (z*y_grp + (b*H + h)*y_seq + t) of y.
struct RopeJob {
  const bf16* x;
  bf16* y;
  long long x_seq, y_seq, x_grp, y_grp;
  long long n;
  int H;
  const int* pos;
  long long pos_grp;
  long long pos0, pos0_grp;
  double inv_freq[64];
};
void rope_inv_freq(int D, double base, double* out);
cudaError_t launch_rope(const RopeJob& j, int D, int B, int groups, cudaStream_t st);
// one CTA whose bounded wait on a barrier nothing completes must give up
// (selftest.cu); synchronous, *gave_up = 1 when it did
cudaError_t run_wait_timeout(unsigned polls, int* gave_up, cudaStream_t st);

// Prefill work split: spans [x0, x1) of a (batch, kv head)'s key rows, which
// are numbered over the context (0..L-1) and then the query region (L..L+n-1,
// n = rows in use once the call's rows are appended).  One CTA per (span,
// batch x kv head, 256-row pair of packed query rows); a span may cross
// context segments (its tiles split at their ends) and run on into the
// query region.
struct PrefillSpan {
  int x0, x1;
};
// Span table size of a prefill launch (kernel parameter): the per-segment
// debug plan needs one span per context segment and one for the query
// region, so a cache has at most kMaxPrefillSpans - 1 segments.
constexpr int kMaxPrefillSpans = 192;

struct PrefillPlan {
  int n_spans;
  PrefillSpan span[kMaxPrefillSpans];
};

// Keys per prefill tile (the tile kernel's BN).
constexpr int kPrefillTileKeys = 128;

// The 128-key tiles of one prefill span [x, x1) of a (batch, kv head)'s key
// rows, numbered over the context (0..L-1) and then the query region (L..).
// A tile never crosses the end of a context segment or of the context; for
// each one: its first row in the TMA map it is read through (the context
// cache, or the query region from row L on), its key count, and for the query
// region the region row of its first key.  The producer and every softmax
// thread walk the same sequence.
struct TileWalk {
  long long x, x1, seg_end;
  int seg;                                          // -1 once in the query region
  __host__ __device__ __forceinline__ void start(long long x0, long long xe, const CacheView& c) {
    x = x0;
    x1 = xe;
    seg = x0 < c.L ? (int)(x0 / c.b) : -1;
    seg_end = seg >= 0 ? ((long long)(seg + 1) * c.b < c.L ? (long long)(seg + 1) * c.b : c.L) : xe;
  }
  __host__ __device__ __forceinline__ int next(const CacheView& c, int bg, int& row, bool& region, int& r0) {
    if (seg >= 0 && x >= seg_end) {
      if (x < c.L) {
        ++seg;
        seg_end = ((long long)(seg + 1) * c.b < c.L ? (long long)(seg + 1) * c.b : c.L);
      } else {
        seg = -1;
        seg_end = x1;
      }
    }
    const long long end = seg_end < x1 ? seg_end : x1;
    const int n = (int)(end - x < kPrefillTileKeys ? end - x : kPrefillTileKeys);
    if (seg >= 0) {
      row = (int)((long long)seg * c.B * c.Hkv * c.b + (long long)bg * seg_len(c, seg) + (x - (long long)seg * c.b));
      region = false;
      r0 = 0;
    } else {
      r0 = (int)(x - c.L);
      row = (int)((long long)bg * c.q_cap + r0);
      region = true;
    }
    x += n;
    return n;
  }
};

// Tiles of span [x0, x1): one term per segment it overlaps, then the region.
__host__ __device__ __forceinline__ int span_tiles(long long x0, long long x1, const CacheView& c) {
  int n = 0;
  long long x = x0;
  while (x < x1 && x < c.L) {
    const int seg = (int)(x / c.b);
    long long e = (long long)(seg + 1) * c.b < c.L ? (long long)(seg + 1) * c.b : c.L;
    if (e > x1) e = x1;
    n += (int)((e - x + kPrefillTileKeys - 1) / kPrefillTileKeys);
    x = e;
  }
  if (x < x1) n += (int)((x1 - x + kPrefillTileKeys - 1) / kPrefillTileKeys);
  return n;
}


// Decode work split: the cached rows of all (batch, kv head) pairs, laid end
// to end, are cut into one balanced span per CTA; each span leaves one part
// per (batch, kv head) it touches, and the new token one more.
struct DecodePlan {
  int ncta;   // CTAs
  int maxp;   // part slots per (batch, kv head)
};
int decode_max_partials(const CacheView& c, int ncta);
// skip: leading context rows of each (batch, kv head) the step leaves out
DecodePlan decode_plan(const CacheView& c, long long len0, int num_sms, long long skip = 0);

// Span of CTA i: rows [span_start(i), span_start(i + 1)) of the R cached rows
// of all (batch, kv head) pairs laid end to end.  Row indices stay below 2^31
// (checked when the cache is made), so both quotients below divide a
// numerator under 2^53 by at most 2^31.  They are taken in double, which is
// exact there: the rounding error of the quotient is below 1 / divisor, the
// least distance of a non-integer quotient from an integer, so its floor is
// the integer quotient.  (A 64-bit integer division costs several times as
// long on the device, ahead of the first TMA load.)  Host and device share
// these two functions, so the host's list of parts is the kernel's.
__host__ __device__ __forceinline__ long long span_start(long long i, long long R, int n) {
  return (long long)floor((double)(i * R) / (double)n);
}
// CTA whose span holds row x (largest i with span_start(i) <= x).
__host__ __device__ __forceinline__ int cta_of(long long x, long long R, int n) {
  return (int)floor((double)((x + 1) * n - 1) / (double)R);
}

// One part of a decode step: the run of (batch, kv head) bg's cached rows
// [first, end) (context rows, then query-region rows from L on) that one CTA
// folds into part slot `slot` of bg.
struct DecodePart {
  int bg, slot;
  long long first, end;
};
void decode_parts(const CacheView& c, long long len0, const DecodePlan& pl, std::vector<DecodePart>& out);

// Prefill plans (star_abi.cu): spans of about equal length over the context
// segments [s0, s1) and, with `query`, the query region's len0 + lq rows; or
// one span per segment and one for the region.
PrefillPlan plan_prefill(const CacheView& v, int num_sms, int lq, long long len0, int s0 = 0, int s1 = -1,
                         bool query = true);
PrefillPlan plan_prefill_per_segment(const CacheView& v, int lq, long long len0);

// TMA maps of the cache, built once per cache.
struct DecodeMaps {
  CUtensorMap k_ctx, v_ctx, k_q, v_q;
  CUtensorMap k8_ctx, v8_ctx, k8_q, v8_q;     // FP8 rows: context, query region
  CUtensorMap ks_ctx, vs_ctx, ks_q, vs_q;     // their per-row scales
};
cudaError_t launch_quantize_ctx_fp8(const CacheView& c, cudaStream_t st);
// FP8 copy of prefill rows: K, V [B][Hkv][lq][D] -> query-region rows len0..len0+lq-1
cudaError_t launch_quantize_qregion_fp8(const CacheView& c, const bf16* K, const bf16* V, int len0, int lq,
                                        cudaStream_t st);
// Builds the cache's TMA maps; returns nullptr, or the name of the map the
// driver rejected.
const char* decode_make_maps(const CacheView& c, DecodeMaps* m);
cudaError_t decode_prepare(int D);   // one-time kernel attributes
// One decode step over each (batch, kv head)'s cached rows past its first
// `skip` context rows, then the query region's len0 rows and, with_token, the
// step's own k, v (appended at region row len0).  o (bf16) and o32 (float32)
// may each be null; lse is written.
cudaError_t launch_decode_step(const CacheView& c, const DecodeMaps& maps, float scale, int len0,
                               const bf16* q, const bf16* k, const bf16* v, bf16* o, float* lse,
                               const DecodePlan& plan, const Scratch& s, cudaStream_t st, long long skip = 0,
                               bool with_token = true, float* o32 = nullptr);

cudaError_t attn_tc_prepare(int D);   // one-time kernel attributes
int prefill_row_pairs(const CacheView& c, int lq);   // 256-row pairs of packed query rows
cudaError_t launch_query_prefill_tc(const CacheView& c, const DecodeMaps& maps, float scale, int lq,
                                    int len0, const bf16* Q, const bf16* Kq, const bf16* Vq, bf16* O,
                                    float* LSE, const PrefillPlan& plan, const Scratch& s,
                                    cudaStream_t st, float* O32 = nullptr, float* Ah = nullptr,
                                    float* sh = nullptr, bool append = true);

// outA (float32) or outB (bf16) may be null
cudaError_t launch_lse_merge(int P, long long R, int D, const float* A, const float* S,
                             float* outA, float* outS, cudaStream_t st, bf16* outB = nullptr);

}  // namespace star
