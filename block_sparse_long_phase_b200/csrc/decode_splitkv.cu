// Phase-2 generation step: split-KV, HBM-streaming attention with a fused
// log-sum-exp merge.
//
// "Star Attention: Efficient LLM Inference over Long Sequences" (analysis
// page), section 3.4, "Phase 2: Query Encoding and Token Generation with
// Distributed Softmax": every context block ("host") computes the local
// attention A_h of the new token and the log of its exponent sum s_h (Step 3);
// the partials are combined with the log-sum-exp rule (Step 5); only the
// query region's cache grows (Step 7).
//
// One GPU plays all the hosts.  The cached keys of every (batch, kv head) --
// its context segments, then its query region -- are laid end to end and cut
// into one balanced span per CTA (one CTA per SM), so each CTA streams the
// same number of bytes whatever the segment sizes.  Inside a CTA:
//   warp 0     TMA producer: 128-key K and V stages (128-byte swizzled boxes)
//              of the span, never crossing a segment, through a 3-slot ring;
//   warps 1-8  consumers: each owns 16 keys of every stage; the G query heads
//              of the kv group are the M rows of a 16x8x16 bf16 MMA (rows G..15
//              zero), online softmax in base 2, fp32 accumulation.
// When a span ends a (batch, kv head) piece, the consumer warps combine their
// states in shared memory into one partial (A, s) of that piece.  The last CTA
// of a (batch, kv head) to finish -- an atomic ticket, no CTA ever waits for
// another -- merges that head's partials together with the new token's own
// part (score q.k, value v, computed on the spot from the step's inputs) and
// writes o and lse.  The producer warp appends the token's k, v to the query
// region (a row no reader of this launch touches) after its last stage.
#include <cuda_bf16.h>
#include <stdio.h>
#include <algorithm>
#include <math.h>
#include <string.h>

#include <mutex>

#include "../../include/star_attention.h"
#include "fp8_row.cuh"
#include "sm100_primitives.cuh"
#include "star_common.cuh"
#include "star_internal.h"
#include "tmap.h"

namespace star {
namespace {

using namespace sm100;

constexpr int KS = 128;                 // keys per bf16 stage (16 per consumer warp)
constexpr int KS8 = 256;                // keys per FP8 context stage (32 per consumer warp)
constexpr int NSTAGE = 3;
constexpr int NCW = 8;                  // consumer warps
constexpr int NTHREADS = 32 * (NCW + 1);

struct StageMeta {
  int n;         // valid keys in the stage
  int bg;        // batch * Hkv + kv head
  int row0;      // first row of the stage in its region's cache (FP8: picks the scales)
  int flush;     // 1: before this stage, flush the previous run (fbg, fslot, frows)
  int end;       // 1: terminal stage (no keys): the CTA's work is done
  int fbg, fslot, frows;
};

struct DecodeArgs {
  CUtensorMap tk_ctx, tv_ctx;   // context cache as [B*Hkv*L][D]
  CUtensorMap tk_q, tv_q;       // query region as [B*Hkv*q_cap][D]
  CUtensorMap tk8, tv8;         // FP8 context cache as [B*Hkv*L][D] bytes, 256-row boxes
  CUtensorMap tkq8, tvq8;       // FP8 query region as [B*Hkv*q_cap][D] bytes
  CUtensorMap tks, tvs;         // FP8 row scales as [ceil(B*Hkv*L / 4)][4] float32
  CUtensorMap tkqs, tvqs;       // ... of the query region, [ceil(B*Hkv*q_cap / 4)][4]
  CacheView c;
  float scale_log2;
  int len0;                     // query-region rows before this step
  int ncta;
  int maxp;                     // partial slots per (batch, kv head)
  long long rpb;                // rows attended per (batch, kv head): L - skip + len0
  long long skip = 0;           // leading context rows of each (batch, kv head) left out
  int with_token = 1;           // append the step's k, v and fold its own score in
  const bf16* q;                // [B][Hq][D]
  const bf16* k;                // [B][Hkv][D] (unused without the token)
  const bf16* v;
  bf16* o;                      // [B][Hq][D] (null: not written)
  float* o32 = nullptr;         // [B][Hq][D] float32 rows (null: not written)
  float* lse;                   // [B][Hq]
  float* partA;                 // [B*Hkv][maxp][G][D]
  float* partS;                 // [B*Hkv][maxp][G]
  long long part_rows;          // rows the scratch holds (partS elements)
  unsigned* tickets;            // [B*Hkv] rows folded into parts (kept at 0 between steps)
  int* err;
};


// Release the partials this CTA wrote (ordered before by the consumer barrier,
// cumulatively) and acquire every other CTA's, in one atomic.
SM100_DEV unsigned atom_add_acq_rel_gpu(unsigned* p, unsigned v) {
  unsigned old;
  asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], %2;\n" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}

SM100_DEV void named_sync(int id, int n) { asm volatile("bar.sync %0, %1;\n" ::"r"(id), "r"(n) : "memory"); }

template <int D, bool FP8 = false>
struct DSmem {
  static constexpr int HALF = KS * 128;               // one 64-column half of a bf16 stage tile
  // K (or V) of one stage: 128 rows of bf16, or in FP8 mode 256 rows of E4M3
  // codes (128- or 64-byte swizzled)
  static constexpr int TILE = FP8 ? KS8 * D : KS * D * 2;
  static constexpr int STAGE = 2 * TILE;
  static constexpr int NST = FP8 ? (D == 128 ? 3 : 6) : NSTAGE;
  // FP8 row scales of a stage: 65 groups of 4 floats starting at the group
  // that holds the stage's first row (260 rows >= 256 + 3)
  static constexpr int SCL_QUADS = KS8 / 4 + 1;
  static constexpr int SCL_BYTES = SCL_QUADS * 16;
  static constexpr int SCL_SLOT = 1152;
  static constexpr int SCL = FP8 ? NST * 2 * SCL_SLOT : 0;
  // 4 rows of O per warp per round; also holds the merge weights (<= 16 x 160)
  static constexpr int COMB = NCW * 4 * 128 * 4;
  static constexpr int BYTES = NST * STAGE + SCL + COMB;
};

SM100_DEV uint32_t pack_f16(float lo, float hi) {
  uint32_t d;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;\n" : "=r"(d) : "f"(hi), "f"(lo));
  return d;
}
SM100_DEV uint32_t e4m3x2_to_f16x2(uint32_t two_codes) {
  uint32_t d;
  const uint16_t a = (uint16_t)two_codes;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;\n" : "=r"(d) : "h"(a));
  return d;
}
SM100_DEV uint32_t bf16x2_to_f16x2(uint32_t v) {
  return pack_f16(__uint_as_float(v << 16), __uint_as_float(v & 0xffff0000u));
}
// Offset of 16-byte chunk `chunk` of row `row` in a stage tile of E4M3 codes
// (rows of D bytes) as TMA writes it: 128-byte swizzle for D = 128, 64-byte
// swizzle for D = 64 (chunk index XOR address bits 7..9, resp. 7..8).
template <int D>
SM100_DEV uint32_t sw8(int row, int chunk) {
  return (uint32_t)(row * D + ((chunk ^ (D == 128 ? (row & 7) : ((row >> 1) & 3))) << 4));
}
// Transpose of an 8x8 matrix of 16-bit values held one row pair per thread.
SM100_DEV uint32_t movmatrix_trans(uint32_t x) {
  uint32_t d;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;\n" : "=r"(d) : "r"(x));
  return d;
}
SM100_DEV void mma_f16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

template <int D, bool FP8, int NG>   // NG: blocks of 8 heads per kv group (G <= 8 NG)
__global__ void __launch_bounds__(NTHREADS, 1) decode_kernel(const __grid_constant__ DecodeArgs a) {
  using S = DSmem<D, FP8>;
  constexpr int NH = D / 64;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* scl = smem + S::NST * S::STAGE;                     // [NST][K, V] row scales (FP8)
  float* comb = reinterpret_cast<float*>(scl + S::SCL);         // [NCW][4][D]
  __shared__ __align__(8) uint64_t bar_full[S::NST];
  __shared__ __align__(8) uint64_t bar_empty[S::NST];
  __shared__ StageMeta meta[S::NST];
  __shared__ float wm[NCW][16], wl[NCW][16];
  __shared__ int s_last, abort_s, cons_abort;

  const CacheView& c = a.c;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = c.G;

  if (tid == 0) {
    for (int i = 0; i < S::NST; ++i) {
      mbar_init(smem_u32(&bar_full[i]), 1);
      mbar_init(smem_u32(&bar_empty[i]), NCW);
    }
    abort_s = 0;
    cons_abort = 0;
    fence_barrier_init();
  }
  __syncthreads();
  auto fail = [&]() {
    *(volatile int*)&abort_s = 1;
    atomicExch(a.err, 1);
  };
  auto aborted = [&]() { return *(volatile int*)&abort_s != 0; };

  if (warp == 0) {
    // ------------------------------ TMA producer ------------------------------
    // The CTA's span of the cached rows (all (batch, kv head) pairs bg laid end
    // to end, bg-major) is cut into runs of one bg each.  A run's partial is
    // flushed at the first stage of the next run (or at the terminal stage),
    // whose meta carries the run's bg, partial slot and row count.
    if (elect_one()) {
      prefetch_tmap(&a.tk_ctx);
      prefetch_tmap(&a.tv_ctx);
      prefetch_tmap(&a.tk_q);
      prefetch_tmap(&a.tv_q);
      if (FP8) {
        prefetch_tmap(&a.tk8);
        prefetch_tmap(&a.tv8);
        prefetch_tmap(&a.tkq8);
        prefetch_tmap(&a.tvq8);
        prefetch_tmap(&a.tks);
        prefetch_tmap(&a.tvs);
        prefetch_tmap(&a.tkqs);
        prefetch_tmap(&a.tvqs);
      }
      const long long R = (long long)c.B * c.Hkv * a.rpb;
      long long x = span_start(blockIdx.x, R, a.ncta);
      const long long x1 = span_start(blockIdx.x + 1, R, a.ncta);
      int last_use[S::NST];
      for (int k = 0; k < S::NST; ++k) last_use[k] = -1;
      int run_bg = -1, run_slot = 0, run_rows = 0;
      bool broke = false;
      for (int st = 0;; ++st) {
        const bool have = x < x1;
        int bg = -1, row = 0;
        long long n = 0;
        bool ctx = false;
        if (have) {
          bg = (int)((unsigned)x / (unsigned)a.rpb);
          const long long off = x - (long long)bg * a.rpb + a.skip;   // key index within bg
          const long long run_end = ((long long)bg + 1) * a.rpb < x1 ? ((long long)bg + 1) * a.rpb : x1;
          long long region_end;
          if (off < c.L) {
            const int seg = (int)((unsigned)off / (unsigned)c.b);
            const long long len = seg_len(c, seg);
            region_end = (long long)seg * c.b + len;
            row = (int)((long long)seg * c.B * c.Hkv * c.b + (long long)bg * len + (off - (long long)seg * c.b));
            ctx = true;
          } else {
            region_end = a.rpb + a.skip;
            row = (int)((long long)bg * c.q_cap + (off - c.L));
          }
          n = FP8 ? KS8 : KS;
          if (region_end - off < n) n = region_end - off;
          if (run_end - x < n) n = run_end - x;
        }
        const int slot = st % S::NST, use = st / S::NST;
        if (use > 0 && !mbar_wait(smem_u32(&bar_empty[slot]), (use - 1) & 1)) {
          fail();
          broke = true;
          break;
        }
        if (aborted()) {
          broke = true;
          break;
        }
        const bool new_run = !have || bg != run_bg;
        StageMeta& md = meta[slot];
        md.n = (int)n;
        md.bg = bg;
        md.row0 = row;
        md.flush = (new_run && run_bg >= 0) ? 1 : 0;
        md.end = have ? 0 : 1;
        md.fbg = run_bg;
        md.fslot = run_slot;
        md.frows = run_rows;
        const uint32_t fb = smem_u32(&bar_full[slot]);
        if (!have) {
          mbar_arrive(fb);                          // terminal stage: meta only
          break;
        }
        if (new_run) {
          run_bg = bg;
          run_slot = (int)blockIdx.x - cta_of((long long)bg * a.rpb, R, a.ncta);   // rank among bg's CTAs
          run_rows = 0;
        }
        mbar_arrive_expect_tx(fb, FP8 ? S::STAGE + 2 * S::SCL_BYTES : S::STAGE);
        const uint32_t dst = smem_u32(smem + slot * S::STAGE);
        if (FP8) {
          const uint32_t sd = smem_u32(scl + slot * 2 * S::SCL_SLOT);
          tma_load_2d(dst, ctx ? &a.tk8 : &a.tkq8, 0, row, fb);
          tma_load_2d(dst + S::TILE, ctx ? &a.tv8 : &a.tvq8, 0, row, fb);
          tma_load_2d(sd, ctx ? &a.tks : &a.tkqs, 0, row >> 2, fb);
          tma_load_2d(sd + S::SCL_SLOT, ctx ? &a.tvs : &a.tvqs, 0, row >> 2, fb);
        } else {
          for (int hf = 0; hf < NH; ++hf) {
            tma_load_2d(dst + hf * S::HALF, ctx ? &a.tk_ctx : &a.tk_q, hf * 64, row, fb);
            tma_load_2d(dst + S::TILE + hf * S::HALF, ctx ? &a.tv_ctx : &a.tv_q, hf * 64, row, fb);
          }
        }
        last_use[slot] = use;
        x += n;
        run_rows += (int)n;
      }
      if (broke)
        for (int k = 0; k < S::NST; ++k)
          if (last_use[k] >= 0) mbar_wait(smem_u32(&bar_full[k]), last_use[k] & 1);
    }
    __syncwarp();
    // The new token's row of the query region (row len0, which no reader of
    // this launch touches) and its FP8 copy for the steps after this one,
    // written by the whole warp once its last stage is issued: off the path
    // the step's time depends on.
    if (!aborted() && a.with_token) {
      for (int bg = blockIdx.x; bg < c.B * c.Hkv; bg += a.ncta) {
        const int bb = bg / c.Hkv, g = bg - (bg / c.Hkv) * c.Hkv;
        const long long qo = q_row_offset(c, bb, g, a.len0);
        const uint4* kn = reinterpret_cast<const uint4*>(a.k + (long long)bg * D);
        const uint4* vn = reinterpret_cast<const uint4*>(a.v + (long long)bg * D);
        if (!STAR_STORE_OK(qo + D - 1, (long long)c.B * c.Hkv * c.q_cap * D, a.err)) continue;
        if (lane < D / 8) reinterpret_cast<uint4*>(c.qK + qo)[lane] = kn[lane];
        else if (lane >= 16 && lane < 16 + D / 8) reinterpret_cast<uint4*>(c.qV + qo)[lane - 16] = vn[lane - 16];
        if (FP8) {
          const long long qrow = (long long)bg * c.q_cap + a.len0;
          quantize_row_warp<D>(a.k + (long long)bg * D, c.qK8 + qrow * D, c.qKs + qrow, lane);
          quantize_row_warp<D>(a.v + (long long)bg * D, c.qV8 + qrow * D, c.qVs + qrow, lane);
        }
      }
    }
    return;   // the producer takes part in no named barrier
  }

  // --------------------------------- consumers --------------------------------
  // Keys are the MMA's M dimension: per warp and stage, S^T = K q^T over the
  // warp's 16 keys (M = 16 keys, N = 8 heads of the group per block of NG,
  // K = 16 columns of d) and O^T += V^T P^T (M = 16 rows of d, N = heads,
  // K = the 16 keys).  With G <= 8 every key costs D/16 MMAs each way.
  // Thread (t = lane/4, c = lane%4) holds, per head block nb, the heads
  // g = 8nb + 2c + e (e = 0, 1): scores of keys t and t+8, O^T rows t and t+8
  // of each 16-row block of d, and the running max / sum of those heads.
  constexpr int SL = FP8 ? 2 : 1;                // slices of 16 keys per warp and stage
  constexpr int KPW = 16 * SL;                   // keys per warp and stage
  const int cw = warp - 1;                       // consumer warp 0..7
  const int ctid = tid - 32;                     // 0..255
  const int t4 = lane >> 2, c4 = lane & 3;
  uint32_t qb[D / 16][NG][2];                    // B fragments of q^T
  float oT[D / 16][NG][4];                       // C fragments of O^T
  float mx[NG][2], ls[NG][2];                    // per head: max (log2 units), partial sum
  int cur_bg = -1;
  auto load_q = [&](int bg) {
    const int bb = bg / c.Hkv, g = bg - (bg / c.Hkv) * c.Hkv;
    const bf16* qg = a.q + ((long long)bb * c.Hq + (long long)g * G) * D;
#pragma unroll
    for (int kd = 0; kd < D / 16; ++kd) {
      // FP8 mode permutes the contraction index inside each 16-column step:
      // k-slots 2c, 2c+1 take columns 4c, 4c+1 and k-slots 2c+8, 2c+9 take
      // 4c+2, 4c+3, the order in which one 32-bit word of a key row holds them
      const int col = FP8 ? 16 * kd + 4 * c4 : 16 * kd + 2 * c4;
      const int hi = FP8 ? 2 : 8;
#pragma unroll
      for (int nb = 0; nb < NG; ++nb) {
        const int h = 8 * nb + t4;
        uint32_t b0 = h < G ? *reinterpret_cast<const uint32_t*>(qg + h * D + col) : 0u;
        uint32_t b1 = h < G ? *reinterpret_cast<const uint32_t*>(qg + h * D + col + hi) : 0u;
        if (FP8) {                                 // the FP8 path multiplies in f16
          b0 = bf16x2_to_f16x2(b0);
          b1 = bf16x2_to_f16x2(b1);
        }
        qb[kd][nb][0] = b0;
        qb[kd][nb][1] = b1;
      }
    }
  };
  auto reset_state = [&]() {
#pragma unroll
    for (int m = 0; m < D / 16; ++m)
#pragma unroll
      for (int nb = 0; nb < NG; ++nb) {
        oT[m][nb][0] = oT[m][nb][1] = oT[m][nb][2] = oT[m][nb][3] = 0.f;
        qb[m][nb][0] = qb[m][nb][1] = 0u;
      }
#pragma unroll
    for (int nb = 0; nb < NG; ++nb) {
      mx[nb][0] = mx[nb][1] = -INFINITY;
      ls[nb][0] = ls[nb][1] = 0.f;
    }
  };
  reset_state();

  // Scale and mask the scores of the warp's SL slices of 16 keys (sk[sl][0/1]:
  // factor on the log2 scale of keys kw + 16 sl + t and + t + 8), update the
  // running max / sum per head, turn scores into p.
  auto softmax_update = [&](float (&s)[SL][NG][4], const float (&sk)[SL][2], int kw, int n) {
#pragma unroll
    for (int sl = 0; sl < SL; ++sl) {
      const bool v0 = kw + 16 * sl + t4 < n, v1 = kw + 16 * sl + t4 + 8 < n;
#pragma unroll
      for (int nb = 0; nb < NG; ++nb) {
        s[sl][nb][0] = v0 ? s[sl][nb][0] * sk[sl][0] : -INFINITY;
        s[sl][nb][1] = v0 ? s[sl][nb][1] * sk[sl][0] : -INFINITY;
        s[sl][nb][2] = v1 ? s[sl][nb][2] * sk[sl][1] : -INFINITY;
        s[sl][nb][3] = v1 ? s[sl][nb][3] * sk[sl][1] : -INFINITY;
      }
    }
    float mn[NG][2];
    bool up = false;
#pragma unroll
    for (int nb = 0; nb < NG; ++nb)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        float v = fmaxf(s[0][nb][e], s[0][nb][2 + e]);
#pragma unroll
        for (int sl = 1; sl < SL; ++sl) v = fmaxf(v, fmaxf(s[sl][nb][e], s[sl][nb][2 + e]));
        v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 4));
        v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 8));
        v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 16));
        mn[nb][e] = v;
        up |= v > mx[nb][e] + 8.f;
      }
    // The exponent base only moves up when a head's maximum grows by more
    // than 2^8, so the accumulator is rarely rescaled.
    if (__any_sync(0xffffffffu, up)) {
#pragma unroll
      for (int nb = 0; nb < NG; ++nb)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const bool u = mn[nb][e] > mx[nb][e] + 8.f;
          const float al = u ? exp2f(mx[nb][e] - mn[nb][e]) : 1.f;
          if (u) mx[nb][e] = mn[nb][e];
          ls[nb][e] *= al;
#pragma unroll
          for (int m = 0; m < D / 16; ++m) {
            oT[m][nb][e] *= al;
            oT[m][nb][2 + e] *= al;
          }
        }
    }
#pragma unroll
    for (int nb = 0; nb < NG; ++nb)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const float base = mx[nb][e] == -INFINITY ? 0.f : mx[nb][e];
#pragma unroll
        for (int sl = 0; sl < SL; ++sl) {
          s[sl][nb][e] = exp2f(s[sl][nb][e] - base);
          s[sl][nb][2 + e] = exp2f(s[sl][nb][2 + e] - base);
          ls[nb][e] += s[sl][nb][e] + s[sl][nb][2 + e];
        }
      }
  };

  // P^T as the B operand of O^T += V^T P^T: the score fragment holds keys t,
  // t+8 x heads 2c, 2c+1; a warp transpose of each 8x8 block gives keys 2c,
  // 2c+1 (+8) x head t.  pv0 / pv1 scale keys t / t+8 (FP8: the V row scale).
  auto p_fragments = [&](const float (&s)[NG][4], float pv0, float pv1, uint32_t (&pb)[NG][2]) {
#pragma unroll
    for (int nb = 0; nb < NG; ++nb) {
      const uint32_t x0 = FP8 ? pack_f16(s[nb][0] * pv0, s[nb][1] * pv0) : pack_bf16(s[nb][0], s[nb][1]);
      const uint32_t x1 = FP8 ? pack_f16(s[nb][2] * pv1, s[nb][3] * pv1) : pack_bf16(s[nb][2], s[nb][3]);
      pb[nb][0] = movmatrix_trans(x0);
      pb[nb][1] = movmatrix_trans(x1);
    }
  };

  // One stage of bf16 keys: K and V fragments straight from the
  // 128-byte-swizzled TMA tiles.
  auto bf16_stage = [&](uint32_t kb, uint32_t vb, int kw, int n, int slot) {
    float s[SL][NG][4], s2[NG][4];               // even / odd column steps: two short chains
#pragma unroll
    for (int nb = 0; nb < NG; ++nb)
#pragma unroll
      for (int e = 0; e < 4; ++e) s[0][nb][e] = s2[nb][e] = 0.f;
#pragma unroll
    for (int kd = 0; kd < D / 16; ++kd) {
      uint32_t af[4];
      const int row = kw + (lane & 7) + ((lane >> 3) & 1) * 8;
      const int ch = 2 * kd + (lane >> 4);
      ldmatrix_x4(kb + (ch >> 3) * S::HALF + row * 128 + (((ch & 7) ^ (row & 7)) << 4), af[0], af[1], af[2],
                  af[3]);
#pragma unroll
      for (int nb = 0; nb < NG; ++nb)
        mma_bf16_16816((kd & 1) ? s2[nb] : s[0][nb], af, qb[kd][nb][0], qb[kd][nb][1]);
    }
#pragma unroll
    for (int nb = 0; nb < NG; ++nb)
#pragma unroll
      for (int e = 0; e < 4; ++e) s[0][nb][e] += s2[nb][e];
    float sk[SL][2];
#pragma unroll
    for (int sl = 0; sl < SL; ++sl) sk[sl][0] = sk[sl][1] = a.scale_log2;
    softmax_update(s, sk, kw, n);
    if (kw + 16 > n) {
      // Keys past the stage's valid count carry p = 0, but 0 * NaN is NaN:
      // clear this warp's V rows there (bytes past the end of a buffer need
      // not be finite).  Each warp reads only its own 16 V rows.
      for (int i = lane; i < 16 * (D / 8); i += 32) {
        const int row = kw + i / (D / 8), ch = i % (D / 8);
        if (row >= n) {
          uint8_t* dst = smem + slot * S::STAGE + S::TILE + (ch >> 3) * S::HALF + row * 128 +
                         (((ch & 7) ^ (row & 7)) << 4);
          *reinterpret_cast<uint4*>(dst) = make_uint4(0u, 0u, 0u, 0u);
        }
      }
      __syncwarp();
    }
    uint32_t pb[NG][2];
    p_fragments(s[0], 1.f, 1.f, pb);
#pragma unroll
    for (int m = 0; m < D / 16; ++m) {
      uint32_t af[4];
      const int row = kw + (lane & 7) + ((lane >> 4) << 3);
      const int ch = 2 * m + ((lane >> 3) & 1);
      ldmatrix_x4_trans(vb + (ch >> 3) * S::HALF + row * 128 + (((ch & 7) ^ (row & 7)) << 4), af[0], af[1],
                        af[2], af[3]);
#pragma unroll
      for (int nb = 0; nb < NG; ++nb) mma_bf16_16816(oT[m][nb], af, pb[nb][0], pb[nb][1]);
    }
    // generic-proxy writes above must be ordered before the next TMA write
    if (kw + 16 > n) fence_proxy_async_smem();
  };

  // One stage in FP8 mode (context segments and query region alike); each
  // warp takes SL = 2 slices of 16 keys (kw + 16 sl ...), whose softmax shares
  // one reduction.  ldmatrix on the swizzled byte tile gives each thread one
  // 32-bit word (4 codes) per 8x16-byte matrix, converted in registers to f16
  // MMA operands.  For K the word holds 4 columns of one key, the A fragment
  // under the permuted contraction order of q.  For V (.trans) it holds 2 keys
  // x 2 columns; a byte permute regroups it into key pairs, and the rows of
  // each 16-row block of O^T follow: row t <-> d = 16m + 2t, row t+8 <->
  // d = 16m + 2t + 1.  Per-row scales: K's on the score, V's on p.
  auto fp8_stage = [&](const StageMeta& m, uint32_t kb, uint32_t vb, const uint8_t* sclp, int kw, int n) {
    float s[SL][NG][4], s2[SL][NG][4];
#pragma unroll
    for (int sl = 0; sl < SL; ++sl)
#pragma unroll
      for (int nb = 0; nb < NG; ++nb)
#pragma unroll
        for (int e = 0; e < 4; ++e) s[sl][nb][e] = s2[sl][nb][e] = 0.f;
#pragma unroll
    for (int sl = 0; sl < SL; ++sl) {
      const int k0 = kw + 16 * sl;
#pragma unroll
      for (int jp = 0; jp < D / 32; ++jp) {
        const int row = k0 + (lane & 7) + ((lane >> 3) & 1) * 8;
        uint32_t r0, r1, r2, r3;
        ldmatrix_x4(kb + sw8<D>(row, 2 * jp + (lane >> 4)), r0, r1, r2, r3);
        const uint32_t af0[4] = {e4m3x2_to_f16x2(r0), e4m3x2_to_f16x2(r1), e4m3x2_to_f16x2(r0 >> 16),
                                 e4m3x2_to_f16x2(r1 >> 16)};
        const uint32_t af1[4] = {e4m3x2_to_f16x2(r2), e4m3x2_to_f16x2(r3), e4m3x2_to_f16x2(r2 >> 16),
                                 e4m3x2_to_f16x2(r3 >> 16)};
#pragma unroll
        for (int nb = 0; nb < NG; ++nb) {
          mma_f16_16816(s[sl][nb], af0, qb[2 * jp][nb][0], qb[2 * jp][nb][1]);
          mma_f16_16816(s2[sl][nb], af1, qb[2 * jp + 1][nb][0], qb[2 * jp + 1][nb][1]);
        }
      }
    }
#pragma unroll
    for (int sl = 0; sl < SL; ++sl)
#pragma unroll
      for (int nb = 0; nb < NG; ++nb)
#pragma unroll
        for (int e = 0; e < 4; ++e) s[sl][nb][e] += s2[sl][nb][e];
    // scales: a box of 4-row groups from the group holding row0
    const float* sks = reinterpret_cast<const float*>(sclp) + (m.row0 & 3);
    const float* svs = reinterpret_cast<const float*>(sclp + S::SCL_SLOT) + (m.row0 & 3);
    float sk[SL][2];
#pragma unroll
    for (int sl = 0; sl < SL; ++sl) {
      const int k0 = kw + 16 * sl + t4;
      sk[sl][0] = a.scale_log2 * sks[k0];
      sk[sl][1] = a.scale_log2 * sks[k0 + 8];
    }
    softmax_update(s, sk, kw, n);
#pragma unroll
    for (int sl = 0; sl < SL; ++sl) {
      const int k0 = kw + 16 * sl;
      uint32_t pb[NG][2];
      p_fragments(s[sl], svs[k0 + t4], svs[k0 + t4 + 8], pb);
#pragma unroll
      for (int jp = 0; jp < D / 32; ++jp) {
        const int row = k0 + (lane & 7) + ((lane >> 3) & 1) * 8;
        uint32_t r0, r1, r2, r3;
        ldmatrix_x4_trans(vb + sw8<D>(row, 2 * jp + (lane >> 4)), r0, r1, r2, r3);
        // r0: keys 2c, 2c+1 x columns 2t, 2t+1 of chunk 2jp; r1: keys 2c+8, 2c+9;
        // r2, r3: the same of chunk 2jp+1.  Regroup to key pairs per column.
        const uint32_t p0 = __byte_perm(r0, 0u, 0x3120), p1 = __byte_perm(r1, 0u, 0x3120);
        const uint32_t p2 = __byte_perm(r2, 0u, 0x3120), p3 = __byte_perm(r3, 0u, 0x3120);
        const uint32_t af0[4] = {e4m3x2_to_f16x2(p0), e4m3x2_to_f16x2(p0 >> 16), e4m3x2_to_f16x2(p1),
                                 e4m3x2_to_f16x2(p1 >> 16)};
        const uint32_t af1[4] = {e4m3x2_to_f16x2(p2), e4m3x2_to_f16x2(p2 >> 16), e4m3x2_to_f16x2(p3),
                                 e4m3x2_to_f16x2(p3 >> 16)};
#pragma unroll
        for (int nb = 0; nb < NG; ++nb) {
          mma_f16_16816(oT[2 * jp][nb], af0, pb[nb][0], pb[nb][1]);
          mma_f16_16816(oT[2 * jp + 1][nb], af1, pb[nb][0], pb[nb][1]);
        }
      }
    }
  };

  // [B*Hkv] cached rows of each (batch, kv head) folded into parts: the CTA
  // that completes rpb rows merges
  unsigned* const done = a.tickets;

  // ---- merge of bg's parts: one per CTA whose span holds rows of bg (slots
  // 0..nspan-1), and the new token.  A thread owns one float4 column of one
  // row and every npg-th part: it loads their A_h and s_h together with its
  // slices of q, k and v (one round trip), folds the parts with a running
  // maximum, and the npg threads of a column combine through shared memory.
  // The row's D/4 consecutive threads (one warp, or half of one at D = 64)
  // sum q.k by shuffles; the npg == 0 thread folds the new token in. -------
  auto merge_bg = [&](int bg) {
    const int bb = bg / c.Hkv, g = bg - (bg / c.Hkv) * c.Hkv;
    const long long R = (long long)c.B * c.Hkv * a.rpb;
    const int nspan = cta_of((long long)bg * a.rpb + a.rpb - 1, R, a.ncta) - cta_of((long long)bg * a.rpb, R, a.ncta) + 1;
    const int cnt = nspan;
    const bool tok = a.with_token != 0;
    const bf16* kn = tok ? a.k + (long long)bg * D : nullptr;
    const bf16* vn = tok ? a.v + (long long)bg * D : nullptr;
    constexpr int NT = 32 * NCW;
    constexpr int KMAX = 11;
    const int nout = G * (D / 4);
    float4* red = reinterpret_cast<float4*>(comb);             // [npg][nb] partial sums
    float* redm = comb + 4 * NT;                               // [npg][nb] their maxima
    float* redl = redm + NT;                                   // [npg][nb] their sums
    for (int ob = 0; ob < nout; ob += NT) {
      const int nb = nout - ob < NT ? nout - ob : NT;
      const int npg = NT / nb;
      const bool active = ctid < nb * npg;
      const int oi = ob + ctid % nb, pg = ctid / nb;
      const int r = oi / (D / 4), d4 = oi - (oi / (D / 4)) * (D / 4);
      const float4* pa = reinterpret_cast<const float4*>(a.partA + ((long long)bg * a.maxp * G + r) * D) + d4;
      const float* ps = a.partS + (long long)bg * a.maxp * G + r;
      const long long pstride = (long long)G * D / 4;
      float M = -INFINITY, L = 0.f;
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
      // the new token: this thread's 4 elements of q_r . k, and of v
      uint2 q2 = make_uint2(0u, 0u), k2 = make_uint2(0u, 0u), v2 = make_uint2(0u, 0u);
      if (active && tok) {
        q2 = *reinterpret_cast<const uint2*>(a.q + ((long long)bb * c.Hq + (long long)g * G + r) * D + 4 * d4);
        k2 = *reinterpret_cast<const uint2*>(kn + 4 * d4);
        v2 = *reinterpret_cast<const uint2*>(vn + 4 * d4);
      }
      for (int p0 = 0; p0 < cnt; p0 += KMAX * npg) {
        float4 v[KMAX];
        float sp[KMAX];
#pragma unroll
        for (int k = 0; k < KMAX; ++k) {
          const int p = p0 + pg + k * npg;
          const bool ok = active && p < cnt;
          v[k] = ok ? __ldcg(pa + p * pstride) : make_float4(0.f, 0.f, 0.f, 0.f);
          sp[k] = ok ? __ldcg(ps + (long long)p * G) : -INFINITY;
        }
        float Mn = M;
#pragma unroll
        for (int k = 0; k < KMAX; ++k) Mn = fmaxf(Mn, sp[k]);
        if (Mn != -INFINITY) {
          const float al = M == -INFINITY ? 0.f : __expf(M - Mn);
          L *= al;
          acc.x *= al;
          acc.y *= al;
          acc.z *= al;
          acc.w *= al;
#pragma unroll
          for (int k = 0; k < KMAX; ++k) {
            const float wk = sp[k] == -INFINITY ? 0.f : __expf(sp[k] - Mn);
            L += wk;
            acc.x += wk * v[k].x;
            acc.y += wk * v[k].y;
            acc.z += wk * v[k].z;
            acc.w += wk * v[k].w;
          }
          M = Mn;
        }
      }
      // (every thread takes part in the shuffles: the groups of D/4 threads are
      // wholly active or wholly idle, nb * npg being a multiple of D/4)
      float qk = __uint_as_float(q2.x << 16) * __uint_as_float(k2.x << 16) +
                 __uint_as_float(q2.x & 0xffff0000u) * __uint_as_float(k2.x & 0xffff0000u) +
                 __uint_as_float(q2.y << 16) * __uint_as_float(k2.y << 16) +
                 __uint_as_float(q2.y & 0xffff0000u) * __uint_as_float(k2.y & 0xffff0000u);
#pragma unroll
      for (int off = D / 8; off > 0; off >>= 1) qk += __shfl_xor_sync(0xffffffffu, qk, off);
      if (active && pg == 0 && tok) {
        const float sn = qk * a.scale_log2 * kLn2;  // natural-log units, like s_h
        const float Mn = fmaxf(M, sn);
        const float al = M == -INFINITY ? 0.f : __expf(M - Mn);
        const float wk = __expf(sn - Mn);
        L = L * al + wk;
        acc.x = acc.x * al + wk * __uint_as_float(v2.x << 16);
        acc.y = acc.y * al + wk * __uint_as_float(v2.x & 0xffff0000u);
        acc.z = acc.z * al + wk * __uint_as_float(v2.y << 16);
        acc.w = acc.w * al + wk * __uint_as_float(v2.y & 0xffff0000u);
        M = Mn;
      }
      if (active) {
        red[pg * nb + (oi - ob)] = acc;
        redm[pg * nb + (oi - ob)] = M;
        redl[pg * nb + (oi - ob)] = L;
      }
      named_sync(1, NT);
      if (active && pg == 0) {
        float Mt = M;
        for (int q2 = 1; q2 < npg; ++q2) Mt = fmaxf(Mt, redm[q2 * nb + (oi - ob)]);
        float Lt = 0.f;
        float4 at = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int q2 = 0; q2 < npg; ++q2) {
          const float mq = redm[q2 * nb + (oi - ob)];
          const float f = mq == -INFINITY ? 0.f : __expf(mq - Mt);
          const float4 u = red[q2 * nb + (oi - ob)];
          Lt += f * redl[q2 * nb + (oi - ob)];
          at.x += f * u.x;
          at.y += f * u.y;
          at.z += f * u.z;
          at.w += f * u.w;
        }
        const float inv = Lt > 0.f ? 1.f / Lt : 0.f;
        const long long orow = (long long)bb * c.Hq + (long long)g * G + r;
        // (no early exit here: every consumer thread must reach the barrier below)
        if (STAR_STORE_OK(orow, (long long)c.B * c.Hq, a.err)) {
          if (a.o) {
            uint2 pk;
            pk.x = pack_bf16(at.x * inv, at.y * inv);
            pk.y = pack_bf16(at.z * inv, at.w * inv);
            *reinterpret_cast<uint2*>(a.o + orow * D + 4 * d4) = pk;
          }
          if (a.o32)
            *reinterpret_cast<float4*>(a.o32 + orow * D + 4 * d4) =
                make_float4(at.x * inv, at.y * inv, at.z * inv, at.w * inv);
          if (d4 == 0) a.lse[orow] = Lt > 0.f ? Mt + __logf(Lt) : -INFINITY;
        }
      }
      named_sync(1, NT);
    }
    if (ctid == 0) done[bg] = 0u;                  // ready for the next step
  };

  // ---- rows of bg now live in partials: count them; the CTA that completes
  // bg merges.  The barrier orders every consumer's partial stores before
  // thread 0's gpu-scope release (cumulative), which precedes the count.
  auto complete = [&](int bg, int rows) {
    named_sync(1, 32 * NCW);
    if (ctid == 0)
      s_last = atom_add_acq_rel_gpu(&done[bg], (unsigned)rows) + (unsigned)rows == (unsigned)a.rpb;
    named_sync(1, 32 * NCW);
    if (s_last) merge_bg(bg);
  };

  // ---- flush: this CTA's run of bg becomes part `pslot` ---------------------
  auto flush_run = [&](int bg, int pslot, int rows) {
#pragma unroll
    for (int nb = 0; nb < NG; ++nb)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        float v = ls[nb][e];
        v += __shfl_xor_sync(0xffffffffu, v, 4);
        v += __shfl_xor_sync(0xffffffffu, v, 8);
        v += __shfl_xor_sync(0xffffffffu, v, 16);
        ls[nb][e] = v;
      }
    if (t4 == 0) {
#pragma unroll
      for (int nb = 0; nb < NG; ++nb)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          wm[cw][8 * nb + 2 * c4 + e] = mx[nb][e];
          wl[cw][8 * nb + 2 * c4 + e] = ls[nb][e];
        }
    }
    for (int rh = 0; rh < G; rh += 4) {            // heads rh .. rh+3 per round
#pragma unroll
      for (int mb = 0; mb < D / 16; ++mb)
#pragma unroll
        for (int nb = 0; nb < NG; ++nb)
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int h = 8 * nb + 2 * c4 + e;
            // rows t, t+8 of O^T block mb (FP8 mode: permuted, see fp8_stage)
            const int d0 = FP8 ? 16 * mb + 2 * t4 : 16 * mb + t4;
            const int d1 = FP8 ? d0 + 1 : d0 + 8;
            if (h >= rh && h < rh + 4) {
              comb[(cw * 4 + h - rh) * D + d0] = oT[mb][nb][e];
              comb[(cw * 4 + h - rh) * D + d1] = oT[mb][nb][2 + e];
            }
          }
      named_sync(1, 32 * NCW);
      const int nrow = G - rh < 4 ? G - rh : 4;
      for (int idx = ctid; idx < nrow * D; idx += 32 * NCW) {
        const int r = idx / D, d = idx - (idx / D) * D, rr = rh + r;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < NCW; ++w) M = fmaxf(M, wm[w][rr]);
        const float base = M == -INFINITY ? 0.f : M;
        float Ls = 0.f, acc = 0.f;
#pragma unroll
        for (int w = 0; w < NCW; ++w) {
          const float f = exp2f(wm[w][rr] - base);
          Ls += f * wl[w][rr];
          acc += f * comb[(w * 4 + r) * D + d];
        }
        const long long pr = ((long long)bg * a.maxp + pslot) * G + rr;
        if (!STAR_STORE_OK(pr, a.part_rows, a.err) || !STAR_STORE_OK(pslot, a.maxp, a.err)) continue;
        a.partA[pr * D + d] = Ls > 0.f ? acc / Ls : 0.f;
        if (d == 0) a.partS[pr] = Ls > 0.f ? (base + log2f(Ls)) * kLn2 : -INFINITY;
      }
      named_sync(1, 32 * NCW);
    }
    reset_state();                             // the run's state now lives in the partial
    cur_bg = -1;
    complete(bg, rows);
  };

  // Warm L2 with the step's q, k and v rows of every (batch, kv head) this
  // CTA's span touches: the flush cleared them out, and whichever CTA merges a
  // pair reads them right after its last stage, on the step's critical path.
  {
    const long long R = (long long)c.B * c.Hkv * a.rpb;
    const long long x0 = span_start(blockIdx.x, R, a.ncta), x1 = span_start(blockIdx.x + 1, R, a.ncta);
    if (x1 > x0) {
      const int bg0 = (int)((unsigned)x0 / (unsigned)a.rpb), bg1 = (int)((unsigned)(x1 - 1) / (unsigned)a.rpb);
      constexpr int kLine = 128;                       // bytes per L2 prefetch
      const int q_lines = G * D * 2 / kLine, kv_lines = D * 2 / kLine;
      const int per_bg = q_lines + (a.with_token ? 2 * kv_lines : 0);
      for (int i = ctid; i < (bg1 - bg0 + 1) * per_bg; i += 32 * NCW) {
        const int bg = bg0 + i / per_bg, l = i % per_bg;
        const int bb = bg / c.Hkv, g = bg - (bg / c.Hkv) * c.Hkv;
        const char* p = l < q_lines
                            ? reinterpret_cast<const char*>(a.q + ((long long)bb * c.Hq + (long long)g * G) * D) + l * kLine
                            : reinterpret_cast<const char*>((l - q_lines < kv_lines ? a.k : a.v) + (long long)bg * D) +
                                  ((l - q_lines) % kv_lines) * kLine;
        asm volatile("prefetch.global.L2 [%0];\n" ::"l"(p));
      }
    }
  }

  for (int st = 0;; ++st) {
    const int slot = st % S::NST, use = st / S::NST;
    // every consumer warp takes the same path: a warp whose bounded wait gave
    // up says so before the barrier, and all of them stop after it
    if (!mbar_wait(smem_u32(&bar_full[slot]), use & 1)) {
      fail();
      if (lane == 0) cons_abort = 1;
    }
    named_sync(2, 32 * NCW);
    if (cons_abort) break;
    const StageMeta m = meta[slot];
    if (m.flush) flush_run(m.fbg, m.fslot, m.frows);
    if (m.end) break;
    if (m.bg != cur_bg) {
      load_q(m.bg);
      cur_bg = m.bg;
    }
    const uint32_t kb = smem_u32(smem + slot * S::STAGE);
    const uint32_t vb = kb + S::TILE;
    const int kw = KPW * cw;   // first key of this warp in the stage
    if (kw < m.n) {            // a warp past the stage's valid keys adds nothing
      if constexpr (FP8) fp8_stage(m, kb, vb, scl + slot * 2 * S::SCL_SLOT, kw, m.n);
      else bf16_stage(kb, vb, kw, m.n, slot);
    }
    if (lane == 0) mbar_arrive(smem_u32(&bar_empty[slot]));
  }
}

}  // namespace

void decode_parts(const CacheView& c, long long len0, const DecodePlan& pl, std::vector<DecodePart>& out) {
  out.clear();
  const long long rpb = c.L + len0;
  const long long R = (long long)c.B * c.Hkv * rpb;
  for (int bg = 0; bg < c.B * c.Hkv; ++bg) {
    const long long lo = (long long)bg * rpb, hi = lo + rpb;
    const int c0 = cta_of(lo, R, pl.ncta), c1 = cta_of(hi - 1, R, pl.ncta);
    for (int i = c0; i <= c1; ++i) {
      const long long x0 = std::max(lo, span_start(i, R, pl.ncta));
      const long long x1 = std::min(hi, span_start(i + 1, R, pl.ncta));
      out.push_back({bg, i - c0, x0 - lo, x1 - lo});
    }
  }
}

int decode_max_partials(const CacheView& c, int ncta) {
  // spans that can touch one (batch, kv head): ceil(ncta / (B * Hkv)), one
  // more where a span straddles two of them, and spare slots
  const int bgs = c.B * c.Hkv;
  return (ncta + bgs - 1) / bgs + 3;
}

DecodePlan decode_plan(const CacheView& c, long long len0, int num_sms, long long skip) {
  DecodePlan pl;
  long long n = (long long)c.B * c.Hkv * (c.L - skip + len0) / 512;   // at least 512 cached rows per CTA
  if (n < 1) n = 1;
  if (n > num_sms) n = num_sms;
  // A whole number of CTAs per (batch, kv head), if that idles at most 4 % of
  // the SMs: no span then crosses from one (batch, kv head) into the next,
  // which would cost it a second flush.
  const long long bgs = (long long)c.B * c.Hkv;
  const long long aligned = n / bgs * bgs;
  if (n == num_sms && aligned > 0 && aligned * 25 >= n * 24) n = aligned;
  pl.ncta = (int)n;
  pl.maxp = decode_max_partials(c, pl.ncta);
  return pl;
}

const char* decode_make_maps(const CacheView& c, DecodeMaps* m) {
  const unsigned long long ctx_rows = (unsigned long long)c.B * c.Hkv * c.L;
  const unsigned long long q_rows = (unsigned long long)c.B * c.Hkv * c.q_cap;
  if (!make_tmap_bf16_2d(&m->k_ctx, c.ctxK, ctx_rows, c.D, KS, 64) ||
      !make_tmap_bf16_2d(&m->v_ctx, c.ctxV, ctx_rows, c.D, KS, 64))
    return "context K/V";
  if (!make_tmap_bf16_2d(&m->k_q, c.qK, q_rows, c.D, KS, 64) ||
      !make_tmap_bf16_2d(&m->v_q, c.qV, q_rows, c.D, KS, 64))
    return "query region K/V";
  if (!c.ctxK8) return nullptr;
  if (!make_tmap_u8_2d(&m->k8_ctx, c.ctxK8, ctx_rows, c.D, KS8) ||
      !make_tmap_u8_2d(&m->v8_ctx, c.ctxV8, ctx_rows, c.D, KS8))
    return "FP8 context K/V";
  // the scale arrays are padded (with zeros) to whole groups of 4 rows
  if (!make_tmap_f32_quads(&m->ks_ctx, c.ctxKs, (ctx_rows + 3) / 4, DSmem<128, true>::SCL_QUADS) ||
      !make_tmap_f32_quads(&m->vs_ctx, c.ctxVs, (ctx_rows + 3) / 4, DSmem<128, true>::SCL_QUADS))
    return "FP8 row scales";
  if (!make_tmap_u8_2d(&m->k8_q, c.qK8, q_rows, c.D, KS8) ||
      !make_tmap_u8_2d(&m->v8_q, c.qV8, q_rows, c.D, KS8))
    return "FP8 query region K/V";
  if (!make_tmap_f32_quads(&m->ks_q, c.qKs, (q_rows + 3) / 4, DSmem<128, true>::SCL_QUADS) ||
      !make_tmap_f32_quads(&m->vs_q, c.qVs, (q_rows + 3) / 4, DSmem<128, true>::SCL_QUADS))
    return "FP8 query region row scales";
  return nullptr;
}

template <int D, bool FP8>
cudaError_t decode_prepare_one() {
  cudaError_t e = cudaFuncSetAttribute(decode_kernel<D, FP8, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       DSmem<D, FP8>::BYTES + 1024);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(decode_kernel<D, FP8, 2>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             DSmem<D, FP8>::BYTES + 1024);
  return e;
}

cudaError_t decode_prepare(int D) {
  cudaError_t e = D == 128 ? decode_prepare_one<128, false>() : decode_prepare_one<64, false>();
  if (e == cudaSuccess) e = D == 128 ? decode_prepare_one<128, true>() : decode_prepare_one<64, true>();
  return e;
}

template <int D, bool FP8>
void launch_decode_kernel(const DecodeArgs& a, int G, int ncta, cudaStream_t st) {
  if (G <= 8)
    decode_kernel<D, FP8, 1><<<ncta, NTHREADS, DSmem<D, FP8>::BYTES + 1024, st>>>(a);
  else
    decode_kernel<D, FP8, 2><<<ncta, NTHREADS, DSmem<D, FP8>::BYTES + 1024, st>>>(a);
}

cudaError_t launch_decode_step(const CacheView& c, const DecodeMaps& maps, float scale, int len0,
                               const bf16* q, const bf16* k, const bf16* v, bf16* o, float* lse,
                               const DecodePlan& plan, const Scratch& s, cudaStream_t st, long long skip,
                               bool with_token, float* o32) {
  if (skip < 0 || skip > c.L || c.L - skip + len0 < 1) return cudaErrorInvalidValue;
  DecodeArgs a;
  a.tk_ctx = maps.k_ctx;
  a.tv_ctx = maps.v_ctx;
  a.tk_q = maps.k_q;
  a.tv_q = maps.v_q;
  a.tk8 = maps.k8_ctx;
  a.tv8 = maps.v8_ctx;
  a.tkq8 = maps.k8_q;
  a.tvq8 = maps.v8_q;
  a.tks = maps.ks_ctx;
  a.tvs = maps.vs_ctx;
  a.tkqs = maps.ks_q;
  a.tvqs = maps.vs_q;
  a.c = c;
  a.scale_log2 = scale * kLog2e;
  a.len0 = len0;
  a.ncta = plan.ncta;
  a.maxp = plan.maxp;
  a.rpb = c.L - skip + len0;
  a.skip = skip;
  a.with_token = with_token ? 1 : 0;
  a.o32 = o32;
  a.q = q;
  a.k = k;
  a.v = v;
  a.o = o;
  a.lse = lse;
  a.partA = s.partA;
  a.partS = s.partS;
  a.part_rows = s.partS_elems;
  a.tickets = s.tickets;
  a.err = s.err;
  const bool fp8 = c.ctxK8 != nullptr;
  if (c.D == 128 && fp8)
    launch_decode_kernel<128, true>(a, c.G, plan.ncta, st);
  else if (c.D == 128)
    launch_decode_kernel<128, false>(a, c.G, plan.ncta, st);
  else if (fp8)
    launch_decode_kernel<64, true>(a, c.G, plan.ncta, st);
  else
    launch_decode_kernel<64, false>(a, c.G, plan.ncta, st);
  return cudaGetLastError();
}

}  // namespace star

// ===========================================================================
// Allocation-free decode step.
//
// Some callers cannot allocate device memory when they run a step: a runtime
// that owns every byte of the GPU through its own pool, or a caller that must
// not touch the CUDA allocator on its serving path.  For them the decode step
// below takes the KV cache as caller-owned buffers and keeps its own split-KV
// scratch (partials, merge tickets, error word) in one file-scope device
// array, reserved when the library is loaded on a GPU and held until exit.
// ===========================================================================
namespace star {
int check_params(const star_params* p);
namespace {

constexpr long long kNoAllocPartA = 1LL << 20;    // floats of partial outputs (4 MiB)
constexpr long long kNoAllocPartS = 1LL << 14;    // floats of partial log-sum-exps (64 KiB)
constexpr long long kNoAllocTickets = 1024;       // merge counters (one per batch x kv head)
constexpr long long kNoAllocFloats = kNoAllocPartA + kNoAllocPartS + kNoAllocTickets + 64;

static __device__ __align__(256) float g_noalloc_scratch[kNoAllocFloats];

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
float* g_noalloc_addr[kMaxDevices];
int g_noalloc_sms[kMaxDevices];

// Device address of the static scratch on `dev` (the current device), looked
// up once per device: in host code the array's name is only a host-side
// stand-in, never a device address.
cudaError_t noalloc_setup(int dev, float** addr, int* sms) {
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_noalloc_addr[dev]) {
    void* p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    int n = 0;
    e = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    e = decode_prepare(64);
    if (e == cudaSuccess) e = decode_prepare(128);
    if (e != cudaSuccess) return e;
    g_noalloc_sms[dev] = n;
    g_noalloc_addr[dev] = static_cast<float*>(p);
  }
  *addr = g_noalloc_addr[dev];
  *sms = g_noalloc_sms[dev];
  return cudaSuccess;
}

}  // namespace
}  // namespace star

extern "C" STAR_API int star_decode_step_noalloc(const star_params* p, long long q_len,
                                                 const void* ctx_k, const void* ctx_v, void* q_k,
                                                 void* q_v, const void* q, const void* k,
                                                 const void* v, void* o, float* lse, void* stream) {
  using namespace star;
  int rc = check_params(p);
  if (rc) return rc;
  if (p->kv_fp8) return set_error(STAR_EINVAL, "the no-alloc decode streams bf16 only (kv_fp8 must be 0)");
  if (!ctx_k || !ctx_v || !q_k || !q_v || !q || !k || !v || !o || !lse)
    return set_error(STAR_EINVAL, "NULL tensor pointer");
  const void* ptrs[] = {ctx_k, ctx_v, q_k, q_v, q, k, v, o, lse};
  for (const void* x : ptrs)
    if (reinterpret_cast<uintptr_t>(x) & 15u) return set_error(STAR_EINVAL, "tensor pointers must be 16-byte aligned");
  if (q_len < 0) return set_error(STAR_EINVAL, "q_len must be >= 0");
  if (q_len + 1 > p->q_cap) return set_error(STAR_ENOSPC, "query region full");
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess || dev < 0 || dev >= kMaxDevices) return set_error(STAR_ECUDA, "cudaGetDevice failed");
  float* base = nullptr;
  int sms = 0;
  e = noalloc_setup(dev, &base, &sms);
  if (e != cudaSuccess) return set_error(STAR_ECUDA, cudaGetErrorString(e));

  CacheView c;
  c.B = p->B; c.Hq = p->Hq; c.Hkv = p->Hkv; c.D = p->D; c.G = p->Hq / p->Hkv;
  c.L = p->L; c.b = p->block; c.b_a = p->anchor;
  c.n_seg = (int)((p->L + p->block - 1) / p->block);
  c.q_cap = p->q_cap;
  c.ctxK = static_cast<bf16*>(const_cast<void*>(ctx_k));
  c.ctxV = static_cast<bf16*>(const_cast<void*>(ctx_v));
  c.qK = static_cast<bf16*>(q_k);
  c.qV = static_cast<bf16*>(q_v);
  c.ctxK8 = nullptr;
  c.ctxV8 = nullptr;
  c.ctxKs = nullptr;
  c.ctxVs = nullptr;
  c.qK8 = nullptr;
  c.qV8 = nullptr;
  c.qKs = nullptr;
  c.qVs = nullptr;
  c.err = nullptr;

  const DecodePlan pl = decode_plan(c, q_len, sms);
  const long long rows = (long long)c.B * c.Hkv * pl.maxp * c.G;
  if (rows * c.D > kNoAllocPartA || rows > kNoAllocPartS || (long long)c.B * c.Hkv > kNoAllocTickets)
    return set_error(STAR_EINVAL, "problem too large for the static decode scratch "
                                  "(B*Hkv*G*D*(ceil(SMs/(B*Hkv))+3) must be <= 1048576 floats, "
                                  "B*Hkv <= 1024)");
  DecodeMaps maps;
  if (const char* bad = decode_make_maps(c, &maps)) {
    char msg[96];
    snprintf(msg, sizeof(msg), "TMA tensor map rejected by the driver: %s", bad);
    return set_error(STAR_EINVAL, msg);
  }
  Scratch sc;
  c.err = reinterpret_cast<int*>(base + kNoAllocPartA + kNoAllocPartS + kNoAllocTickets);
  sc.partA = base;
  sc.partS = base + kNoAllocPartA;
  sc.tickets = reinterpret_cast<unsigned*>(base + kNoAllocPartA + kNoAllocPartS);
  sc.err = reinterpret_cast<int*>(base + kNoAllocPartA + kNoAllocPartS + kNoAllocTickets);
  sc.partA_elems = kNoAllocPartA;
  sc.partS_elems = kNoAllocPartS;
  sc.n_tickets = (int)kNoAllocTickets;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // the merge tickets must start at zero (a step that gave up a wait may have
  // left some behind); the error word next to them is left as it is, so an
  // abandoned wait stays visible until star_noalloc_device_error reads it
  e = cudaMemsetAsync(sc.tickets, 0, kNoAllocTickets * sizeof(unsigned), st);
  if (e == cudaSuccess)
    e = launch_decode_step(c, maps, p->scale > 0.f ? p->scale : 1.0f / sqrtf((float)p->D), (int)q_len,
                           static_cast<const bf16*>(q), static_cast<const bf16*>(k),
                           static_cast<const bf16*>(v), static_cast<bf16*>(o), lse, pl, sc, st);
  if (e != cudaSuccess) return set_error(STAR_ECUDA, cudaGetErrorString(e));
  return STAR_OK;
}

// Reads and clears the error word of the static decode scratch on the current
// device, after the work already queued on `stream`.
extern "C" STAR_API int star_noalloc_device_error(int* flag, void* stream) {
  using namespace star;
  if (!flag) return set_error(STAR_EINVAL, "flag is NULL");
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess || dev < 0 || dev >= kMaxDevices) return set_error(STAR_ECUDA, "cudaGetDevice failed");
  float* base = nullptr;
  int sms = 0;
  e = noalloc_setup(dev, &base, &sms);
  if (e != cudaSuccess) return set_error(STAR_ECUDA, cudaGetErrorString(e));
  unsigned* tickets = reinterpret_cast<unsigned*>(base + kNoAllocPartA + kNoAllocPartS);
  int* err = reinterpret_cast<int*>(base + kNoAllocPartA + kNoAllocPartS + kNoAllocTickets);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int h = 0;
  e = cudaMemcpyAsync(&h, err, sizeof(int), cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e == cudaSuccess && h) e = cudaMemsetAsync(err, 0, sizeof(int), st);
  if (e == cudaSuccess && h) e = cudaMemsetAsync(tickets, 0, kNoAllocTickets * sizeof(unsigned), st);
  if (e == cudaSuccess && h) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return set_error(STAR_ECUDA, cudaGetErrorString(e));
  *flag = h;
  return STAR_OK;
}
