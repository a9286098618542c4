// Tensor-core attention tile kernel for sm_100a (tcgen05 + TMEM + TMA),
// warp-specialised.  Two operations share it:
//
// * Phase-1 context encoding -- "Star Attention: Efficient LLM Inference over
//   Long Sequences" (analysis page), section 3.4, "Phase 1: Context Encoding
//   with Anchor Blocks": block i >= 1 is prefixed with the anchor and encoded
//   with causal attention over [anchor | block i] (Steps 2 and 4); block 0 is
//   encoded on its own; only the block's own K/V is kept in the cache (Step
//   5).  The augmented block is never materialised: a CTA streams the anchor's
//   K/V tiles [0, b_a) with no mask and then its own block's tiles up to the
//   diagonal with a causal mask.  CTA work item: one 128-row query tile of one
//   block for TWO q heads of the same kv group (GQA), so each K/V tile fetched
//   by TMA feeds two S = Q K^T and two O += P V MMAs; both heads share the mask.
// * Phase-2 query prefill -- same page, "Phase 2: Query Encoding and Token
//   Generation with Distributed Softmax", Step 3: the query rows attend to one
//   key chunk (a slice of a context segment, fully visible, or the query
//   region, causal) and leave that chunk's local (A_h, s_h) in fp32 for the
//   merge (Step 5).  The G q heads x lq query rows of one kv head are
//   contiguous, so a CTA takes two 128-row tiles of those packed rows.
//
// Roles (12 warps):
//   warp 0      TMA producer: Q0/Q1 once, then K_j, V_j into a 4-slot ring
//   warp 1      MMA issuer (one thread) and TMEM owner
//   warps 2-3   phase 1: copy the tile's own K/V rows into the block's segment
//   warps 4-7   softmax for tile 0: one S row per thread, P back into TMEM
//   warps 8-11  softmax for tile 1
// TMEM (512 columns): S0 [0,128) S1 [128,256) O0 [256,256+D) O1 [256+D,256+2D);
// P_i (bf16) overwrites the first 64 columns of S_i.  tcgen05.mma ops issued by
// the one MMA thread run in order, so S_i(j+1) is written only after
// O_i += P_i(j) V_j has read P_i(j), and a commit that fires for S_i(j+1) also
// guarantees O_i is stable, which is when its softmax warps may rescale it.
//
// Online softmax in base 2 with log2(e) folded into the scale; the running
// maximum used for the exponentials is only raised when a row's maximum
// grows by more than 2^8, so O rarely needs a TMEM read-modify-write.
#include <cuda_bf16.h>
#include <math.h>
#include <string.h>

#include <algorithm>
#include <vector>

#include "sm100_primitives.cuh"
#include "star_common.cuh"
#include "star_internal.h"
#include "tmap.h"

namespace star {
namespace {

using namespace sm100;

constexpr int BM = 128;          // query rows per tile
constexpr int BN = 128;          // keys per K/V tile
static_assert(BN == kPrefillTileKeys, "the prefill tile walk uses the kernel's tile length");
constexpr int NBUF = 4;          // K/V ring slots, phase 1
constexpr int NBUF_PF = 5;       // prefill: its tiles stream from HBM, one more in flight
constexpr int NTHREADS = 384;
// Register split between the warpgroups (setmaxnreg): warpgroup 0 (producer,
// MMA issuer, cache copy) drops to kRegsWG0 per thread and the two softmax
// warpgroups rise to kRegsSoftmax.  The pool is what the CTA was launched
// with (NTHREADS x the kernel's register count, 168 under these launch
// bounds): attn_tc_prepare refuses a build whose count is below kRegsPool,
// since an increase the pool cannot grant would never return.
constexpr int kRegsWG0 = 120;
constexpr int kRegsSoftmax = 192;
constexpr int kRegsPool = 4 * 32 * kRegsWG0 + 8 * 32 * kRegsSoftmax;
static_assert(kRegsPool == NTHREADS * 168, "register split must add up to the launch's registers");
static_assert(kRegsWG0 % 8 == 0 && kRegsSoftmax % 8 == 0, "setmaxnreg takes multiples of 8");
constexpr float kRescaleThreshold = 8.0f;   // log2 units

struct CtxTcArgs {
  CUtensorMap tq;   // phase 1: Q as [B*Hq*L][D]; prefill: query rows as [B*Hq*lq][D]
  CUtensorMap tk;   // phase 1: K as [B*Hkv*L][D]; prefill: context cache as [B*Hkv*L][D]
  CUtensorMap tv;
  CUtensorMap tkq;  // prefill: query region as [B*Hkv*q_cap][D]; phase 1: anchor keys as
                    // [(n-1)*B*Hkv*b_a][D] (anchor_keys 1) or [B*Hkv*b_a][D] (anchor_keys 2)
  CUtensorMap tvq;  // prefill: query region V; phase 1, anchor_keys 2: anchor V [B*Hkv*b_a][D]
  CacheView c;
  float scale_log2;
  const bf16* K;
  const bf16* V;
  bf16* O;
  float* LSE;
  float* O32;         // phase 1, debug: the rows before their bf16 rounding (null: none)
  const int4* work;   // phase 1: (b*Hkv + g, head pair, block, q tile)
  int* err;
  int anchor_keys;    // phase 1: 1 -- block i >= 1 reads its anchor's K tiles from tkq;
                      // 2 -- every block, 0 included, follows an anchor held outside this
                      //      context: its K and V tiles from tkq and tvq
  // prefill
  int lq, len0, row_pairs;
  float* partA;
  float* partS;
  long long part_rows;   // rows the scratch holds (partS elements)
  int wait_first;        // prefill without the append kernel: wait for the previous kernel before any load
  PrefillPlan plan;
};
static_assert(sizeof(CtxTcArgs) <= 4096, "kernel parameters beyond 4 KB");

SM100_DEV float ex2(float x) {
  float y;
  asm volatile("ex2.approx.ftz.f32 %0, %1;\n" : "=f"(y) : "f"(x));
  return y;
}
// Packed fp32 pair arithmetic of sm_100 (one instruction for two lanes of work).
SM100_DEV void ffma2(float& d0, float& d1, float a0, float a1, float b0, float b1, float c0, float c1) {
  asm("{\n .reg .b64 ra, rb, rc, rd;\n"
      " mov.b64 ra, {%2, %3};\n mov.b64 rb, {%4, %5};\n mov.b64 rc, {%6, %7};\n"
      " fma.rn.f32x2 rd, ra, rb, rc;\n mov.b64 {%0, %1}, rd;\n}\n"
      : "=f"(d0), "=f"(d1)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1), "f"(c0), "f"(c1));
}
SM100_DEV void fadd2(float& d0, float& d1, float a0, float a1, float b0, float b1) {
  asm("{\n .reg .b64 ra, rb, rd;\n"
      " mov.b64 ra, {%2, %3};\n mov.b64 rb, {%4, %5};\n"
      " add.rn.f32x2 rd, ra, rb;\n mov.b64 {%0, %1}, rd;\n}\n"
      : "=f"(d0), "=f"(d1)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}
SM100_DEV float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;\n" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

template <int D, int NB>
struct Smem {
  static constexpr int TILE = BM * D * 2;           // one Q or K/V tile, bytes
  static constexpr int HALF = BM * 128;             // one 64-column (128 B) half
  static constexpr int Q0 = 0;
  static constexpr int Q1 = TILE;
  static constexpr int RING = 2 * TILE;
  static constexpr int BYTES = RING + NB * TILE;    // + barriers in static smem
};
static_assert(Smem<128, NBUF_PF>::BYTES + 1024 <= 227 * 1024, "prefill ring beyond shared memory");

template <int D, bool PF>
__global__ void __launch_bounds__(NTHREADS, 1) attn_tc_kernel(const __grid_constant__ CtxTcArgs a) {
  constexpr int NBUF = PF ? NBUF_PF : ::star::NBUF;
  using S = Smem<D, NBUF>;
  constexpr int NH = D / 64;                          // 128-byte halves per row
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  __shared__ __align__(8) uint64_t bar_q_full;
  __shared__ __align__(8) uint64_t bar_kv_full[NBUF];
  __shared__ __align__(8) uint64_t bar_kv_empty[NBUF];
  __shared__ __align__(8) uint64_t bar_s_full[2];
  __shared__ __align__(8) uint64_t bar_p_full[2];
  __shared__ __align__(8) uint64_t bar_o_full;
  __shared__ uint32_t tmem_base_s;
  __shared__ int abort_s;

  const CacheView& c = a.c;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  // ---- work item ------------------------------------------------------------
  int bg, bb, g, h0 = 0, nq, blk = 0, n_rows0, n_rows1, n_anchor = 0, n_kv, chunk = 0;
  long long bstart = 0, t0 = 0, kv_row0, qrow0;
  if (!PF) {
    const int4 w = a.work[blockIdx.x];
    bg = w.x;
    bb = bg / c.Hkv;
    g = bg - bb * c.Hkv;
    h0 = g * c.G + 2 * w.y;
    nq = (h0 + 1 < (g + 1) * c.G) ? 2 : 1;
    blk = w.z;
    bstart = (long long)blk * c.b;
    const long long bend = bstart + c.b < c.L ? bstart + c.b : c.L;
    t0 = bstart + (long long)w.w * BM;
    n_rows0 = n_rows1 = (int)((bend - t0) < BM ? (bend - t0) : BM);
    n_anchor = (blk > 0 || a.anchor_keys == 2) ? (c.b_a + BN - 1) / BN : 0;
    n_kv = n_anchor + w.w + 1;
    kv_row0 = (long long)bg * c.L;                          // (b, g, token 0) in the K/V maps
    qrow0 = ((long long)bb * c.Hq + h0) * c.L + t0;         // Q0's first row; Q1 is one head later
  } else {
    const int bgs = c.B * c.Hkv;
    const int pair = blockIdx.x % a.row_pairs;
    bg = (blockIdx.x / a.row_pairs) % bgs;
    chunk = blockIdx.x / (a.row_pairs * bgs);
    bb = bg / c.Hkv;
    g = bg - bb * c.Hkv;
    const int rows_total = c.G * a.lq;
    const int r0 = pair * 2 * BM;
    nq = r0 + BM < rows_total ? 2 : 1;
    n_rows0 = rows_total - r0 < BM ? rows_total - r0 : BM;
    n_rows1 = rows_total - r0 - BM < BM ? rows_total - r0 - BM : BM;
    t0 = r0;                                                // packed row of Q0's first row
    n_kv = span_tiles(a.plan.span[chunk].x0, a.plan.span[chunk].x1, c);
    kv_row0 = 0;
    qrow0 = ((long long)bb * c.Hq + (long long)g * c.G) * a.lq + r0;   // Q1 is 128 rows later
  }

  if (tid == 0) {
    mbar_init(smem_u32(&bar_q_full), 1);
    for (int i = 0; i < NBUF; ++i) {
      mbar_init(smem_u32(&bar_kv_full[i]), 1);
      mbar_init(smem_u32(&bar_kv_empty[i]), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&bar_s_full[i]), 1);
      mbar_init(smem_u32(&bar_p_full[i]), 128);
    }
    mbar_init(smem_u32(&bar_o_full), 1);
    abort_s = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&tmem_base_s), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (PF) griddep_launch();
  const uint32_t tmem = tmem_base_s;
  auto fail = [&]() {
    abort_s = 1;
    atomicExch(a.err, 1);
  };

  if (warp < 4) {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;\n" ::"n"(kRegsWG0));
  if (warp == 0) {
    // ------------------------------ TMA producer -----------------------------
    if (elect_one()) {
      const CUtensorMap* mk = &a.tk;
      const CUtensorMap* mv = &a.tv;
      prefetch_tmap(&a.tq);
      prefetch_tmap(mk);
      prefetch_tmap(mv);
      TileWalk walk;
      if (PF) {
        walk.start(a.plan.span[chunk].x0, a.plan.span[chunk].x1, c);
        if (a.plan.span[chunk].x1 > c.L) {
          prefetch_tmap(&a.tkq);
          prefetch_tmap(&a.tvq);
        }
      }
      int pf_row = 0;
      bool pf_region = false, region_ready = false;
      const bool own_anchor = !PF && a.anchor_keys == 1 && blk > 0;   // per-block anchor keys
      const bool ext_anchor = !PF && a.anchor_keys == 2;                // anchor K, V outside
      if (own_anchor || ext_anchor) prefetch_tmap(&a.tkq);
      if (ext_anchor) prefetch_tmap(&a.tvq);
      if (PF && a.wait_first) {
        griddep_wait();                                 // inputs written by the kernel before this one
        region_ready = true;
      }
      const uint32_t qb = smem_u32(&bar_q_full);
      mbar_arrive_expect_tx(qb, nq * S::TILE);
      for (int q = 0; q < nq; ++q) {
        const int qrow = (int)(qrow0 + (PF ? (long long)q * BM : (long long)q * c.L));
        for (int hf = 0; hf < NH; ++hf)
          tma_load_2d(smem_u32(smem + (q ? S::Q1 : S::Q0) + hf * S::HALF), &a.tq, hf * 64, qrow, qb);
      }
      int last_use[NBUF];
#pragma unroll
      for (int k = 0; k < NBUF; ++k) last_use[k] = -1;
      for (int i = 0; i < 2 * n_kv; ++i) {
        const int j = i >> 1, slot = i % NBUF, use = i / NBUF;
        if (use > 0 && !mbar_wait(smem_u32(&bar_kv_empty[slot]), (use - 1) & 1)) { fail(); break; }
        if (*(volatile int*)&abort_s) break;
        const long long tok = PF ? 0 : (j < n_anchor ? (long long)j * BN : bstart + (long long)(j - n_anchor) * BN);
        int row = (int)(kv_row0 + tok);
        const CUtensorMap* m = (i & 1) ? mv : mk;
        if (PF) {
          if (!(i & 1)) {                                  // K comes first: step to the next tile
            int r0u;
            walk.next(c, bg, pf_row, pf_region, r0u);
          }
          row = pf_row;
          if (pf_region) {
            m = (i & 1) ? &a.tvq : &a.tkq;
            if (!region_ready) {
              griddep_wait();                           // the append kernel's rows are written
              region_ready = true;
            }
          }
        }
        if (own_anchor && !(i & 1) && j < n_anchor) {
          // K of block blk's anchor: rows of Ka[blk - 1] for this (batch, kv head)
          m = &a.tkq;
          row = (int)((((long long)(blk - 1) * c.B * c.Hkv) + bg) * c.b_a + tok);
        }
        if (ext_anchor && j < n_anchor) {
          // the anchor's K / V rows for this (batch, kv head)
          m = (i & 1) ? &a.tvq : &a.tkq;
          row = (int)((long long)bg * c.b_a + tok);
        }
        const uint32_t fb = smem_u32(&bar_kv_full[slot]);
        mbar_arrive_expect_tx(fb, S::TILE);
        for (int hf = 0; hf < NH; ++hf)
          tma_load_2d(smem_u32(smem + S::RING + slot * S::TILE + hf * S::HALF), m, hf * 64, row, fb);
        last_use[slot] = use;
      }
      if (*(volatile int*)&abort_s) {
        // let every copy this CTA started land before its shared memory is released
        mbar_wait(qb, 0);
        for (int k = 0; k < NBUF; ++k)
          if (last_use[k] >= 0) mbar_wait(smem_u32(&bar_kv_full[k]), last_use[k] & 1);
      }
    }
  } else if (warp == 1) {
    // ------------------------------ MMA issuer -------------------------------
    if (elect_one()) {
      const uint32_t id_qk = idesc_bf16_f32(BM, BN, false);
      const uint32_t id_pv = idesc_bf16_f32(BM, D, true);
      const uint32_t sO[2] = {tmem + 256, tmem + 256 + D};
      const uint32_t sS[2] = {tmem, tmem + 128};
      // Issue order per K/V tile j (two heads):
      //   PV0(j), S0(j+1), PV1(j), S1(j+1)
      // so the tensor core computes head 0's next scores while head 1's
      // softmax still runs, and the other way round.
      // Descriptors are built once; an MMA then costs one add (the start
      // address is the low field, and every offset stays inside it).
      // Q1 follows Q0 and the ring slots follow each other at TILE bytes.
      const uint64_t dq0 = smem_desc_sw128(smem_u32(smem + S::Q0), 16, 1024);
      const uint64_t dk0 = smem_desc_sw128(smem_u32(smem + S::RING), 16, 1024);
      const uint64_t dv0 = smem_desc_sw128(smem_u32(smem + S::RING), S::HALF, 1024);
      constexpr uint64_t kTileStep = S::TILE >> 4;
      auto issue_s = [&](int q, int slot) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t off = (uint64_t)(((kk >> 2) * S::HALF + (kk & 3) * 32) >> 4);
          mma_ss(sS[q], dq0 + q * kTileStep + off, dk0 + slot * kTileStep + off, id_qk, kk > 0);
        }
        mma_commit(smem_u32(&bar_s_full[q]));
      };
      auto issue_pv = [&](int q, int slot, int j) {
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk)
          mma_ts(sO[q], sS[q] + kk * 8, dv0 + slot * kTileStep + (uint64_t)((kk * 2048) >> 4), id_pv,
                 (j > 0 || kk > 0) ? 1u : 0u);
      };
      bool ok = mbar_wait(smem_u32(&bar_q_full), 0) && mbar_wait(smem_u32(&bar_kv_full[0]), 0);
      if (!ok) fail();
      if (ok) {
        tc_fence_after();
        for (int q = 0; q < nq; ++q) issue_s(q, 0);
        mma_commit(smem_u32(&bar_kv_empty[0]));
      }
      for (int j = 0; ok && j < n_kv; ++j) {
        const int iv = 2 * j + 1, ik = 2 * j + 2;       // ring indices of V_j and K_{j+1}
        const bool more = j + 1 < n_kv;
        if (!mbar_wait(smem_u32(&bar_kv_full[iv % NBUF]), (iv / NBUF) & 1)) { fail(); break; }
        if (more && !mbar_wait(smem_u32(&bar_kv_full[ik % NBUF]), (ik / NBUF) & 1)) { fail(); break; }
        for (int q = 0; q < nq; ++q) {
          if (!mbar_spin(smem_u32(&bar_p_full[q]), j & 1)) { fail(); ok = false; break; }
          tc_fence_after();
          issue_pv(q, iv % NBUF, j);
          if (more) issue_s(q, ik % NBUF);
        }
        if (!ok) break;
        mma_commit(smem_u32(&bar_kv_empty[iv % NBUF]));
        if (more) mma_commit(smem_u32(&bar_kv_empty[ik % NBUF]));
        if (*(volatile int*)&abort_s) break;
      }
      mma_commit(smem_u32(&bar_o_full));
    }
  } else if (warp < 4) {
    // ---------------- cache segment write (anchor KV discarded) ---------------
    if (!PF && h0 == g * c.G) {
      const int n_rows = n_rows0;
      const long long len = seg_len(c, blk);
      const long long sbase = (long long)blk * c.B * c.Hkv * (long long)c.b * D +
                              ((long long)bg * len + (t0 - bstart)) * D;
      const long long gbase = (kv_row0 + t0) * D;
      constexpr int CPR = D / 8;
      const long long kv_elems = (long long)c.B * c.Hkv * c.L * D;
      for (int i = tid - 64; i < n_rows * CPR; i += 64) {
        const int r = i / CPR, ch = i - (i / CPR) * CPR;
        if (!STAR_STORE_OK(sbase + (long long)r * D + ch * 8 + 7, kv_elems, a.err) ||
            !STAR_STORE_OK(gbase + (long long)r * D + ch * 8 + 7, kv_elems, a.err))
          continue;
        const uint4 kv = *reinterpret_cast<const uint4*>(a.K + gbase + (long long)r * D + ch * 8);
        const uint4 vv = *reinterpret_cast<const uint4*>(a.V + gbase + (long long)r * D + ch * 8);
        *reinterpret_cast<uint4*>(c.ctxK + sbase + (long long)r * D + ch * 8) = kv;
        *reinterpret_cast<uint4*>(c.ctxV + sbase + (long long)r * D + ch * 8) = vv;
      }
    }
  }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;\n" ::"n"(kRegsSoftmax));
    // ------------------------------ softmax ----------------------------------
    const int q = (warp - 4) >> 2;                    // head 0 or 1 of the pair
    if (q < nq) {
      const int r = ((warp & 3) << 5) | lane;         // tile row owned by this thread
      const uint32_t lane_off = (uint32_t)((warp & 3) << 5) << 16;
      const uint32_t tS = tmem + lane_off + q * 128;
      const uint32_t tO = tmem + lane_off + 256 + q * D;
      const long long pos = t0 + (PF ? q * BM : 0) + r;  // token (phase 1) / packed row (prefill)
      const int n_rows = q ? (n_rows1 > 0 ? n_rows1 : 0) : n_rows0;
      // prefill: this row sees query-region rows 0..len0 + (its query index)
      TileWalk walk;
      long long q_lim = 0;
      if (PF) {
        walk.start(a.plan.span[chunk].x0, a.plan.span[chunk].x1, c);
        q_lim = a.len0 + (pos % a.lq) + 1;
      }
      float m_used = -INFINITY, l = 0.f;
      const float sl2 = a.scale_log2;
      for (int j = 0; j < n_kv; ++j) {
        if (!mbar_wait(smem_u32(&bar_s_full[q]), j & 1)) { fail(); break; }
        tc_fence_after();
        uint32_t s[BN];
#pragma unroll
        for (int cc = 0; cc < BN / 32; ++cc) tmem_ld32(tS + cc * 32, *reinterpret_cast<uint32_t(*)[32]>(&s[cc * 32]));
        tmem_wait_ld();
        // mask: phase 1 -- anchor tail (keys >= b_a) and the causal diagonal;
        // prefill -- chunk tail, or the causal query region
        const bool anchor = !PF && j < n_anchor;
        long long k0 = anchor ? (long long)j * BN : bstart + (long long)(j - n_anchor) * BN;
        long long lim = anchor ? (long long)c.b_a : pos + 1;     // keys < lim visible
        if (PF) {
          // the tile's keys are [0, n) of the walk; in the query region only
          // those up to this row's own position
          int row_u, r0;
          bool region;
          const int n = walk.next(c, bg, row_u, region, r0);
          k0 = 0;
          lim = region ? (q_lim - r0 < n ? q_lim - r0 : n) : n;
        }
        if (k0 + BN > lim) {
          const int nvis = (int)(lim - k0 < 0 ? 0 : lim - k0);   // visible columns: [0, nvis)
#pragma unroll
          for (int i = 0; i < BN; ++i)
            if (i >= nvis) s[i] = __float_as_uint(-INFINITY);
        }
        // row maximum: eight independent chains of 3-input max, then a tree
        float mk[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) mk[k] = fmaxf(__uint_as_float(s[2 * k]), __uint_as_float(s[2 * k + 1]));
#pragma unroll
        for (int i = 16; i < BN; i += 16)
#pragma unroll
          for (int k = 0; k < 8; ++k)
            mk[k] = fmax3(mk[k], __uint_as_float(s[i + 2 * k]), __uint_as_float(s[i + 2 * k + 1]));
        const float mx = fmaxf(fmax3(mk[0], mk[1], mk[2]), fmax3(fmax3(mk[3], mk[4], mk[5]), mk[6], mk[7]));
        const float m_tile = mx * sl2;
        const bool need = m_tile > m_used + kRescaleThreshold;
        float alpha = 1.f;
        if (need) {
          alpha = ex2(m_used - m_tile);               // 0 when m_used is -inf
          m_used = m_tile;
        }
        if (__any_sync(0xffffffffu, need) && j > 0) {
          // O_i is stable here (see header); rescale this warp's rows.
#pragma unroll 1
          for (int cc = 0; cc < D / 32; ++cc) {
            uint32_t o[32];
            tmem_ld32(tO + cc * 32, o);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
            tmem_st32(tO + cc * 32, o);
          }
        }
        l *= alpha;
        const float base = m_used == -INFINITY ? 0.f : m_used;
        // P = 2^(s*scale - base): packed-pair FMA, ex2, four packed row-sum chains
        float ra[4] = {0.f, 0.f, 0.f, 0.f}, rb[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int cc = 0; cc < BN / 32; ++cc) {
          uint32_t p[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            float x0, x1;
            ffma2(x0, x1, __uint_as_float(s[cc * 32 + 2 * i]), __uint_as_float(s[cc * 32 + 2 * i + 1]),
                  sl2, sl2, -base, -base);
            const float e0 = ex2(x0), e1 = ex2(x1);
            fadd2(ra[i & 3], rb[i & 3], ra[i & 3], rb[i & 3], e0, e1);
            p[i] = pack_bf16(e0, e1);
          }
          tmem_st16(tS + cc * 16, p);
        }
        const float rs = (ra[0] + rb[0]) + (ra[1] + rb[1]) + ((ra[2] + rb[2]) + (ra[3] + rb[3]));
        l += rs;
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(smem_u32(&bar_p_full[q]));
      }
      // ---- epilogue -------------------------------------------------------------
      // phase 1: O / l in bf16 and LSE = (m + log2 l) ln 2;  prefill: the chunk's
      // fp32 partial (A_h, s_h) of every packed row.
      const bool ok = mbar_wait(smem_u32(&bar_o_full), 0);
      if (!ok) fail();
      tc_fence_after();
      const float inv = l > 0.f ? 1.f / l : 0.f;
      const float lse = l > 0.f ? (m_used + log2f(l)) * kLn2 : -INFINITY;
      if (!PF) {
        const int h = h0 + q;
        const long long orow_i = ((long long)bb * c.Hq + h) * c.L + pos;
        const bool row_ok = r >= n_rows || STAR_STORE_OK(orow_i, (long long)c.B * c.Hq * c.L, a.err);
        bf16* orow = a.O + orow_i * D;
#pragma unroll 1
        for (int cc = 0; cc < D / 32; ++cc) {
          uint32_t o[32];
          tmem_ld32(tO + cc * 32, o);
          tmem_wait_ld();
          if (r < n_rows && row_ok) {
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * inv);
            uint32_t pk[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) pk[i] = pack_bf16(__uint_as_float(o[2 * i]), __uint_as_float(o[2 * i + 1]));
#pragma unroll
            for (int v = 0; v < 4; ++v)
              reinterpret_cast<uint4*>(orow + cc * 32)[v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
            if (a.O32) {
              float4* o32 = reinterpret_cast<float4*>(a.O32 + orow_i * D + cc * 32);
#pragma unroll
              for (int v = 0; v < 8; ++v)
                o32[v] = make_float4(__uint_as_float(o[4 * v]), __uint_as_float(o[4 * v + 1]),
                                     __uint_as_float(o[4 * v + 2]), __uint_as_float(o[4 * v + 3]));
            }
          }
        }
        if (r < n_rows && row_ok) a.LSE[orow_i] = lse;
      } else {
        const long long prow = ((long long)bg * a.plan.n_spans + chunk) * (c.G * a.lq) + pos;
        const bool row_ok = r >= n_rows || STAR_STORE_OK(prow, a.part_rows, a.err);
        float* arow = a.partA + prow * D;
#pragma unroll 1
        for (int cc = 0; cc < D / 32; ++cc) {
          uint32_t o[32];
          tmem_ld32(tO + cc * 32, o);
          tmem_wait_ld();
          if (r < n_rows && row_ok) {
#pragma unroll
            for (int v = 0; v < 8; ++v)
              reinterpret_cast<float4*>(arow + cc * 32)[v] =
                  make_float4(__uint_as_float(o[4 * v]) * inv, __uint_as_float(o[4 * v + 1]) * inv,
                              __uint_as_float(o[4 * v + 2]) * inv, __uint_as_float(o[4 * v + 3]) * inv);
          }
        }
        if (r < n_rows && row_ok) a.partS[prow] = lse;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace

// Work list for the tensor-core phase-1 kernel: (b*Hkv + g, head pair, block,
// q tile) for every 128-row tile; the order is set by ctx_tc_fill_work below.
size_t ctx_tc_work_count(const CacheView& c) {
  const int pairs = (c.G + 1) / 2;
  size_t n = 0;
  for (int blk = 0; blk < c.n_seg; ++blk) n += (size_t)((seg_len(c, blk) + BM - 1) / BM);
  return n * c.B * c.Hkv * pairs;
}

void ctx_tc_fill_work(const CacheView& c, int4* out) {
  const int pairs = (c.G + 1) / 2;
  const int BG = c.B * c.Hkv;
  // Work units (block, batch x kv head), last block first, are packed into
  // groups whose K/V (the block's rows plus the anchor rows it reads) stays
  // under kGroupBytes, about two thirds of the 126 MB L2.  Inside a group the
  // longest tile goes first.  The CTAs that run together then re-read one
  // group's K/V from L2 instead of streaming every head's from HBM (one
  // global longest-first order spans all heads of all batch entries: 268 MB
  // of K/V at four 32K-token sequences), and the short tiles of block 0 close
  // the launch.
  constexpr long long kGroupBytes = 80ll << 20;
  std::vector<int> group((size_t)c.n_seg * BG);
  int g = 0;
  long long used = 0;
  for (int blk = c.n_seg - 1; blk >= 0; --blk) {
    const long long unit = (seg_len(c, blk) + (blk > 0 ? c.b_a : 0)) * c.D * 2ll * (long long)sizeof(bf16);
    if (used > 0 && used + unit * BG > kGroupBytes && unit * BG <= kGroupBytes) {
      ++g;                                   // a block that fits a group of its own is not split
      used = 0;
    }
    for (int bg = 0; bg < BG; ++bg) {
      if (used > 0 && used + unit > kGroupBytes) {
        ++g;
        used = 0;
      }
      used += unit;
      group[(size_t)blk * BG + bg] = g;
    }
  }
  struct Item { int group; long long cost; int4 v; };
  std::vector<Item> items;
  for (int blk = 0; blk < c.n_seg; ++blk) {
    const long long tiles = (seg_len(c, blk) + BM - 1) / BM;
    const long long anchor_tiles = blk > 0 ? (c.b_a + BN - 1) / BN : 0;
    for (int qt = 0; qt < tiles; ++qt)
      for (int bg = 0; bg < BG; ++bg)
        for (int hp = 0; hp < pairs; ++hp)
          items.push_back({group[(size_t)blk * BG + bg], anchor_tiles + qt + 1, make_int4(bg, hp, blk, qt)});
  }
  std::stable_sort(items.begin(), items.end(), [](const Item& x, const Item& y) {
    if (x.group != y.group) return x.group < y.group;
    return x.cost > y.cost;
  });
  for (size_t i = 0; i < items.size(); ++i) out[i] = items[i].v;
}

void ctx_tc_fill_units(const CacheView& c, int num_sms, std::vector<CtxUnit>& units, int4* out) {
  const int pairs = (c.G + 1) / 2;
  const int BG = c.B * c.Hkv;
  units.clear();
  int off = 0;
  for (int blk = 0; blk < c.n_seg; ++blk) {
    const long long tiles = (seg_len(c, blk) + BM - 1) / BM;
    // equal units of at least one wave of CTAs each (the units run on two
    // streams, so one unit's tail overlaps the next unit's start): the largest
    // divisor of B*Hkv that keeps a unit at num_sms CTAs or more
    const long long per_bg = tiles * pairs;
    int parts = 1;
    for (int d = 1; d <= BG; ++d)
      if (BG % d == 0 && per_bg * (BG / d) >= num_sms) parts = d;
    for (int k = 0; k < parts; ++k) {
      CtxUnit u;
      u.blk = blk;
      u.bg0 = (int)((long long)BG * k / parts);
      u.bg1 = (int)((long long)BG * (k + 1) / parts);
      u.off = off;
      // longest tile (last one, most K/V tiles) first
      for (long long qt = tiles - 1; qt >= 0; --qt)
        for (int bg = u.bg0; bg < u.bg1; ++bg)
          for (int hp = 0; hp < pairs; ++hp) out[off++] = make_int4(bg, hp, blk, (int)qt);
      u.n = off - u.off;
      units.push_back(u);
    }
  }
}

template <int D, bool PF>
constexpr int smem_bytes() {
  return Smem<D, PF ? NBUF_PF : NBUF>::BYTES + 1024;
}

template <int D, bool PF>
cudaError_t check_reg_pool() {
  cudaFuncAttributes fa;
  cudaError_t e = cudaFuncGetAttributes(&fa, attn_tc_kernel<D, PF>);
  if (e != cudaSuccess) return e;
  return fa.numRegs * NTHREADS >= kRegsPool ? cudaSuccess : cudaErrorInvalidConfiguration;
}

cudaError_t attn_tc_prepare(int D) {
  cudaError_t e = D == 128 ? check_reg_pool<128, false>() : check_reg_pool<64, false>();
  if (e == cudaSuccess) e = D == 128 ? check_reg_pool<128, true>() : check_reg_pool<64, true>();
  if (e != cudaSuccess) return e;
  if (D == 128) {
    e = cudaFuncSetAttribute(attn_tc_kernel<128, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             smem_bytes<128, false>());
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(attn_tc_kernel<128, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               smem_bytes<128, true>());
  } else {
    e = cudaFuncSetAttribute(attn_tc_kernel<64, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             smem_bytes<64, false>());
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(attn_tc_kernel<64, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               smem_bytes<64, true>());
  }
  return e;
}

cudaError_t launch_ctx_encode_tc(const CacheView& c, float scale, const bf16* Q, const bf16* K,
                                 const bf16* V, bf16* O, float* LSE, const int4* work, int n_work,
                                 int* err, cudaStream_t st, const bf16* Ka, float* O32, const bf16* Va) {
  if (n_work == 0) return cudaSuccess;
  CtxTcArgs a;
  memset(&a, 0, sizeof(a));
  const unsigned long long qrows = (unsigned long long)c.B * c.Hq * c.L;
  const unsigned long long kvrows = (unsigned long long)c.B * c.Hkv * c.L;
  if (!make_tmap_bf16_2d(&a.tq, Q, qrows, c.D, BM, 64) || !make_tmap_bf16_2d(&a.tk, K, kvrows, c.D, BN, 64) ||
      !make_tmap_bf16_2d(&a.tv, V, kvrows, c.D, BN, 64))
    return cudaErrorInvalidValue;
  if (Ka && Va) {
    // every block follows the anchor Ka, Va [B][Hkv][b_a][D] (no anchor: plain blocks)
    if (c.b_a > 0) {
      const unsigned long long arows = (unsigned long long)c.B * c.Hkv * c.b_a;
      if (!make_tmap_bf16_2d(&a.tkq, Ka, arows, c.D, BN, 64) || !make_tmap_bf16_2d(&a.tvq, Va, arows, c.D, BN, 64))
        return cudaErrorInvalidValue;
      a.anchor_keys = 2;
    }
  } else if (Ka && c.n_seg > 1 && c.b_a > 0) {
    const unsigned long long karows = (unsigned long long)(c.n_seg - 1) * c.B * c.Hkv * c.b_a;
    if (!make_tmap_bf16_2d(&a.tkq, Ka, karows, c.D, BN, 64)) return cudaErrorInvalidValue;
    a.anchor_keys = 1;
  }
  a.c = c;
  a.scale_log2 = scale * kLog2e;
  a.K = K;
  a.V = V;
  a.O = O;
  a.LSE = LSE;
  a.O32 = O32;
  a.work = work;
  a.err = err;
  if (c.D == 128)
    attn_tc_kernel<128, false><<<n_work, NTHREADS, smem_bytes<128, false>(), st>>>(a);
  else
    attn_tc_kernel<64, false><<<n_work, NTHREADS, smem_bytes<64, false>(), st>>>(a);
  return cudaGetLastError();
}

// ---- query prefill ------------------------------------------------------------
namespace {

// Append this call's query K/V rows to the query region (rows len0..len0+lq-1).
__global__ void __launch_bounds__(256) query_append_kernel(CacheView c, int lq, int len0,
                                                           const uint4* __restrict__ K,
                                                           const uint4* __restrict__ V) {
  griddep_launch();                                           // the tile kernel waits for these rows itself
  const int cpr = c.D / 8;                                    // 16-byte chunks per row
  const long long n = (long long)c.B * c.Hkv * lq * cpr;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (long long)gridDim.x * blockDim.x) {
    const long long row = i / cpr;
    const int ch = (int)(i - row * cpr);
    const int bg = (int)(row / lq), t = (int)(row - (long long)bg * lq);
    const long long dst = (((long long)bg * c.q_cap) + len0 + t) * cpr + ch;
    if (!STAR_STORE_OK(dst, (long long)c.B * c.Hkv * c.q_cap * cpr, c.err)) continue;
    reinterpret_cast<uint4*>(c.qK)[dst] = K[i];
    reinterpret_cast<uint4*>(c.qV)[dst] = V[i];
  }
}

// Merge the chunks' partials of every packed query row and scatter to O / LSE.
// One warp per row: lane p holds the s of chunks p, p + 32, ... (one load
// each, all in flight together), the maximum and the total come from warp
// reductions, the chunk weights go through shared memory, and the lanes then
// accumulate their D/32 columns over the chunks, eight chunks' loads at a time.
// Debug outputs (null in the normal path): O32, the merged rows in float32;
// Ah / sh, every chunk's partial in [chunk][B][Hq][lq] row order.  O may be
// null when only the float32 rows are wanted (a partial over part of the cache).
constexpr int kMergeWarps = 4;
constexpr int kSPerLane = (kMaxPrefillSpans + 31) / 32;
template <int D>
__global__ void __launch_bounds__(32 * kMergeWarps) prefill_merge_kernel(CacheView c, int lq, int n_chunks,
                                                                        long long part_rows,
                                                                        const float* __restrict__ partA,
                                                                        const float* __restrict__ partS,
                                                                        bf16* __restrict__ O,
                                                                        float* __restrict__ LSE,
                                                                        float* __restrict__ O32,
                                                                        float* __restrict__ Ah,
                                                                        float* __restrict__ sh) {
  __shared__ float wgt[kMergeWarps][kSPerLane * 32];
  griddep_wait();                                    // the tile kernel's partials are complete
  const int rows_total = c.G * lq;
  const int wid = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long gw = (long long)blockIdx.x * kMergeWarps + wid;
  if (gw >= (long long)c.B * c.Hkv * rows_total) return;
  const long long bg = gw / rows_total;
  const int m = (int)(gw - bg * rows_total);
  const int bb = (int)(bg / c.Hkv), g = (int)(bg - (long long)bb * c.Hkv);
  const int h = g * c.G + m / lq;
  const int rr = m % lq;
  const long long orow_i = ((long long)bb * c.Hq + h) * lq + rr;   // row of O / LSE
  const long long prow0 = bg * n_chunks * rows_total + m;          // chunk p's row: prow0 + p * rows_total
  if (!STAR_STORE_OK(orow_i, (long long)c.B * c.Hq * lq, c.err) ||
      (n_chunks > 0 && !STAR_STORE_OK(prow0 + (long long)(n_chunks - 1) * rows_total, part_rows, c.err)))
    return;
  float sv[kSPerLane];
  float mx = -INFINITY;
#pragma unroll
  for (int k = 0; k < kSPerLane; ++k) {
    const int p = lane + 32 * k;
    sv[k] = p < n_chunks ? partS[prow0 + (long long)p * rows_total] : -INFINITY;
    mx = fmaxf(mx, sv[k]);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
  const float base = mx == -INFINITY ? 0.f : mx;
  float tot = 0.f;
#pragma unroll
  for (int k = 0; k < kSPerLane; ++k) tot += sv[k] == -INFINITY ? 0.f : __expf(sv[k] - base);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) tot += __shfl_xor_sync(0xffffffffu, tot, off);
  const float lse = mx == -INFINITY ? -INFINITY : base + __logf(tot);
  const long long prow_stride = (long long)c.B * c.Hq * lq;        // rows per chunk in Ah / sh
#pragma unroll
  for (int k = 0; k < kSPerLane; ++k) {
    const int p = lane + 32 * k;
    if (p < n_chunks) {
      wgt[wid][p] = sv[k] == -INFINITY ? 0.f : __expf(sv[k] - lse);
      if (sh) sh[p * prow_stride + orow_i] = sv[k];
    }
  }
  __syncwarp();
  constexpr int PER = D / 32;
  float acc[PER];
#pragma unroll
  for (int i = 0; i < PER; ++i) acc[i] = 0.f;
  constexpr int U = 8;
  for (int p0 = 0; p0 < n_chunks; p0 += U) {
    float v[U][PER];
#pragma unroll
    for (int u = 0; u < U; ++u)
#pragma unroll
      for (int i = 0; i < PER; ++i)
        v[u][i] = p0 + u < n_chunks ? partA[(prow0 + (long long)(p0 + u) * rows_total) * D + lane + 32 * i] : 0.f;
#pragma unroll
    for (int u = 0; u < U; ++u) {
      if (p0 + u >= n_chunks) break;
      const float w = wgt[wid][p0 + u];
#pragma unroll
      for (int i = 0; i < PER; ++i) {
        acc[i] += w * v[u][i];
        if (Ah) Ah[((p0 + u) * prow_stride + orow_i) * D + lane + 32 * i] = v[u][i];
      }
    }
  }
  if (O) {
    bf16* orow = O + orow_i * D;
#pragma unroll
    for (int i = 0; i < PER; ++i) orow[lane + 32 * i] = __float2bfloat16_rn(acc[i]);
  }
  if (O32) {
#pragma unroll
    for (int i = 0; i < PER; ++i) O32[orow_i * D + lane + 32 * i] = acc[i];
  }
  if (lane == 0) LSE[orow_i] = lse;
}

}  // namespace

int prefill_row_pairs(const CacheView& c, int lq) { return (c.G * lq + 2 * BM - 1) / (2 * BM); }

cudaError_t launch_query_prefill_tc(const CacheView& c, const DecodeMaps& maps, float scale, int lq,
                                    int len0, const bf16* Q, const bf16* Kq, const bf16* Vq, bf16* O,
                                    float* LSE, const PrefillPlan& plan, const Scratch& s,
                                    cudaStream_t st, float* O32, float* Ah, float* sh, bool append) {
  CtxTcArgs a;
  memset(&a, 0, sizeof(a));
  const unsigned long long qrows = (unsigned long long)c.B * c.Hq * lq;
  if (!make_tmap_bf16_2d(&a.tq, Q, qrows, c.D, BM, 64)) return cudaErrorInvalidValue;
  a.tk = maps.k_ctx;
  a.tv = maps.v_ctx;
  a.tkq = maps.k_q;
  a.tvq = maps.v_q;
  a.c = c;
  a.scale_log2 = scale * kLog2e;
  a.err = s.err;
  a.lq = lq;
  a.len0 = len0;
  a.row_pairs = prefill_row_pairs(c, lq);
  a.partA = s.partA;
  a.partS = s.partS;
  a.part_rows = s.partS_elems;
  a.plan = plan;
  a.wait_first = append ? 0 : 1;
  if (append) {
    const long long n16 = (long long)c.B * c.Hkv * lq * (c.D / 8);
    const int agrid = (int)((n16 + 255) / 256 < 1024 ? (n16 + 255) / 256 : 1024);
    query_append_kernel<<<agrid, 256, 0, st>>>(c, lq, len0, reinterpret_cast<const uint4*>(Kq),
                                               reinterpret_cast<const uint4*>(Vq));
  }
  // The tile kernel and the merge are launched as programmatic dependents of
  // the kernel before them: each starts while that one drains and waits for
  // its results where it reads them (griddep_wait).
  cudaLaunchAttribute pdl[1];
  pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  pdl[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.stream = st;
  cfg.attrs = pdl;
  cfg.numAttrs = 1;
  cudaError_t e = cudaSuccess;
  const int grid = c.B * c.Hkv * a.row_pairs * plan.n_spans;
  if (grid > 0) {
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(NTHREADS);
    cfg.dynamicSmemBytes = c.D == 128 ? smem_bytes<128, true>() : smem_bytes<64, true>();
    e = c.D == 128 ? cudaLaunchKernelEx(&cfg, attn_tc_kernel<128, true>, a)
                   : cudaLaunchKernelEx(&cfg, attn_tc_kernel<64, true>, a);
    if (e != cudaSuccess) return e;
  }
  const long long rows = (long long)c.B * c.Hkv * c.G * lq;
  cfg.gridDim = dim3((unsigned)((rows + kMergeWarps - 1) / kMergeWarps));
  cfg.blockDim = dim3(32 * kMergeWarps);
  cfg.dynamicSmemBytes = 0;
  const int n_spans = plan.n_spans;
  const long long part_rows = s.partS_elems;
  const float* pA = s.partA;
  const float* pS = s.partS;
  e = c.D == 128 ? cudaLaunchKernelEx(&cfg, prefill_merge_kernel<128>, c, lq, n_spans, part_rows, pA, pS, O, LSE, O32, Ah, sh)
                 : cudaLaunchKernelEx(&cfg, prefill_merge_kernel<64>, c, lq, n_spans, part_rows, pA, pS, O, LSE, O32, Ah, sh);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace star
