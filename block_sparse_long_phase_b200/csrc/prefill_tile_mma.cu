// Phase-2 query-prefill partials: flash-style attention tile kernel on
// warp-level bf16 MMA (mma.sync m16n8k16).
//
// "Star Attention: Efficient LLM Inference over Long Sequences" (analysis
// page), section 3.4, "Phase 2: Query Encoding and Token Generation with
// Distributed Softmax", Step 3: every context block computes the local
// attention A_h of the query rows over its own cache, with the log of its
// exponent sum s_h; the query region is one more partition, attended causally.
// A CTA takes 64 packed query rows of one kv group (the G q heads x lq rows of
// one kv head are contiguous in Q) against one key chunk -- a slice of a
// context segment (fully visible) or the query region (causal) -- streaming
// 64-key K/V tiles through double-buffered cp.async stages in XOR-swizzled
// shared memory with an online softmax (exp2, log2(e) folded into the scale)
// and fp32 accumulation, and writes (A_h, s_h) of that chunk in fp32.  A
// second kernel merges the chunks' partials per row (Step 5).
#include <cuda_bf16.h>
#include <math.h>

#include "star_common.cuh"
#include "star_internal.h"

namespace star {
namespace {

constexpr int BM = 64;
constexpr int BN = 64;
constexpr int NTHREADS = 128;

struct TileArgs {
  CacheView c;
  float scale_log2;
  const bf16* Q;  // query rows [B][Hq][lq][D]
  const bf16* K;  // this call's query K [B][Hkv][lq][D]
  const bf16* V;
  int lq, len0;
  float* partA;
  float* partS;
  PrefillPlan plan;
};

template <int D>
__global__ void __launch_bounds__(NTHREADS) prefill_tile_kernel(const __grid_constant__ TileArgs a) {
  constexpr int CPR = D / 8;                 // 16-byte chunks per row
  constexpr int TILE_BYTES = BM * D * 2;     // BM == BN
  constexpr int NT_O = D / 8;                // output n-tiles
  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t* sQ = smem;
  uint8_t* sK = smem + TILE_BYTES;           // 2 stages
  uint8_t* sV = sK + 2 * TILE_BYTES;         // 2 stages

  const CacheView& c = a.c;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  // ---- work item: (batch*kv head, key chunk, 64-row tile) -------------------
  const int per_bg = a.plan.row_tiles * a.plan.n_chunks;
  const int bg = blockIdx.x / per_bg;
  const int rem = blockIdx.x - bg * per_bg;
  const int chunk_id = rem / a.plan.row_tiles;
  const int rt = rem - chunk_id * a.plan.row_tiles;
  const int bb = bg / c.Hkv;
  const int g = bg - bb * c.Hkv;
  const int rows_total = c.G * a.lq;
  const long long row0 = (long long)rt * BM;
  const int n_rows = (int)(rows_total - row0 < BM ? rows_total - row0 : BM);
  const bf16* qptr = a.Q + (((long long)bb * c.Hq + (long long)g * c.G) * a.lq + row0) * D;
  const long long nk = a.plan.chunk[chunk_id].len;   // keys in this chunk
  const int n_tiles = (int)((nk + BN - 1) / BN);

  // Row pointer of key j of the chunk (K when v == false, V otherwise).
  auto key_row = [&](long long j, bool v) -> const bf16* {
    const PrefillChunk ch = a.plan.chunk[chunk_id];
    if (ch.seg >= 0) {
      const bf16* base = v ? c.ctxV : c.ctxK;
      return base + ctx_row_offset(c, bb, g, (long long)ch.seg * c.b + ch.start + j);
    }
    if (j < a.len0) return (v ? c.qV : c.qK) + q_row_offset(c, bb, g, j);
    const bf16* base = v ? a.V : a.K;
    return base + (((long long)bb * c.Hkv + g) * a.lq + (j - a.len0)) * D;
  };

  auto load_tile = [&](int stage, int t) {
    const long long j0 = (long long)t * BN;
    const uint32_t dk = smem_u32(sK + stage * TILE_BYTES);
    const uint32_t dv = smem_u32(sV + stage * TILE_BYTES);
    for (int i = tid; i < BN * CPR; i += NTHREADS) {
      const int row = i / CPR, ch = i - (i / CPR) * CPR;
      const long long j = j0 + row;
      const bool ok = j < nk;
      const bf16* kp = ok ? key_row(j, false) : qptr;
      const bf16* vp = ok ? key_row(j, true) : qptr;
      cp_async16(dk + swz(row, ch, CPR), kp + ch * 8, ok ? 16 : 0);
      cp_async16(dv + swz(row, ch, CPR), vp + ch * 8, ok ? 16 : 0);
    }
  };

  // ---- Q tile + first K/V tile ---------------------------------------------
  for (int i = tid; i < BM * CPR; i += NTHREADS) {
    const int row = i / CPR, ch = i - (i / CPR) * CPR;
    const bool ok = row < n_rows;
    cp_async16(smem_u32(sQ) + swz(row, ch, CPR), qptr + (long long)(ok ? row : 0) * D + ch * 8,
               ok ? 16 : 0);
  }
  if (n_tiles > 0) load_tile(0, 0);
  cp_async_commit();

  // Per-thread rows inside the tile: r_a = warp*16 + lane/4, r_b = r_a + 8.
  const int ra = warp * 16 + (lane >> 2);
  const int rb = ra + 8;
  // Causal position of each row in the query region.
  const long long pos_a = a.len0 + (row0 + ra) % a.lq;
  const long long pos_b = a.len0 + (row0 + rb) % a.lq;
  const bool causal = a.plan.chunk[chunk_id].seg < 0;

  uint32_t qa[D / 16][4];
  float o[NT_O][4];
#pragma unroll
  for (int n = 0; n < NT_O; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
  float m_a = -INFINITY, m_b = -INFINITY, l_a = 0.f, l_b = 0.f;

  for (int t = 0; t < n_tiles; ++t) {
    const int stage = t & 1;
    if (t + 1 < n_tiles) load_tile(stage ^ 1, t + 1);
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    if (t == 0) {
#pragma unroll
      for (int kd = 0; kd < D / 16; ++kd) {
        const int row = warp * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
        const int ch = 2 * kd + (lane >> 4);
        ldmatrix_x4(smem_u32(sQ) + swz(row, ch, CPR), qa[kd][0], qa[kd][1], qa[kd][2], qa[kd][3]);
      }
    }
    const uint32_t kbase = smem_u32(sK + stage * TILE_BYTES);
    const uint32_t vbase = smem_u32(sV + stage * TILE_BYTES);

    // S = Q K^T for 16 rows x 64 keys per warp.
    float s[8][4];
#pragma unroll
    for (int n = 0; n < 8; ++n) s[n][0] = s[n][1] = s[n][2] = s[n][3] = 0.f;
#pragma unroll
    for (int kd = 0; kd < D / 16; ++kd) {
#pragma unroll
      for (int jn = 0; jn < 4; ++jn) {
        const int row = 16 * jn + (lane & 7) + ((lane >> 4) << 3);
        const int ch = 2 * kd + ((lane >> 3) & 1);
        uint32_t b0, b1, b2, b3;
        ldmatrix_x4(kbase + swz(row, ch, CPR), b0, b1, b2, b3);
        mma_bf16_16816(s[2 * jn], qa[kd], b0, b1);
        mma_bf16_16816(s[2 * jn + 1], qa[kd], b2, b3);
      }
    }

    // Scale into log2 units and mask.
    const long long j0 = (long long)t * BN;
    const bool need_mask = (j0 + BN > nk) || causal;
#pragma unroll
    for (int n = 0; n < 8; ++n) {
#pragma unroll
      for (int e = 0; e < 4; ++e) s[n][e] *= a.scale_log2;
    }
    if (need_mask) {
      const long long kpos0 = j0;
#pragma unroll
      for (int n = 0; n < 8; ++n) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int col = 8 * n + 2 * (lane & 3) + (e & 1);
          const long long j = j0 + col;
          const long long pos = (e < 2) ? pos_a : pos_b;
          bool vis = j < nk;
          if (causal) vis = vis && (kpos0 + col <= pos);
          if (!vis) s[n][e] = -INFINITY;
        }
      }
    }

    // Online softmax.
    float mx_a = -INFINITY, mx_b = -INFINITY;
#pragma unroll
    for (int n = 0; n < 8; ++n) {
      mx_a = fmaxf(mx_a, fmaxf(s[n][0], s[n][1]));
      mx_b = fmaxf(mx_b, fmaxf(s[n][2], s[n][3]));
    }
    mx_a = fmaxf(mx_a, __shfl_xor_sync(0xffffffffu, mx_a, 1));
    mx_a = fmaxf(mx_a, __shfl_xor_sync(0xffffffffu, mx_a, 2));
    mx_b = fmaxf(mx_b, __shfl_xor_sync(0xffffffffu, mx_b, 1));
    mx_b = fmaxf(mx_b, __shfl_xor_sync(0xffffffffu, mx_b, 2));
    const float mn_a = fmaxf(m_a, mx_a), mn_b = fmaxf(m_b, mx_b);
    const float base_a = mn_a == -INFINITY ? 0.f : mn_a;
    const float base_b = mn_b == -INFINITY ? 0.f : mn_b;
    const float al_a = exp2f(m_a - base_a), al_b = exp2f(m_b - base_b);
    m_a = mn_a;
    m_b = mn_b;
    float rs_a = 0.f, rs_b = 0.f;
#pragma unroll
    for (int n = 0; n < 8; ++n) {
      s[n][0] = exp2f(s[n][0] - base_a);
      s[n][1] = exp2f(s[n][1] - base_a);
      s[n][2] = exp2f(s[n][2] - base_b);
      s[n][3] = exp2f(s[n][3] - base_b);
      rs_a += s[n][0] + s[n][1];
      rs_b += s[n][2] + s[n][3];
    }
    l_a = l_a * al_a + rs_a;
    l_b = l_b * al_b + rs_b;
#pragma unroll
    for (int n = 0; n < NT_O; ++n) {
      o[n][0] *= al_a;
      o[n][1] *= al_a;
      o[n][2] *= al_b;
      o[n][3] *= al_b;
    }

    // O += P V.
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      uint32_t pa[4];
      pa[0] = pack_bf16(s[2 * kk][0], s[2 * kk][1]);
      pa[1] = pack_bf16(s[2 * kk][2], s[2 * kk][3]);
      pa[2] = pack_bf16(s[2 * kk + 1][0], s[2 * kk + 1][1]);
      pa[3] = pack_bf16(s[2 * kk + 1][2], s[2 * kk + 1][3]);
#pragma unroll
      for (int j = 0; j < D / 16; ++j) {
        const int row = 16 * kk + (lane & 7) + ((lane >> 3) & 1) * 8;
        const int ch = 2 * j + (lane >> 4);
        uint32_t b0, b1, b2, b3;
        ldmatrix_x4_trans(vbase + swz(row, ch, CPR), b0, b1, b2, b3);
        mma_bf16_16816(o[2 * j], pa, b0, b1);
        mma_bf16_16816(o[2 * j + 1], pa, b2, b3);
      }
    }
    __syncthreads();
  }
  cp_async_wait<0>();

  // ---- epilogue --------------------------------------------------------------
  l_a += __shfl_xor_sync(0xffffffffu, l_a, 1);
  l_a += __shfl_xor_sync(0xffffffffu, l_a, 2);
  l_b += __shfl_xor_sync(0xffffffffu, l_b, 1);
  l_b += __shfl_xor_sync(0xffffffffu, l_b, 2);
  const float inv_a = l_a > 0.f ? 1.f / l_a : 0.f;
  const float inv_b = l_b > 0.f ? 1.f / l_b : 0.f;
  const float lse_a = l_a > 0.f ? (m_a + log2f(l_a)) * kLn2 : -INFINITY;
  const float lse_b = l_b > 0.f ? (m_b + log2f(l_b)) * kLn2 : -INFINITY;
  const int cq = 2 * (lane & 3);

  {
    const long long pbase = ((long long)bg * a.plan.n_chunks + chunk_id) * rows_total;
    if (ra < n_rows) {
      float* pa_ = a.partA + (pbase + row0 + ra) * D;
#pragma unroll
      for (int n = 0; n < NT_O; ++n)
        *reinterpret_cast<float2*>(pa_ + 8 * n + cq) = make_float2(o[n][0] * inv_a, o[n][1] * inv_a);
      if ((lane & 3) == 0) a.partS[pbase + row0 + ra] = lse_a;
    }
    if (rb < n_rows) {
      float* pb_ = a.partA + (pbase + row0 + rb) * D;
#pragma unroll
      for (int n = 0; n < NT_O; ++n)
        *reinterpret_cast<float2*>(pb_ + 8 * n + cq) = make_float2(o[n][2] * inv_b, o[n][3] * inv_b);
      if ((lane & 3) == 0) a.partS[pbase + row0 + rb] = lse_b;
    }
    // Append this call's query K/V to the query region (one writer per
    // (batch, kv head); readers in this launch take those rows from the input).
    if (a.plan.chunk[chunk_id].seg < 0 && row0 == 0) {
      const bf16* ks = a.K + (long long)bg * a.lq * D;
      const bf16* vs = a.V + (long long)bg * a.lq * D;
      bf16* kd = c.qK + q_row_offset(c, bb, g, a.len0);
      bf16* vd = c.qV + q_row_offset(c, bb, g, a.len0);
      for (int i = tid; i < a.lq * CPR; i += NTHREADS) {
        reinterpret_cast<uint4*>(kd)[i] = reinterpret_cast<const uint4*>(ks)[i];
        reinterpret_cast<uint4*>(vd)[i] = reinterpret_cast<const uint4*>(vs)[i];
      }
    }
  }
}

// Merge the prefill partials of every packed row and scatter to O / LSE.
template <int D>
__global__ void __launch_bounds__(128) prefill_merge_kernel(CacheView c, int lq, int n_chunks,
                                                            const float* __restrict__ partA,
                                                            const float* __restrict__ partS,
                                                            bf16* __restrict__ O,
                                                            float* __restrict__ LSE) {
  const int rows_total = c.G * lq;
  const long long gw = (long long)blockIdx.x * 4 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (gw >= (long long)c.B * c.Hkv * rows_total) return;
  const long long bg = gw / rows_total;
  const int m = (int)(gw - bg * rows_total);
  const int bb = (int)(bg / c.Hkv), g = (int)(bg - (long long)bb * c.Hkv);
  float mx = -INFINITY;
  for (int p = 0; p < n_chunks; ++p) mx = fmaxf(mx, partS[(bg * n_chunks + p) * rows_total + m]);
  const float base = mx == -INFINITY ? 0.f : mx;
  float tot = 0.f;
  for (int p = 0; p < n_chunks; ++p) tot += __expf(partS[(bg * n_chunks + p) * rows_total + m] - base);
  const float lse = mx == -INFINITY ? -INFINITY : base + __logf(tot);
  constexpr int PER = D / 32;
  float acc[PER];
#pragma unroll
  for (int i = 0; i < PER; ++i) acc[i] = 0.f;
  for (int p = 0; p < n_chunks; ++p) {
    const long long r = (bg * n_chunks + p) * rows_total + m;
    const float s = partS[r];
    if (s == -INFINITY) continue;
    const float w = __expf(s - lse);
#pragma unroll
    for (int i = 0; i < PER; ++i) acc[i] += w * partA[r * D + lane + 32 * i];
  }
  const int h = g * c.G + m / lq;
  const int rr = m % lq;
  bf16* orow = O + (((long long)bb * c.Hq + h) * lq + rr) * D;
#pragma unroll
  for (int i = 0; i < PER; ++i) orow[lane + 32 * i] = __float2bfloat16_rn(acc[i]);
  if (lane == 0) LSE[((long long)bb * c.Hq + h) * lq + rr] = lse;
}

template <int D>
cudaError_t launch_tile(const TileArgs& a, int grid, cudaStream_t st) {
  const int smem = 5 * BM * D * 2;
  cudaError_t e = cudaFuncSetAttribute(prefill_tile_kernel<D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  prefill_tile_kernel<D><<<grid, NTHREADS, smem, st>>>(a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_query_prefill_mma(const CacheView& c, float scale, int lq, int len0,
                                     const bf16* Q, const bf16* Kq, const bf16* Vq, bf16* O,
                                     float* LSE, const PrefillPlan& plan, const Scratch& s,
                                     cudaStream_t st) {
  TileArgs a{};
  a.c = c;
  a.scale_log2 = scale * kLog2e;
  a.Q = Q;
  a.K = Kq;
  a.V = Vq;
  a.lq = lq;
  a.len0 = len0;
  a.partA = s.partA;
  a.partS = s.partS;
  a.plan = plan;
  const int grid = c.B * c.Hkv * plan.row_tiles * plan.n_chunks;
  cudaError_t e = (c.D == 128) ? launch_tile<128>(a, grid, st) : launch_tile<64>(a, grid, st);
  if (e != cudaSuccess) return e;
  const long long rows = (long long)c.B * c.Hkv * c.G * lq;
  const int mgrid = (int)((rows + 3) / 4);
  if (c.D == 128)
    prefill_merge_kernel<128><<<mgrid, 128, 0, st>>>(c, lq, plan.n_chunks, s.partA, s.partS, O, LSE);
  else
    prefill_merge_kernel<64><<<mgrid, 128, 0, st>>>(c, lq, plan.n_chunks, s.partA, s.partS, O, LSE);
  return cudaGetLastError();
}

}  // namespace star
