// Phase-2 generation step: split-KV HBM-streaming attention with a fused
// log-sum-exp merge.
//
// "Star Attention: Efficient LLM Inference over Long Sequences" (analysis
// page), section 3.4, "Phase 2: Query Encoding and Token Generation with
// Distributed Softmax": every context block ("host") computes the local
// attention A_h and its exponent sum s_h for the new token (Step 3), the
// partials are combined with the log-sum-exp rule (Step 5), and only the query
// region's cache grows (Step 7).  On one GPU each CTA plays a "host" for one
// contiguous chunk of the (batch, kv head)'s key sequence
// [context segments | query region | new token]; chunks are sized so that the
// grid is two CTAs per SM.  The last CTA of each (batch, kv head) to finish --
// chosen by an atomic ticket, no CTA ever waits for another -- merges that
// head's partials and writes the output.
//
// Inside a CTA: the G query heads that share the kv head are the M rows of a
// 16x8x16 bf16 MMA (rows G..15 are zero), K/V stream through a 3-stage
// cp.async ring of 64-key stages in XOR-swizzled shared memory, and each of
// the 4 warps owns 16 keys of every stage with its own online softmax; the
// warps' states are combined in shared memory at the end.
#include <cuda_bf16.h>
#include <math.h>

#include "star_common.cuh"
#include "star_internal.h"

namespace star {
namespace {

constexpr int KS = 64;        // keys per stage
constexpr int NSTAGE = 3;
constexpr int NTHREADS = 128;

struct DecodeArgs {
  CacheView c;
  float scale_log2;
  int len0;                   // query-region rows before this step
  int cph;                    // chunks per (batch, kv head)
  int chunk_rows;
  const bf16* q;              // [B][Hq][D]
  const bf16* k;              // [B][Hkv][D]
  const bf16* v;
  bf16* o;                    // [B][Hq][D]
  float* lse;                 // [B][Hq]
  float* partA;               // [B*Hkv][cph][G][D]
  float* partS;               // [B*Hkv][cph][G]
  unsigned* tickets;          // [B*Hkv]
};

template <int D>
__global__ void __launch_bounds__(NTHREADS) decode_kernel(const __grid_constant__ DecodeArgs a) {
  constexpr int CPR = D / 8;
  constexpr int STAGE_BYTES = KS * D * 2;
  constexpr int NT_O = D / 8;
  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t* sQ = smem;                               // 16 x D bf16
  uint8_t* sK = smem + 16 * D * 2;                  // NSTAGE stages
  uint8_t* sV = sK + NSTAGE * STAGE_BYTES;
  __shared__ int s_last;

  const CacheView& c = a.c;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int bg = blockIdx.x / a.cph;
  const int chunk = blockIdx.x - bg * a.cph;
  const int bb = bg / c.Hkv, g = bg - bb * c.Hkv;
  const int G = c.G;
  const int Lc = (int)c.L;
  const int n_keys_total = Lc + a.len0 + 1;
  const int j_begin = chunk * a.chunk_rows;
  int j_end = j_begin + a.chunk_rows;
  if (j_end > n_keys_total) j_end = n_keys_total;
  const int nk = j_end > j_begin ? j_end - j_begin : 0;
  const int n_st = (nk + KS - 1) / KS;

  const bf16* knew = a.k + (long long)bg * D;
  const bf16* vnew = a.v + (long long)bg * D;

  // Append the new token to the query region (readers in this launch take it
  // from the input, so the write order does not matter).
  if (chunk == a.cph - 1 && tid < CPR) {
    const long long off = q_row_offset(c, bb, g, a.len0);
    reinterpret_cast<uint4*>(c.qK + off)[tid] = reinterpret_cast<const uint4*>(knew)[tid];
    reinterpret_cast<uint4*>(c.qV + off)[tid] = reinterpret_cast<const uint4*>(vnew)[tid];
  }

  auto row_ptr = [&](int j, bool v) -> const bf16* {
    if (j < Lc) {
      const int seg = j / c.b;
      const int off = j - seg * c.b;
      const long long len = seg_len(c, seg);
      const long long base = (long long)seg * c.B * c.Hkv * (long long)c.b * D +
                             (((long long)bb * c.Hkv + g) * len + off) * D;
      return (v ? c.ctxV : c.ctxK) + base;
    }
    if (j < Lc + a.len0) return (v ? c.qV : c.qK) + q_row_offset(c, bb, g, j - Lc);
    return v ? vnew : knew;
  };
  auto load_stage = [&](int slot, int st) {
    const int j0 = j_begin + st * KS;
    const uint32_t dk = smem_u32(sK + slot * STAGE_BYTES);
    const uint32_t dv = smem_u32(sV + slot * STAGE_BYTES);
    for (int i = tid; i < KS * CPR; i += NTHREADS) {
      const int row = i / CPR, ch = i - (i / CPR) * CPR;
      const int j = j0 + row;
      const bool ok = j < j_end;
      const bf16* kp = ok ? row_ptr(j, false) : knew;
      const bf16* vp = ok ? row_ptr(j, true) : vnew;
      cp_async16(dk + swz(row, ch, CPR), kp + ch * 8, ok ? 16 : 0);
      cp_async16(dv + swz(row, ch, CPR), vp + ch * 8, ok ? 16 : 0);
    }
  };

  // Q rows 0..G-1 of this kv group, zero beyond.
  for (int i = tid; i < 16 * CPR; i += NTHREADS) {
    const int row = i / CPR, ch = i - (i / CPR) * CPR;
    const bool ok = row < G;
    const bf16* src = a.q + ((long long)bb * c.Hq + g * G + (ok ? row : 0)) * D + ch * 8;
    cp_async16(smem_u32(sQ) + swz(row, ch, CPR), src, ok ? 16 : 0);
  }
#pragma unroll
  for (int s = 0; s < NSTAGE - 1; ++s) {
    if (s < n_st) load_stage(s, s);
    cp_async_commit();
  }

  uint32_t qa[D / 16][4];
  float o[NT_O][4];
#pragma unroll
  for (int n = 0; n < NT_O; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
  float m_a = -INFINITY, m_b = -INFINITY, l_a = 0.f, l_b = 0.f;

  for (int st = 0; st < n_st; ++st) {
    const int slot = st % NSTAGE;
    if (st + NSTAGE - 1 < n_st) load_stage((st + NSTAGE - 1) % NSTAGE, st + NSTAGE - 1);
    cp_async_commit();
    cp_async_wait<NSTAGE - 1>();
    __syncthreads();
    if (st == 0) {
#pragma unroll
      for (int kd = 0; kd < D / 16; ++kd) {
        const int row = (lane & 7) + ((lane >> 3) & 1) * 8;
        const int ch = 2 * kd + (lane >> 4);
        ldmatrix_x4(smem_u32(sQ) + swz(row, ch, CPR), qa[kd][0], qa[kd][1], qa[kd][2], qa[kd][3]);
      }
    }
    const uint32_t kbase = smem_u32(sK + slot * STAGE_BYTES);
    const uint32_t vbase = smem_u32(sV + slot * STAGE_BYTES);
    float s[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
    for (int kd = 0; kd < D / 16; ++kd) {
      const int row = 16 * warp + (lane & 7) + ((lane >> 4) << 3);
      const int ch = 2 * kd + ((lane >> 3) & 1);
      uint32_t b0, b1, b2, b3;
      ldmatrix_x4(kbase + swz(row, ch, CPR), b0, b1, b2, b3);
      mma_bf16_16816(s[0], qa[kd], b0, b1);
      mma_bf16_16816(s[1], qa[kd], b2, b3);
    }
    const int jw = j_begin + st * KS + 16 * warp;   // first key of this warp
#pragma unroll
    for (int n = 0; n < 2; ++n) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int j = jw + 8 * n + 2 * (lane & 3) + (e & 1);
        s[n][e] = j < j_end ? s[n][e] * a.scale_log2 : -INFINITY;
      }
    }
    float mx_a = fmaxf(fmaxf(s[0][0], s[0][1]), fmaxf(s[1][0], s[1][1]));
    float mx_b = fmaxf(fmaxf(s[0][2], s[0][3]), fmaxf(s[1][2], s[1][3]));
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
#pragma unroll
    for (int n = 0; n < 2; ++n) {
      s[n][0] = exp2f(s[n][0] - base_a);
      s[n][1] = exp2f(s[n][1] - base_a);
      s[n][2] = exp2f(s[n][2] - base_b);
      s[n][3] = exp2f(s[n][3] - base_b);
    }
    l_a = l_a * al_a + s[0][0] + s[0][1] + s[1][0] + s[1][1];
    l_b = l_b * al_b + s[0][2] + s[0][3] + s[1][2] + s[1][3];
    uint32_t pa[4];
    pa[0] = pack_bf16(s[0][0], s[0][1]);
    pa[1] = pack_bf16(s[0][2], s[0][3]);
    pa[2] = pack_bf16(s[1][0], s[1][1]);
    pa[3] = pack_bf16(s[1][2], s[1][3]);
#pragma unroll
    for (int j = 0; j < D / 16; ++j) {
      o[2 * j][0] *= al_a;
      o[2 * j][1] *= al_a;
      o[2 * j][2] *= al_b;
      o[2 * j][3] *= al_b;
      o[2 * j + 1][0] *= al_a;
      o[2 * j + 1][1] *= al_a;
      o[2 * j + 1][2] *= al_b;
      o[2 * j + 1][3] *= al_b;
      const int row = 16 * warp + (lane & 7) + ((lane >> 3) & 1) * 8;
      const int ch = 2 * j + (lane >> 4);
      uint32_t b0, b1, b2, b3;
      ldmatrix_x4_trans(vbase + swz(row, ch, CPR), b0, b1, b2, b3);
      mma_bf16_16816(o[2 * j], pa, b0, b1);
      mma_bf16_16816(o[2 * j + 1], pa, b2, b3);
    }
    __syncthreads();
  }
  cp_async_wait<0>();
  __syncthreads();

  // ---- combine the 4 warps (shared memory reuses the K ring) ---------------
  l_a += __shfl_xor_sync(0xffffffffu, l_a, 1);
  l_a += __shfl_xor_sync(0xffffffffu, l_a, 2);
  l_b += __shfl_xor_sync(0xffffffffu, l_b, 1);
  l_b += __shfl_xor_sync(0xffffffffu, l_b, 2);
  float* wm = reinterpret_cast<float*>(sK);          // [4][16]
  float* wl = wm + 4 * 16;                            // [4][16]
  float* wo = wl + 4 * 16;                            // [4][16][D]
  const int ra = lane >> 2, rb = ra + 8, cq = 2 * (lane & 3);
  if ((lane & 3) == 0) {
    wm[warp * 16 + ra] = m_a;
    wm[warp * 16 + rb] = m_b;
    wl[warp * 16 + ra] = l_a;
    wl[warp * 16 + rb] = l_b;
  }
#pragma unroll
  for (int n = 0; n < NT_O; ++n) {
    wo[(warp * 16 + ra) * D + 8 * n + cq] = o[n][0];
    wo[(warp * 16 + ra) * D + 8 * n + cq + 1] = o[n][1];
    wo[(warp * 16 + rb) * D + 8 * n + cq] = o[n][2];
    wo[(warp * 16 + rb) * D + 8 * n + cq + 1] = o[n][3];
  }
  __syncthreads();
  const long long pbase = ((long long)bg * a.cph + chunk) * G;
  for (int idx = tid; idx < G * D; idx += NTHREADS) {
    const int r = idx / D, d = idx - (idx / D) * D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < 4; ++w) M = fmaxf(M, wm[w * 16 + r]);
    const float base = M == -INFINITY ? 0.f : M;
    float Lsum = 0.f, acc = 0.f;
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const float f = exp2f(wm[w * 16 + r] - base);
      Lsum += f * wl[w * 16 + r];
      acc += f * wo[(w * 16 + r) * D + d];
    }
    a.partA[(pbase + r) * D + d] = Lsum > 0.f ? acc / Lsum : 0.f;
    if (d == 0) a.partS[pbase + r] = Lsum > 0.f ? (base + log2f(Lsum)) * kLn2 : -INFINITY;
  }

  // ---- last CTA of this (batch, kv head) merges ----------------------------
  __threadfence();
  __syncthreads();
  if (tid == 0) s_last = (atomicAdd(&a.tickets[bg], 1u) == (unsigned)(a.cph - 1));
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  float* wts = reinterpret_cast<float*>(sV);          // [G][cph] merge weights
  float* lse_s = wts + G * a.cph;                     // [G]
  if (tid < G) {
    const int r = tid;
    float M = -INFINITY;
    for (int p = 0; p < a.cph; ++p)
      M = fmaxf(M, __ldcg(a.partS + ((long long)bg * a.cph + p) * G + r));
    const float base = M == -INFINITY ? 0.f : M;
    float tot = 0.f;
    for (int p = 0; p < a.cph; ++p)
      tot += __expf(__ldcg(a.partS + ((long long)bg * a.cph + p) * G + r) - base);
    const float l = M == -INFINITY ? -INFINITY : base + __logf(tot);
    lse_s[r] = l;
    for (int p = 0; p < a.cph; ++p) {
      const float sp = __ldcg(a.partS + ((long long)bg * a.cph + p) * G + r);
      wts[r * a.cph + p] = sp == -INFINITY ? 0.f : __expf(sp - l);
    }
  }
  __syncthreads();
  for (int idx = tid; idx < G * D; idx += NTHREADS) {
    const int r = idx / D, d = idx - (idx / D) * D;
    float acc = 0.f;
    for (int p = 0; p < a.cph; ++p) {
      const float w = wts[r * a.cph + p];
      if (w != 0.f) acc += w * __ldcg(a.partA + (((long long)bg * a.cph + p) * G + r) * D + d);
    }
    const long long orow = (long long)bb * c.Hq + g * G + r;
    a.o[orow * D + d] = __float2bfloat16_rn(acc);
    if (d == 0) a.lse[orow] = lse_s[r];
  }
  if (tid == 0) a.tickets[bg] = 0u;   // ready for the next step
}

}  // namespace

cudaError_t launch_decode_step(const CacheView& c, float scale, int len0, const bf16* q,
                               const bf16* k, const bf16* v, bf16* o, float* lse,
                               const DecodePlan& plan, const Scratch& s, cudaStream_t st) {
  DecodeArgs a{};
  a.c = c;
  a.scale_log2 = scale * kLog2e;
  a.len0 = len0;
  a.cph = plan.chunks_per_head;
  a.chunk_rows = (int)plan.chunk_rows;
  a.q = q;
  a.k = k;
  a.v = v;
  a.o = o;
  a.lse = lse;
  a.partA = s.partA;
  a.partS = s.partS;
  a.tickets = s.tickets;
  const int grid = c.B * c.Hkv * plan.chunks_per_head;
  cudaError_t e;
  if (c.D == 128) {
    const int smem = 16 * 128 * 2 + 2 * NSTAGE * KS * 128 * 2;
    e = cudaFuncSetAttribute(decode_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    decode_kernel<128><<<grid, NTHREADS, smem, st>>>(a);
  } else {
    const int smem = 16 * 64 * 2 + 2 * NSTAGE * KS * 64 * 2;
    e = cudaFuncSetAttribute(decode_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    decode_kernel<64><<<grid, NTHREADS, smem, st>>>(a);
  }
  return cudaGetLastError();
}

}  // namespace star
