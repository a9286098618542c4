// Standalone phase-2 merge of per-partition partials.
//
// "Star Attention: Efficient LLM Inference over Long Sequences" (analysis
// page), section 3.4, "Phase 2", Step 5, and the "NVIDIA/Star-Attention"
// README, "Phase 2": with s_h carried as the log of the partition's exponent
// sum, s = log sum_h exp(s_h) and A = sum_h exp(s_h - s) A_h (the README's
// s_h / s_global weights written in log space, the maximum subtracted first).
// Memory-bound: one warp per row streams the row's P partial vectors once.
#include <math.h>

#include "star_common.cuh"
#include "star_internal.h"

namespace star {
namespace {

constexpr int ROWS_PER_CTA = 8;

// outA (float32) and outB (bf16, rounded to nearest even once) may each be null.
__global__ void __launch_bounds__(32 * ROWS_PER_CTA)
    lse_merge_kernel(int P, long long R, int D, const float* __restrict__ A,
                     const float* __restrict__ S, float* __restrict__ outA,
                     bf16* __restrict__ outB, float* __restrict__ outS) {
  const long long r = (long long)blockIdx.x * ROWS_PER_CTA + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (r >= R) return;
  // Row maximum and total in one pass (online), lanes split the parts.
  float m = -INFINITY, tot = 0.f;
  for (int p = lane; p < P; p += 32) {
    const float s = S[(long long)p * R + r];
    if (s == -INFINITY) continue;
    if (s > m) {
      tot = tot * __expf(m - s) + 1.f;
      m = s;
    } else {
      tot += __expf(s - m);
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    const float mo = __shfl_xor_sync(0xffffffffu, m, off);
    const float to = __shfl_xor_sync(0xffffffffu, tot, off);
    const float mn = fmaxf(m, mo);
    const float base = mn == -INFINITY ? 0.f : mn;
    tot = (m == -INFINITY ? 0.f : tot * __expf(m - base)) +
          (mo == -INFINITY ? 0.f : to * __expf(mo - base));
    m = mn;
  }
  const float lse = m == -INFINITY ? -INFINITY : m + __logf(tot);
  for (int d0 = 0; d0 < D; d0 += 128) {
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    for (int p = 0; p < P; ++p) {
      const float s = S[(long long)p * R + r];
      if (s == -INFINITY) continue;
      const float w = __expf(s - lse);
      const float* row = A + ((long long)p * R + r) * D;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int d = d0 + lane + 32 * i;
        if (d < D) acc[i] += w * row[d];
      }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int d = d0 + lane + 32 * i;
      if (d < D && outA) outA[r * D + d] = acc[i];
      if (d < D && outB) outB[r * D + d] = __float2bfloat16_rn(acc[i]);
    }
  }
  if (lane == 0) outS[r] = lse;
}

}  // namespace

cudaError_t launch_lse_merge(int P, long long R, int D, const float* A, const float* S,
                             float* outA, float* outS, cudaStream_t st, bf16* outB) {
  if (R == 0) return cudaSuccess;
  const long long grid = (R + ROWS_PER_CTA - 1) / ROWS_PER_CTA;
  lse_merge_kernel<<<(unsigned)grid, 32 * ROWS_PER_CTA, 0, st>>>(P, R, D, A, S, outA, outB, outS);
  return cudaGetLastError();
}

}  // namespace star
