// RoPE front end of the Star Attention path and the anchor keys of each block.
//
// "Star Attention: Efficient LLM Inference over Long Sequences", Phase 1
// Step 2: the anchor tokens prepended to block i keep their original position
// IDs while the block's own tokens keep theirs; the position-ID ablation of
// Section 4.1 (Table 4) gives the anchor the first block's IDs (the method),
// the previous block's, or random ones.  With rotary embeddings that means
// every block i >= 1 sees the anchor's keys rotated at its own set of IDs.
//
// Rotation: each adjacent pair (x_2k, x_2k+1) turns by pos * base^(-2k/D).
// The inverse frequencies come from the host in double; the angle is formed
// and reduced to [-pi, pi] in double (positions reach 2^20 and beyond, where
// a float angle would be off by a large fraction of a radian), and only the
// reduced angle goes through sincosf.  HBM-bound: every element is read and
// written once; a CTA holds the cos/sin of 16 positions in shared memory and
// applies them to every head of its batch entry.
#include <cuda_bf16.h>
#include <math.h>
#include <stdint.h>

#include "star_common.cuh"
#include "star_internal.h"

namespace star {
namespace {

constexpr int kTP = 16;                      // positions per CTA
constexpr double kTwoPi = 6.283185307179586476925286766559;

template <int D>
__global__ void __launch_bounds__(256) rope_kernel(const __grid_constant__ RopeJob j) {
  __shared__ float2 cs[kTP][D / 2];
  const long long t0 = (long long)blockIdx.x * kTP;
  const int b = blockIdx.y, grp = blockIdx.z;
  const int np = (int)(j.n - t0 < kTP ? j.n - t0 : kTP);
  for (int i = threadIdx.x; i < kTP * (D / 2); i += blockDim.x) {
    const int t = i / (D / 2), k = i - (i / (D / 2)) * (D / 2);
    if (t < np) {
      const long long p = j.pos ? (long long)j.pos[(long long)grp * j.pos_grp + t0 + t]
                                : j.pos0 + (long long)grp * j.pos0_grp + t0 + t;
      const double a = (double)p * j.inv_freq[k];
      const double r = a - kTwoPi * rint(a * (1.0 / kTwoPi));
      float s, c;
      sincosf((float)r, &s, &c);
      cs[t][k] = make_float2(c, s);
    }
  }
  __syncthreads();
  constexpr int VPR = D / 8;                 // 16-byte vectors (4 pairs) per row
  const int total = j.H * np * VPR;
  for (int i = threadIdx.x; i < total; i += blockDim.x) {
    const int v = i % VPR, r = i / VPR, t = r % np, h = r / np;
    const long long xrow = (long long)grp * j.x_grp + ((long long)b * j.H + h) * j.x_seq + t0 + t;
    const long long yrow = (long long)grp * j.y_grp + ((long long)b * j.H + h) * j.y_seq + t0 + t;
    const uint4 u = *reinterpret_cast<const uint4*>(j.x + xrow * D + v * 8);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
    uint32_t o[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 f = cs[t][v * 4 + e];
      const float x0 = __uint_as_float(w[e] << 16), x1 = __uint_as_float(w[e] & 0xffff0000u);
      o[e] = pack_bf16(x0 * f.x - x1 * f.y, x0 * f.y + x1 * f.x);
    }
    *reinterpret_cast<uint4*>(j.y + yrow * D + v * 8) = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

}  // namespace

void rope_inv_freq(int D, double base, double* out) {
  for (int k = 0; k < D / 2; ++k) out[k] = pow(base, -2.0 * k / D);
}

cudaError_t launch_rope(const RopeJob& j, int D, int B, int groups, cudaStream_t st) {
  if (j.n <= 0 || B <= 0 || groups <= 0) return cudaSuccess;
  const dim3 grid((unsigned)((j.n + kTP - 1) / kTP), (unsigned)B, (unsigned)groups);
  if (D == 128)
    rope_kernel<128><<<grid, 256, 0, st>>>(j);
  else
    rope_kernel<64><<<grid, 256, 0, st>>>(j);
  return cudaGetLastError();
}

}  // namespace star
