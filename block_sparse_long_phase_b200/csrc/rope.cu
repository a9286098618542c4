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
// written once; a thread computes the cos/sin of its 4 pairs at one position
// and applies them to that slice of every head of its batch entry (of every
// other head at D = 64).
#include <cuda_bf16.h>
#include <math.h>
#include <stdint.h>

#include "star_common.cuh"
#include "star_internal.h"

namespace star {
namespace {

// A CTA turns 16 positions of every head: one thread per (position, 16-byte
// vector) slot at D = 128, two heads side by side at D = 64.  (Four-position
// CTAs, for a shorter last wave, measured slower: 107 registers, 2 CTAs/SM.)
template <int D>
constexpr int kTP = 16;
constexpr double kTwoPi = 6.283185307179586476925286766559;

template <int D>
__global__ void __launch_bounds__(256) rope_kernel(const __grid_constant__ RopeJob j) {
  // Thread = (position t, 16-byte vector v of 4 pairs); it turns that vector
  // of every head, so its 4 (cos, sin) pairs are computed once, in registers.
  constexpr int VPR = D / 8;                 // 16-byte vectors per row
  constexpr int TV = kTP<D> * VPR;           // (position, vector) slots of a CTA
  constexpr int HS = 256 / TV;               // heads taken side by side
  constexpr int kU = 8;                      // loads in flight per thread
  const int tv = threadIdx.x % TV, hs = threadIdx.x / TV;
  const int t = tv / VPR, v = tv % VPR;
  const long long tok = (long long)blockIdx.x * kTP<D> + t;
  const int b = blockIdx.y, grp = blockIdx.z;
  if (tok >= j.n) return;
  const long long p = j.pos ? (long long)j.pos[(long long)grp * j.pos_grp + tok]
                            : j.pos0 + (long long)grp * j.pos0_grp + tok;
  float2 cv[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const double a = (double)p * j.inv_freq[4 * v + e];
    const double r = a - kTwoPi * rint(a * (1.0 / kTwoPi));
    sincosf((float)r, &cv[e].y, &cv[e].x);
  }
  const bf16* x = j.x + ((long long)grp * j.x_grp + (long long)b * j.H * j.x_seq + tok) * D + v * 8;
  bf16* y = j.y + ((long long)grp * j.y_grp + (long long)b * j.H * j.y_seq + tok) * D + v * 8;
  const long long xs = j.x_seq * D, ys = j.y_seq * D;
  for (int h0 = hs; h0 < j.H; h0 += kU * HS) {
    uint4 u[kU];
#pragma unroll
    for (int q = 0; q < kU; ++q) {
      const int h = h0 + q * HS;
      if (h < j.H) u[q] = *reinterpret_cast<const uint4*>(x + h * xs);
    }
#pragma unroll
    for (int q = 0; q < kU; ++q) {
      const int h = h0 + q * HS;
      if (h < j.H) {
        const uint32_t w[4] = {u[q].x, u[q].y, u[q].z, u[q].w};
        uint32_t o[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float x0 = __uint_as_float(w[e] << 16), x1 = __uint_as_float(w[e] & 0xffff0000u);
          o[e] = pack_bf16(x0 * cv[e].x - x1 * cv[e].y, x0 * cv[e].y + x1 * cv[e].x);
        }
        *reinterpret_cast<uint4*>(y + h * ys) = make_uint4(o[0], o[1], o[2], o[3]);
      }
    }
  }
}

}  // namespace

void rope_inv_freq(int D, double base, double* out) {
  for (int k = 0; k < D / 2; ++k) out[k] = pow(base, -2.0 * k / D);
}

cudaError_t launch_rope(const RopeJob& j, int D, int B, int groups, cudaStream_t st) {
  if (j.n <= 0 || B <= 0 || groups <= 0) return cudaSuccess;
  const int tp = D == 128 ? kTP<128> : kTP<64>;
  const dim3 grid((unsigned)((j.n + tp - 1) / tp), (unsigned)B, (unsigned)groups);
  if (D == 128)
    rope_kernel<128><<<grid, 256, 0, st>>>(j);
  else
    rope_kernel<64><<<grid, 256, 0, st>>>(j);
  return cudaGetLastError();
}

}  // namespace star
