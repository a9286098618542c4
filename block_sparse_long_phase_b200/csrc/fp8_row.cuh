// One warp quantises one cache row of D values to E4M3 with its own scale:
// s = max|x| / 448 (1 when max|x| <= 1e-30), codes = e4m3_rn(x * (1/s)), all
// in float32 with IEEE division and rounding to nearest even, so |x/s| <= 448
// and nothing saturates.
#pragma once
#include <cuda_bf16.h>
#include <stdint.h>

namespace star {

__device__ __forceinline__ uint16_t e4m3x2_rn(float lo, float hi) {
  uint16_t d;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;\n" : "=h"(d) : "f"(hi), "f"(lo));
  return d;
}

template <int D>
__device__ __forceinline__ void quantize_row_warp(const __nv_bfloat16* __restrict__ src,
                                                  uint8_t* __restrict__ dst, float* __restrict__ scale,
                                                  int lane) {
  constexpr int PER = D / 32;                     // values per lane (4 or 2)
  float x[PER];
#pragma unroll
  for (int i = 0; i < PER; ++i) x[i] = __bfloat162float(src[lane * PER + i]);
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < PER; ++i) amax = fmaxf(amax, fabsf(x[i]));
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
  const float s = amax > 1e-30f ? __fdiv_rn(amax, 448.0f) : 1.0f;
  const float inv = __fdiv_rn(1.0f, s);
#pragma unroll
  for (int i = 0; i < PER; i += 2)
    *reinterpret_cast<uint16_t*>(dst + lane * PER + i) = e4m3x2_rn(__fmul_rn(x[i], inv), __fmul_rn(x[i + 1], inv));
  if (lane == 0) *scale = s;
}

}  // namespace star
