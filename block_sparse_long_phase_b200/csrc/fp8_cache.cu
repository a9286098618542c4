// FP8 (E4M3) copy of the context KV cache, read by the decode step.
//
// The pages call KV-cache quantisation orthogonal to the method and define
// none; this is the build's own scheme.  Every cached row (one token of one kv
// head) gets the scale s = max|x| / 448 (1 when max|x| <= 1e-30) and codes
// e4m3_rn(x * (1/s)), computed in float32 with IEEE division and rounding to
// nearest even, so |x/s| <= 448 and nothing saturates.  HBM-bound: one warp
// per row reads the bf16 row once and writes D bytes and one scale.
#include <cuda_bf16.h>
#include <stdint.h>

#include "star_common.cuh"
#include "star_internal.h"

namespace star {
namespace {

__device__ __forceinline__ uint16_t e4m3x2(float lo, float hi) {
  uint16_t d;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;\n" : "=h"(d) : "f"(hi), "f"(lo));
  return d;
}

template <int D>
__global__ void __launch_bounds__(256) quantize_rows_kernel(const bf16* __restrict__ src,
                                                            uint8_t* __restrict__ dst,
                                                            float* __restrict__ scale, long long rows) {
  constexpr int PER = D / 32;                     // values per lane (4 or 2)
  const long long row = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  float x[PER];
  const bf16* r = src + row * D + lane * PER;
#pragma unroll
  for (int i = 0; i < PER; ++i) x[i] = __bfloat162float(r[i]);
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < PER; ++i) amax = fmaxf(amax, fabsf(x[i]));
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
  const float s = amax > 1e-30f ? __fdiv_rn(amax, 448.0f) : 1.0f;
  const float inv = __fdiv_rn(1.0f, s);
  uint8_t* o = dst + row * D + lane * PER;
#pragma unroll
  for (int i = 0; i < PER; i += 2) {
    const uint16_t c = e4m3x2(__fmul_rn(x[i], inv), __fmul_rn(x[i + 1], inv));
    *reinterpret_cast<uint16_t*>(o + i) = c;
  }
  if (lane == 0) scale[row] = s;
}

}  // namespace

cudaError_t launch_quantize_ctx_fp8(const CacheView& c, cudaStream_t st) {
  const long long rows = (long long)c.B * c.Hkv * c.L;
  const unsigned grid = (unsigned)((rows + 7) / 8);
  if (c.D == 128) {
    quantize_rows_kernel<128><<<grid, 256, 0, st>>>(c.ctxK, c.ctxK8, c.ctxKs, rows);
    quantize_rows_kernel<128><<<grid, 256, 0, st>>>(c.ctxV, c.ctxV8, c.ctxVs, rows);
  } else {
    quantize_rows_kernel<64><<<grid, 256, 0, st>>>(c.ctxK, c.ctxK8, c.ctxKs, rows);
    quantize_rows_kernel<64><<<grid, 256, 0, st>>>(c.ctxV, c.ctxV8, c.ctxVs, rows);
  }
  return cudaGetLastError();
}

}  // namespace star
