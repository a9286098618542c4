// FP8 (E4M3) copy of the KV cache, read by the decode step.
//
// The pages call KV-cache quantisation orthogonal to the method and define
// none; this is the build's own scheme (fp8_row.cuh): one float32 scale per
// cached row (one token of one kv head).  The context rows are quantised once
// after phase 1; query-region rows as a prefill appends them (a decode step
// quantises its own new row).  HBM-bound: one warp per row reads the bf16 row
// once and writes D bytes and one scale.
#include <cuda_bf16.h>
#include <stdint.h>

#include "fp8_row.cuh"
#include "star_common.cuh"
#include "star_internal.h"

namespace star {
namespace {

// rows [0, rows) of src -> same rows of dst / scale
template <int D>
__global__ void __launch_bounds__(256) quantize_rows_kernel(const bf16* __restrict__ src,
                                                            uint8_t* __restrict__ dst,
                                                            float* __restrict__ scale, long long rows) {
  const long long row = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
  if (row >= rows) return;
  quantize_row_warp<D>(src + row * D, dst + row * D, scale + row, threadIdx.x & 31);
}

// prefill rows: input row (bg, r) of [B*Hkv][lq][D] -> query-region row
// bg * q_cap + len0 + r
template <int D>
__global__ void __launch_bounds__(256) quantize_qrows_kernel(const bf16* __restrict__ src,
                                                             uint8_t* __restrict__ dst,
                                                             float* __restrict__ scale, int bgs, int lq,
                                                             int q_cap, int len0, int* err) {
  const long long row = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
  if (row >= (long long)bgs * lq) return;
  const long long bg = row / lq, r = row - bg * lq;
  const long long out = bg * q_cap + len0 + r;
  if (!STAR_STORE_OK(out, (long long)bgs * q_cap, err)) return;
  quantize_row_warp<D>(src + row * D, dst + out * D, scale + out, threadIdx.x & 31);
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

cudaError_t launch_quantize_qregion_fp8(const CacheView& c, const bf16* K, const bf16* V, int len0, int lq,
                                        cudaStream_t st) {
  const int bgs = c.B * c.Hkv;
  const unsigned grid = (unsigned)(((long long)bgs * lq + 7) / 8);
  if (grid == 0) return cudaSuccess;
  if (c.D == 128) {
    quantize_qrows_kernel<128><<<grid, 256, 0, st>>>(K, c.qK8, c.qKs, bgs, lq, c.q_cap, len0, c.err);
    quantize_qrows_kernel<128><<<grid, 256, 0, st>>>(V, c.qV8, c.qVs, bgs, lq, c.q_cap, len0, c.err);
  } else {
    quantize_qrows_kernel<64><<<grid, 256, 0, st>>>(K, c.qK8, c.qKs, bgs, lq, c.q_cap, len0, c.err);
    quantize_qrows_kernel<64><<<grid, 256, 0, st>>>(V, c.qV8, c.qVs, bgs, lq, c.q_cap, len0, c.err);
  }
  return cudaGetLastError();
}

}  // namespace star
