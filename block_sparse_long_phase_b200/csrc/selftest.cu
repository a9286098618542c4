// Self-test of the failure path of the pipelined kernels: a bounded mbarrier
// wait that runs out makes the kernel set its error word and return, and the
// context stays usable.  The test kernel waits on a barrier nothing arrives
// on, so its wait must give up; it is the same wait (sm100::mbar_wait) the
// phase-1, prefill and decode kernels use, with a short limit.
#include <cuda_runtime.h>

#include "sm100_primitives.cuh"
#include "star_common.cuh"
#include "star_internal.h"

namespace star {
namespace {

using namespace sm100;

__device__ int g_selftest_err;

__global__ void wait_timeout_kernel(unsigned polls) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0 && !mbar_wait(smem_u32(&bar), 0, polls)) atomicExch(&g_selftest_err, 1);
}

}  // namespace

cudaError_t run_wait_timeout(unsigned polls, int* gave_up, cudaStream_t st) {
  const int zero = 0;
  cudaError_t e = cudaMemcpyToSymbolAsync(g_selftest_err, &zero, sizeof(int), 0, cudaMemcpyHostToDevice, st);
  if (e != cudaSuccess) return e;
  wait_timeout_kernel<<<1, 32, 0, st>>>(polls);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  e = cudaMemcpyFromSymbolAsync(gave_up, g_selftest_err, sizeof(int), 0, cudaMemcpyDeviceToHost, st);
  if (e != cudaSuccess) return e;
  return cudaStreamSynchronize(st);
}

}  // namespace star
