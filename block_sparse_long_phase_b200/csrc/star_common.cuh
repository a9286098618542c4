// Shared device helpers for the libstar kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#define STAR_DEVICE __device__ __forceinline__

namespace star {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// Bounds-checked build (nvcc -DSTAR_CHECK_BOUNDS, lib/libstar_checked.so): a
// kernel checks each global index it computes for a store (and for the cache
// rows phase 1 copies) against the size of the buffer; a bad index sets the
// cache's error word to 2 and the access is skipped.  The normal build
// compiles the checks away.
STAR_DEVICE bool store_ok(long long idx, long long n, int* err) {
  if (idx >= 0 && idx < n) return true;
  if (err) atomicExch(err, 2);
  return false;
}
#ifdef STAR_CHECK_BOUNDS
#define STAR_STORE_OK(idx, n, err) ::star::store_ok((long long)(idx), (long long)(n), (err))
#else
// (the operands are named, never evaluated, so the unchecked build sees them used)
#define STAR_STORE_OK(idx, n, err) ((void)sizeof((idx) + (n)), (void)sizeof(err), true)
#endif

STAR_DEVICE uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// 16-byte async global->shared copy; src_bytes = 0 fills the 16 bytes with 0.
STAR_DEVICE void cp_async16(uint32_t dst, const void* src, int src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src),
               "r"(src_bytes));
}
STAR_DEVICE void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
template <int N>
STAR_DEVICE void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N));
}

STAR_DEVICE void ldmatrix_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                             uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
STAR_DEVICE void ldmatrix_x4_trans(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                   uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

// D = A(16x16 bf16, row) * B(16x8 bf16, col) + D, fp32 accumulate.
STAR_DEVICE void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

STAR_DEVICE uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

STAR_DEVICE float fast_exp2(float x) { return exp2f(x); }

// Byte offset of 16-byte chunk `chunk` of row `row` in a [rows][chunks_per_row]
// tile whose chunk index is XOR-swizzled with the row's low 3 bits, so eight
// consecutive rows at one logical chunk hit eight different bank groups.
STAR_DEVICE uint32_t swz(int row, int chunk, int chunks_per_row) {
  return static_cast<uint32_t>((row * chunks_per_row + (chunk ^ (row & 7))) * 16);
}

}  // namespace star
