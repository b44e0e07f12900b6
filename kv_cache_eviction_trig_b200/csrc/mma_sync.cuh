// Warp-level tensor-core helpers shared by the kernels that read 2-D TMA tiles
// (128-byte swizzle, boxes of 64 bf16 dims per row) straight from shared memory:
// ldmatrix loads and the bf16 m16n8k16 MMA with float32 accumulators.
//
// Fragment layout of mma m16n8k16 (r0 = lane / 4, k0 = 2 (lane % 4)):
//   A (16 x 16, row-major)  a0 = A[r0][k0, k0+1]   a1 = A[r0+8][k0, k0+1]
//                           a2 = A[r0][k0+8, k0+9] a3 = A[r0+8][k0+8, k0+9]
//   B (16 x 8)              b0 = B[k0, k0+1][r0]   b1 = B[k0+8, k0+9][r0]
//   C (16 x 8, float)       c0 = C[r0][k0] c1 = C[r0][k0+1] c2 = C[r0+8][k0] c3 = C[r0+8][k0+1]
// (each bf16 pair packed low element first).
#pragma once

#include "tria_internal.cuh"

namespace tria {

// Address of the 16-byte unit holding dims [dim, dim + 8) of row `row` of a tile
// stored as 128-byte-swizzled TMA boxes of 64 dims, BOXB bytes per box.
template <int BOXB>
__device__ __forceinline__ uint32_t swz(uint32_t base, int row, int dim) {
  return base + (uint32_t)(dim >> 6) * BOXB + (uint32_t)row * 128u +
         ((uint32_t)(((dim >> 3) & 7) ^ (row & 7)) << 4);
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr));
}
__device__ __forceinline__ void ldsm_x2(uint32_t addr, uint32_t (&r)[2]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0, %1}, [%2];"
               : "=r"(r[0]), "=r"(r[1]) : "r"(addr));
}
__device__ __forceinline__ void mma_bf16(float (&c)[4], const uint32_t (&a)[4], const uint32_t (&b)[2]) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, "
      "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

// Two floats rounded to a bf16 pair (a in the low half).
__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(b), "f"(a));
  return r;
}

}  // namespace tria
