// Warp-level tensor-core products for the small dense contractions beside the attention
// kernel (decode-step append, split merge): m16n8k16 bf16 x bf16 -> f32 with ldmatrix
// fragment loads.  These products have 8 to 32 rows; on them a tcgen05.mma (which costs
// about the same issue time whatever its shape) would spend more time issuing than the
// warp-level form spends computing.
#pragma once

#include <stdint.h>

namespace mla {
namespace wmma16 {

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// Four 8x8 b16 matrices; lane l supplies the address of row (l % 8) of matrix (l / 8).
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

// d += a * b;  a: 16x16 row-major fragment, b: 16x8 column fragment, d: 16x8 f32.
__device__ __forceinline__ void mma_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// A fragment (rows m0..m0+15, k0..k0+15) of a row-major bf16 tile with row stride `ld`
// elements.
__device__ __forceinline__ void load_a(uint32_t (&a)[4], const __nv_bfloat16* tile, int ld, int m0, int k0, int lane) {
  const __nv_bfloat16* p = tile + (size_t)(m0 + (lane & 15)) * ld + k0 + ((lane >> 4) << 3);
  ldsm_x4(smem_addr(p), a[0], a[1], a[2], a[3]);
}

// B fragments of two adjacent n-tiles (k0..k0+15, n0..n0+15) of a row-major [k][n] bf16
// tile with row stride `ld`: (b[0], b[1]) for n0..n0+7 and (b[2], b[3]) for n0+8..n0+15.
__device__ __forceinline__ void load_b2(uint32_t (&b)[4], const __nv_bfloat16* tile, int ld, int k0, int n0, int lane) {
  const __nv_bfloat16* p = tile + (size_t)(k0 + (lane & 15)) * ld + n0 + ((lane >> 4) << 3);
  ldsm_x4_t(smem_addr(p), b[0], b[1], b[2], b[3]);
}

}  // namespace wmma16
}  // namespace mla
