// Device helpers shared by the kernels: element conversion and the error word.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "mla_internal.h"


namespace mla {

__device__ __forceinline__ float to_f32(float v) { return v; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 v) { return __bfloat162float(v); }

template <typename T> __device__ __forceinline__ T from_f32(float v);
template <> __device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float v) {
  return __float2bfloat16_rn(v);
}

// Round a double directly to the storage type (one rounding).
template <typename T> __device__ __forceinline__ T from_f64(double v);
template <> __device__ __forceinline__ float from_f64<float>(double v) { return __double2float_rn(v); }
template <> __device__ __forceinline__ __nv_bfloat16 from_f64<__nv_bfloat16>(double v) {
  return __double2bfloat16(v);  // single round-to-nearest-even from double
}

// Read-only global load (non-coherent path): tells the compiler the source cannot alias
// shared memory, so loads are not serialised behind shared-memory stores.
template <typename T> __device__ __forceinline__ float ldg_f32(const T* p) { return to_f32(__ldg(p)); }

// Stages a tile of `rows` x `cols` elements of T into shared memory as float
// (dst[r * dst_ld + c]), row r starting at row_ptr(r).  Each thread issues a batch of up to
// 8 loads before it uses any (16-byte vectors when `vec`: every row start 16-byte aligned
// and cols a multiple of 16 / sizeof(T)), so a batch costs one memory round trip.
template <typename T, typename RowPtr>
__device__ __forceinline__ void stage_rows_f32(float* dst, int dst_ld, int rows, int cols, bool vec, RowPtr row_ptr) {
  const int tid = threadIdx.x, nt = blockDim.x;
  if (vec) {
    constexpr int VEC = 16 / sizeof(T);
    const int vpr = cols / VEC, nv = rows * vpr;
    for (int base = 0; base < nv; base += 8 * nt) {
      uint4 r[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const int v = base + tid + k * nt;
        if (v < nv) r[k] = __ldg(reinterpret_cast<const uint4*>(row_ptr(v / vpr) + (v % vpr) * VEC));
      }
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const int v = base + tid + k * nt;
        if (v < nv) {
          const T* e = reinterpret_cast<const T*>(&r[k]);
          float* d = dst + (v / vpr) * dst_ld + (v % vpr) * VEC;
#pragma unroll
          for (int t = 0; t < VEC; ++t) d[t] = to_f32(e[t]);
        }
      }
    }
  } else {
    const int n = rows * cols;
    for (int base = 0; base < n; base += 8 * nt) {
      float f[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const int i = base + tid + k * nt;
        f[k] = i < n ? to_f32(__ldg(row_ptr(i / cols) + i % cols)) : 0.f;
      }
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const int i = base + tid + k * nt;
        if (i < n) dst[(i / cols) * dst_ld + i % cols] = f[k];
      }
    }
  }
}

// Programmatic dependent launch.  pdl_wait() returns once the preceding kernel in the
// stream has completed and its writes are visible (at once when the launch carries no
// programmatic dependency); pdl_trigger() lets the next kernel start launching.  Every
// kernel of the library waits before its first global write and before reading anything
// an earlier kernel produced, and triggers only after that wait, so completion stays
// ordered along the stream.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

__device__ __forceinline__ void raise_error(int32_t* err, int32_t bit) {
  if (err) atomicOr(err, bit);
}

// int4 two's-complement nibble -> int
__device__ __forceinline__ int nib_to_int(uint32_t n) { return (int)((n ^ 8u) & 15u) - 8; }

constexpr float kLog2e = 1.4426950408889634f;

// sin and cos of the RoPE angle p * theta.  The angle is formed and reduced to [-pi, pi] in
// float64 by Cody and Waite's two-constant reduction (2 pi = hi + lo, hi with 31 significant
// bits so that k * hi is exact for |k| < 2^20, i.e. angles below ~6.5e6 rad), and the
// float32 sincos of the reduced angle follows: about 3e-7 absolute error, far below the
// rounding of the bf16 / f32 values it rotates.
__device__ __forceinline__ void rope_sincos(int p, double theta, float* s, float* c) {
  const double a = (double)p * theta;
  const double k = rint(a * 0.15915494309189535);   // 1 / (2 pi)
  double r = fma(-k, 6.2831853069365025, a);        // hi part of 2 pi
  r = fma(-k, 2.430840202602477e-10, r);            // lo part
  sincosf((float)r, s, c);
}

}  // namespace mla
