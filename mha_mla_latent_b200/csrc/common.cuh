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

__device__ __forceinline__ void raise_error(int32_t* err, int32_t bit) {
  if (err) atomicOr(err, bit);
}

// int4 two's-complement nibble -> int
__device__ __forceinline__ int nib_to_int(uint32_t n) { return (int)((n ^ 8u) & 15u) - 8; }

constexpr float kLog2e = 1.4426950408889634f;

}  // namespace mla
