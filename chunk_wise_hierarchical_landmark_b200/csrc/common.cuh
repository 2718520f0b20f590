// Device helpers shared by the HiLS kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace hils {

// Error word written by device-side checks (debug mode).  Codes match the
// hils_status values they are reported as.
enum : uint32_t { DEV_OK = 0, DEV_BAD_INDEX = 5, DEV_TIMEOUT = 6 };

template <typename T>
__device__ __forceinline__ float to_f(T x);
template <>
__device__ __forceinline__ float to_f<float>(float x) { return x; }
template <>
__device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 x) {
  return __bfloat162float(x);
}

template <typename T>
__device__ __forceinline__ T from_f(float x);
template <>
__device__ __forceinline__ float from_f<float>(float x) { return x; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

// Selection key: a larger key ranks first.  The upper word orders scores
// (an order-preserving map of the fp32 bits), the lower word orders chunk
// ids descending, so that among equal scores the lower chunk id ranks first.
// Adding +0.0f turns -0.0 into +0.0 so that the two zeros tie.
// Three-input maximum (one sm_100 instruction).
__device__ __forceinline__ float max3f(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

__device__ __forceinline__ uint64_t sel_key(float s, int c) {
  uint32_t b = __float_as_uint(s + 0.0f);
  b = (b & 0x80000000u) ? ~b : (b | 0x80000000u);
  return ((uint64_t)b << 32) | (uint64_t)(0xFFFFFFFFu - (uint32_t)c);
}
__device__ __forceinline__ float key_score(uint64_t key) {
  uint32_t b = (uint32_t)(key >> 32);
  b = (b & 0x80000000u) ? (b & 0x7FFFFFFFu) : ~b;
  return __uint_as_float(b);
}
__device__ __forceinline__ int key_chunk(uint64_t key) {
  return (int)(0xFFFFFFFFu - (uint32_t)key);
}

__device__ __forceinline__ void report(uint32_t *err, uint32_t code) {
  if (err) atomicCAS(err, DEV_OK, code);
}

}  // namespace hils
