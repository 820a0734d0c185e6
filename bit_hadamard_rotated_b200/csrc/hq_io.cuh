// hq_io.cuh -- typed loads for the rotation prologues: fp16/bf16/fp32 rows to
// fp32 registers, 16-byte vectors where the chunk allows, and sign flips.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

namespace hq {

template <typename T>
__device__ __forceinline__ float to_f32(T v);
template <>
__device__ __forceinline__ float to_f32<float>(float v) {
  return v;
}
template <>
__device__ __forceinline__ float to_f32<__half>(__half v) {
  return __half2float(v);
}
template <>
__device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 v) {
  return __bfloat162float(v);
}

template <typename T>
__device__ __forceinline__ T from_f32(float v);
template <>
__device__ __forceinline__ float from_f32<float>(float v) {
  return v;
}
template <>
__device__ __forceinline__ __half from_f32<__half>(float v) {
  return __float2half_rn(v);
}
template <>
__device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float v) {
  return __float2bfloat16_rn(v);
}

// Load E consecutive elements (16-byte vectors when the chunk allows it).
template <typename T, int E>
__device__ __forceinline__ void load_chunk(const T* p, float (&v)[E]) {
  constexpr int BYTES = E * sizeof(T);
  if constexpr (BYTES % 16 == 0) {
    constexpr int NV = BYTES / 16;
    constexpr int PER = 16 / sizeof(T);
#pragma unroll
    for (int i = 0; i < NV; ++i) {
      const uint4 u = __ldg(reinterpret_cast<const uint4*>(p) + i);
      const T* t = reinterpret_cast<const T*>(&u);
#pragma unroll
      for (int j = 0; j < PER; ++j) v[i * PER + j] = to_f32<T>(t[j]);
    }
  } else {
#pragma unroll
    for (int e = 0; e < E; ++e) v[e] = to_f32<T>(p[e]);
  }
}

template <int E>
__device__ __forceinline__ void apply_signs(const int8_t* s, float (&v)[E]) {
  if (s == nullptr) return;
  if constexpr (E % 16 == 0) {
#pragma unroll
    for (int i = 0; i < E / 16; ++i) {
      const uint4 u = __ldg(reinterpret_cast<const uint4*>(s) + i);
      const int8_t* b = reinterpret_cast<const int8_t*>(&u);
#pragma unroll
      for (int j = 0; j < 16; ++j) v[16 * i + j] = b[j] < 0 ? -v[16 * i + j] : v[16 * i + j];
    }
  } else {
#pragma unroll
    for (int e = 0; e < E; ++e) v[e] = s[e] < 0 ? -v[e] : v[e];
  }
}

}  // namespace hq
