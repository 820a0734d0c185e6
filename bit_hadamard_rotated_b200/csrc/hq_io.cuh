// hq_io.cuh -- typed loads for the rotation prologues: fp16/bf16/fp32 rows to
// fp32 registers, 16-byte vectors where the chunk allows, and sign flips.
#pragma once

#include <type_traits>

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

// The signs of a thread's chunk of E consecutive values as a bit mask (bit
// e set: value e flips), read with the widest aligned loads (the sign vector
// is 16-byte aligned and the chunk starts at a multiple of E).  The signs are
// weights, so kernels read them before griddepcontrol.wait.
template <int E>
using SignMask = typename std::conditional<(E <= 32), uint32_t, unsigned long long>::type;

template <int E>
__device__ __forceinline__ SignMask<E> sign_bits(const int8_t* s) {
  static_assert(E <= 64, "one bit per value");
  using Mk = SignMask<E>;
  if (s == nullptr) return Mk(0);
  Mk m = 0;
  if constexpr (E % 16 == 0) {
#pragma unroll
    for (int i = 0; i < E / 16; ++i) {
      const uint4 u = __ldg(reinterpret_cast<const uint4*>(s) + i);
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int j = 0; j < 16; ++j) m |= static_cast<Mk>(w[j >> 2] >> (8 * (j & 3) + 7) & 1u) << (16 * i + j);
    }
  } else if constexpr (E == 8) {
    const uint2 u = __ldg(reinterpret_cast<const uint2*>(s));
#pragma unroll
    for (int j = 0; j < 8; ++j) m |= (((j < 4) ? u.x : u.y) >> (8 * (j & 3) + 7) & 1u) << j;
  } else if constexpr (E == 4) {
    const uint32_t u = __ldg(reinterpret_cast<const uint32_t*>(s));
#pragma unroll
    for (int j = 0; j < 4; ++j) m |= (u >> (8 * j + 7) & 1u) << j;
  } else {
#pragma unroll
    for (int e = 0; e < E; ++e) m |= (s[e] < 0 ? 1u : 0u) << e;
  }
  return m;
}

template <int E>
__device__ __forceinline__ void flip_signs(SignMask<E> m, float (&v)[E]) {
#pragma unroll
  for (int e = 0; e < E; ++e) v[e] = (m >> e & 1u) ? -v[e] : v[e];
}

}  // namespace hq
