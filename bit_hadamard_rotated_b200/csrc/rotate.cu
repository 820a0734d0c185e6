// rotate.cu -- the random-sign Hadamard rotation x' = H_K diag(s) x / sqrt(K)
// ("group-128 GPTQ in a Hadamard-rotated basis", rotation signs in small.bin:
// LLaDA2.2-mini Orin-Nano model card, Properties table and file list).
//
// Two kernels share fwht_block:
//   rotate_rows_kernel  -- hq_rotate: one CTA per row, natural-order output.
//   prep_gemv_kernel    -- the GEMV's activation operand: one CTA per batch
//                          row; writes x' in fp16, reordered into the m16n8k16
//                          B-fragment order of the packed-code decode
//                          (hq_layout.cuh) and pre-scaled by 2^-a, plus the
//                          per-(group, column) correction sum_k (1024 +
//                          zero 2^a_k) B_k that removes the decode's offsets.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "fwht.cuh"
#include "hq_common.cuh"
#include "hq_internal.h"
#include "hq_launch.cuh"
#include "hq_layout.cuh"

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

template <int LOGK, typename InT, typename OutT>
__global__ void __launch_bounds__(FwhtShape<LOGK>::THREADS)
    rotate_rows_kernel(const InT* __restrict__ x, OutT* __restrict__ out,
                       const int8_t* __restrict__ signs, float inv_sqrt_k) {
  using S = FwhtShape<LOGK>;
  extern __shared__ float buf[];
  pdl_launch_dependents();
  pdl_wait();
  const int tid = threadIdx.x;
  const size_t row = blockIdx.x;
  float v[S::E];
  load_chunk<InT, S::E>(x + row * S::K + tid * S::E, v);
  apply_signs<S::E>(signs ? signs + tid * S::E : nullptr, v);
  fwht_block<LOGK>(v, buf);
  OutT* o = out + row * S::K + tid * S::E;
#pragma unroll
  for (int e = 0; e < S::E; ++e) o[e] = from_f32<OutT>(buf[fwht_pad(tid * S::E + e)] * inv_sqrt_k);
}

// xs layout (halves): xs[((S * N + n) * 4 + t) * 4 + r], S = 8*G + s the MMA
// step, t the lane's k-quad, r the B-fragment element.  corr[G * N + n].
template <int BITS, int LOGK>
__global__ void __launch_bounds__(FwhtShape<LOGK>::THREADS)
    prep_gemv_kernel(const __half* __restrict__ x, const int8_t* __restrict__ signs,
                     uint16_t* __restrict__ xs, float* __restrict__ corr, int N, int zero,
                     float inv_sqrt_k) {
  using S = FwhtShape<LOGK>;
  extern __shared__ float buf[];
  pdl_launch_dependents();
  pdl_wait();
  const int tid = threadIdx.x;
  const int n = blockIdx.x;
  float v[S::E];
  load_chunk<__half, S::E>(x + static_cast<size_t>(n) * S::K + tid * S::E, v);
  apply_signs<S::E>(signs ? signs + tid * S::E : nullptr, v);
  fwht_block<LOGK>(v, buf);

  const int lane = tid & 31, warp = tid >> 5;
  const int s = lane >> 2, t = lane & 3;
  constexpr int G = S::K / kGroup;
  for (int g = warp; g < G; g += S::W) {
    uint16_t hv[4];
    float part = 0.f;
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const PairDesc pd = Pairs<BITS>::get(2 * s + (r >> 1));
      const int code = (r & 1) ? pd.c_hi : pd.c_lo;
      const int a = (r & 1) ? pd.a_hi : pd.a_lo;
      const int k = kGroup * g + 32 * t + code;
      const __half xh = __float2half_rn(buf[fwht_pad(k)] * inv_sqrt_k);
      const __half b = __float2half_rn(__half2float(xh) * __int_as_float((127 - a) << 23));
      hv[r] = __half_as_ushort(b);
      part += static_cast<float>(1024 + (zero << a)) * __half2float(b);
    }
#pragma unroll
    for (int m = 16; m >= 1; m >>= 1) part += __shfl_xor_sync(0xffffffffu, part, m);
    const int Sg = 8 * g + s;
    uint2 pk;
    pk.x = static_cast<uint32_t>(hv[0]) | (static_cast<uint32_t>(hv[1]) << 16);
    pk.y = static_cast<uint32_t>(hv[2]) | (static_cast<uint32_t>(hv[3]) << 16);
    *reinterpret_cast<uint2*>(xs + ((static_cast<size_t>(Sg) * N + n) * 4 + t) * 4) = pk;
    if (lane == 0) corr[g * N + n] = part;
  }
}

// ---------------------------------------------------------------- launchers
template <int LOGK, typename InT, typename OutT>
static cudaError_t rotate_launch_t(const void* x, void* out, int n_rows, const int8_t* signs,
                                   cudaStream_t st) {
  using S = FwhtShape<LOGK>;
  const float inv = static_cast<float>(1.0 / sqrt(static_cast<double>(S::K)));
  return launch_pdl(rotate_rows_kernel<LOGK, InT, OutT>, dim3(n_rows), dim3(S::THREADS),
                    S::SMEM_FLOATS * sizeof(float), st, true, static_cast<const InT*>(x),
                    static_cast<OutT*>(out), signs, inv);
}

template <int LOGK, typename InT>
static cudaError_t rotate_launch_in(hq_dtype od, const void* x, void* out, int n_rows,
                                    const int8_t* signs, cudaStream_t st) {
  switch (od) {
    case HQ_F16: return rotate_launch_t<LOGK, InT, __half>(x, out, n_rows, signs, st);
    case HQ_BF16: return rotate_launch_t<LOGK, InT, __nv_bfloat16>(x, out, n_rows, signs, st);
    default: return rotate_launch_t<LOGK, InT, float>(x, out, n_rows, signs, st);
  }
}

template <int LOGK>
static cudaError_t rotate_launch_k(hq_dtype id, hq_dtype od, const void* x, void* out,
                                   int n_rows, const int8_t* signs, cudaStream_t st) {
  switch (id) {
    case HQ_F16: return rotate_launch_in<LOGK, __half>(od, x, out, n_rows, signs, st);
    case HQ_BF16: return rotate_launch_in<LOGK, __nv_bfloat16>(od, x, out, n_rows, signs, st);
    default: return rotate_launch_in<LOGK, float>(od, x, out, n_rows, signs, st);
  }
}

cudaError_t launch_rotate(hq_dtype id, hq_dtype od, const void* x, void* out, int n_rows, int K,
                          const int8_t* signs, cudaStream_t st) {
  switch (K) {
    case 32: return rotate_launch_k<5>(id, od, x, out, n_rows, signs, st);
    case 64: return rotate_launch_k<6>(id, od, x, out, n_rows, signs, st);
    case 128: return rotate_launch_k<7>(id, od, x, out, n_rows, signs, st);
    case 256: return rotate_launch_k<8>(id, od, x, out, n_rows, signs, st);
    case 512: return rotate_launch_k<9>(id, od, x, out, n_rows, signs, st);
    case 1024: return rotate_launch_k<10>(id, od, x, out, n_rows, signs, st);
    case 2048: return rotate_launch_k<11>(id, od, x, out, n_rows, signs, st);
    case 4096: return rotate_launch_k<12>(id, od, x, out, n_rows, signs, st);
    case 8192: return rotate_launch_k<13>(id, od, x, out, n_rows, signs, st);
    case 16384: return rotate_launch_k<14>(id, od, x, out, n_rows, signs, st);
    case 32768: return rotate_launch_k<15>(id, od, x, out, n_rows, signs, st);
    default: return cudaErrorInvalidValue;
  }
}

template <int BITS, int LOGK>
static cudaError_t prep_launch_t(const __half* x, const int8_t* signs, uint16_t* xs, float* corr,
                                 int N, int zero, cudaStream_t st) {
  using S = FwhtShape<LOGK>;
  const float inv = static_cast<float>(1.0 / sqrt(static_cast<double>(S::K)));
  return launch_pdl(prep_gemv_kernel<BITS, LOGK>, dim3(N), dim3(S::THREADS),
                    S::SMEM_FLOATS * sizeof(float), st, true, x, signs, xs, corr, N, zero, inv);
}

template <int BITS>
static cudaError_t prep_launch_b(int K, const __half* x, const int8_t* signs, uint16_t* xs,
                                 float* corr, int N, int zero, cudaStream_t st) {
  switch (K) {
    case 128: return prep_launch_t<BITS, 7>(x, signs, xs, corr, N, zero, st);
    case 256: return prep_launch_t<BITS, 8>(x, signs, xs, corr, N, zero, st);
    case 512: return prep_launch_t<BITS, 9>(x, signs, xs, corr, N, zero, st);
    case 1024: return prep_launch_t<BITS, 10>(x, signs, xs, corr, N, zero, st);
    case 2048: return prep_launch_t<BITS, 11>(x, signs, xs, corr, N, zero, st);
    case 4096: return prep_launch_t<BITS, 12>(x, signs, xs, corr, N, zero, st);
    case 8192: return prep_launch_t<BITS, 13>(x, signs, xs, corr, N, zero, st);
    case 16384: return prep_launch_t<BITS, 14>(x, signs, xs, corr, N, zero, st);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_prep_gemv(int bits, int K, const __half* x, const int8_t* signs, uint16_t* xs,
                             float* corr, int N, int zero, cudaStream_t st) {
  switch (bits) {
    case 2: return prep_launch_b<2>(K, x, signs, xs, corr, N, zero, st);
    case 3: return prep_launch_b<3>(K, x, signs, xs, corr, N, zero, st);
    case 4: return prep_launch_b<4>(K, x, signs, xs, corr, N, zero, st);
    case 8: return prep_launch_b<8>(K, x, signs, xs, corr, N, zero, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace hq
