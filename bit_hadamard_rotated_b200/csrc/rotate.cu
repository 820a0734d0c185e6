// rotate.cu -- the random-sign Hadamard rotation x' = H_K diag(s) x / sqrt(K)
// ("group-128 GPTQ in a Hadamard-rotated basis", rotation signs in small.bin:
// LLaDA2.2-mini Orin-Nano model card, Properties table and file list).
//
// rotate_rows_kernel (hq_rotate): one CTA per row, fp32 butterflies
// (fwht.cuh), one rounding to the output type, natural-order output.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "fwht.cuh"
#include "hq_common.cuh"
#include "hq_internal.h"
#include "hq_launch.cuh"
#include "hq_io.cuh"

namespace hq {

template <int LOGK, typename InT, typename OutT>
__global__ void __launch_bounds__(FwhtShape<LOGK>::THREADS)
    rotate_rows_kernel(const InT* __restrict__ x, OutT* __restrict__ out,
                       const int8_t* __restrict__ signs, float inv_sqrt_k) {
  using S = FwhtShape<LOGK>;
  extern __shared__ float buf[];
  pdl_launch_dependents();
  const int tid = threadIdx.x;
  const size_t row = blockIdx.x;
  const auto neg = sign_bits<S::E>(signs ? signs + tid * S::E : nullptr);
  pdl_wait();
  float v[S::E];
  load_chunk<InT, S::E>(x + row * S::K + tid * S::E, v);
  flip_signs<S::E>(neg, v);
  fwht_block<LOGK, 5>(v, buf);
  OutT* o = out + row * S::K + tid * S::E;
#pragma unroll
  for (int e = 0; e < S::E; ++e) o[e] = from_f32<OutT>(buf[fwht_pad(tid * S::E + e)] * inv_sqrt_k);
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

}  // namespace hq
