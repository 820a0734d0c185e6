// quantize.cu -- hq_quantize: the rotated round-to-nearest packer that turns
// real-valued weights into this library's packed format ("group-128 GPTQ in a
// Hadamard-rotated basis": LLaDA2.2-mini Orin-Nano model card, Properties
// table; weights "behind a random Hadamard rotation": Qwen3.8-27B Pingala-8
// 2-bit card, "What this is"), without GPTQ's calibration-driven rounding:
//   r       = H_K diag(s) W[m] / sqrt(K)                 (fp64)
//   scale_g = fp16(min(2 max_{k in g} |r_k| / (2^b - 1), 65504))
//   q_k     = clamp(rint(r_k / scale_g) + 2^(b-1), 0, 2^b - 1)   (2^(b-1) if scale_g = 0)
// packed as hq_linear reads it, with zero point 2^(b-1).
//
// Offline work, so it is written for exactness rather than speed: the rotation
// runs in fp64, so a code differs from an fp64 reference only where r_k /
// scale_g lies within rounding noise of a half-integer.  One CTA per (row,
// half of 16384 values): H_{2n} = [[H_n, H_n], [H_n, -H_n]] in natural order,
// so CTA c of a row of K = 2n > 16384 transforms u_lo + (-1)^c u_hi with an
// n-point transform and writes outputs c n .. c n + n - 1.  The n values sit in
// shared memory as doubles (128 KiB at n = 16384); butterfly stages run over
// it with a barrier between stages.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "hq_common.cuh"
#include "hq_internal.h"
#include "hq_io.cuh"
#include "hq_launch.cuh"

namespace hq {
namespace {

constexpr int kQThreads = 512;
constexpr int kQMaxN = 16384;  // values per CTA

template <typename T>
__device__ __forceinline__ double load_f64(const T* p) {
  return static_cast<double>(to_f32<T>(*p));
}

template <typename T>
__global__ void __launch_bounds__(kQThreads)
    quantize_kernel(const T* __restrict__ W, int K, int bits, const int8_t* __restrict__ signs,
                    double inv_sqrt_k, uint32_t* __restrict__ qw, uint16_t* __restrict__ scales) {
  extern __shared__ __align__(16) uint8_t smem[];
  const int n = K < kQMaxN ? K : kQMaxN;  // transform length of this CTA
  const int parts = K / n;
  const int m = blockIdx.x / parts, c = blockIdx.x % parts;
  double* buf = reinterpret_cast<double*>(smem);
  uint8_t* codes = smem + static_cast<size_t>(n) * sizeof(double);
  const int tid = threadIdx.x;
  const T* row = W + static_cast<size_t>(m) * K;
  auto sgn = [&](int i) { return signs != nullptr && signs[i] < 0 ? -1.0 : 1.0; };
  // u = diag(s) W[m]; for K = 2n: u_lo + (-1)^c u_hi (the first butterfly stage)
  for (int i = tid; i < n; i += kQThreads) {
    double v = sgn(i) * load_f64(row + i);
    if (parts == 2) {
      const double h = sgn(n + i) * load_f64(row + n + i);
      v = c == 0 ? v + h : v - h;
    }
    buf[i] = v;
  }
  __syncthreads();
  // n-point Sylvester transform: at stride h, (a, b) -> (a + b, a - b)
  for (int h = 1; h < n; h <<= 1) {
    for (int j = tid; j < n / 2; j += kQThreads) {
      const int i = (j / h) * 2 * h + (j % h);
      const double a = buf[i], b = buf[i + h];
      buf[i] = a + b;
      buf[i + h] = a - b;
    }
    __syncthreads();
  }
  // per group of 128: scale and codes (one warp per group, 4 values a lane)
  const int warp = tid >> 5, lane = tid & 31;
  const int zero = 1 << (bits - 1), qmax = (1 << bits) - 1;
  const int G = K / kGroup, g0 = c * (n / kGroup);
  for (int gl = warp; gl < n / kGroup; gl += kQThreads / 32) {
    double r[4];
    double amax = 0.0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      r[i] = buf[gl * kGroup + 32 * i + lane] * inv_sqrt_k;
      amax = fmax(amax, fabs(r[i]));
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) amax = fmax(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    const double want = fmin(2.0 * amax / static_cast<double>(qmax), 65504.0);
    const __half s16 = __double2half(want);
    const double s = static_cast<double>(__half2float(s16));
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      int q = zero;
      if (s > 0.0) {
        q = static_cast<int>(rint(r[i] / s)) + zero;
        q = q < 0 ? 0 : (q > qmax ? qmax : q);
      }
      codes[gl * kGroup + 32 * i + lane] = static_cast<uint8_t>(q);
    }
    if (lane == 0) scales[static_cast<size_t>(m) * G + g0 + gl] = __half_as_ushort(s16);
  }
  __syncthreads();
  // pack: word w of this CTA's part holds stream bits [32 w, 32 w + 32) of
  // its codes (a group is 4 bits words, so parts start on word boundaries)
  const int words = n * bits / 32;
  uint32_t* out = qw + static_cast<size_t>(m) * (K * bits / 32) + static_cast<size_t>(c) * words;
  for (int w = tid; w < words; w += kQThreads) {
    const int b0 = 32 * w;
    uint32_t v = 0;
    for (int j = b0 / bits; j * bits < b0 + 32; ++j) {
      const int sh = j * bits - b0;  // may be negative for a code straddling in from below
      const uint32_t cj = codes[j];
      v |= sh >= 0 ? cj << sh : cj >> (-sh);
    }
    out[w] = v;
  }
}

template <typename T>
cudaError_t quantize_launch(const void* W, int M, int K, int bits, const int8_t* signs,
                            uint32_t* qw, uint16_t* scales, cudaStream_t st) {
  const int n = K < kQMaxN ? K : kQMaxN;
  const size_t smem = static_cast<size_t>(n) * (sizeof(double) + 1);
  const double inv = 1.0 / sqrt(static_cast<double>(K));
  const unsigned grid = static_cast<unsigned>(M) * static_cast<unsigned>(K / n);
  return launch_pdl(quantize_kernel<T>, dim3(grid), dim3(kQThreads), smem, st, false,
                    static_cast<const T*>(W), K, bits, signs, inv, qw, scales);
}

}  // namespace
}  // namespace hq

using namespace hq;

extern "C" hq_status hq_quantize(const void* W, hq_dtype w_dtype, int M, int K, int bits,
                                 const int8_t* signs, uint32_t* qweight, uint16_t* scales,
                                 hq_stream_t stream) {
  auto aligned = [](const void* p, uintptr_t a) {
    return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0;
  };
  if (w_dtype < HQ_F16 || w_dtype > HQ_F32) return HQ_ERR_INVALID_ARG;
  if (M < 0 || K <= 0 || M > (1 << 24)) return HQ_ERR_INVALID_ARG;
  if (!(bits == 2 || bits == 3 || bits == 4 || bits == 8)) {
    return (bits >= 1 && bits <= 8) ? HQ_ERR_UNSUPPORTED : HQ_ERR_INVALID_ARG;
  }
  if ((K & (K - 1)) != 0 || K < 128 || K > 32768) return HQ_ERR_UNSUPPORTED;
  if (M == 0) return HQ_OK;
  if (!W || !qweight || !scales) return HQ_ERR_INVALID_ARG;
  if (!aligned(W, 16) || !aligned(qweight, 16) || !aligned(scales, 16) ||
      (signs && !aligned(signs, 16))) {
    return HQ_ERR_INVALID_ARG;
  }
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e;
  switch (w_dtype) {
    case HQ_F16: e = quantize_launch<__half>(W, M, K, bits, signs, qweight, scales, st); break;
    case HQ_BF16: e = quantize_launch<__nv_bfloat16>(W, M, K, bits, signs, qweight, scales, st); break;
    default: e = quantize_launch<float>(W, M, K, bits, signs, qweight, scales, st); break;
  }
  if (e != cudaSuccess) {
    (void)cudaGetLastError();
    return HQ_ERR_CUDA;
  }
  return HQ_OK;
}
