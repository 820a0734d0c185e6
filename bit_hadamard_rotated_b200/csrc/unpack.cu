// unpack.cu -- hq_unpack_codes: one byte per code from the packed
// little-endian bit stream (code j at stream bits [bits*j, bits*j + bits)).
// Test-facing: it exposes the exact code layout the matmul kernels decode.
#include <algorithm>

#include "hq_common.cuh"
#include "hq_internal.h"
#include "hq_launch.cuh"

namespace hq {

__global__ void unpack_kernel(const uint32_t* __restrict__ words, int bits, size_t n,
                              size_t n_words, uint8_t* __restrict__ out) {
  pdl_launch_dependents();
  pdl_wait();
  const uint32_t mask = (1u << bits) - 1u;
  for (size_t j = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; j < n;
       j += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const size_t bit = j * static_cast<size_t>(bits);
    const size_t w = bit >> 5;
    const uint32_t off = static_cast<uint32_t>(bit & 31);
    uint32_t v = words[w] >> off;
    if (off + bits > 32 && w + 1 < n_words) v |= words[w + 1] << (32 - off);
    out[j] = static_cast<uint8_t>(v & mask);
  }
}

cudaError_t launch_unpack(const uint32_t* packed, int bits, size_t n, uint8_t* out,
                          cudaStream_t st) {
  const size_t n_words = (n * static_cast<size_t>(bits) + 31) / 32;
  const size_t blocks = std::min<size_t>((n + 255) / 256, 148 * 16);
  return launch_pdl(unpack_kernel, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, st, true,
                    packed, bits, n, n_words, out);
}

// Bits 0, 2, .., 30 of x gathered into bits 0..15.
__device__ __forceinline__ uint32_t even_bits(uint32_t x) {
  x &= 0x55555555u;
  x = (x | (x >> 1)) & 0x33333333u;
  x = (x | (x >> 2)) & 0x0F0F0F0Fu;
  x = (x | (x >> 4)) & 0x00FF00FFu;
  return (x | (x >> 8)) & 0x0000FFFFu;
}

// One thread per 32-code span: packed words (codes 0..15, 16..31) -> the
// span's plane words (bit 0 of each code, then bit 1).
__global__ void to_bitplanes_kernel(const uint2* __restrict__ packed, size_t spans, uint2* __restrict__ planes) {
  pdl_launch_dependents();
  pdl_wait();
  for (size_t j = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; j < spans;
       j += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const uint2 w = packed[j];
    planes[j] = make_uint2(even_bits(w.x) | (even_bits(w.y) << 16), even_bits(w.x >> 1) | (even_bits(w.y >> 1) << 16));
  }
}

}  // namespace hq

extern "C" hq_status hq_to_bitplanes(const uint32_t* packed, size_t n_codes, uint32_t* planes,
                                     hq_stream_t stream) {
  if (n_codes % 32 != 0) return HQ_ERR_INVALID_ARG;
  if (n_codes == 0) return HQ_OK;
  if (!packed || !planes || (reinterpret_cast<uintptr_t>(packed) & 7) || (reinterpret_cast<uintptr_t>(planes) & 7)) {
    return HQ_ERR_INVALID_ARG;
  }
  const size_t spans = n_codes / 32;
  const size_t blocks = std::min<size_t>((spans + 255) / 256, 148 * 16);
  const cudaError_t e = hq::launch_pdl(hq::to_bitplanes_kernel, dim3(static_cast<unsigned>(blocks)), dim3(256), 0,
                                       reinterpret_cast<cudaStream_t>(stream), true,
                                       reinterpret_cast<const uint2*>(packed), spans, reinterpret_cast<uint2*>(planes));
  if (e != cudaSuccess) {
    (void)cudaGetLastError();
    return HQ_ERR_CUDA;
  }
  return HQ_OK;
}
