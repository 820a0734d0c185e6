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

}  // namespace hq
