// hq_internal.h -- host-side declarations shared by the libhq translation units.
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/hq.h"

namespace hq {

// Bits OR-ed into the workspace status word by device code.
enum : uint32_t {
  HQ_DEV_TIMEOUT = 1u,
  HQ_DEV_BAD_EXPERT = 2u,
  HQ_DEV_BAD_BITS = 4u,
  HQ_DEV_BAD_ZERO = 8u,
};

// Counts every kernel launch libhq enqueues (hq_launch_count).
void note_launch();

cudaError_t launch_rotate(hq_dtype id, hq_dtype od, const void* x, void* out, int n_rows, int K,
                          const int8_t* signs, cudaStream_t st);

cudaError_t launch_prep_gemv(int bits, int K, const __half* x, const int8_t* signs, uint16_t* xs,
                             float* corr, int N, int zero, cudaStream_t st);

struct GemvArgs {
  int bits, M, K, N, zero;
  const uint32_t* q;
  const uint16_t* scales;
  const uint16_t* xs;
  const float* corr;
  float* y;  // [N][M] block of outputs, row stride ldy
  int ldy;
  uint32_t* status;
};

// Shared memory the GEMV needs for a column block of nb <= 8 rows (0 if the
// tile does not fit in one CTA).
size_t gemv_smem_bytes(int bits, int K, int nb);
cudaError_t launch_gemv(const GemvArgs& a, cudaStream_t st);

cudaError_t launch_unpack(const uint32_t* packed, int bits, size_t n, uint8_t* out,
                          cudaStream_t st);

}  // namespace hq
