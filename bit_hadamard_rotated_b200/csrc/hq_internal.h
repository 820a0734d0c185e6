// hq_internal.h -- host-side declarations shared by the libhq translation units.
#pragma once

#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "hq.h"

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
// True (and one fewer pending) if hq_set_test_fault asked for a withheld copy.
bool take_test_fault();

cudaError_t launch_rotate(hq_dtype id, hq_dtype od, const void* x, void* out, int n_rows, int K,
                          const int8_t* signs, cudaStream_t st);

struct GemvArgs {
  int bits, M, K, N, zero;
  const uint32_t* q;
  const uint16_t* scales;
  const uint16_t* x;    // [N][K] fp16 activations (not rotated)
  const int8_t* signs;  // [K] or NULL
  float* y;             // [N][M] block of outputs, row stride ldy
  int ldy;
  uint32_t* status;
  void* xg;       // gemv_scratch_bytes(K, N) bytes, 16-byte aligned: prep output
  const uint8_t* zeros = nullptr;  // per-group zero points [M][K/128], or nullptr: zero
  bool zero_frac = false;           // use zero_f (a fractional zero point) instead of zero
  bool planes = false;              // 2-bit codes in the bit-plane layout
  float zero_f = 0.f;
  uint32_t* sync = nullptr;  // two words, zero between calls: the 32-row GEMV's rotation gate
};

// Shared memory the GEMV needs for a batch block of nb <= 8 rows, with or
// without per-group zero points (0 if no ring configuration fits in one CTA).
size_t gemv_smem_bytes(int bits, int K, int nb, bool pgz);
// Scratch for the rotated activations of one GEMV launch of nb <= 8 columns.
size_t gemv_scratch_bytes(int K, int nb);
// Streaming multiprocessors of the current device (148 if the query fails).
int sm_count();
// One GEMV launch, preceded by a rotation (prep) launch unless the GEMV CTAs
// rotate the batch themselves (gemv_launches tells which: 1 or 2).
cudaError_t launch_gemv(const GemvArgs& a, cudaStream_t st);
int gemv_launches(int K, int nb);

// A 2D tiled TMA tensor map over a row-major [rows][inner] matrix of `dtype`
// elements (row stride in bytes, a multiple of 16); box = box_inner x box_rows
// elements; no multicast.  cudaErrorNotSupported if the driver entry point is
// missing, cudaErrorInvalidValue if the driver rejects the description.
cudaError_t tensor_map_2d(CUtensorMap* map, CUtensorMapDataType dtype, const void* base, uint64_t inner,
                          uint64_t rows, uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_rows,
                          CUtensorMapSwizzle swizzle);
// The same over a 3-D view: dims and box innermost first, byte strides of
// dims 1 and 2 (each a multiple of 16; they need not increase).
cudaError_t tensor_map_3d(CUtensorMap* map, CUtensorMapDataType dtype, const void* base,
                          const uint64_t (&dims)[3], const uint64_t (&strides_bytes)[2],
                          const uint32_t (&box)[3], CUtensorMapSwizzle swizzle);

// The 32-row GEMV for batches up to 16 (gemv32.cu): whether a launch shape
// fits (K >= 1024, the scalar zero point, at most 16 tiles per CTA), the
// scratch for its prep output, and one prep + GEMV launch pair.
bool gemv32_supported(int bits, int M, int K, int N);
int gemv32_launches(int bits, int M, int K, int N);
size_t gemv32_scratch_bytes(int K, int N);
cudaError_t launch_gemv32(const GemvArgs& a, cudaStream_t st);

// Tensor-core path (tcgen05) for larger batches.
struct TcArgs {
  int bits, M, K, N, zero;
  const uint32_t* q;
  const uint16_t* scales;
  const uint16_t* x;
  const int8_t* signs;
  float* y;
  int ldy;
  uint32_t* status;
  void* xp;  // workspace: tc_xp_bytes(bits, K, N) bytes, 256-byte aligned
  uint32_t* counters;  // kTcCounterBytes, zero between calls (every call leaves them zero)
};
// Arrival counters of the tensor-core GEMM's tiles shared by two CTAs (one
// per CTA boundary; at most kMaxTcGrid CTAs).
constexpr int kMaxTcGrid = 160;
constexpr size_t kTcCounterBytes = 1024;
static_assert(kMaxTcGrid * 4 <= static_cast<int>(kTcCounterBytes), "counter region");
// Largest batch block per GEMM launch for this width and K (0: path unavailable).
int tc_col_block(int bits, int K);
// Workspace bytes for the rotated activation images of a batch and the
// partial sums of tiles shared by two CTAs.
size_t tc_xp_bytes(int bits, int K, int batch);
// Kernel launches of one tensor-core hq_linear call (prep + one GEMM per block).
int tc_launches(int bits, int K, int batch);
cudaError_t launch_linear_tc(const TcArgs& a, cudaStream_t st);

cudaError_t launch_unpack(const uint32_t* packed, int bits, size_t n, uint8_t* out,
                          cudaStream_t st);

}  // namespace hq
