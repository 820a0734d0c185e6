// hq_api.cu -- the C ABI of libhq: argument validation, workspace layout and
// kernel dispatch.  Every check happens on the host before any launch; no
// entry point allocates or frees memory.
#include <algorithm>
#include <atomic>
#include <cstdint>

#include "hq_internal.h"

namespace hq {

static std::atomic<uint64_t> g_launches{0};
// Batch from which hq_linear uses the tensor-core GEMM; 0 = automatic.
static std::atomic<int> g_tc_min_batch{0};
// Batch from which hq_linear uses the 32-row GEMV (up to batch 16); 0 = automatic.
static std::atomic<int> g_g32_min_batch{0};

void note_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

// GEMV launches that still have to withhold one copy (hq_set_test_fault).
static std::atomic<int> g_test_faults{0};

bool take_test_fault() {
  int n = g_test_faults.load(std::memory_order_relaxed);
  while (n > 0) {
    if (g_test_faults.compare_exchange_weak(n, n - 1, std::memory_order_relaxed)) return true;
  }
  return false;
}

static bool aligned(const void* p, uintptr_t a) {
  return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0;
}
static bool is_pow2(long v) { return v > 0 && (v & (v - 1)) == 0; }
static size_t align256(size_t v) { return (v + 255) & ~static_cast<size_t>(255); }

constexpr size_t kStatusBytes = 256;
// Words of the counter region (after the tensor-core GEMM's per-CTA-boundary
// counters) that the 32-row GEMV's rotation gate uses.
constexpr int kG32SyncWord = 192;
static_assert(kG32SyncWord >= kMaxTcGrid && (kG32SyncWord + 2) * 4 <= static_cast<int>(kTcCounterBytes),
              "gate words inside the counter region, past the tensor-core counters");
constexpr int kMaxColBlock = 8;

static hq_status from_cuda(cudaError_t e) {
  if (e == cudaSuccess) return HQ_OK;
  (void)cudaGetLastError();  // clear a non-sticky launch error
  return HQ_ERR_CUDA;
}

static hq_status check_weight(const hq_weight* w) {
  if (w == nullptr) return HQ_ERR_INVALID_ARG;
  if (w->M <= 0 || w->K <= 0 || w->M > (1 << 28)) return HQ_ERR_INVALID_ARG;
  if (!(w->bits == 2 || w->bits == 3 || w->bits == 4 || w->bits == 8)) {
    return (w->bits >= 1 && w->bits <= 8) ? HQ_ERR_UNSUPPORTED : HQ_ERR_INVALID_ARG;
  }
  if (!is_pow2(w->K) || w->K < 128 || w->K > 32768) return HQ_ERR_UNSUPPORTED;
  if (w->zero < 0 || w->zero >= (1 << w->bits)) return HQ_ERR_INVALID_ARG;
  if (w->qweight == nullptr || w->scales == nullptr) return HQ_ERR_INVALID_ARG;
  if (!aligned(w->qweight, 16) || !aligned(w->scales, 16)) return HQ_ERR_INVALID_ARG;
  if (w->signs != nullptr && !aligned(w->signs, 16)) return HQ_ERR_INVALID_ARG;
  if (w->zeros != nullptr && !aligned(w->zeros, 16)) return HQ_ERR_INVALID_ARG;
  if (w->layout != HQ_LAYOUT_PACKED && w->layout != HQ_LAYOUT_BITPLANES) return HQ_ERR_INVALID_ARG;
  if (w->layout == HQ_LAYOUT_BITPLANES && w->bits != 2) return HQ_ERR_UNSUPPORTED;
  return HQ_OK;
}

// Largest GEMV batch block whose ring plan fits in one CTA.
static int gemv_col_block(int bits, int K, bool pgz) {
  for (int nb = kMaxColBlock; nb >= 1; nb >>= 1) {
    if (gemv_smem_bytes(bits, K, nb, pgz) != 0) return nb;
  }
  return 0;
}

// The batch-8 GEMV stages its activation fragments (2 K bytes per column) in
// shared memory for the whole of K and reads them from there once per 16-row
// tile; the 32-row GEMV stages K in slices and reads them once per 32 rows,
// with its rotation in the same launch.  Batch sweeps on B200 (12288 x 4096,
// 8192^2, 28672 x 8192, 4096^2) put the switch at batch 4 for 8-bit rows,
// 5 for 3/4-bit rows and 6 for 2-bit rows (9 above 16384 rows, where the
// batch-8 GEMV's long tile ranges keep it ahead); up to batch 16, then the
// tensor-core GEMM.
static int g32_auto_min_batch(const hq_weight* w) {
  return w->bits == 8 ? 4 : w->bits >= 3 ? 5 : (w->M > 16384 ? 9 : 6);
}
// Where the 32-row GEMV does not apply: the tensor-core GEMM from batch 5 for
// 3/4/8-bit codes with K >= 8192 (its shared-memory rings stay deep where the
// batch-8 GEMV's become shallow), else from batch 9.
static int tc_auto_min_batch(const hq_weight* w) { return (w->bits >= 3 && w->K >= 8192) ? 5 : 9; }

static bool tc_fits(const hq_weight* w) {
  return w->zeros == nullptr && w->layout == HQ_LAYOUT_PACKED && tc_col_block(w->bits, w->K) > 0;
}

static hq_path path_of(const hq_weight* w, int batch) {
  const int tc_min = g_tc_min_batch.load(std::memory_order_relaxed);
  if (tc_min > 0 && batch >= tc_min && tc_fits(w)) return HQ_PATH_TENSOR;
  int g32_min = g_g32_min_batch.load(std::memory_order_relaxed);
  if (g32_min == 0) g32_min = g32_auto_min_batch(w);
  if (batch >= g32_min && batch <= 16 && w->zeros == nullptr &&
      gemv32_supported(w->bits, w->M, w->K, batch)) {
    return HQ_PATH_GEMV32;
  }
  if (tc_min == 0 && batch >= tc_auto_min_batch(w) && tc_fits(w)) return HQ_PATH_TENSOR;
  return HQ_PATH_GEMV;
}

static bool use_tc(const hq_weight* w, int batch) { return path_of(w, batch) == HQ_PATH_TENSOR; }

// hq_linear workspace: [status 256 B] [tensor-core tile counters 1 KiB, zero
// between calls] [on the tensor-core path the rotated activation images
// (batch rounded up to whole batch blocks, x K fp16) and the partial sums of
// tiles shared by two CTAs; on the GEMV path the rotated activations of one
// batch block in fragment order (blocks run in turn)].  The counters sit at a
// fixed offset that neither path writes anything else to, so calls of any
// width and batch can share the workspace.
struct LinearWs {
  uint32_t* status;
  uint32_t* counters;
  void* xp;
  size_t bytes;
};

static LinearWs linear_ws(void* base, const hq_weight* w, int batch) {
  LinearWs l{};
  const int nb = gemv_col_block(w->bits, w->K, w->zeros != nullptr);
  const hq_path path = batch > 0 ? path_of(w, batch) : HQ_PATH_GEMV;
  const size_t xp_bytes =
      path == HQ_PATH_TENSOR   ? align256(tc_xp_bytes(w->bits, w->K, batch))
      : path == HQ_PATH_GEMV32 ? align256(gemv32_scratch_bytes(w->K, batch))
                               : align256(gemv_scratch_bytes(w->K, nb > 0 ? std::min(nb, std::max(batch, 1)) : 1));
  uint8_t* b = static_cast<uint8_t*>(base);
  l.status = reinterpret_cast<uint32_t*>(b);
  l.counters = reinterpret_cast<uint32_t*>(b + kStatusBytes);
  l.xp = b + kStatusBytes + kTcCounterBytes;
  l.bytes = kStatusBytes + kTcCounterBytes + xp_bytes;
  return l;
}

}  // namespace hq

using namespace hq;

extern "C" {

const char* hq_status_string(hq_status s) {
  switch (s) {
    case HQ_OK: return "HQ_OK";
    case HQ_ERR_INVALID_ARG: return "HQ_ERR_INVALID_ARG: bad pointer, size, alignment or value";
    case HQ_ERR_UNSUPPORTED: return "HQ_ERR_UNSUPPORTED: valid but not implemented";
    case HQ_ERR_WORKSPACE: return "HQ_ERR_WORKSPACE: workspace missing, misaligned or too small";
    case HQ_ERR_CUDA: return "HQ_ERR_CUDA: a CUDA launch or runtime call failed";
    case HQ_ERR_DATA: return "HQ_ERR_DATA: device data out of range";
    case HQ_ERR_TIMEOUT: return "HQ_ERR_TIMEOUT: a bounded device-side wait ran out";
  }
  return "HQ_ERR_UNKNOWN";
}

uint64_t hq_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

int hq_set_test_fault(int n) {
  if (n < 0) return g_test_faults.load();
  return g_test_faults.exchange(n);
}

int hq_set_tc_min_batch(int n) {
  if (n < 0) return g_tc_min_batch.load();
  return g_tc_min_batch.exchange(n);
}

int hq_set_gemv32_min_batch(int n) {
  if (n < 0) return g_g32_min_batch.load();
  return g_g32_min_batch.exchange(n);
}

int hq_linear_path(const hq_weight* w, int batch) {
  if (check_weight(w) != HQ_OK || batch <= 0) return -1;
  return static_cast<int>(path_of(w, batch));
}

hq_status hq_rotate(const void* x, hq_dtype x_dtype, void* x_rot, hq_dtype out_dtype, int n_rows,
                    int K, const int8_t* signs, hq_stream_t stream) {
  if (n_rows < 0) return HQ_ERR_INVALID_ARG;
  if (x_dtype < HQ_F16 || x_dtype > HQ_F32 || out_dtype < HQ_F16 || out_dtype > HQ_F32) {
    return HQ_ERR_INVALID_ARG;
  }
  if (K <= 0) return HQ_ERR_INVALID_ARG;
  if (!is_pow2(K) || K < 32 || K > 32768) return HQ_ERR_UNSUPPORTED;
  if (n_rows == 0) return HQ_OK;
  if (x == nullptr || x_rot == nullptr) return HQ_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(x_rot, 16)) return HQ_ERR_INVALID_ARG;
  if (signs != nullptr && !aligned(signs, 16)) return HQ_ERR_INVALID_ARG;
  if (n_rows > 0x7fffffff / 2) return HQ_ERR_INVALID_ARG;
  return from_cuda(launch_rotate(x_dtype, out_dtype, x, x_rot, n_rows, K, signs,
                                 reinterpret_cast<cudaStream_t>(stream)));
}

size_t hq_linear_workspace_size(const hq_weight* w, int batch) {
  if (check_weight(w) != HQ_OK || batch < 0) return 0;
  return linear_ws(nullptr, w, batch).bytes;
}

int hq_linear_uses_tensor_cores(const hq_weight* w, int batch) {
  if (check_weight(w) != HQ_OK || batch <= 0) return -1;
  return use_tc(w, batch) ? 1 : 0;
}

int hq_linear_launches(const hq_weight* w, int batch) {
  if (check_weight(w) != HQ_OK || batch <= 0) return 0;
  const hq_path path = path_of(w, batch);
  if (path == HQ_PATH_TENSOR) return tc_launches(w->bits, w->K, batch);
  if (path == HQ_PATH_GEMV32) return gemv32_launches(w->bits, w->M, w->K, batch);
  const int nb = gemv_col_block(w->bits, w->K, w->zeros != nullptr);
  if (nb == 0) return 0;
  int n = 0;
  for (int n0 = 0; n0 < batch; n0 += nb) n += gemv_launches(w->K, std::min(nb, batch - n0));
  return n;
}

hq_status hq_linear(const hq_weight* w, const uint16_t* x, int batch, float* y, void* workspace,
                    size_t ws_bytes, hq_stream_t stream) {
  const hq_status ws_ok = check_weight(w);
  if (ws_ok != HQ_OK) return ws_ok;
  if (batch < 0 || batch > 65535) return HQ_ERR_INVALID_ARG;
  if (batch == 0) return HQ_OK;
  if (x == nullptr || y == nullptr) return HQ_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(y, 16)) return HQ_ERR_INVALID_ARG;
  const LinearWs l = linear_ws(workspace, w, batch);
  if (workspace == nullptr || !aligned(workspace, 256) || ws_bytes < l.bytes) {
    return HQ_ERR_WORKSPACE;
  }
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const hq_path path = path_of(w, batch);
  if (path == HQ_PATH_GEMV32) {
    GemvArgs a;
    a.bits = w->bits;
    a.M = w->M;
    a.K = w->K;
    a.N = batch;
    a.zero = w->zero;
    a.q = w->qweight;
    a.scales = w->scales;
    a.x = x;
    a.signs = w->signs;
    a.y = y;
    a.ldy = w->M;
    a.status = l.status;
    a.xg = l.xp;
    a.planes = w->layout == HQ_LAYOUT_BITPLANES;
    a.sync = l.counters + kG32SyncWord;
    return from_cuda(launch_gemv32(a, st));
  }
  if (path == HQ_PATH_TENSOR) {
    TcArgs a;
    a.bits = w->bits;
    a.M = w->M;
    a.K = w->K;
    a.N = batch;
    a.zero = w->zero;
    a.q = w->qweight;
    a.scales = w->scales;
    a.x = x;
    a.signs = w->signs;
    a.y = y;
    a.ldy = w->M;
    a.status = l.status;
    a.xp = l.xp;
    a.counters = l.counters;
    return from_cuda(launch_linear_tc(a, st));
  }
  const int nb = gemv_col_block(w->bits, w->K, w->zeros != nullptr);
  if (nb == 0) return HQ_ERR_UNSUPPORTED;
  for (int n0 = 0; n0 < batch; n0 += nb) {
    GemvArgs a;
    a.bits = w->bits;
    a.M = w->M;
    a.K = w->K;
    a.N = batch - n0 < nb ? batch - n0 : nb;
    a.zero = w->zero;
    a.q = w->qweight;
    a.scales = w->scales;
    a.x = x + static_cast<size_t>(n0) * w->K;
    a.signs = w->signs;
    a.y = y + static_cast<size_t>(n0) * w->M;
    a.ldy = w->M;
    a.status = l.status;
    a.xg = l.xp;
    a.zeros = w->zeros;
    a.planes = w->layout == HQ_LAYOUT_BITPLANES;
    const cudaError_t e = launch_gemv(a, st);
    if (e != cudaSuccess) return from_cuda(e);
  }
  return HQ_OK;
}

hq_status hq_check_status(void* workspace, hq_stream_t stream) {
  if (workspace == nullptr || !aligned(workspace, 256)) return HQ_ERR_WORKSPACE;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return from_cuda(cudaErrorUnknown);
  uint32_t v = 0;
  if (cudaMemcpy(&v, workspace, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess) {
    return from_cuda(cudaErrorUnknown);
  }
  if (v == 0) return HQ_OK;
  if (cudaMemset(workspace, 0, sizeof(v)) != cudaSuccess) return from_cuda(cudaErrorUnknown);
  if (v & HQ_DEV_TIMEOUT) return HQ_ERR_TIMEOUT;
  return HQ_ERR_DATA;
}

hq_status hq_unpack_codes(const uint32_t* packed, int bits, size_t n_codes, uint8_t* codes_out,
                          hq_stream_t stream) {
  if (bits < 1 || bits > 8) return HQ_ERR_INVALID_ARG;
  if (n_codes == 0) return HQ_OK;
  if (packed == nullptr || codes_out == nullptr || !aligned(packed, 4)) return HQ_ERR_INVALID_ARG;
  return from_cuda(
      launch_unpack(packed, bits, n_codes, codes_out, reinterpret_cast<cudaStream_t>(stream)));
}

}  // extern "C"

