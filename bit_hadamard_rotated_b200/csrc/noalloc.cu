// noalloc.cu -- hq_linear_noalloc: the rotated low-bit linear with its scratch
// memory in a fixed, file-scope device array instead of a caller workspace.
//
// Who needs it: callers that cannot allocate device memory for a workspace.
// A plug-in running inside another program's process may find the device heap
// owned by that program's pool allocator, with no way to add buffers of its
// own; a latency-critical loop cannot afford cudaMalloc, which may
// synchronise the device and takes unbounded time; and a thin foreign-language
// binding may have device pointers to its tensors but no allocator to manage a
// scratch buffer's lifetime.  This entry point needs nothing beyond the
// weight, input and output buffers.
//
// Costs of that convenience:
//   * every GPU that loads the library keeps kScratchBytes (512 KiB) of device
//     memory until the process exits;
//   * every batch runs the GEMV kernels in blocks of up to 8 columns: the
//     tensor-core path would need a batch-sized activation buffer;
//   * every call shares the one array, so calls that overlap on the GPU (two
//     streams, or two host threads) race on it and must be serialised by the
//     caller;
//   * device-side wait timeouts are recorded in the array's status word, which
//     the next call clears: hq_linear_noalloc_check_status reads (and clears)
//     what the last call recorded.
#include "hq_internal.h"

namespace hq {
namespace {

constexpr size_t kScratchBytes = size_t{512} << 10;  // 512 KiB in total
constexpr size_t kStatus = 256;                      // status word, kept zero
// Rotated activations of one batch block: at most 332 KiB (K = 16384 with 8
// columns; K = 32768 runs blocks of at most 2).
constexpr size_t kXgBytes = kScratchBytes - kStatus;

// The scratch: [status][rotated activations of the current batch block].
// Static storage starts zeroed; each call clears the status word.
__device__ __align__(256) uint8_t g_noalloc_scratch[kScratchBytes];

// Device address of the array in the current context.  The host-side name of
// a __device__ variable is not a device address, and the address belongs to a
// CUDA context, not to a device ordinal: a host that binds its own
// (non-primary) context, or a cudaDeviceReset that reloads the module, gives
// the array a new address.  So it is looked up on every call; the lookup is a
// runtime query that allocates nothing.  The first lookup in a context loads
// the library's device code there, which is why the first call belongs before
// any stream capture.
cudaError_t scratch_in_current_context(uint8_t** out) {
  void* p = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
  if (e != cudaSuccess) return e;
  *out = static_cast<uint8_t*>(p);
  return cudaSuccess;
}

}  // namespace
}  // namespace hq

using namespace hq;

extern "C" hq_status hq_linear_noalloc(const hq_weight* w, const uint16_t* x, int batch, float* y,
                                       hq_stream_t stream) {
  auto aligned = [](const void* p, uintptr_t a) {
    return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0;
  };
  auto pow2 = [](int v) { return v > 0 && (v & (v - 1)) == 0; };
  if (w == nullptr || w->M <= 0 || w->K <= 0 || w->M > (1 << 28)) return HQ_ERR_INVALID_ARG;
  if (!(w->bits == 2 || w->bits == 3 || w->bits == 4 || w->bits == 8)) {
    return (w->bits >= 1 && w->bits <= 8) ? HQ_ERR_UNSUPPORTED : HQ_ERR_INVALID_ARG;
  }
  if (!pow2(w->K) || w->K < 128 || w->K > 32768) return HQ_ERR_UNSUPPORTED;
  if (w->zero < 0 || w->zero >= (1 << w->bits)) return HQ_ERR_INVALID_ARG;
  if (!w->qweight || !w->scales || !aligned(w->qweight, 16) || !aligned(w->scales, 16) ||
      (w->signs && !aligned(w->signs, 16)) || (w->zeros && !aligned(w->zeros, 16))) {
    return HQ_ERR_INVALID_ARG;
  }
  if (w->layout != HQ_LAYOUT_PACKED && w->layout != HQ_LAYOUT_BITPLANES) return HQ_ERR_INVALID_ARG;
  if (w->layout == HQ_LAYOUT_BITPLANES && w->bits != 2) return HQ_ERR_UNSUPPORTED;
  if (batch < 0 || batch > 65535) return HQ_ERR_INVALID_ARG;
  if (batch == 0) return HQ_OK;
  if (!x || !y || !aligned(x, 16) || !aligned(y, 16)) return HQ_ERR_INVALID_ARG;
  int nb = 0;
  for (int b = 8; b >= 1 && nb == 0; b >>= 1) {
    if (gemv_smem_bytes(w->bits, w->K, b, w->zeros != nullptr) != 0) nb = b;
  }
  if (nb == 0) return HQ_ERR_UNSUPPORTED;
  // beyond what the fixed scratch holds (cannot happen for a supported K)
  if (gemv_scratch_bytes(w->K, nb) > kXgBytes) return HQ_ERR_WORKSPACE;

  uint8_t* scratch = nullptr;
  if (scratch_in_current_context(&scratch) != cudaSuccess) {
    (void)cudaGetLastError();
    return HQ_ERR_CUDA;
  }
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(scratch, 0, kStatus, st) != cudaSuccess) {
    (void)cudaGetLastError();
    return HQ_ERR_CUDA;
  }
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
    a.status = reinterpret_cast<uint32_t*>(scratch);
    a.xg = scratch + kStatus;
    a.zeros = w->zeros;
    a.planes = w->layout == HQ_LAYOUT_BITPLANES;
    if (launch_gemv(a, st) != cudaSuccess) {
      (void)cudaGetLastError();
      return HQ_ERR_CUDA;
    }
  }
  return HQ_OK;
}

// The status word is the first word of the scratch: every call clears it
// before its kernels run, so after a synchronisation it holds what the last
// call's kernels recorded.
extern "C" hq_status hq_linear_noalloc_check_status(hq_stream_t stream) {
  uint8_t* scratch = nullptr;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  uint32_t v = 0;
  if (scratch_in_current_context(&scratch) != cudaSuccess ||
      cudaMemcpyAsync(&v, scratch, sizeof(v), cudaMemcpyDeviceToHost, st) != cudaSuccess ||
      cudaStreamSynchronize(st) != cudaSuccess) {
    (void)cudaGetLastError();
    return HQ_ERR_CUDA;
  }
  if (v == 0) return HQ_OK;
  if (cudaMemsetAsync(scratch, 0, sizeof(v), st) != cudaSuccess || cudaStreamSynchronize(st) != cudaSuccess) {
    (void)cudaGetLastError();
    return HQ_ERR_CUDA;
  }
  return (v & HQ_DEV_TIMEOUT) ? HQ_ERR_TIMEOUT : HQ_ERR_DATA;
}
