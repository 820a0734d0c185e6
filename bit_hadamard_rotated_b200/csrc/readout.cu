// readout.cu -- hq_readout_topk: the screened top-k readout over an 8-bit
// lm_head kept as high and low nibble planes (lm_head_split.bin, "the same
// codes split into high/low nibble planes, used by the engine's screened
// readout": LLaDA2.2-mini Orin-Nano model card, file list and Properties
// table), and hq_split_nibbles, which makes the planes from 8-bit codes.
//
// The pages give no screening rule; this library's (the oracle implements the
// same one): with q = 16 hi + lo, zero point z and x' the rotated input,
//   screen  e[m]  = sum_k s (16 hi + 7.5 - z) x'_k        (the high plane only)
//   spread  sd[m] = sqrt(21.25 sum_k s^2 x'_k^2)          (the low nibbles' term,
//                   were they independent and uniform on 0..15)
//   L = e - beta sd,  U = e + beta sd,  tau = the topk-th largest L,
//   candidates: U >= tau; exact logits for those; the topk largest returned.
// On the GPU the threshold is taken from a histogram of the top 11 bits of L
// (the lower edge of the bin holding the topk-th largest): a lower tau, so a
// superset of the rule's candidates, whose extra rows cost only their exact
// logits (2 K bytes each).
//
// Launches: hq_rotate's kernel (x' in fp32), the small-batch GEMV over the
// high plane (4-bit codes, fractional zero point (z - 7.5) / 16: e / 16),
// ro_bounds_kernel (sd, U and the histogram of L), ro_refine_kernel
// (threshold, candidates, their exact logits from both planes, appended to a
// list) and ro_final_kernel (radix selection of the topk-th largest exact
// logit, sort of the entries at or above it, output; leaves the counters at
// zero for the next call).
#include <cuda_fp16.h>

#include <algorithm>

#include "hq_common.cuh"
#include "hq_internal.h"
#include "hq_launch.cuh"

namespace hq {
namespace ro {

constexpr int kHistBits = 11;  // top bits of the order-preserving key in the coarse histogram
constexpr int kHist = 1 << kHistBits;
constexpr int kFinalCap = 2048;  // entries the final CTA sorts in shared memory
constexpr int kRankMax = 512;    // lists up to this long are ranked directly (count^2 compares)
constexpr int kMaxTopk = 256;
constexpr int kMaxBatch = 8;
constexpr int kBoundsThreads = 256;
constexpr int kRefineWarps = 8;
constexpr int kFinalThreads = 1024;

// Order-preserving map of a float to a uint32 (larger float, larger key).
__device__ __forceinline__ uint32_t fkey(float f) {
  const uint32_t b = __float_as_uint(f);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
__device__ __forceinline__ float funkey(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

struct Ws {
  uint32_t* status;
  void* xg;        // the GEMV's scratch
  float* xr;       // [N][K] rotated input, fp32
  float* e16;      // [N][V] e / 16 from the high-plane GEMV
  float* U;        // [N][V]
  uint32_t* hist;  // [N][kHist] histogram of L's top bits (zero between calls)
  uint32_t* cnt;   // [N] candidates listed (zero between calls)
  uint32_t* done;  // [N] bounds CTAs finished (zero between calls)
  float* tau;      // [N] candidate threshold (lower edge of the topk-th largest L's bin)
  float2* list;    // [N][V] (exact logit, row as int bits)
};

struct Dims {
  int V, K, N, zero, topk;
  float beta;
};

static size_t a256(size_t v) { return (v + 255) & ~static_cast<size_t>(255); }

struct Plan {
  size_t off[8];
  size_t bytes;
};

static Plan plan(int V, int K, int N) {
  Plan p{};
  const size_t sizes[8] = {
      256,
      gemv_scratch_bytes(K, std::min(N, kMaxBatch)),
      4 * static_cast<size_t>(N) * K,
      4 * static_cast<size_t>(N) * V,
      4 * static_cast<size_t>(N) * V,
      4 * static_cast<size_t>(N) * kHist,
      4 * 3 * static_cast<size_t>(kMaxBatch),  // cnt [N], done [N], tau [N] (kMaxBatch each)
      8 * static_cast<size_t>(N) * V,
  };
  size_t o = 0;
  for (int i = 0; i < 8; ++i) {
    p.off[i] = o;
    o += a256(sizes[i]);
  }
  p.bytes = o;
  return p;
}

static Ws carve(void* base, const Plan& pl) {
  uint8_t* b = static_cast<uint8_t*>(base);
  Ws w;
  w.status = reinterpret_cast<uint32_t*>(b + pl.off[0]);
  w.xg = b + pl.off[1];
  w.xr = reinterpret_cast<float*>(b + pl.off[2]);
  w.e16 = reinterpret_cast<float*>(b + pl.off[3]);
  w.U = reinterpret_cast<float*>(b + pl.off[4]);
  w.hist = reinterpret_cast<uint32_t*>(b + pl.off[5]);
  w.cnt = reinterpret_cast<uint32_t*>(b + pl.off[6]);
  w.done = w.cnt + kMaxBatch;
  w.tau = reinterpret_cast<float*>(w.cnt + 2 * kMaxBatch);
  w.list = reinterpret_cast<float2*>(b + pl.off[7]);
  return w;
}

// Grid (ceil(V / 256), N): per row m of batch row n, sd, L and U; U stored, the
// top 11 bits of L's key counted (shared-memory histogram, then merged).
// The bin (of kHist, counted from the top) holding the need-th largest key,
// and the number of entries in the bins above it: one warp, two rounds of
// loads (each lane sums 64 bins; then the crossing lane's 64 bins, two per
// lane), with inclusive scans across the lanes.
__device__ __forceinline__ void top_bin(const uint32_t* h, uint32_t need, int lane, int* bin_out,
                                        uint32_t* above_out) {
  const int hi_bin = kHist - 64 * lane - 1;  // lane l: bins [hi_bin - 63, hi_bin]
  uint32_t c = 0;
  const uint4* g4 = reinterpret_cast<const uint4*>(h + hi_bin - 63);
#pragma unroll
  for (int b = 0; b < 16; ++b) {
    const uint4 v = __ldcg(g4 + b);
    c += v.x + v.y + v.z + v.w;
  }
  uint32_t incl = c;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  const int first = __ffs(__ballot_sync(0xffffffffu, incl >= need)) - 1;  // crossing lane
  const uint32_t base = __shfl_sync(0xffffffffu, incl - c, first);       // entries above its bins
  const int top = kHist - 64 * first - 1;
  // lane j: bins top - 2 j and top - 2 j - 1
  const uint32_t b0 = __ldcg(h + top - 2 * lane), b1 = __ldcg(h + top - 2 * lane - 1);
  uint32_t pair = b0 + b1, inc2 = pair;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, inc2, o);
    if (lane >= o) inc2 += y;
  }
  const uint32_t before_pair = base + inc2 - pair;  // entries above bin top - 2 j
  const int j = __ffs(__ballot_sync(0xffffffffu, base + inc2 >= need)) - 1;
  const uint32_t bp = __shfl_sync(0xffffffffu, before_pair, j);
  const uint32_t first_of_pair = __shfl_sync(0xffffffffu, b0, j);
  const bool in_first = bp + first_of_pair >= need;
  *bin_out = in_first ? top - 2 * j : top - 2 * j - 1;
  *above_out = in_first ? bp : bp + first_of_pair;
}

__global__ void __launch_bounds__(kBoundsThreads)
    ro_bounds_kernel(const uint16_t* __restrict__ scales, Ws w, Dims d) {
  __shared__ float x2[256];     // sum of x'^2 over each group (G <= 256)
  __shared__ uint32_t hist[kHist];
  pdl_launch_dependents();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int n = blockIdx.y;
  const int G = d.K / kGroup;
  for (int i = tid; i < kHist; i += kBoundsThreads) hist[i] = 0u;
  pdl_wait();  // x' and e / 16 come from the previous kernels
  const float* xr = w.xr + static_cast<size_t>(n) * d.K;
  for (int g = warp; g < G; g += kBoundsThreads / 32) {
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float v = xr[kGroup * g + 32 * i + lane];
      s = fmaf(v, v, s);
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (lane == 0) x2[g] = s;
  }
  __syncthreads();
  const int m = blockIdx.x * kBoundsThreads + tid;
  if (m < d.V) {
    const __half* sr = reinterpret_cast<const __half*>(scales) + static_cast<size_t>(m) * G;
    float var = 0.f;
    for (int g = 0; g < G; ++g) {
      const float s = __half2float(sr[g]);
      var = fmaf(s * s, x2[g], var);
    }
    const float sd = sqrtf(21.25f * var);
    const float e = 16.f * w.e16[static_cast<size_t>(n) * d.V + m];
    w.U[static_cast<size_t>(n) * d.V + m] = e + d.beta * sd;
    atomicAdd(&hist[fkey(e - d.beta * sd) >> (32 - kHistBits)], 1u);
  }
  __syncthreads();
  uint32_t* gh = w.hist + static_cast<size_t>(n) * kHist;
  for (int i = tid; i < kHist; i += kBoundsThreads) {
    if (hist[i] != 0u) atomicAdd(&gh[i], hist[i]);
  }
  // the last CTA of the row to finish finds the threshold once (every other
  // CTA's histogram adds are visible after its fence and counter increment)
  __shared__ bool s_last;
  __threadfence();
  __syncthreads();
  if (tid == 0) s_last = atomicAdd(w.done + n, 1u) == gridDim.x - 1;
  __syncthreads();
  if (s_last && warp == 0) {
    __threadfence();
    int bin;
    uint32_t above;
    top_bin(gh, static_cast<uint32_t>(d.topk), lane, &bin, &above);
    if (lane == 0) {
      w.tau[n] = funkey(static_cast<uint32_t>(bin) << (32 - kHistBits));
      w.done[n] = 0u;
    }
  }
}

// Grid (ceil(V / (32 warps)), N): warp 0 first finds the threshold (the lower
// edge of the histogram bin holding the topk-th largest L); then each warp
// takes 32 rows, and for every row with U >= threshold computes its exact
// logit from both planes and appends (logit, row) to the batch row's list.
__global__ void __launch_bounds__(kRefineWarps * 32)
    ro_refine_kernel(const uint32_t* __restrict__ hi, const uint32_t* __restrict__ lo,
                     const uint16_t* __restrict__ scales, Ws w, Dims d) {
  pdl_launch_dependents();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int n = blockIdx.y;
  pdl_wait();
  const float tau = w.tau[n];
  const int words = d.K / 8;  // uint32 words of a 4-bit plane row
  const int G = d.K / kGroup;
  const float* xr = w.xr + static_cast<size_t>(n) * d.K;
  const int m0 = (blockIdx.x * kRefineWarps + warp) * 32;
  const int mine = m0 + lane;
  const bool cand = mine < d.V && w.U[static_cast<size_t>(n) * d.V + mine] >= tau;
  unsigned todo = __ballot_sync(0xffffffffu, cand);
  while (todo != 0u) {
    const int r = __ffs(todo) - 1;
    todo &= todo - 1u;
    const int m = m0 + r;
    const uint32_t* hr = hi + static_cast<size_t>(m) * words;
    const uint32_t* lr = lo + static_cast<size_t>(m) * words;
    const __half* sr = reinterpret_cast<const __half*>(scales) + static_cast<size_t>(m) * G;
    float acc = 0.f;
    // the loads of 8 iterations are independent: unrolled, they are issued
    // together (one round trip to L2 per 8 instead of one per iteration)
#pragma unroll 8
    for (int wd = lane; wd < words; wd += 32) {
      const uint32_t h = hr[wd], l = lr[wd];
      const float4 xa = *reinterpret_cast<const float4*>(xr + 8 * wd);
      const float4 xb = *reinterpret_cast<const float4*>(xr + 8 * wd + 4);
      const float xv[8] = {xa.x, xa.y, xa.z, xa.w, xb.x, xb.y, xb.z, xb.w};
      float part = 0.f;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int q = 16 * static_cast<int>((h >> (4 * j)) & 15u) + static_cast<int>((l >> (4 * j)) & 15u);
        part = fmaf(static_cast<float>(q - d.zero), xv[j], part);
      }
      acc = fmaf(__half2float(sr[wd >> 4]), part, acc);  // 16 words per 128-code group
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) {
      const uint32_t at = atomicAdd(w.cnt + n, 1u);
      w.list[static_cast<size_t>(n) * d.V + at] = make_float2(acc, __int_as_float(m));
    }
  }
}

// Entry order of the final sort: larger logit first, then the lower row.
__device__ __forceinline__ bool before(float2 a, float2 b) {
  return a.x > b.x || (a.x == b.x && __float_as_int(a.y) < __float_as_int(b.y));
}

// One CTA per batch row: the topk-th largest exact logit among the listed
// candidates (radix selection on the order-preserving keys, 11 + 11 + 10
// bits), the entries at or above it sorted in shared memory (bitonic), the
// first topk written out; the row's counters are cleared for the next call.
__global__ void __launch_bounds__(kFinalThreads)
    ro_final_kernel(Ws w, Dims d, int32_t* __restrict__ ids, float* __restrict__ out) {
  __shared__ __align__(16) uint32_t hist[kHist];
  __shared__ float2 keep[kFinalCap];
  __shared__ uint32_t s_prefix, s_need, s_kept;
  pdl_launch_dependents();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int n = blockIdx.x;
  pdl_wait();
  const uint32_t count = w.cnt[n];
  const float2* lst = w.list + static_cast<size_t>(n) * d.V;
  if (count <= static_cast<uint32_t>(kRankMax)) {
    // a short list: every candidate's rank is the number of entries before
    // it in (logit descending, row ascending), a total order, so the ranks
    // 0 .. topk - 1 are the output positions
    for (uint32_t i = tid; i < count; i += kFinalThreads) keep[i] = lst[i];
    __syncthreads();
    for (uint32_t i = tid; i < count; i += kFinalThreads) {
      const float2 v = keep[i];
      uint32_t rank = 0;
      for (uint32_t j = 0; j < count; ++j) rank += before(keep[j], v) ? 1u : 0u;
      if (rank < static_cast<uint32_t>(d.topk)) {
        ids[static_cast<size_t>(n) * d.topk + rank] = __float_as_int(v.y);
        out[static_cast<size_t>(n) * d.topk + rank] = v.x;
      }
    }
    uint32_t* gh = w.hist + static_cast<size_t>(n) * kHist;
    for (int i = tid; i < kHist; i += kFinalThreads) gh[i] = 0u;
    if (tid == 0) w.cnt[n] = 0u;
    return;
  }
  uint32_t prefix = 0u, pmask = 0u;
  if (tid == 0) {
    s_need = static_cast<uint32_t>(d.topk);
    s_kept = 0u;
  }
  const int shifts[3] = {21, 10, 0}, widths[3] = {11, 11, 10};
  for (int pass = 0; pass < 3; ++pass) {
    const int sh = shifts[pass];
    const uint32_t bmask = (1u << widths[pass]) - 1u;
    for (int i = tid; i < kHist; i += kFinalThreads) hist[i] = 0u;
    __syncthreads();
    for (uint32_t i = tid; i < count; i += kFinalThreads) {
      const uint32_t k = fkey(lst[i].x);
      if ((k & pmask) == prefix) atomicAdd(&hist[(k >> sh) & bmask], 1u);
    }
    __syncthreads();
    if (warp == 0) {
      // the bin from the top where the count reaches s_need: each lane sums
      // per = nb / 32 bins, a scan across lanes finds the crossing lane, then
      // its bins (per / 32 a lane) are scanned the same way
      const int nb = static_cast<int>(bmask) + 1, per = nb / 32;
      const int top = nb - per * lane - 1;
      uint32_t c = 0;
      for (int b = 0; b < per; b += 4) {
        const uint4 v = *reinterpret_cast<const uint4*>(&hist[top - per + 1 + b]);
        c += v.x + v.y + v.z + v.w;
      }
      uint32_t incl = c;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      const uint32_t need = s_need;
      const int first = __ffs(__ballot_sync(0xffffffffu, incl >= need)) - 1;
      const uint32_t base = __shfl_sync(0xffffffffu, incl - c, first);
      const int ftop = nb - per * first - 1;
      const int q = per / 32;  // bins per lane in the second scan (1 or 2)
      uint32_t bv[2] = {0u, 0u}, own = 0u;
      for (int k = 0; k < q; ++k) {
        bv[k] = hist[ftop - q * lane - k];
        own += bv[k];
      }
      uint32_t inc2 = own;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, inc2, o);
        if (lane >= o) inc2 += y;
      }
      const int j = __ffs(__ballot_sync(0xffffffffu, base + inc2 >= need)) - 1;
      if (lane == j) {
        uint32_t acc = base + inc2 - own;  // entries above this lane's bins
        int bin = ftop - q * lane;
        for (int k = 0; k < q; ++k) {
          bin = ftop - q * lane - k;
          if (acc + bv[k] >= need) break;
          acc += bv[k];
        }
        s_need = need - acc;
        s_prefix = prefix | (static_cast<uint32_t>(bin) << sh);
      }
    }
    __syncthreads();
    prefix = s_prefix;
    pmask |= bmask << sh;
    __syncthreads();
  }
  // prefix is now the key of the topk-th largest logit: keep every entry at or above it
  for (uint32_t i = tid; i < count; i += kFinalThreads) {
    const float2 v = lst[i];
    if (fkey(v.x) >= prefix) {
      const uint32_t at = atomicAdd(&s_kept, 1u);
      if (at < kFinalCap) keep[at] = v;
    }
  }
  __syncthreads();
  const int kept = min(static_cast<int>(s_kept), kFinalCap);
  int size = 1;
  while (size < kept) size <<= 1;
  for (int i = kept + tid; i < size; i += kFinalThreads) keep[i] = make_float2(-INFINITY, __int_as_float(0x7FFFFFFF));
  __syncthreads();
  for (int k = 2; k <= size; k <<= 1) {
    for (int j = k >> 1; j > 0; j >>= 1) {
      for (int i = tid; i < size; i += kFinalThreads) {
        const int p = i ^ j;
        if (p > i) {
          const bool up = (i & k) == 0;
          const float2 a = keep[i], b = keep[p];
          if (up ? before(b, a) : before(a, b)) {
            keep[i] = b;
            keep[p] = a;
          }
        }
      }
      __syncthreads();
    }
  }
  for (int i = tid; i < d.topk; i += kFinalThreads) {
    const float2 v = keep[i];
    ids[static_cast<size_t>(n) * d.topk + i] = __float_as_int(v.y);
    out[static_cast<size_t>(n) * d.topk + i] = v.x;
  }
  // counters back at zero for the next call on this workspace
  uint32_t* gh = w.hist + static_cast<size_t>(n) * kHist;
  for (int i = tid; i < kHist; i += kFinalThreads) gh[i] = 0u;
  if (tid == 0) w.cnt[n] = 0u;
}

// hi / lo planes of 8-bit codes: thread i makes word i of each plane (codes
// 8i..8i+7) from words 2i and 2i + 1 of the 8-bit matrix (row-major, whole
// rows of K / 4 and K / 8 words).
__global__ void split_nibbles_kernel(const uint32_t* __restrict__ q8, uint32_t* __restrict__ hi,
                                     uint32_t* __restrict__ lo, size_t n_words) {
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n_words;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const uint32_t a = q8[2 * i], b = q8[2 * i + 1];
    // byte j of a (code j) -> nibble j: compress the low nibbles of the bytes
    auto squeeze = [](uint32_t v) {  // v: a nibble in the low half of each byte
      v = (v | (v >> 4)) & 0x00FF00FFu;
      return (v | (v >> 8)) & 0x0000FFFFu;
    };
    lo[i] = squeeze(a & 0x0F0F0F0Fu) | (squeeze(b & 0x0F0F0F0Fu) << 16);
    hi[i] = squeeze((a >> 4) & 0x0F0F0F0Fu) | (squeeze((b >> 4) & 0x0F0F0F0Fu) << 16);
  }
}

}  // namespace ro
}  // namespace hq

using namespace hq;

extern "C" {

static bool ro_weight_ok(const hq_readout_weight* r) {
  auto al = [](const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; };
  return r != nullptr && r->V >= 1 && r->K >= 128 && r->K <= 32768 && (r->K & (r->K - 1)) == 0 &&
         r->zero >= 0 && r->zero < 256 && r->hi && r->lo && r->scales && al(r->hi, 16) && al(r->lo, 16) &&
         al(r->scales, 16) && (r->signs == nullptr || al(r->signs, 16)) && r->V <= (1 << 28);
}

size_t hq_readout_workspace_size(const hq_readout_weight* r, int batch) {
  if (!ro_weight_ok(r) || batch < 1 || batch > ro::kMaxBatch) return 0;
  return ro::plan(r->V, r->K, batch).bytes;
}

hq_status hq_readout_topk(const hq_readout_weight* r, const uint16_t* x, int batch, int topk,
                          float beta, int32_t* ids, float* logits, void* workspace,
                          size_t ws_bytes, hq_stream_t stream) {
  auto al = [](const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; };
  if (r == nullptr) return HQ_ERR_INVALID_ARG;
  if (r->K < 128 || r->K > 32768 || (r->K & (r->K - 1)) != 0) return HQ_ERR_UNSUPPORTED;
  if (!ro_weight_ok(r)) return HQ_ERR_INVALID_ARG;
  if (batch < 0 || batch > ro::kMaxBatch) return batch < 0 ? HQ_ERR_INVALID_ARG : HQ_ERR_UNSUPPORTED;
  if (batch == 0) return HQ_OK;
  if (topk < 1 || topk > ro::kMaxTopk || topk > r->V) return HQ_ERR_INVALID_ARG;
  if (!(beta >= 0.f) || !(beta < 1e30f)) return HQ_ERR_INVALID_ARG;
  if (!x || !ids || !logits || !al(x, 16) || !al(ids, 4) || !al(logits, 4)) return HQ_ERR_INVALID_ARG;
  const ro::Plan pl = ro::plan(r->V, r->K, batch);
  if (!workspace || !al(workspace, 256) || ws_bytes < pl.bytes) return HQ_ERR_WORKSPACE;
  const ro::Ws w = ro::carve(workspace, pl);
  const ro::Dims d{r->V, r->K, batch, r->zero, topk, beta};
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = launch_rotate(HQ_F16, HQ_F32, x, w.xr, batch, r->K, r->signs, st);
  if (e == cudaSuccess) {
    GemvArgs a;
    a.bits = 4;
    a.M = r->V;
    a.K = r->K;
    a.N = batch;
    a.zero = 0;
    a.zero_frac = true;
    a.zero_f = (static_cast<float>(r->zero) - 7.5f) / 16.f;  // exact in fp32
    a.q = r->hi;
    a.scales = r->scales;
    a.x = x;
    a.signs = r->signs;
    a.y = w.e16;
    a.ldy = r->V;
    a.status = w.status;
    a.xg = w.xg;
    e = launch_gemv(a, st);
  }
  if (e == cudaSuccess) {
    const dim3 grid((r->V + ro::kBoundsThreads - 1) / ro::kBoundsThreads, batch);
    e = launch_pdl(ro::ro_bounds_kernel, grid, dim3(ro::kBoundsThreads), 0, st, true, r->scales, w, d);
  }
  if (e == cudaSuccess) {
    const int rows_per_cta = 32 * ro::kRefineWarps;
    const dim3 grid((r->V + rows_per_cta - 1) / rows_per_cta, batch);
    e = launch_pdl(ro::ro_refine_kernel, grid, dim3(ro::kRefineWarps * 32), 0, st, true, r->hi, r->lo,
                   r->scales, w, d);
  }
  if (e == cudaSuccess) {
    e = launch_pdl(ro::ro_final_kernel, dim3(batch), dim3(ro::kFinalThreads), 0, st, true, w, d, ids, logits);
  }
  if (e != cudaSuccess) {
    (void)cudaGetLastError();
    return HQ_ERR_CUDA;
  }
  return HQ_OK;
}

hq_status hq_split_nibbles(const uint32_t* q8, int rows, int K, uint32_t* hi, uint32_t* lo,
                           hq_stream_t stream) {
  auto al = [](const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; };
  if (rows < 0 || K <= 0 || K % 8 != 0) return HQ_ERR_INVALID_ARG;
  if (rows == 0) return HQ_OK;
  if (!q8 || !hi || !lo || !al(q8, 8) || !al(hi, 4) || !al(lo, 4)) return HQ_ERR_INVALID_ARG;
  const size_t n_words = static_cast<size_t>(rows) * (K / 8);
  const unsigned blocks = static_cast<unsigned>(std::min<size_t>((n_words + 255) / 256, 148 * 16));
  note_launch();
  ro::split_nibbles_kernel<<<blocks, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(q8, hi, lo, n_words);
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? HQ_OK : HQ_ERR_CUDA;
}

}  // extern "C"
