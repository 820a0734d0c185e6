// gemv.cu -- fused unpack-dequant GEMV over packed low-bit codes, batch <= 8.
//
// y[n][m] = sum_k scale[m][k/128] (q[m][k] - zero) x'[n][k] for a 16-row tile
// per CTA.  The decode of packed weights is the bytes-bound part of decoding
// ("decode is per-byte neutral": Laguna-S-2.1 gridbook card, "Reading it
// honestly"), so the kernel is built to stream codes at HBM rate:
//   * the CTA's 4 warps split the tile's K range; each warp pulls its 16 rows
//     x (K/4) codes into shared memory with one bulk (TMA) copy per row,
//     issued before griddepcontrol.wait so that the copies overlap the
//     previous kernel (the activations are the only dependent input);
//   * rows land at a padded stride that keeps the lanes' bundle loads free of
//     bank conflicts;
//   * each lane turns 32 codes into 16 fp16 pairs with one LOP3/PRMT per pair
//     (hq_layout.cuh) and feeds mma.sync m16n8k16 with fp32 accumulation: A =
//     the decoded tile, B = x' (pre-scaled, fragment-ordered by the prep
//     kernel), 8 MMAs per 128-code group, accumulator initialised with the
//     group's offset correction; the group scale multiplies the fp32 sum;
//   * the 4 warps' partial sums are added in a fixed order (deterministic).
#include <algorithm>

#include "hq_common.cuh"
#include "hq_internal.h"
#include "hq_launch.cuh"
#include "hq_layout.cuh"

namespace hq {

struct GemvKParams {
  const uint32_t* q;
  const __half* scales;
  const uint16_t* xs;
  const float* corr;
  float* y;
  uint32_t* status;
  int M, K, N, zero, ldy;
  int row_words;  // K * BITS / 32
  int stride;     // bytes between rows of a warp's slice in shared memory
  int xs_bytes;   // N * K * 2
  int corr_off, codes_off, red_off, bar_off;
};

constexpr int kGemvWarps = 4;
constexpr int kGemvRows = 16;

template <int BITS>
__global__ void __launch_bounds__(kGemvWarps * 32) gemv_kernel(const GemvKParams p) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, t = lane & 3;
  const int G = p.K >> 7;
  const int m0 = blockIdx.x * kGemvRows;
  const int rows_valid = min(kGemvRows, p.M - m0);
  const int G0 = (warp * G) / kGemvWarps, G1 = ((warp + 1) * G) / kGemvWarps;
  const uint32_t slice = static_cast<uint32_t>(G1 - G0) * 16u * BITS;

  uint16_t* xs_s = reinterpret_cast<uint16_t*>(smem);
  float* corr_s = reinterpret_cast<float*>(smem + p.corr_off);
  uint8_t* codes_w = smem + p.codes_off + warp * kGemvRows * p.stride;
  float4* red = reinterpret_cast<float4*>(smem + p.red_off);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + p.bar_off);

  if (tid == 0) {
    for (int i = 0; i <= kGemvWarps; ++i) mbar_init(&bars[i], 1);
    fence_mbar_init();
  }
  __syncthreads();
  pdl_launch_dependents();

  // Weights do not depend on earlier kernels: start their copies now.
  if (slice > 0) {
    if (lane == 0) mbar_arrive_expect_tx(&bars[warp], rows_valid * slice);
    __syncwarp();
    if (lane < rows_valid) {
      const uint8_t* src = reinterpret_cast<const uint8_t*>(
                               p.q + static_cast<size_t>(m0 + lane) * p.row_words) +
                           static_cast<size_t>(G0) * 16 * BITS;
      bulk_g2s(codes_w + lane * p.stride, src, slice, &bars[warp]);
    }
  }
  pdl_wait();
  if (tid == 0) {
    mbar_arrive_expect_tx(&bars[kGemvWarps], p.xs_bytes);
    bulk_g2s(xs_s, p.xs, p.xs_bytes, &bars[kGemvWarps]);
  }
  for (int i = tid; i < G * p.N; i += kGemvWarps * 32) corr_s[i] = p.corr[i];
  __syncthreads();

  bool ok = mbar_wait(&bars[kGemvWarps], 0);
  if (slice > 0) ok = mbar_wait(&bars[warp], 0) && ok;

  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  if (ok) {
    const bool ra = g < rows_valid, rb = g + 8 < rows_valid;
    const __half* sca = p.scales + static_cast<size_t>(m0 + g) * G;
    const __half* scb = p.scales + static_cast<size_t>(m0 + g + 8) * G;
    const bool n0 = 2 * t < p.N, n1 = 2 * t + 1 < p.N;
    const bool has_b = g < p.N;
    const uint8_t* rowa = codes_w + g * p.stride + t * 4 * BITS;
    const uint8_t* rowb = codes_w + (g + 8) * p.stride + t * 4 * BITS;
    const int xs_step = p.N * 16;  // halves between consecutive MMA steps
#pragma unroll 1
    for (int gi = G0; gi < G1; ++gi) {
      const int off = (gi - G0) * 16 * BITS;
      uint32_t wa[BITS], wb[BITS];
      load_bundle<BITS>(rowa + off, wa);
      load_bundle<BITS>(rowb + off, wb);
      const float sa = ra ? __half2float(sca[gi]) : 0.f;
      const float sb = rb ? __half2float(scb[gi]) : 0.f;
      const float k0 = n0 ? -corr_s[gi * p.N + 2 * t] : 0.f;
      const float k1 = n1 ? -corr_s[gi * p.N + 2 * t + 1] : 0.f;
      uint32_t Pa[16], Pb[16];
      decode16<BITS>(wa, Pa);
      decode16<BITS>(wb, Pb);
      float cg[4] = {k0, k1, k0, k1};
      const uint16_t* xb = xs_s + (static_cast<size_t>(8 * gi) * p.N + g) * 16 + t * 4;
#pragma unroll
      for (int s = 0; s < 8; ++s) {
        uint32_t b0 = 0u, b1 = 0u;
        if (has_b) {
          const uint2 bb = *reinterpret_cast<const uint2*>(xb + s * xs_step);
          b0 = bb.x;
          b1 = bb.y;
        }
        const uint32_t a[4] = {Pa[2 * s], Pb[2 * s], Pa[2 * s + 1], Pb[2 * s + 1]};
        mma_16816(cg, a, b0, b1, cg);
      }
      acc[0] = fmaf(sa, cg[0], acc[0]);
      acc[1] = fmaf(sa, cg[1], acc[1]);
      acc[2] = fmaf(sb, cg[2], acc[2]);
      acc[3] = fmaf(sb, cg[3], acc[3]);
    }
  } else {
    if (lane == 0) record_error(p.status, HQ_DEV_TIMEOUT);
    // Give copies still in flight one more bounded chance to land before
    // this CTA's shared memory is released.
    if (slice > 0) (void)mbar_wait(&bars[warp], 0);
    if (tid == 0) (void)mbar_wait(&bars[kGemvWarps], 0);
  }

  red[warp * 32 + lane] = make_float4(acc[0], acc[1], acc[2], acc[3]);
  const bool all_ok = __syncthreads_and(ok) != 0;
  if (warp == 0 && all_ok) {
    float4 s = red[lane];
#pragma unroll
    for (int w = 1; w < kGemvWarps; ++w) {
      const float4 u = red[w * 32 + lane];
      s.x += u.x;
      s.y += u.y;
      s.z += u.z;
      s.w += u.w;
    }
    const int ma = m0 + g, mb = m0 + g + 8;
    const int c0 = 2 * t, c1 = 2 * t + 1;
    if (g < rows_valid) {
      if (c0 < p.N) p.y[static_cast<size_t>(c0) * p.ldy + ma] = s.x;
      if (c1 < p.N) p.y[static_cast<size_t>(c1) * p.ldy + ma] = s.y;
    }
    if (g + 8 < rows_valid) {
      if (c0 < p.N) p.y[static_cast<size_t>(c0) * p.ldy + mb] = s.z;
      if (c1 < p.N) p.y[static_cast<size_t>(c1) * p.ldy + mb] = s.w;
    }
  }
}

struct GemvPlan {
  int stride, xs_bytes, corr_off, codes_off, red_off, bar_off;
  size_t smem;
};

static GemvPlan gemv_plan(int bits, int K, int nb) {
  GemvPlan pl{};
  const int G = K / kGroup;
  const int ng_max = (G + kGemvWarps - 1) / kGemvWarps;
  const int slice = ng_max * 16 * bits;
  const int words = slice / 4;
  const int pad_w = ((bank_target_words(bits) - words) % 32 + 32) % 32;
  pl.stride = slice + 4 * pad_w;
  pl.xs_bytes = nb * K * 2;
  pl.corr_off = (pl.xs_bytes + 15) & ~15;
  pl.codes_off = (pl.corr_off + G * nb * 4 + 127) & ~127;
  pl.red_off = pl.codes_off + kGemvWarps * kGemvRows * pl.stride;
  pl.bar_off = pl.red_off + kGemvWarps * 32 * 16;
  pl.smem = static_cast<size_t>(pl.bar_off) + 8 * (kGemvWarps + 1);
  return pl;
}

constexpr size_t kMaxSmem = 227 * 1024;

size_t gemv_smem_bytes(int bits, int K, int nb) {
  const GemvPlan pl = gemv_plan(bits, K, nb);
  return pl.smem <= kMaxSmem ? pl.smem : 0;
}

cudaError_t launch_gemv(const GemvArgs& a, cudaStream_t st) {
  const GemvPlan pl = gemv_plan(a.bits, a.K, a.N);
  if (pl.smem > kMaxSmem) return cudaErrorInvalidValue;
  GemvKParams p;
  p.q = a.q;
  p.scales = reinterpret_cast<const __half*>(a.scales);
  p.xs = a.xs;
  p.corr = a.corr;
  p.y = a.y;
  p.status = a.status;
  p.M = a.M;
  p.K = a.K;
  p.N = a.N;
  p.zero = a.zero;
  p.ldy = a.ldy;
  p.row_words = a.K * a.bits / 32;
  p.stride = pl.stride;
  p.xs_bytes = pl.xs_bytes;
  p.corr_off = pl.corr_off;
  p.codes_off = pl.codes_off;
  p.red_off = pl.red_off;
  p.bar_off = pl.bar_off;
  const dim3 grid((a.M + kGemvRows - 1) / kGemvRows);
  const dim3 block(kGemvWarps * 32);
  switch (a.bits) {
    case 2: return launch_pdl(gemv_kernel<2>, grid, block, pl.smem, st, true, p);
    case 3: return launch_pdl(gemv_kernel<3>, grid, block, pl.smem, st, true, p);
    case 4: return launch_pdl(gemv_kernel<4>, grid, block, pl.smem, st, true, p);
    case 8: return launch_pdl(gemv_kernel<8>, grid, block, pl.smem, st, true, p);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace hq
