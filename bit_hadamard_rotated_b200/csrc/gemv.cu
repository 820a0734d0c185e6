// gemv.cu -- fused rotate + unpack-dequant GEMV over packed low-bit codes,
// batch <= 8 per launch.
//
//   y[n][m] = sum_k scale[m][k/128] (q[m][k] - zero) x'[n][k],
//   x'[n]   = H_K diag(s) x[n] / sqrt(K).
//
// Decoding is bound by weight bytes ("decode is per-byte neutral": Laguna-S-2.1
// gridbook card, "Reading it honestly"), so the kernel is shaped to stream the
// packed codes at HBM rate with the rotation and all dequantisation on chip:
//
//   * Persistent grid, one CTA of 8 warps per SM.  The work is the list of
//     (16-row tile, 128-code group) units; every warp owns one contiguous
//     range of ~U/(8 * #SMs) units, so the load is balanced to one group.
//   * Each warp streams its range through a private ring of NS shared-memory
//     slots.  A slot holds up to CH groups of 16 rows (one bulk/TMA copy per
//     row, rows at a bank-conflict-free padded stride) and the matching fp16
//     scales (one more bulk copy per row), all completing on one mbarrier.
//     The first NS copies are issued before griddepcontrol.wait: weights do not
//     depend on earlier kernels, so they overlap the previous kernel's tail.
//   * Meanwhile the CTA rotates its N activation rows in fp32 (fwht.cuh) and
//     stores x' as fp16 in the order of the MMA B fragments (hq_layout.cuh).
//   * Per group: each lane decodes 2 x 32 codes into exact fp16 (q - zero)
//     pairs (one LOP3/PRMT + one HFMA2 per pair), 8 mma.sync m16n8k16 with
//     fp32 accumulation in two independent chains, then acc += scale * sum.
//   * A tile split between warps is finished by whichever contributor arrives
//     last at the tile's counter: it adds all contributors' partial sums in
//     warp order (deterministic, no waiting) and resets the counter.
#include <algorithm>

#include "fwht.cuh"
#include "hq_common.cuh"
#include "hq_internal.h"
#include "hq_io.cuh"
#include "hq_launch.cuh"
#include "hq_layout.cuh"

namespace hq {

constexpr int kWarps = 8;
constexpr int kRows = 16;

struct GemvParams {
  const uint32_t* q;
  const uint16_t* scales;
  const __half* x;
  const int8_t* signs;
  float* y;
  uint32_t* status;
  float4* part;   // [GWmax][2][32] partial tiles
  uint32_t* cnt;  // [n_tiles] arrival counters, zero between launches
  int M, N, ldy;
  uint32_t U;  // units = n_tiles * G
  uint32_t GW;  // active warps
  int CH, NS, stride, slot_bytes, buf_off, ring_off, bar_off;
  float inv_sqrt_k;
  uint32_t add[16];
};

__device__ __forceinline__ uint32_t unit_begin(uint32_t gw, uint32_t U, uint32_t GW) {
  return static_cast<uint32_t>((static_cast<uint64_t>(gw) * U) / GW);
}
// Warp whose range contains unit u.
__device__ __forceinline__ uint32_t unit_owner(uint32_t u, uint32_t U, uint32_t GW) {
  return static_cast<uint32_t>((static_cast<uint64_t>(u) * GW + GW - 1) / U);
}

template <int BITS, int LOGK>
__global__ void __launch_bounds__(kWarps * 32, 1) gemv_kernel(const __grid_constant__ GemvParams p) {
  using FS = FwhtShape<LOGK, 3>;
  constexpr int K = 1 << LOGK;
  constexpr int G = K / kGroup;
  constexpr int GB = 16 * BITS;  // bytes of one group of one row
  extern __shared__ __align__(128) uint8_t smem[];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, t = lane & 3;
  const uint32_t gw = blockIdx.x * kWarps + warp;
  const bool active = gw < p.GW;
  const uint32_t u0 = active ? unit_begin(gw, p.U, p.GW) : 0u;
  const uint32_t u1 = active ? unit_begin(gw + 1, p.U, p.GW) : 0u;
  const int row_words = K * BITS / 32;

  uint16_t* xs = reinterpret_cast<uint16_t*>(smem);
  float* buf = reinterpret_cast<float*>(smem + p.buf_off);
  uint8_t* ring = smem + p.ring_off + warp * p.NS * p.slot_bytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + p.bar_off) + warp * p.NS;

  if (lane == 0) {
    for (int i = 0; i < p.NS; ++i) mbar_init(&bars[i], 1);
    fence_mbar_init();
  }
  __syncthreads();
  pdl_launch_dependents();

  // ---- producer side of the warp's ring: one chunk = up to CH groups of a tile
  uint32_t ui = u0;
  int issued = 0;
  auto issue = [&](int slot) {
    const uint32_t tile = ui / G, g0 = ui % G;
    const uint32_t len = min(static_cast<uint32_t>(p.CH), min(G - g0, u1 - ui));
    const int m0 = tile * kRows;
    const int rv = min(kRows, p.M - m0);
    uint8_t* base = ring + slot * p.slot_bytes;
    uint8_t* sdst = base + kRows * p.stride;
    const uint32_t cbytes = len * GB;
    uint32_t total = rv * cbytes;
    uint32_t sg0 = 0, sbytes = 0;
    bool tile_bulk = false;
    if constexpr (G >= 8) {
      sg0 = g0 & ~7u;
      sbytes = (((g0 + len + 7u) & ~7u) - sg0) * 2u;
      total += rv * sbytes;
    } else {
      tile_bulk = ((rv * G * 2) % 16) == 0;
      if (tile_bulk) total += rv * G * 2;
    }
    if (lane == 0) mbar_arrive_expect_tx(&bars[slot], total);
    __syncwarp();
    if (lane < rv) {
      const uint8_t* src = reinterpret_cast<const uint8_t*>(
                               p.q + static_cast<size_t>(m0 + lane) * row_words) +
                           static_cast<size_t>(g0) * GB;
      bulk_g2s(base + lane * p.stride, src, cbytes, &bars[slot]);
    }
    if constexpr (G >= 8) {
      const int r = lane - 16;
      if (r >= 0 && r < rv) {
        bulk_g2s(sdst + r * 32, p.scales + static_cast<size_t>(m0 + r) * G + sg0, sbytes,
                 &bars[slot]);
      }
    } else {
      if (tile_bulk) {
        if (lane == 16) {
          bulk_g2s(sdst, p.scales + static_cast<size_t>(m0) * G, rv * G * 2, &bars[slot]);
        }
      } else {
        uint16_t* sd = reinterpret_cast<uint16_t*>(sdst);
        for (int i = lane; i < rv * G; i += 32) sd[i] = p.scales[static_cast<size_t>(m0) * G + i];
      }
    }
    ui += len;
    ++issued;
  };
  for (int s = 0; s < p.NS && ui < u1; ++s) issue(s);

  // ---- rotate the activations (depends on the previous kernel)
  pdl_wait();
  for (int n = 0; n < p.N; ++n) {
    float v[FS::E];
    if (tid < FS::THREADS) {
      load_chunk<__half, FS::E>(p.x + static_cast<size_t>(n) * K + tid * FS::E, v);
      apply_signs<FS::E>(p.signs ? p.signs + tid * FS::E : nullptr, v);
    }
    fwht_block<LOGK, 3>(v, buf);
    for (int qd = tid; qd < K / 4; qd += kWarps * 32) {
      const int S = qd >> 2, tt = qd & 3;
      uint16_t hv[4];
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const PairDesc pd = Pairs<BITS>::get(2 * (S & 7) + (r >> 1));
        const int k = kGroup * (S >> 3) + 32 * tt + ((r & 1) ? pd.c_hi : pd.c_lo);
        hv[r] = __half_as_ushort(__float2half_rn(buf[fwht_pad(k)] * p.inv_sqrt_k));
      }
      uint2 pk;
      pk.x = hv[0] | (static_cast<uint32_t>(hv[1]) << 16);
      pk.y = hv[2] | (static_cast<uint32_t>(hv[3]) << 16);
      *reinterpret_cast<uint2*>(xs + ((static_cast<size_t>(S) * p.N + n) * 4 + tt) * 4) = pk;
    }
    __syncthreads();
  }

  // ---- consumer: decode + MMA over the warp's units
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  int tile_start = -1;
  int consumed = 0;
  bool ok = true;
  const bool has_b = g < p.N;
  const int xs_step = p.N * 16;
  uint32_t uc = u0;
  while (uc < u1) {
    const uint32_t tile = uc / G, g0 = uc % G;
    const uint32_t len = min(static_cast<uint32_t>(p.CH), min(G - g0, u1 - uc));
    const int slot = consumed % p.NS;
    if (!mbar_wait(&bars[slot], (consumed / p.NS) & 1)) {
      ok = false;
      break;
    }
    __syncwarp();
    if (tile_start < 0) tile_start = static_cast<int>(g0);
    const uint8_t* base = ring + slot * p.slot_bytes;
    const __half* sc = reinterpret_cast<const __half*>(base + kRows * p.stride);
    const uint8_t* rowa = base + g * p.stride + t * 4 * BITS;
    const uint8_t* rowb = base + (g + 8) * p.stride + t * 4 * BITS;
    const uint32_t sg0 = (G >= 8) ? (g0 & ~7u) : 0u;
    const int sstride = (G >= 8) ? 16 : G;
#pragma unroll 1
    for (uint32_t j = 0; j < len; ++j) {
      const uint32_t gi = g0 + j;
      uint32_t wa[BITS], wb[BITS];
      load_bundle<BITS>(rowa + j * GB, wa);
      load_bundle<BITS>(rowb + j * GB, wb);
      const float sa = __half2float(sc[g * sstride + (gi - sg0)]);
      const float sb = __half2float(sc[(g + 8) * sstride + (gi - sg0)]);
      uint32_t Pa[16], Pb[16];
      decode16_exact<BITS>(wa, p.add, Pa);
      decode16_exact<BITS>(wb, p.add, Pb);
      float c0[4] = {0.f, 0.f, 0.f, 0.f}, c1[4] = {0.f, 0.f, 0.f, 0.f};
      const uint16_t* xb = xs + (static_cast<size_t>(8 * gi) * p.N + g) * 16 + t * 4;
#pragma unroll
      for (int s = 0; s < 8; ++s) {
        uint32_t b0 = 0u, b1 = 0u;
        if (has_b) {
          const uint2 bb = *reinterpret_cast<const uint2*>(xb + s * xs_step);
          b0 = bb.x;
          b1 = bb.y;
        }
        const uint32_t a[4] = {Pa[2 * s], Pb[2 * s], Pa[2 * s + 1], Pb[2 * s + 1]};
        if (s & 1) {
          mma_16816(c1, a, b0, b1, c1);
        } else {
          mma_16816(c0, a, b0, b1, c0);
        }
      }
      acc[0] = fmaf(sa, c0[0] + c1[0], acc[0]);
      acc[1] = fmaf(sa, c0[1] + c1[1], acc[1]);
      acc[2] = fmaf(sb, c0[2] + c1[2], acc[2]);
      acc[3] = fmaf(sb, c0[3] + c1[3], acc[3]);
    }
    __syncwarp();
    fence_proxy_async_smem();
    if (ui < u1) issue(slot);
    uc += len;
    ++consumed;

    if (g0 + len == G || uc >= u1) {
      // ---- finish this warp's part of the tile
      const int m0 = tile * kRows;
      const int rv = min(kRows, p.M - m0);
      const bool full = tile_start == 0 && g0 + len == G;
      float4 out = make_float4(acc[0], acc[1], acc[2], acc[3]);
      bool store = full;
      if (!full) {
        const int which = (tile == u0 / G) ? 0 : 1;
        p.part[(static_cast<size_t>(gw) * 2 + which) * 32 + lane] = out;
        __threadfence();
        __syncwarp();
        uint32_t old = 0;
        if (lane == 0) old = atomicAdd(&p.cnt[tile], 1u);
        old = __shfl_sync(0xffffffffu, old, 0);
        const uint32_t gwf = unit_owner(tile * G, p.U, p.GW);
        const uint32_t gwl = unit_owner(tile * G + G - 1, p.U, p.GW);
        if (old == gwl - gwf) {
          __threadfence();
          out = make_float4(0.f, 0.f, 0.f, 0.f);
          for (uint32_t c = gwf; c <= gwl; ++c) {
            const int wc = (tile == unit_begin(c, p.U, p.GW) / G) ? 0 : 1;
            const float4 v = __ldcg(&p.part[(static_cast<size_t>(c) * 2 + wc) * 32 + lane]);
            out.x += v.x;
            out.y += v.y;
            out.z += v.z;
            out.w += v.w;
          }
          if (lane == 0) p.cnt[tile] = 0u;
          store = true;
        }
      }
      if (store) {
        const int c0 = 2 * t, c1 = 2 * t + 1;
        if (g < rv) {
          if (c0 < p.N) p.y[static_cast<size_t>(c0) * p.ldy + m0 + g] = out.x;
          if (c1 < p.N) p.y[static_cast<size_t>(c1) * p.ldy + m0 + g] = out.y;
        }
        if (g + 8 < rv) {
          if (c0 < p.N) p.y[static_cast<size_t>(c0) * p.ldy + m0 + g + 8] = out.z;
          if (c1 < p.N) p.y[static_cast<size_t>(c1) * p.ldy + m0 + g + 8] = out.w;
        }
      }
      acc[0] = acc[1] = acc[2] = acc[3] = 0.f;
      tile_start = -1;
    }
  }
  if (!ok) {
    if (lane == 0) record_error(p.status, HQ_DEV_TIMEOUT);
    // Let copies still in flight land before the CTA's shared memory is released.
    for (int k = consumed; k < issued; ++k) (void)mbar_wait(&bars[k % p.NS], (k / p.NS) & 1);
  }
}

// ---------------------------------------------------------------- host planning
struct GemvPlan {
  int CH = 0, NS = 0, stride = 0, slot_bytes = 0, buf_off = 0, ring_off = 0, bar_off = 0;
  size_t smem = 0;
};

constexpr size_t kMaxSmem = 227 * 1024;

static GemvPlan gemv_plan(int bits, int K, int nb) {
  GemvPlan best;
  const int G = K / kGroup;
  const size_t xs = static_cast<size_t>(nb) * K * 2;
  const size_t buf_off = (xs + 127) & ~static_cast<size_t>(127);
  const size_t buf = static_cast<size_t>(K + K / 32) * 4;
  const size_t ring_off = (buf_off + buf + 127) & ~static_cast<size_t>(127);
  for (int CH : {8, 4, 2, 1}) {
    const int ch = std::min(CH, G);
    const int row = ch * 16 * bits;
    const int pad_w = ((bank_target_words(bits) - row / 4) % 32 + 32) % 32;
    const int stride = row + 4 * pad_w;
    const int sbytes = G >= 8 ? kRows * 32 : ((kRows * G * 2 + 15) & ~15);
    const int slot = kRows * stride + sbytes;
    for (int NS : {4, 3, 2}) {
      const size_t bar_off = ring_off + static_cast<size_t>(kWarps) * NS * slot;
      const size_t smem = bar_off + static_cast<size_t>(kWarps) * NS * 8;
      if (smem > kMaxSmem) continue;
      if (static_cast<long>(ch) * NS > static_cast<long>(best.CH) * best.NS) {
        best.CH = ch;
        best.NS = NS;
        best.stride = stride;
        best.slot_bytes = slot;
        best.buf_off = static_cast<int>(buf_off);
        best.ring_off = static_cast<int>(ring_off);
        best.bar_off = static_cast<int>(bar_off);
        best.smem = smem;
      }
      break;  // the largest NS that fits for this CH
    }
  }
  return best;
}

size_t gemv_smem_bytes(int bits, int K, int nb) { return gemv_plan(bits, K, nb).smem; }

int gemv_max_warps() {
  static int sms = 0;
  if (sms == 0) {
    int dev = 0, v = 0;
    if (cudaGetDevice(&dev) == cudaSuccess &&
        cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && v > 0) {
      sms = v;
    } else {
      (void)cudaGetLastError();
      return 148 * kWarps;
    }
  }
  return sms * kWarps;
}

template <int BITS>
static void fill_addends(GemvParams& p, int zero) {
  for (int i = 0; i < 16; ++i) p.add[i] = pair_addend<BITS>(i, zero);
}

template <int BITS>
static cudaError_t gemv_launch_b(int K, GemvParams& p, size_t smem, unsigned grid,
                                 cudaStream_t st) {
  const dim3 g(grid), b(kWarps * 32);
  switch (K) {
    case 128: return launch_pdl(gemv_kernel<BITS, 7>, g, b, smem, st, true, p);
    case 256: return launch_pdl(gemv_kernel<BITS, 8>, g, b, smem, st, true, p);
    case 512: return launch_pdl(gemv_kernel<BITS, 9>, g, b, smem, st, true, p);
    case 1024: return launch_pdl(gemv_kernel<BITS, 10>, g, b, smem, st, true, p);
    case 2048: return launch_pdl(gemv_kernel<BITS, 11>, g, b, smem, st, true, p);
    case 4096: return launch_pdl(gemv_kernel<BITS, 12>, g, b, smem, st, true, p);
    case 8192: return launch_pdl(gemv_kernel<BITS, 13>, g, b, smem, st, true, p);
    case 16384: return launch_pdl(gemv_kernel<BITS, 14>, g, b, smem, st, true, p);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_gemv(const GemvArgs& a, cudaStream_t st) {
  const GemvPlan pl = gemv_plan(a.bits, a.K, a.N);
  if (pl.smem == 0) return cudaErrorInvalidValue;
  const int G = a.K / kGroup;
  const uint32_t n_tiles = static_cast<uint32_t>((a.M + kRows - 1) / kRows);
  const uint32_t U = n_tiles * static_cast<uint32_t>(G);
  const int max_warps = gemv_max_warps();
  const uint32_t grid = std::min<uint32_t>(max_warps / kWarps, (U + kWarps - 1) / kWarps);
  GemvParams p{};
  p.q = a.q;
  p.scales = a.scales;
  p.x = reinterpret_cast<const __half*>(a.x);
  p.signs = a.signs;
  p.y = a.y;
  p.status = a.status;
  p.part = reinterpret_cast<float4*>(a.part);
  p.cnt = a.cnt;
  p.M = a.M;
  p.N = a.N;
  p.ldy = a.ldy;
  p.U = U;
  p.GW = std::min<uint32_t>(grid * kWarps, U);
  p.CH = pl.CH;
  p.NS = pl.NS;
  p.stride = pl.stride;
  p.slot_bytes = pl.slot_bytes;
  p.buf_off = pl.buf_off;
  p.ring_off = pl.ring_off;
  p.bar_off = pl.bar_off;
  p.inv_sqrt_k = static_cast<float>(1.0 / sqrt(static_cast<double>(a.K)));
  switch (a.bits) {
    case 2: fill_addends<2>(p, a.zero); return gemv_launch_b<2>(a.K, p, pl.smem, grid, st);
    case 3: fill_addends<3>(p, a.zero); return gemv_launch_b<3>(a.K, p, pl.smem, grid, st);
    case 4: fill_addends<4>(p, a.zero); return gemv_launch_b<4>(a.K, p, pl.smem, grid, st);
    case 8: fill_addends<8>(p, a.zero); return gemv_launch_b<8>(a.K, p, pl.smem, grid, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace hq
