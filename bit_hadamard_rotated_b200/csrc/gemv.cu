// gemv.cu -- unpack-dequant GEMV over packed low-bit codes, batch <= 8 per
// launch, with the rotation of the activations fused in or in a prep kernel.
//
//   y[n][m] = sum_k scale[m][k/128] (q[m][k] - zero) x'[n][k],
//   x'[n]   = H_K diag(s) x[n] / sqrt(K).
//
// At small batch the cost is set by the weight bytes (decode speed follows the
// bytes streamed: Laguna-S-2.1 gridbook card, "Reading it honestly"), so the
// GEMV is shaped to stream packed codes at HBM rate with all dequantisation
// on chip:
//
//   * The rotation x' = H diag(s) x / sqrt(K) runs in fp32 (fwht.cuh), and x'
//     is written as fp16 in the order of the MMA B fragments, each value
//     scaled by the 2^-a of its code field (hq_layout.cuh) and by a power of
//     two 2^e of its row that puts the row's largest |x'| just below 2^14
//     (so small activations do not fall into fp16's subnormal range; the
//     output is multiplied by 2^(24-e), exactly), plus the zero-point term
//     -zero * sum_k x'_k * 2^(e-24) of each group: for one or
//     two rows of K <= 8192 by every GEMV CTA itself, after its first weight
//     copies are on their way (one launch per call); otherwise by
//     gemv_prep_kernel (one CTA per batch row) before the GEMV.
//   * gemv_kernel: persistent grid, one 16-warp CTA per SM.  The work is the
//     list of (16-row tile, 128-code group) units; each CTA owns a contiguous
//     range of whole tiles and its warps split that range evenly.
//   * Each warp streams its range through a private ring of shared-memory
//     slots of about 4 KiB of codes (CH groups of 16 rows, plus scales),
//     moved by TMA copies issued by lane 0 that complete on one mbarrier per
//     slot (transaction bytes).  The first slots are requested
//     before griddepcontrol.wait: weights do not depend on earlier kernels.
//     Full slots of codes arrive as one 3-D TMA box ([CH groups][16 rows]
//     [16 bits bytes]), a slot's scales as one or two 2-D boxes.
//   * Per group: each lane masks 2 x 32 codes into exact subnormal fp16 pairs
//     (one LOP3/PRMT per pair), runs 8 mma.sync m16n8k16 with fp32
//     accumulation in two chains (one starting at the zero-point term), then
//     acc += (scale * 2^24) * sum.
//   * A tile split between warps of the CTA is summed in warp order through
//     shared memory after one __syncthreads (deterministic); no tile is split
//     between CTAs, so no global exchange is needed.
#include <algorithm>

#include "fwht.cuh"
#include "hq_common.cuh"
#include "hq_internal.h"
#include "hq_io.cuh"
#include "hq_launch.cuh"
#include "hq_layout.cuh"
#include "gemv_frag.cuh"

namespace hq {


struct GemvParams {
  CUtensorMap qmap3;  // codes as [G][M][16 bits bytes]; box CH groups x 16 rows (one slot)
  CUtensorMap smap;  // scales as fp16 [M][K/128]; box 8 x 16 rows (K >= 1024 only)
  CUtensorMap zmap;  // per-group zero points as uint8 [M][K/128]; box 16 x 16 rows (K >= 2048)
  const uint8_t* zeros;  // per-group zero points, or nullptr for the scalar zero
  const uint32_t* q;
  const uint16_t* scales;
  const __half* x;
  const int8_t* signs;
  float* y;
  uint32_t* status;
  int M, N, ldy;
  uint32_t U;       // units = n_tiles * G
  uint32_t tq, tr;  // tiles per CTA: n_tiles = tq * grid + tr
  float zero;  // the zero point (fractional only for the screened readout's high plane)
  int withhold;  // test of the error path: CTA 0's last warp never requests its second chunk
  int planes;    // 2-bit codes in the bit-plane layout
  const uint8_t* xg;  // prep output: x' fragments [N][G][4][64 B] fp16, zq [G][16] fp32, fac [8] fp32
  float inv_sqrt_k;
  int NS, slot_bytes, zc_off, buf_off, ring_off, bar_off;
};

// Batches whose rotation the GEMV CTAs compute themselves (no prep launch):
// a row or two of at most 8192 values, a few microseconds of fp32 work that
// overlaps the first weight copies.
__host__ __device__ constexpr bool gemv_fused_rotation(int K, int nb) { return nb <= 2 && K <= 8192; }


// Groups per ring slot (a "chunk", one 16-row tile): about 4 KiB of codes at
// 2, 3 and 4 bits (8, 4, 4 groups), 2 groups of 8-bit codes; never more than
// the G groups of a row.  Slot-shape sweeps on B200 (batch 1) put slots of
// about 4 KiB at 1.3-2x the rate of many small ones.
__host__ __device__ constexpr int gemv_ch_max(int bits, int G) {
  return (bits == 2 ? 8 : bits == 8 ? 2 : 4) < G ? (bits == 2 ? 8 : bits == 8 ? 2 : 4) : G;
}

// The FWHT a fused GEMV CTA (16 warps) runs on one row: the 512-thread shape
// for K >= 512, else the prep kernel's (at most 8 warps).
template <int LOGK, bool WIDE = (LOGK >= 9)>
struct FusedFwht;
template <int LOGK>
struct FusedFwht<LOGK, true> {
  static constexpr int E = Fwht512<LOGK>::E, THREADS = 512;
  static __device__ __forceinline__ void run(float (&v)[E], float* buf, float* red) {
    fwht_block512<LOGK>(v, buf, red);
  }
};
template <int LOGK>
struct FusedFwht<LOGK, false> {
  static constexpr int E = FwhtShape<LOGK, 3>::E, THREADS = FwhtShape<LOGK, 3>::THREADS;
  static __device__ __forceinline__ void run(float (&v)[E], float* buf, float* red) {
    fwht_block<LOGK, 3>(v, buf, red);
  }
};

// The CH scales of a lane's row for one chunk, as fp16 bit pairs: CH = 8, 4,
// 2, 1 -> one 16-, 8-, 4- or 2-byte shared-memory load.
template <int CH>
struct ScaleVec {
  uint32_t h[(CH + 1) / 2];
  __device__ __forceinline__ void load(const uint8_t* p) {
    if constexpr (CH == 8) {
      const uint4 v = *reinterpret_cast<const uint4*>(p);
      h[0] = v.x; h[1] = v.y; h[2] = v.z; h[3] = v.w;
    } else if constexpr (CH == 4) {
      const uint2 v = *reinterpret_cast<const uint2*>(p);
      h[0] = v.x; h[1] = v.y;
    } else if constexpr (CH == 2) {
      h[0] = *reinterpret_cast<const uint32_t*>(p);
    } else {
      h[0] = *reinterpret_cast<const uint16_t*>(p);
    }
  }
  __device__ __forceinline__ float get(int j) const {
    const uint32_t w = h[j >> 1];
    return __half2float(__ushort_as_half(static_cast<unsigned short>((j & 1) ? (w >> 16) : (w & 0xFFFFu))));
  }
};


// The CH per-group zero points of a lane's row for one chunk (uint8 each):
// one 8-, 4-, 2- or 1-byte shared-memory load.
template <int CH>
struct ZeroVec {
  uint32_t h[(CH + 3) / 4];
  __device__ __forceinline__ void load(const uint8_t* p) {
    if constexpr (CH == 8) {
      const uint2 v = *reinterpret_cast<const uint2*>(p);
      h[0] = v.x; h[1] = v.y;
    } else if constexpr (CH == 4) {
      h[0] = *reinterpret_cast<const uint32_t*>(p);
    } else if constexpr (CH == 2) {
      h[0] = *reinterpret_cast<const uint16_t*>(p);
    } else {
      h[0] = *p;
    }
  }
  __device__ __forceinline__ float get(int j) const {
    return static_cast<float>((h[j >> 2] >> (8 * (j & 3))) & 0xFFu);
  }
};

// The lane's two 32-code bundles (rows g and g + 8) of group j of a slot.
template <int BITS>
__device__ __forceinline__ void load_pair_rows(const uint8_t* ra, int j, int g, int t, uint32_t (&wa)[BITS],
                                               uint32_t (&wb)[BITS]) {
  constexpr int GB = 16 * BITS;
  if constexpr (BITS == 8) {
    const int sw = g & 7;
    const uint4 a0 = *reinterpret_cast<const uint4*>(ra + j * kRows * GB + (((2 * t) ^ sw) << 4));
    const uint4 a1 = *reinterpret_cast<const uint4*>(ra + j * kRows * GB + (((2 * t + 1) ^ sw) << 4));
    const uint4 b0 = *reinterpret_cast<const uint4*>(ra + j * kRows * GB + 8 * GB + (((2 * t) ^ sw) << 4));
    const uint4 b1 = *reinterpret_cast<const uint4*>(ra + j * kRows * GB + 8 * GB + (((2 * t + 1) ^ sw) << 4));
    wa[0] = a0.x; wa[1] = a0.y; wa[2] = a0.z; wa[3] = a0.w;
    wa[4] = a1.x; wa[5] = a1.y; wa[6] = a1.z; wa[7] = a1.w;
    wb[0] = b0.x; wb[1] = b0.y; wb[2] = b0.z; wb[3] = b0.w;
    wb[4] = b1.x; wb[5] = b1.y; wb[6] = b1.z; wb[7] = b1.w;
  } else {
    load_bundle<BITS>(ra + j * kRows * GB, wa);
    load_bundle<BITS>(ra + j * kRows * GB + 8 * GB, wb);
  }
}

// One chunk of a warp: CH groups of one 16-row tile from a full slot.  Per
// group: the lane's two 32-code bundles (rows g, g + 8) decode into 16 + 16
// fp16 pairs, 8 MMAs (m16n8k16) run in one chain started at the group's
// zero-point term, and acc += scale * chain (per row).  Groups are taken two
// at a time with their chains interleaved, so that each MMA's latency is
// covered by the other chain's, and each MMA's four A registers are masked
// out of the code words right before it (measured ~5 % faster than decoding
// a group's 32 registers first).
template <int BITS, int CH, bool PGZ, bool PL = false>
__device__ __forceinline__ void gemv_chunk(const uint8_t* base, const uint8_t* sca, const uint8_t* scb,
                                           const uint8_t* zra, const uint8_t* zrb, const float4* zq4,
                                           const uint8_t* const (&xb)[4], int g, int t, float (&acc)[4]) {
  constexpr int JP = CH >= 2 ? 2 : 1;  // groups in flight
  ScaleVec<CH> sva, svb;
  sva.load(sca);
  svb.load(scb);
  ZeroVec<CH> zva, zvb;
  if constexpr (PGZ) {
    zva.load(zra);
    zvb.load(zrb);
  }
  // row g of group j at base + j 16 GB + g GB (row g + 8 at + 8 GB); lane t
  // owns bytes [4 t BITS, 4 (t + 1) BITS) of the row (8-bit: 16-byte chunks
  // 2t, 2t + 1 in the 128-byte swizzle, XOR row % 8)
  const uint8_t* ra = base + g * (16 * BITS) + (BITS == 8 ? 0 : t * 4 * BITS);
#pragma unroll
  for (int j0 = 0; j0 < CH; j0 += JP) {
    uint32_t wa[JP][BITS], wb[JP][BITS];
    uint4 bq[JP][4];
    float c[JP][4];
#pragma unroll
    for (int q = 0; q < JP; ++q) {
      load_pair_rows<BITS>(ra, j0 + q, g, t, wa[q], wb[q]);
      if constexpr (PL) {
        plane_bundle(wa[q]);
        plane_bundle(wb[q]);
      }
      const float4 z = zq4[(j0 + q) * 4];
      if constexpr (PGZ) {
        // the group's zero-point term of each row: its zero times -sum x'
        const float za = zva.get(j0 + q), zb = zvb.get(j0 + q);
        c[q][0] = za * z.x;
        c[q][1] = za * z.y;
        c[q][2] = zb * z.z;
        c[q][3] = zb * z.w;
      } else {
        c[q][0] = z.x;
        c[q][1] = z.y;
        c[q][2] = z.z;
        c[q][3] = z.w;
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) bq[q][i] = *reinterpret_cast<const uint4*>(xb[i] + (j0 + q) * kXsGroup);
    }
    DecodeViews<BITS> Va[JP], Vb[JP];
#pragma unroll
    for (int q = 0; q < JP; ++q) {
      Va[q].init(wa[q]);
      Vb[q].init(wb[q]);
    }
#pragma unroll
    for (int s = 0; s < 8; ++s) {
#pragma unroll
      for (int q = 0; q < JP; ++q) {
        const uint32_t b0 = (s & 1) ? bq[q][s >> 1].z : bq[q][s >> 1].x;
        const uint32_t b1 = (s & 1) ? bq[q][s >> 1].w : bq[q][s >> 1].y;
        const uint32_t a[4] = {Va[q].pair(2 * s), Vb[q].pair(2 * s), Va[q].pair(2 * s + 1), Vb[q].pair(2 * s + 1)};
        mma_16816_acc(c[q], a, b0, b1);
      }
    }
#pragma unroll
    for (int q = 0; q < JP; ++q) {
      const float sa = sva.get(j0 + q), sb = svb.get(j0 + q);
      acc[0] = fmaf(sa, c[q][0], acc[0]);
      acc[1] = fmaf(sa, c[q][1], acc[1]);
      acc[2] = fmaf(sb, c[q][2], acc[2]);
      acc[3] = fmaf(sb, c[q][3], acc[3]);
    }
  }
}

template <int BITS, int LOGK, bool FUSED, int CH>
__global__ void __launch_bounds__(kWarps * 32, 1) gemv_kernel(const __grid_constant__ GemvParams p) {
  constexpr int K = 1 << LOGK;
  constexpr int G = K / kGroup;
  constexpr int GB = 16 * BITS;  // bytes of one group of one row
  static_assert(G % CH == 0 && (G < 8 || 8 % CH == 0), "chunks tile the row and an 8-group scale block");
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // TMA boxes in the 128-byte swizzle need 1 KiB-aligned slots: round the
  // base up (the launch asks for 1 KiB more than the plan)
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, t = lane & 3;
  // the CTA owns whole tiles, units [cb, ce): the first tr CTAs tq + 1
  // tiles, the others tq; its warps split them into contiguous ranges of
  // whole chunks (a tile is never shared with another CTA: a cross-CTA sum
  // would put global memory round trips at the end of every CTA)
  const uint32_t c = blockIdx.x;
  const uint32_t cb = (c * p.tq + min(c, p.tr)) * G;
  const uint32_t ce = cb + (p.tq + (c < p.tr ? 1u : 0u)) * G;
  const uint32_t nch = (ce - cb) / CH;  // chunks of the CTA
  auto wbeg = [&](uint32_t w) { return cb + static_cast<uint32_t>((static_cast<uint64_t>(w) * nch) / kWarps) * CH; };
  const uint32_t u0 = wbeg(warp);
  const uint32_t u1 = wbeg(warp + 1);

  uint16_t* xs = reinterpret_cast<uint16_t*>(smem);
  float* zq = reinterpret_cast<float*>(smem + p.zc_off);
  float* fac = zq + G * 16;  // per-column output factors 2^(24 - e)
  // the rings are slot-major: slot s of warp w at (s kWarps + w) slot_bytes,
  // so the last slot of every warp forms one block (the fused rotation's
  // FWHT buffer until that slot is first filled)
  const int ring_stride = kWarps * p.slot_bytes;
  uint8_t* ring = smem + p.ring_off + warp * p.slot_bytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + p.bar_off) + warp * p.NS;
  // slot: [CH groups][16 rows][16 bits bytes] codes (one TMA box; 8-bit rows
  // in the 128-byte swizzle), then the scales: K >= 1024: the tile's [16 rows]
  // [8 halves] of the aligned block of 8 groups holding the chunk; K < 1024:
  // the tile's [16 rows][G halves]; then, with per-group zero points, the
  // zeros: K >= 2048: the tile's [16 rows][16 bytes] of the aligned block of
  // 16 groups holding the chunk; K < 2048: the tile's [16 rows][G bytes]
  constexpr int sc_off = CH * kRows * GB;
  constexpr int z_off = sc_off + (G >= 8 ? kRows * 16 : ((kRows * G * 2 + 15) & ~15));
  const bool pgz = p.zeros != nullptr;
  const bool planes = p.planes != 0;

  if (tid == 0) {
    prefetch_tensormap(&p.qmap3);
    if constexpr (G >= 8) prefetch_tensormap(&p.smap);
    if constexpr (G >= 16) {
      if (pgz) prefetch_tensormap(&p.zmap);
    }
  }
  if (lane == 0) {
    for (int i = 0; i < p.NS; ++i) mbar_init(&bars[i], 1);
    fence_mbar_init();
  }
  __syncthreads();
  pdl_launch_dependents();

  // ---- producer side of the warp's ring (lane 0): a chunk is one 3-D TMA
  // box of codes plus one box (or span) of scales, all completing on the
  // slot's barrier (rows past M read as zero)
  uint32_t ui = u0;
  int issued = 0;
  // a chunk whose copy was never requested (hq_set_test_fault): its wait runs
  // out and is not drained
  const int withheld = (p.withhold && blockIdx.x == 0 && warp == kWarps - 1) ? 1 : -1;
  auto issue = [&](int slot) {
    const uint32_t tile = ui / G, g0 = ui % G;
    const int m0 = tile * kRows;
    uint8_t* base = ring + slot * ring_stride;
    if (lane == 0 && issued != withheld) {
      // bytes the slot's barrier expects; plain-copied remainders are written
      // before the arrival, which releases them to the consumers
      uint32_t bytes = CH * kRows * GB;
      int s_bulk = 0, z_bulk = 0;
      const uint8_t* s_src = reinterpret_cast<const uint8_t*>(p.scales) + static_cast<size_t>(m0) * G * 2;
      const uint8_t* z_src = pgz ? p.zeros + static_cast<size_t>(m0) * G : nullptr;
      if constexpr (G >= 8) {
        bytes += kRows * 16;
      } else {
        // the tile's scales are one contiguous span; bulk-copy its 16-byte
        // multiple, plain-copy the rest (only a last, partial tile has one)
        const int span = min(kRows, p.M - m0) * G * 2;
        s_bulk = span & ~15;
        bytes += s_bulk;
        for (int i = s_bulk; i < span; i += 2) {
          *reinterpret_cast<uint16_t*>(base + sc_off + i) = *reinterpret_cast<const uint16_t*>(s_src + i);
        }
      }
      if (pgz) {
        if constexpr (G >= 16) {
          bytes += kRows * 16;
        } else {
          const int span = min(kRows, p.M - m0) * G;
          z_bulk = span & ~15;
          bytes += z_bulk;
          for (int i = z_bulk; i < span; ++i) base[z_off + i] = z_src[i];
        }
      }
      mbar_arrive_expect_tx(&bars[slot], bytes);
      if constexpr (G >= 8) {
        tma_load_2d(base + sc_off, &p.smap, static_cast<int>(g0 & ~7u), m0, &bars[slot]);
      } else {
        if (s_bulk > 0) bulk_g2s(base + sc_off, s_src, s_bulk, &bars[slot]);
      }
      if (pgz) {
        if constexpr (G >= 16) {
          tma_load_2d(base + z_off, &p.zmap, static_cast<int>(g0 & ~15u), m0, &bars[slot]);
        } else {
          if (z_bulk > 0) bulk_g2s(base + z_off, z_src, z_bulk, &bars[slot]);
        }
      }
      tma_load_3d(base, &p.qmap3, 0, m0, static_cast<int>(g0), &bars[slot]);
    }
    ui += CH;
    ++issued;
  };
  // all slots now, or (fused rotation) all but the last, whose memory the
  // rotation uses first
  for (int s = 0; s < (FUSED ? p.NS - 1 : p.NS) && ui < u1; ++s) issue(s);

  // ---- the rotated activations and zero-point terms
  if constexpr (FUSED) {
    // rotate each row here while the first slots are in flight (all 16 warps
    // for K >= 512); the signs are weights, read before the wait
    using FS = FusedFwht<LOGK>;
    static_assert(FS::E <= 32, "one sign bit per register");
    // bit e: value e of this thread's chunk flips sign
    const SignMask<FS::E> neg =
        tid < FS::THREADS ? sign_bits<FS::E>(p.signs ? p.signs + tid * FS::E : nullptr) : 0u;
    float* buf = reinterpret_cast<float*>(smem + p.ring_off + (p.NS - 1) * ring_stride);
    const FragLane<BITS> fl(lane, p.planes != 0);
    zq_clear_absent(zq, G, p.N, tid, kWarps * 32);
    float* red = fac + 8;
    pdl_wait();
    for (int n = 0; n < p.N; ++n) {
      float v[FS::E];
      if (tid < FS::THREADS) {
        load_chunk<__half, FS::E>(p.x + static_cast<size_t>(n) * K + tid * FS::E, v);
        flip_signs<FS::E>(neg, v);
      }
      FS::run(v, buf, red);
      const int e = row_scale_exp(red_max(red, FS::THREADS / 32) * p.inv_sqrt_k);
      if (tid == 0) fac[n] = pow2f(24 - e);
      const float sc = p.inv_sqrt_k * pow2f(e);
      put_groups<BITS, (G + kWarps - 1) / kWarps>(fl, buf, warp, kWarps, n, G, sc, pgz ? 1.f : p.zero, xs, zq,
                                                  lane);
      // buf becomes a TMA destination after the loop: order this thread's
      // accesses to it before that copy (generic -> async proxy)
      fence_proxy_async_smem();
      __syncthreads();  // buf and red are reused by the next row; xs, zq, fac are complete
    }
    if (ui < u1) issue(p.NS - 1);  // the FWHT buffer is free: the warp's last slot

  } else {
    // from the prep kernel
    pdl_wait();
    const int xs_bytes = static_cast<int>(gemv_xs_bytes(G, p.N));
    for (int i = tid * 16; i < xs_bytes; i += kWarps * 32 * 16) {
      cp_async16(smem + i, p.xg + i, 16);
    }
    for (int i = tid * 16; i < G * 16 * 4; i += kWarps * 32 * 16) {
      cp_async16(smem + p.zc_off + i, p.xg + xs_bytes + i, 16);
    }
    if (tid < 2) cp_async16(fac + 4 * tid, p.xg + xs_bytes + G * 16 * 4 + 16 * tid, 16);
    asm volatile("cp.async.wait_all;" ::: "memory");
    __syncthreads();
  }

  // ---- consumer: decode + MMA over the warp's chunks
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  // Tiles this warp covers only in part: its first (0) and last (1), with
  // their partial sums (scaled to the output), kept in registers until the
  // loop ends and then left in the warp's own (by then idle) ring memory.
  int ptile0 = -1, ptile1 = -1;
  float4 psum0 = make_float4(0.f, 0.f, 0.f, 0.f), psum1 = psum0;
  int tile_start = -1;
  int consumed = 0;
  bool ok = true;
  const int N = p.N, M = p.M, ldy = p.ldy, NS = p.NS;
  const bool n0 = 2 * t < N, n1 = 2 * t + 1 < N;
  // lane's B-fragment stream: its column's blocks; lanes of absent columns
  // read column 0's (their output columns of the MMA are never stored, and a
  // column of the product depends on that column of B alone)
  const uint8_t* xs_lane = reinterpret_cast<const uint8_t*>(xs) + (g < N ? g : 0) * gemv_xs_col(G) + t * kXsBlock;
  const int rot[4] = {(t & 3) << 4, ((t + 1) & 3) << 4, ((t + 2) & 3) << 4, ((t + 3) & 3) << 4};
  const float4* zq_lane = reinterpret_cast<const float4*>(zq) + t;  // + 4 per group
  const uint32_t first_tile = u0 / G;
  // output factors of the lane's columns 2t, 2t + 1 (unused where absent)
  const float f0 = fac[2 * t], f1 = fac[2 * t + 1];
  uint32_t uc = u0;

  auto store_tile = [&](uint32_t tile, const float4& o) {
    const int m0 = tile * kRows;
    const int rv = min(kRows, M - m0);
    if (g < rv) {
      if (n0) p.y[static_cast<size_t>(2 * t) * ldy + m0 + g] = o.x;
      if (n1) p.y[static_cast<size_t>(2 * t + 1) * ldy + m0 + g] = o.y;
    }
    if (g + 8 < rv) {
      if (n0) p.y[static_cast<size_t>(2 * t) * ldy + m0 + g + 8] = o.z;
      if (n1) p.y[static_cast<size_t>(2 * t + 1) * ldy + m0 + g + 8] = o.w;
    }
  };
  int slot = 0;
  uint32_t sph = 0;  // phase parity of the current ring round
  while (uc < u1) {
    const uint32_t tile = uc / G, g0 = uc % G;
    if (!mbar_wait(&bars[slot], sph)) {
      ok = false;
      break;
    }
    __syncwarp();
    if (tile_start < 0) tile_start = static_cast<int>(g0);
    const uint8_t* base = ring + slot * ring_stride;
    const uint8_t* sc = base + sc_off;
    const uint8_t* sca;
    const uint8_t* scb;
    if constexpr (G >= 8) {
      sca = sc + g * 16 + (g0 & 7u) * 2;
      scb = sc + (g + 8) * 16 + (g0 & 7u) * 2;
    } else {
      sca = sc + g * G * 2 + g0 * 2;
      scb = sc + (g + 8) * G * 2 + g0 * 2;
    }
    const uint8_t* const xb[4] = {xs_lane + g0 * kXsGroup + rot[0], xs_lane + g0 * kXsGroup + rot[1],
                                  xs_lane + g0 * kXsGroup + rot[2], xs_lane + g0 * kXsGroup + rot[3]};
    if (pgz) {
      const uint8_t* zr = base + z_off;
      const uint8_t* zra = G >= 16 ? zr + g * 16 + (g0 & 15u) : zr + g * G + g0;
      const uint8_t* zrb = G >= 16 ? zr + (g + 8) * 16 + (g0 & 15u) : zr + (g + 8) * G + g0;
      if (BITS == 2 && planes) {
        gemv_chunk<BITS, CH, true, BITS == 2>(base, sca, scb, zra, zrb, zq_lane + g0 * 4, xb, g, t, acc);
      } else {
        gemv_chunk<BITS, CH, true>(base, sca, scb, zra, zrb, zq_lane + g0 * 4, xb, g, t, acc);
      }
    } else if (BITS == 2 && planes) {
      gemv_chunk<BITS, CH, false, BITS == 2>(base, sca, scb, nullptr, nullptr, zq_lane + g0 * 4, xb, g, t, acc);
    } else {
      gemv_chunk<BITS, CH, false>(base, sca, scb, nullptr, nullptr, zq_lane + g0 * 4, xb, g, t, acc);
    }
    __syncwarp();
    if (ui < u1) issue(slot);
    uc += CH;
    ++consumed;
    if (++slot == NS) {
      slot = 0;
      sph ^= 1u;
    }

    if (g0 + CH == G || uc >= u1) {
      // ---- this warp's part of the tile is done
      const bool full = tile_start == 0 && g0 + CH == G;
      const float4 o = make_float4(acc[0] * f0, acc[1] * f1, acc[2] * f0, acc[3] * f1);
      if (full) {
        store_tile(tile, o);
      } else {
        if (tile == first_tile) {
          ptile0 = static_cast<int>(tile);
          psum0 = o;
        } else {
          ptile1 = static_cast<int>(tile);
          psum1 = o;
        }
      }
      acc[0] = acc[1] = acc[2] = acc[3] = 0.f;
      tile_start = -1;
    }
  }
  // ---- tiles split between warps: the first contributing warp adds the
  // CTA's partials in warp order (shared memory) and stores the tile.
  // Partial sums: the first 512 bytes of the warp's slots 0 and 1 (a slot is
  // at least 640 bytes; the warp's copies have all been consumed).
  auto sp_slot = [&](uint32_t w, int which) {
    return reinterpret_cast<float4*>(smem + p.ring_off + which * ring_stride + w * p.slot_bytes) + lane;
  };
  if (ok) {
    *sp_slot(warp, 0) = psum0;
    *sp_slot(warp, 1) = psum1;
  }
  __syncthreads();
  if (ok) {
#pragma unroll
    for (int which = 0; which < 2; ++which) {
      const int tl = which == 0 ? ptile0 : ptile1;
      if (tl < 0 || (which == 1 && tl == ptile0)) continue;
      const uint32_t tile = static_cast<uint32_t>(tl);
      const uint32_t tf = tile * G, tz = tile * G + G - 1;
      // the ranges are contiguous: the warp whose range holds the tile's
      // first unit adds; the later contributors are the next non-empty
      // warps whose ranges start inside the tile (the tile is their first)
      if (tf < u0) continue;
      float4 o = which == 0 ? psum0 : psum1;
      for (uint32_t w = warp + 1; w < static_cast<uint32_t>(kWarps); ++w) {
        const uint32_t wb = wbeg(w);
        if (wb > tz) break;
        if (wb == wbeg(w + 1)) continue;  // empty range
        const float4 q4 = *sp_slot(w, 0);
        o.x += q4.x;
        o.y += q4.y;
        o.z += q4.z;
        o.w += q4.w;
      }
      store_tile(tile, o);
    }
  }
  if (!ok) {
    if (lane == 0) record_error(p.status, HQ_DEV_TIMEOUT);
    // Let copies still in flight land before the CTA's shared memory is released.
    for (int k = consumed; k < issued; ++k) {
      if (k != withheld) (void)mbar_wait(&bars[k % p.NS], (k / p.NS) & 1);
    }
  }
}

// ---------------------------------------------------------------- host planning
struct GemvPlan {
  int CH = 0, NS = 0, slot_bytes = 0, zc_off = 0, buf_off = 0, ring_off = 0, bar_off = 0;
  size_t smem = 0;
};

// One 16-warp CTA per SM (its registers fill the SM), up to all of the
// shared memory.
constexpr size_t kMaxSmem = 227 * 1024;
constexpr int kMaxNS = 4;

static GemvPlan gemv_plan_shape(int bits, int K, int nb, int ch, int ns, bool pgz, size_t budget) {
  GemvPlan pl;
  const int G = K / kGroup;
  const size_t xs = gemv_xs_bytes(G, nb);
  const size_t zc_off = (xs + 15) & ~static_cast<size_t>(15);
  // ring on a 1 KiB boundary; slots on 1 KiB (8-bit: the 128-byte swizzle
  // atom) or 128-byte boundaries (TMA destinations)
  const size_t ring_off = (zc_off + gemv_zq_bytes(G) + kZcTail + 1023) & ~static_cast<size_t>(1023);
  const int sc_bytes = G >= 8 ? kRows * 16 : ((kRows * G * 2 + 15) & ~15);
  const int z_bytes = pgz ? (G >= 16 ? kRows * 16 : kRows * G) : 0;
  const int align = bits == 8 ? 1024 : 128;
  const int slot = (ch * kRows * 16 * bits + sc_bytes + z_bytes + align - 1) & ~(align - 1);
  // a fused rotation's FWHT buffer (K floats + one pad word per 32) is the
  // last slot of every warp, before that slot is first filled
  if (gemv_fused_rotation(K, nb) &&
      static_cast<size_t>(kWarps) * slot < (static_cast<size_t>(K) + K / 32) * 4 + 16 * 4) {
    return pl;
  }
  const size_t buf_off = ring_off + static_cast<size_t>(kWarps) * (ns - 1) * slot;
  const size_t bar_off = ring_off + static_cast<size_t>(kWarps) * ns * slot;
  // + 1 KiB: the kernel rounds the shared-memory base up to 1 KiB
  const size_t smem = bar_off + static_cast<size_t>(kWarps) * ns * 8 + 1024;
  if (smem > budget) return pl;
  pl.CH = ch;
  pl.NS = ns;
  pl.slot_bytes = slot;
  pl.zc_off = static_cast<int>(zc_off);
  pl.buf_off = static_cast<int>(buf_off);
  pl.ring_off = static_cast<int>(ring_off);
  pl.bar_off = static_cast<int>(bar_off);
  pl.smem = smem;
  return pl;
}

// Chunk lengths the kernels are built for: the full one (gemv_ch_max) and
// half of it; the deepest ring (2 to 4 slots a warp) of the longer chunk that
// fits, else of the shorter one.
static GemvPlan gemv_plan(int bits, int K, int nb, bool pgz) {
  const int G = K / kGroup;
  const int chf = gemv_ch_max(bits, G);
  for (int ch : {chf, chf > 1 ? chf / 2 : 0}) {
    if (ch == 0) break;
    for (int ns = kMaxNS; ns >= 2; --ns) {
      const GemvPlan pl = gemv_plan_shape(bits, K, nb, ch, ns, pgz, kMaxSmem);
      if (pl.smem != 0) return pl;
    }
  }
  return GemvPlan{};
}

size_t gemv_smem_bytes(int bits, int K, int nb, bool pgz) { return gemv_plan(bits, K, nb, pgz).smem; }

int sm_count() {
  static int sms = 0;
  if (sms == 0) {
    int dev = 0, v = 0;
    if (cudaGetDevice(&dev) == cudaSuccess &&
        cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && v > 0) {
      sms = v;
    } else {
      (void)cudaGetLastError();
      return 148;
    }
  }
  return sms;
}

template <int BITS, int LOGK, bool FUSED>
static cudaError_t gemv_launch_ch(int ch, GemvParams& p, size_t smem, unsigned grid, cudaStream_t st) {
  constexpr int CHF = gemv_ch_max(BITS, (1 << LOGK) / kGroup);
  const dim3 g(grid), b(kWarps * 32);
  if (ch == CHF) return launch_pdl(gemv_kernel<BITS, LOGK, FUSED, CHF>, g, b, smem, st, true, p);
  if constexpr (CHF > 1) {
    if (ch == CHF / 2) return launch_pdl(gemv_kernel<BITS, LOGK, FUSED, CHF / 2>, g, b, smem, st, true, p);
  }
  return cudaErrorInvalidValue;
}

template <int BITS, bool FUSED>
static cudaError_t gemv_launch_f(int K, int ch, GemvParams& p, size_t smem, unsigned grid,
                                 cudaStream_t st) {
  switch (K) {
    case 128: return gemv_launch_ch<BITS, 7, FUSED>(ch, p, smem, grid, st);
    case 256: return gemv_launch_ch<BITS, 8, FUSED>(ch, p, smem, grid, st);
    case 512: return gemv_launch_ch<BITS, 9, FUSED>(ch, p, smem, grid, st);
    case 1024: return gemv_launch_ch<BITS, 10, FUSED>(ch, p, smem, grid, st);
    case 2048: return gemv_launch_ch<BITS, 11, FUSED>(ch, p, smem, grid, st);
    case 4096: return gemv_launch_ch<BITS, 12, FUSED>(ch, p, smem, grid, st);
    case 8192: return gemv_launch_ch<BITS, 13, FUSED>(ch, p, smem, grid, st);
    default:
      if constexpr (!FUSED) {
        if (K == 16384) return gemv_launch_ch<BITS, 14, false>(ch, p, smem, grid, st);
        if (K == 32768) return gemv_launch_ch<BITS, 15, false>(ch, p, smem, grid, st);
      }
      return cudaErrorInvalidValue;
  }
}

template <int BITS>
static cudaError_t gemv_launch_b(int K, int nb, int ch, GemvParams& p, size_t smem, unsigned grid,
                                 cudaStream_t st) {
  return gemv_fused_rotation(K, nb) ? gemv_launch_f<BITS, true>(K, ch, p, smem, grid, st)
                                    : gemv_launch_f<BITS, false>(K, ch, p, smem, grid, st);
}

int gemv_launches(int K, int nb) { return gemv_fused_rotation(K, nb) ? 1 : 2; }

size_t gemv_scratch_bytes(int K, int nb) { return gemv_xg_bytes(K / kGroup, nb); }

// The zero point the kernels apply: the integer one, or a fractional override.
static float gemv_zero(const GemvArgs& a) { return a.zero_frac ? a.zero_f : static_cast<float>(a.zero); }

template <int BITS>
static cudaError_t gemv_prep_b(int K, const GemvArgs& a, cudaStream_t st) {
  const dim3 g(a.N);
  const float inv = static_cast<float>(1.0 / sqrt(static_cast<double>(K)));
  const __half* x = reinterpret_cast<const __half*>(a.x);
  uint8_t* xg = static_cast<uint8_t*>(a.xg);
#define HQ_PREP(LK)                                                                          \
  launch_pdl(gemv_prep_kernel<BITS, LK>, g, dim3(prep_warps(LK) * 32),                         \
             (FwhtShape<LK, prep_logw(LK)>::SMEM_FLOATS + 32) * sizeof(float), st, true, x, a.signs, \
             xg, a.N, a.zeros != nullptr ? 1.f : gemv_zero(a), inv, a.planes ? 1 : 0)
  switch (K) {
    case 128: return HQ_PREP(7);
    case 256: return HQ_PREP(8);
    case 512: return HQ_PREP(9);
    case 1024: return HQ_PREP(10);
    case 2048: return HQ_PREP(11);
    case 4096: return HQ_PREP(12);
    case 8192: return HQ_PREP(13);
    case 16384: return HQ_PREP(14);
    case 32768: return HQ_PREP(15);
    default: return cudaErrorInvalidValue;
  }
#undef HQ_PREP
}

cudaError_t launch_gemv(const GemvArgs& a, cudaStream_t st) {
  const GemvPlan pl = gemv_plan(a.bits, a.K, a.N, a.zeros != nullptr);
  if (pl.smem == 0) return cudaErrorInvalidValue;
  const bool fused = gemv_fused_rotation(a.K, a.N);
  cudaError_t e = cudaSuccess;
  if (!fused) {
    switch (a.bits) {
      case 2: e = gemv_prep_b<2>(a.K, a, st); break;
      case 3: e = gemv_prep_b<3>(a.K, a, st); break;
      case 4: e = gemv_prep_b<4>(a.K, a, st); break;
      case 8: e = gemv_prep_b<8>(a.K, a, st); break;
      default: return cudaErrorInvalidValue;
    }
    if (e != cudaSuccess) return e;
  }
  const int G = a.K / kGroup;
  const uint32_t n_tiles = static_cast<uint32_t>((a.M + kRows - 1) / kRows);
  GemvParams p{};
  const uint64_t row_bytes = static_cast<uint64_t>(a.K) * a.bits / 8;
  {
    // the codes viewed as [G][M][16 bits] bytes (group stride 16 bits bytes):
    // one box = a full slot of CH groups x 16 rows, laid out [CH][16][16 bits]
    // (8-bit rows are 128 bytes: 128-byte swizzle for conflict-free reads)
    const uint64_t gb = 16ull * a.bits;
    const uint64_t dims[3] = {gb, static_cast<uint64_t>(a.M), static_cast<uint64_t>(G)};
    const uint64_t strides[2] = {row_bytes, gb};
    const uint32_t box[3] = {static_cast<uint32_t>(gb), static_cast<uint32_t>(kRows),
                             static_cast<uint32_t>(pl.CH)};
    e = tensor_map_3d(&p.qmap3, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.q, dims, strides, box,
                      a.bits == 8 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE);
    if (e != cudaSuccess) return e;
  }
  if (a.zeros != nullptr && G >= 16) {  // zeros [M][G] uint8, one box = 16 groups x 16 rows
    e = tensor_map_2d(&p.zmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.zeros, static_cast<uint64_t>(G),
                      static_cast<uint64_t>(a.M), static_cast<uint64_t>(G), 16, kRows,
                      CU_TENSOR_MAP_SWIZZLE_NONE);
    if (e != cudaSuccess) return e;
  }
  if (G >= 8) {  // scales [M][G] fp16, one box = 8 groups x 16 rows
    e = tensor_map_2d(&p.smap, CU_TENSOR_MAP_DATA_TYPE_UINT16, a.scales, static_cast<uint64_t>(G),
                      static_cast<uint64_t>(a.M), static_cast<uint64_t>(G) * 2, 8, kRows,
                      CU_TENSOR_MAP_SWIZZLE_NONE);
    if (e != cudaSuccess) return e;
  }
  const uint32_t U = n_tiles * static_cast<uint32_t>(G);
  // one CTA per SM, each owning whole tiles (at least one)
  const uint32_t grid = std::min<uint32_t>(static_cast<uint32_t>(sm_count()), n_tiles);
  p.q = a.q;
  p.scales = a.scales;
  p.x = reinterpret_cast<const __half*>(a.x);
  p.signs = a.signs;
  p.y = a.y;
  p.status = a.status;
  p.M = a.M;
  p.N = a.N;
  p.ldy = a.ldy;
  p.U = U;
  p.tq = n_tiles / grid;
  p.tr = n_tiles % grid;
  p.NS = pl.NS;
  p.slot_bytes = pl.slot_bytes;
  p.zc_off = pl.zc_off;
  p.buf_off = pl.buf_off;
  p.inv_sqrt_k = static_cast<float>(1.0 / sqrt(static_cast<double>(a.K)));
  p.xg = static_cast<const uint8_t*>(a.xg);
  p.zero = gemv_zero(a);
  p.zeros = a.zeros;
  p.planes = a.planes ? 1 : 0;
  p.withhold = take_test_fault() ? 1 : 0;
  p.ring_off = pl.ring_off;
  p.bar_off = pl.bar_off;
  switch (a.bits) {
    case 2: return gemv_launch_b<2>(a.K, a.N, pl.CH, p, pl.smem, grid, st);
    case 3: return gemv_launch_b<3>(a.K, a.N, pl.CH, p, pl.smem, grid, st);
    case 4: return gemv_launch_b<4>(a.K, a.N, pl.CH, p, pl.smem, grid, st);
    case 8: return gemv_launch_b<8>(a.K, a.N, pl.CH, p, pl.smem, grid, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace hq
