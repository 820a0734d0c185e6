// gemv32.cu -- unpack-dequant GEMV over 32-row tiles for batches of up to 16
// columns (two 8-column MMA blocks), the rotated activations staged in shared
// memory one K slice at a time.
//
//   y[n][m] = sum_k scale[m][k/128] (q[m][k] - zero) x'[n][k],
//   x'[n]   = H_K diag(s) x[n] / sqrt(K)     (gemv_prep_kernel, gemv_frag.cuh)
//
// Between batch 8 and 16 the path is still bound by the weight stream and the
// decode, not by a dense contraction: a group's 2 x 32 codes per lane are
// masked into fp16 A fragments once (hq_layout.cuh) and feed one m16n8k16 MMA
// per 8-column block, so the decode is shared by all columns.  What changes
// against the batch-8 GEMV (gemv.cu) is where the activations live:
//
//   * x' of 16 columns is 2 K x 16 bytes (256 KB at K = 8192), more than a
//     CTA's shared memory.  Each CTA therefore walks K in S slices of GS
//     groups: slice s holds the B fragments of groups [s GS, (s + 1) GS) of
//     every column plus the scales of the CTA's tiles for those groups, two
//     slice buffers are resident, and the buffer of slice s is refilled with
//     slice s + 2 by the last warp to finish slice s (a shared-memory arrival
//     count; no warp waits for another except through the buffers).
//   * Tiles are 32 rows (two m16 tiles) so each B fragment loaded from shared
//     memory feeds two MMAs; 16 columns' B fragments are 4x the code bytes,
//     and this halves that shared-memory traffic per code.
//   * The CTA owns a contiguous range of whole tiles.  In every slice its
//     (tile, group) units are split between the 16 warps in the same
//     contiguous ranges, so a warp meets the same (at most two) tiles in every
//     slice and keeps their sums in registers across slices; tiles split
//     between warps are added in warp order through shared memory at the end
//     (deterministic, no atomics on data).
//   * Each warp streams its units (one group of one tile: 32 rows x 16 bits
//     bytes) through a private ring of TMA slots, issued ahead across slice
//     boundaries; weights do not depend on earlier kernels, so the first
//     slots are requested before griddepcontrol.wait.
//   * For K <= 8192 and at least as many CTAs as batch rows, the batch is
//     rotated inside the launch: CTA n < N rotates row n (the GEMV's 512-thread
//     FWHT and fragment writer, gemv_frag.cuh) into the workspace and counts
//     it on a counter there; every CTA waits (bounded) until all N rows are
//     in, and the last CTA past that gate puts the counter words back to zero.
//     All CTAs are resident at once (one per SM, grid <= SMs).  Otherwise
//     gemv_prep_kernel runs first.
//
// Every wait is bounded (hq_common.cuh); a CTA that gives up records
// HQ_DEV_TIMEOUT, lets its copies in flight land and stores nothing.
#include <algorithm>

#include "gemv_frag.cuh"
#include "hq_launch.cuh"

namespace hq {

constexpr int kTRows = 32;           // rows of a tile: two m16 MMA tiles
constexpr int kMaxTilesPerCta = 16;  // so that a warp's range of a slice spans at most two tiles

struct G32Params {
  CUtensorMap qmap;  // codes as [G][M][16 bits bytes]; box 1 group x 32 rows (one slot)
  CUtensorMap smap;  // scales fp16 [M][G]; box GS groups x 32 rows
  const uint8_t* xg;  // prep output: fragments [N][xs col], zq [G][NB][16] fp32, fac [8 NB] fp32
  float* y;
  uint32_t* status;
  int M, N, ldy, G;
  uint32_t tq, tr;  // tiles per CTA: tq, one more for the first tr CTAs
  int S, GS;        // K slices and groups per slice
  int NS;           // ring slots per warp
  int slot_bytes;   // 32 rows x 16 bits bytes
  int xcol;         // bytes between columns in a slice buffer (GS 256 + 64: an odd multiple of 64)
  int xbuf_bytes;   // one slice buffer: [N][xcol] fragments, then scales [tiles][32 rows][GS] fp16
  int scale_off;    // offset of the scales inside a slice buffer
  int x_off, ring_off, bar_off;  // zq + fac at offset 0
  // rotation inside the kernel (K <= 8192, grid >= N): CTA n < N rotates row
  // n into xg, then every CTA waits until the N rows are published (sync[0]
  // counts them, sync[1] counts the CTAs past the gate; the last resets both)
  int fused, logk, planes;
  const __half* x;
  const int8_t* signs;
  float zero, inv_sqrt_k;
  uint32_t* sync;
  int withhold;  // test of the error path: CTA 0 does not publish its rotated row
};

// Row n of the batch, rotated by this CTA (512 threads) and written to xg in
// the prep layout: column n's fragments, its zero-point terms and output
// factor; CTA 0 also clears the absent columns' terms.  buf: the FWHT's
// shared-memory buffer (K + K/32 + 16 floats).
template <int BITS, int NB, int LOGK>
__device__ __forceinline__ void g32_rotate_row(const G32Params& p, int n, float* buf) {
  using FS = Fwht512<LOGK>;
  constexpr int K = 1 << LOGK, G = K / kGroup;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  uint8_t* xg = const_cast<uint8_t*>(p.xg);
  uint16_t* xs = reinterpret_cast<uint16_t*>(xg);
  float* zq = reinterpret_cast<float*>(xg + gemv_xs_bytes(G, p.N));
  float* fac = zq + G * 16 * NB;
  float* red = buf + FS::SMEM_FLOATS;
  const FragLane<BITS> fl(lane, p.planes != 0);
  const SignMask<FS::E> neg = sign_bits<FS::E>(p.signs ? p.signs + tid * FS::E : nullptr);
  pdl_wait();  // x is the previous kernel's output; xg may still be read by it
  if (n == 0) zq_clear_absent<NB>(zq, G, p.N, tid, kWarps * 32);
  float v[FS::E];
  load_chunk<__half, FS::E>(p.x + static_cast<size_t>(n) * K + tid * FS::E, v);
  flip_signs<FS::E>(neg, v);
  fwht_block512<LOGK>(v, buf, red);
  const int e = row_scale_exp(red_max(red, kWarps) * p.inv_sqrt_k);
  if (tid == 0) fac[n] = pow2f(24 - e);
  const float sc = p.inv_sqrt_k * pow2f(e);
  put_groups<BITS, (G + kWarps - 1) / kWarps, NB>(fl, buf, warp, kWarps, n, G, sc, p.zero, xs, zq, lane);
}

// Slice s lives in buffer s & 1 (its (s >> 1)-th fill).
template <int BITS, int NB, bool PL>
__global__ void __launch_bounds__(kWarps * 32, 1) gemv32_kernel(const __grid_constant__ G32Params p) {
  constexpr int GB = 16 * BITS;  // bytes of one group of one row
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, t = lane & 3;
  const int G = p.G, GS = p.GS, S = p.S, NS = p.NS, N = p.N;
  const uint32_t c = blockIdx.x;
  const int tile0 = static_cast<int>(c * p.tq + min(c, p.tr));
  const int ntile = static_cast<int>(p.tq + (c < p.tr ? 1u : 0u));
  // the warp's units of every slice: [a, b) of the ntile * GS (tile, group)
  // units, tile-major; the warps with a non-empty range arrive on the slice
  // counters
  const int nunit = ntile * GS;
  auto wbeg = [&](int w) { return (w * nunit) / kWarps; };
  const int a = wbeg(warp), b = wbeg(warp + 1), len = b - a;
  const int n_busy = min(kWarps, nunit);  // warps with work (ranges are balanced)
  const int tA = len > 0 ? a / GS : -1, tB = len > 0 ? (b - 1) / GS : -1;

  float* zq = reinterpret_cast<float*>(smem);
  const float* fac = zq + G * NB * 16;
  uint8_t* xbuf = smem + p.x_off;
  uint64_t* xbar = reinterpret_cast<uint64_t*>(smem + p.bar_off);  // [2]
  uint32_t* xcnt = reinterpret_cast<uint32_t*>(smem + p.bar_off + 16);  // [2] arrivals, [2] last slice issued
  int* xlast = reinterpret_cast<int*>(smem + p.bar_off + 24);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + p.bar_off + 32) + warp * NS;
  const int ring_stride = kWarps * p.slot_bytes;
  uint8_t* ring = smem + p.ring_off + warp * p.slot_bytes;

  if (tid == 0) {
    prefetch_tensormap(&p.qmap);
    prefetch_tensormap(&p.smap);
    mbar_init(&xbar[0], 1);
    mbar_init(&xbar[1], 1);
    xcnt[0] = xcnt[1] = 0u;
    xlast[0] = xlast[1] = -1;
    fence_mbar_init();
  }
  if (lane == 0) {
    for (int i = 0; i < NS; ++i) mbar_init(&bars[i], 1);
    fence_mbar_init();
  }
  __syncthreads();
  pdl_launch_dependents();

  // ---- the warp's code ring (lane 0 issues): unit i of its sequence is
  // slice i / len, unit a + i % len of that slice
  const int total = S * len;
  const int tl_a = len > 0 ? a / GS : 0, gl_a = len > 0 ? a - tl_a * GS : 0;  // the range's first unit
  int issued = 0;
  int i_s = 0, i_u = a, i_tl = tl_a, i_gl = gl_a;  // the next unit to request (slice, unit, tile, group)
  auto issue = [&](int slot) {
    if (lane == 0) {
      mbar_arrive_expect_tx(&bars[slot], kTRows * GB);
      tma_load_3d(ring + slot * ring_stride, &p.qmap, 0, (tile0 + i_tl) * kTRows, i_s * GS + i_gl, &bars[slot]);
    }
    ++issued;
    if (++i_u == b) {
      i_u = a;
      i_tl = tl_a;
      i_gl = gl_a;
      ++i_s;
    } else if (++i_gl == GS) {
      i_gl = 0;
      ++i_tl;
    }
  };
  for (int s = 0; s < NS && issued < total; ++s) issue(s);

  // ---- slice s into buffer s & 1 (one whole warp): the columns' fragments
  // of its groups (one bulk copy per column, lanes 0..N-1) and the tiles'
  // scales (one box per tile, lanes 16..16+ntile-1; rows past M read as zero)
  auto issue_slice = [&](int s) {
    uint8_t* xb = xbuf + (s & 1) * p.xbuf_bytes;
    const uint32_t frag = static_cast<uint32_t>(GS) * 4 * kXsBlock;
    if (lane == 0) {
      xlast[s & 1] = s;
      mbar_arrive_expect_tx(&xbar[s & 1], static_cast<uint32_t>(N) * frag +
                                              static_cast<uint32_t>(ntile) * kTRows * GS * 2);
    }
    __syncwarp();
    if (lane < N) {
      bulk_g2s(xb + lane * p.xcol, p.xg + lane * gemv_xs_col(G) + static_cast<size_t>(s) * frag, frag,
               &xbar[s & 1]);
    }
    if (lane >= 16 && lane - 16 < ntile) {
      const int tl = lane - 16;
      tma_load_2d(xb + p.scale_off + tl * kTRows * GS * 2, &p.smap, s * GS, (tile0 + tl) * kTRows, &xbar[s & 1]);
    }
  };

  bool ok = true;
  if (p.fused) {
    if (static_cast<int>(c) < N) {
      // rotate row c (the FWHT buffer is the slice buffers' memory, unused
      // until the gate), publish it for every CTA's bulk copies (async proxy)
      float* buf = reinterpret_cast<float*>(xbuf);
      switch (p.logk) {
        case 10: g32_rotate_row<BITS, NB, 10>(p, c, buf); break;
        case 11: g32_rotate_row<BITS, NB, 11>(p, c, buf); break;
        case 12: g32_rotate_row<BITS, NB, 12>(p, c, buf); break;
        default: g32_rotate_row<BITS, NB, 13>(p, c, buf); break;
      }
      asm volatile("fence.proxy.async.global;" ::: "memory");
      __syncthreads();
      if (tid == 0 && !(p.withhold && c == 0)) {
        __threadfence();
        atomicAdd(p.sync, 1u);
      }
    } else {
      pdl_wait();
    }
    // the gate: all N rows published
    bool passed = true;
    if (tid == 0) {
      passed = wait_count(p.sync, static_cast<uint32_t>(N));
      if (passed && atomicAdd(p.sync + 1, 1u) == gridDim.x - 1) {
        atomicExch(p.sync, 0u);
        atomicExch(p.sync + 1, 0u);
      }
    }
    ok = __syncthreads_and(passed) != 0;
    // the FWHT's generic accesses to the slice buffers come before the
    // bulk copies into them; the published rows are read by bulk copies
    fence_proxy_async_smem();
    asm volatile("fence.proxy.async.global;" ::: "memory");
    __syncthreads();
  } else {
    pdl_wait();  // the prep output is the previous kernel's
  }
  if (ok) {
    // zero-point terms and output factors, contiguous after the fragments
    const int zbytes = G * NB * 64 + 32 * NB;
    const uint8_t* src = p.xg + gemv_xs_bytes(G, N);
    for (int i = tid * 16; i < zbytes; i += kWarps * 32 * 16) cp_async16(smem + i, src + i, 16);
    if (warp == 0) {
      issue_slice(0);
      if (S > 1) issue_slice(1);
    }
  }
  asm volatile("cp.async.wait_all;" ::: "memory");
  __syncthreads();

  // ---- consumer
  float accA[2][NB][4], accB[2][NB][4];
#pragma unroll
  for (int r = 0; r < 2; ++r) {
#pragma unroll
    for (int nb = 0; nb < NB; ++nb) {
#pragma unroll
      for (int i = 0; i < 4; ++i) accA[r][nb][i] = accB[r][nb][i] = 0.f;
    }
  }
  // shared-window addresses: the lane's B-fragment stream of block nb is
  // column 8 nb + g (column 0's for absent columns, whose outputs are never
  // stored), k-quad t
  const uint32_t s_base = smem_u32(smem);
  uint32_t xl[NB];
#pragma unroll
  for (int nb = 0; nb < NB; ++nb) {
    const int col = 8 * nb + g;
    xl[nb] = static_cast<uint32_t>((col < N ? col : 0) * p.xcol + t * kXsBlock);
  }
  const uint32_t rot[4] = {(t & 3u) << 4, ((t + 1) & 3u) << 4, ((t + 2) & 3u) << 4, ((t + 3) & 3u) << 4};
  const uint32_t zq_s = s_base + t * 16;  // + (group NB + nb) 64
  const uint32_t ring_s = s_base + p.ring_off + warp * p.slot_bytes;
  // the lane's bytes of its rows g + 8 r (8-bit rows: 16-byte chunks 2t, 2t + 1
  // in the 128-byte swizzle, XOR row % 8 = g % 8)
  const uint32_t row_s = static_cast<uint32_t>(g * GB + (BITS == 8 ? 0 : t * 4 * BITS));

  int slot = 0, consumed = 0;
  uint32_t sph = 0;
  for (int s = 0; s < S && ok; ++s) {
    const uint32_t xb_s = s_base + p.x_off + (s & 1) * p.xbuf_bytes;
    if (len > 0) ok = __all_sync(0xffffffffu, mbar_wait(&xbar[s & 1], (s >> 1) & 1));
    int tl = tl_a, gl = gl_a;  // the unit's tile and group in the slice
    for (int u = a; ok && u < b; ++u, (++gl == GS ? (gl = 0, ++tl) : 0)) {
      ok = __all_sync(0xffffffffu, mbar_wait(&bars[slot], sph));
      if (!ok) break;
      const uint32_t codes = ring_s + slot * ring_stride + row_s;
      // the lane's 32-code bundle of row g + 8 r (r < 4: tiles 0 and 1)
      auto load_row = [&](int r, uint32_t (&wr)[BITS]) {
        const uint32_t ra = codes + r * 8 * GB;
        if constexpr (BITS == 8) {
          const uint32_t sw = g & 7;
          const uint4 v0 = lds128(ra + (((2 * t) ^ sw) << 4));
          const uint4 v1 = lds128(ra + (((2 * t + 1) ^ sw) << 4));
          wr[0] = v0.x; wr[1] = v0.y; wr[2] = v0.z; wr[3] = v0.w;
          wr[4] = v1.x; wr[5] = v1.y; wr[6] = v1.z; wr[7] = v1.w;
        } else if constexpr (BITS == 4) {
          const uint4 v = lds128(ra);
          wr[0] = v.x; wr[1] = v.y; wr[2] = v.z; wr[3] = v.w;
        } else if constexpr (BITS == 3) {
          wr[0] = lds32(ra);
          wr[1] = lds32(ra + 4);
          wr[2] = lds32(ra + 8);
        } else {
          const uint2 v = lds64(ra);
          wr[0] = v.x; wr[1] = v.y;
        }
        if constexpr (PL) plane_bundle(wr);
      };
      // B fragments of the group (both tiles' MMAs read them) and the
      // zero-point terms of the blocks' columns
      uint4 bq[NB][4];
      float4 z[NB];
      const int ga = s * GS + gl;  // the group in the row
#pragma unroll
      for (int nb = 0; nb < NB; ++nb) {
#pragma unroll
        for (int i = 0; i < 4; ++i) bq[nb][i] = lds128(xb_s + xl[nb] + gl * (4 * kXsBlock) + rot[i]);
        z[nb] = lds128f(zq_s + (ga * NB + nb) * 64);
      }
      // the chains start at the zero-point terms (C of the first MMA)
      float zc[NB][4], cc[2][NB][4];
#pragma unroll
      for (int nb = 0; nb < NB; ++nb) {
        zc[nb][0] = z[nb].x;
        zc[nb][1] = z[nb].y;
        zc[nb][2] = z[nb].z;
        zc[nb][3] = z[nb].w;
      }
      if constexpr (BITS == 3 || BITS == 8) {
        // 16 (3-bit) or 8 (8-bit) registers per decoded bundle: one tile at a time
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          uint32_t w[2][BITS];
          load_row(2 * r, w[0]);
          load_row(2 * r + 1, w[1]);
          DecodeViews<BITS> Va, Vb;
          Va.init(w[0]);
          Vb.init(w[1]);
#pragma unroll
          for (int st = 0; st < 8; ++st) {
            const uint32_t av[4] = {Va.pair(2 * st), Vb.pair(2 * st), Va.pair(2 * st + 1), Vb.pair(2 * st + 1)};
#pragma unroll
            for (int nb = 0; nb < NB; ++nb) {
              const uint32_t b0 = (st & 1) ? bq[nb][st >> 1].z : bq[nb][st >> 1].x;
              const uint32_t b1 = (st & 1) ? bq[nb][st >> 1].w : bq[nb][st >> 1].y;
              if (st == 0) {
                mma_16816(cc[r][nb], av, b0, b1, zc[nb]);
              } else {
                mma_16816_acc(cc[r][nb], av, b0, b1);
              }
            }
          }
        }
      } else {
        // both tiles' chains interleaved step by step (2 NB chains in flight)
        DecodeViews<BITS> V[4];
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          uint32_t w[BITS];
          load_row(r, w);
          V[r].init(w);
        }
#pragma unroll
        for (int st = 0; st < 8; ++st) {
#pragma unroll
          for (int r = 0; r < 2; ++r) {
            const uint32_t av[4] = {V[2 * r].pair(2 * st), V[2 * r + 1].pair(2 * st), V[2 * r].pair(2 * st + 1),
                                    V[2 * r + 1].pair(2 * st + 1)};
#pragma unroll
            for (int nb = 0; nb < NB; ++nb) {
              const uint32_t b0 = (st & 1) ? bq[nb][st >> 1].z : bq[nb][st >> 1].x;
              const uint32_t b1 = (st & 1) ? bq[nb][st >> 1].w : bq[nb][st >> 1].y;
              if (st == 0) {
                mma_16816(cc[r][nb], av, b0, b1, zc[nb]);
              } else {
                mma_16816_acc(cc[r][nb], av, b0, b1);
              }
            }
          }
        }
      }
      // acc += scale * chain, per row (rows g + 8 r of the tile)
      const uint32_t sc = xb_s + p.scale_off + (tl * kTRows * GS + gl) * 2;
      float sv[4];
#pragma unroll
      for (int r = 0; r < 4; ++r) sv[r] = __half2float(__ushort_as_half(lds16(sc + (g + 8 * r) * GS * 2)));
      __syncwarp();
      if (issued < total) issue(slot);
      ++consumed;
      if (++slot == NS) {
        slot = 0;
        sph ^= 1u;
      }
      if (tl == tA) {
#pragma unroll
        for (int r = 0; r < 2; ++r) {
#pragma unroll
          for (int nb = 0; nb < NB; ++nb) {
            accA[r][nb][0] = fmaf(sv[2 * r], cc[r][nb][0], accA[r][nb][0]);
            accA[r][nb][1] = fmaf(sv[2 * r], cc[r][nb][1], accA[r][nb][1]);
            accA[r][nb][2] = fmaf(sv[2 * r + 1], cc[r][nb][2], accA[r][nb][2]);
            accA[r][nb][3] = fmaf(sv[2 * r + 1], cc[r][nb][3], accA[r][nb][3]);
          }
        }
      } else {
#pragma unroll
        for (int r = 0; r < 2; ++r) {
#pragma unroll
          for (int nb = 0; nb < NB; ++nb) {
            accB[r][nb][0] = fmaf(sv[2 * r], cc[r][nb][0], accB[r][nb][0]);
            accB[r][nb][1] = fmaf(sv[2 * r], cc[r][nb][1], accB[r][nb][1]);
            accB[r][nb][2] = fmaf(sv[2 * r + 1], cc[r][nb][2], accB[r][nb][2]);
            accB[r][nb][3] = fmaf(sv[2 * r + 1], cc[r][nb][3], accB[r][nb][3]);
          }
        }
      }
    }
    if (!ok || len == 0) continue;
    // this warp is done with slice s: order its reads of the buffer before
    // the refill (an async-proxy write), then count it; the last of the busy
    // warps refills the buffer with slice s + 2
    fence_proxy_async_smem();
    __syncwarp();
    uint32_t last = 0;
    if (lane == 0) {
      __threadfence_block();
      const uint32_t old = atomicAdd(&xcnt[s & 1], 1u);
      last = old + 1u == static_cast<uint32_t>(((s >> 1) + 1) * n_busy) && s + 2 < S;
      if (last) __threadfence_block();
    }
    if (__shfl_sync(0xffffffffu, last, 0)) issue_slice(s + 2);
  }

  // ---- end: every warp has consumed its units (or given up)
  const bool all_ok = __syncthreads_and(ok) != 0;
  if (!all_ok) {
    if (lane == 0 && !ok) record_error(p.status, HQ_DEV_TIMEOUT);
    // let copies still in flight land before the CTA's shared memory is released
    for (int k = consumed; k < issued; ++k) (void)mbar_wait(&bars[k % NS], (k / NS) & 1);
    if (tid == 0) {
      for (int bb = 0; bb < 2; ++bb) {
        if (xlast[bb] >= 0) (void)mbar_wait(&xbar[bb], (xlast[bb] >> 1) & 1);
      }
    }
    return;
  }
  // tiles split between warps: each warp leaves its sums of tiles tA and tB
  // (rings and slice buffers are idle now), the warp whose range holds a
  // tile's first unit adds the later contributors in warp order and stores
  float4* xch = reinterpret_cast<float4*>(smem + p.x_off);  // [warp][2][2 NB][32 lanes]
  auto xslot = [&](int w, int which, int i) { return xch + ((w * 2 + which) * 2 * NB + i) * 32 + lane; };
#pragma unroll
  for (int r = 0; r < 2; ++r) {
#pragma unroll
    for (int nb = 0; nb < NB; ++nb) {
      *xslot(warp, 0, r * NB + nb) = make_float4(accA[r][nb][0], accA[r][nb][1], accA[r][nb][2], accA[r][nb][3]);
      *xslot(warp, 1, r * NB + nb) = make_float4(accB[r][nb][0], accB[r][nb][1], accB[r][nb][2], accB[r][nb][3]);
    }
  }
  __syncthreads();
#pragma unroll
  for (int which = 0; which < 2; ++which) {
    const int tl = which == 0 ? tA : tB;
    if (tl < 0 || (which == 1 && tB == tA)) continue;
    if (tl * GS < a) continue;  // an earlier warp holds the tile's first unit
#pragma unroll
    for (int r = 0; r < 2; ++r) {
#pragma unroll
      for (int nb = 0; nb < NB; ++nb) {
        float4 o = *xslot(warp, which, r * NB + nb);
        for (int w2 = warp + 1; w2 < kWarps; ++w2) {
          const int a2 = wbeg(w2);
          if (a2 >= (tl + 1) * GS) break;
          if (a2 == wbeg(w2 + 1)) continue;  // empty range
          const float4 q4 = *xslot(w2, 0, r * NB + nb);  // the tile is the later warp's first
          o.x += q4.x;
          o.y += q4.y;
          o.z += q4.z;
          o.w += q4.w;
        }
        const int n0 = 8 * nb + 2 * t;
        const int m0 = (tile0 + tl) * kTRows + 16 * r + g;
        const float f0 = fac[n0], f1 = fac[n0 + 1];
        if (m0 < p.M) {
          if (n0 < N) p.y[static_cast<size_t>(n0) * p.ldy + m0] = o.x * f0;
          if (n0 + 1 < N) p.y[static_cast<size_t>(n0 + 1) * p.ldy + m0] = o.y * f1;
        }
        if (m0 + 8 < p.M) {
          if (n0 < N) p.y[static_cast<size_t>(n0) * p.ldy + m0 + 8] = o.z * f0;
          if (n0 + 1 < N) p.y[static_cast<size_t>(n0 + 1) * p.ldy + m0 + 8] = o.w * f1;
        }
      }
    }
  }
}

// ---------------------------------------------------------------- host planning
struct G32Plan {
  int NB = 0, GS = 0, S = 0, NS = 0, slot_bytes = 0, xcol = 0, xbuf_bytes = 0, scale_off = 0;
  int x_off = 0, ring_off = 0, bar_off = 0;
  uint32_t grid = 0, tq = 0, tr = 0;
  size_t smem = 0;
  bool fused = false;
};

constexpr size_t kG32MaxSmem = 227 * 1024;
constexpr int kG32MaxNS = 8;
constexpr int kG32MinFlight = 64 * 1024;

static size_t up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// The slice length and ring depth: the longer slice (16 groups: half the
// slice hand-offs, each a refill the warps may wait for) while its ring keeps
// at least kG32MinFlight code bytes in flight per CTA, else the shape with the
// most in flight; none if no shape fits or a CTA would own more than
// kMaxTilesPerCta tiles.
static G32Plan g32_plan(int bits, int M, int K, int N) {
  G32Plan best;
  const bool fused_k = K >= 1024 && K <= 8192;
  const int G = K / kGroup;
  if (N < 1 || N > 16 || G < 8 || M < 1) return best;
  const int NB = gemv_blocks(N);
  const uint32_t tiles = static_cast<uint32_t>((M + kTRows - 1) / kTRows);
  const uint32_t grid = std::min<uint32_t>(static_cast<uint32_t>(sm_count()), tiles);
  const uint32_t tq = tiles / grid, tr = tiles % grid;
  const int tmax = static_cast<int>(tq + (tr ? 1 : 0));
  if (tmax > kMaxTilesPerCta) return best;
  // the rotation runs in the kernel when every row has a CTA; its FWHT buffer
  // (K + K/32 + 16 floats) borrows the slice buffers' memory
  const bool fused = fused_k && grid >= static_cast<uint32_t>(N);
  const size_t fwht = fused ? (static_cast<size_t>(K) + K / 32 + 16) * 4 : 0;
  const int slot = kTRows * 16 * bits;
  const size_t x_off = up(static_cast<size_t>(G) * NB * 64 + 32 * NB, 1024);
  const size_t xch = static_cast<size_t>(kWarps) * 2 * 2 * NB * 32 * 16;
  for (int GS : {16, 8}) {
    if (G % GS != 0) continue;
    const int S = G / GS;
    const int xcol = GS * 4 * kXsBlock + 64;
    const size_t scale_off = up(static_cast<size_t>(N) * xcol, 128);
    const size_t xbuf = up(scale_off + static_cast<size_t>(tmax) * kTRows * GS * 2, 128);
    const size_t ring_off = up(x_off + std::max((S > 1 ? 2 : 1) * xbuf, fwht), 1024);
    for (int ns = kG32MaxNS; ns >= 2; --ns) {
      const size_t bar_off = ring_off + static_cast<size_t>(kWarps) * ns * slot;
      const size_t smem = bar_off + 32 + static_cast<size_t>(kWarps) * ns * 8 + 1024;
      if (smem > kG32MaxSmem || bar_off - x_off < xch) continue;
      const bool keep = best.smem != 0 && kWarps * best.NS * best.slot_bytes >= kG32MinFlight;
      if (best.smem == 0 || (!keep && ns * slot > best.NS * best.slot_bytes)) {
        best.NB = NB;
        best.GS = GS;
        best.S = S;
        best.NS = ns;
        best.slot_bytes = slot;
        best.xcol = xcol;
        best.xbuf_bytes = static_cast<int>(xbuf);
        best.scale_off = static_cast<int>(scale_off);
        best.x_off = static_cast<int>(x_off);
        best.ring_off = static_cast<int>(ring_off);
        best.bar_off = static_cast<int>(bar_off);
        best.grid = grid;
        best.tq = tq;
        best.tr = tr;
        best.smem = smem;
        best.fused = fused;
      }
      break;
    }
  }
  return best;
}

bool gemv32_supported(int bits, int M, int K, int N) { return g32_plan(bits, M, K, N).smem != 0; }

int gemv32_launches(int bits, int M, int K, int N) {
  const G32Plan pl = g32_plan(bits, M, K, N);
  return pl.smem == 0 ? 0 : pl.fused ? 1 : 2;
}

size_t gemv32_scratch_bytes(int K, int N) { return gemv_xg_bytes(K / kGroup, N); }

template <int BITS, int NB>
static cudaError_t g32_prep(int K, const GemvArgs& a, cudaStream_t st) {
  const dim3 g(a.N);
  const float inv = static_cast<float>(1.0 / sqrt(static_cast<double>(K)));
  const __half* x = reinterpret_cast<const __half*>(a.x);
  uint8_t* xg = static_cast<uint8_t*>(a.xg);
#define HQ_PREP32(LK)                                                                                 \
  launch_pdl(gemv_prep_kernel<BITS, LK, NB>, g, dim3(prep_warps(LK) * 32),                              \
             (FwhtShape<LK, prep_logw(LK)>::SMEM_FLOATS + 32) * sizeof(float), st, true, x, a.signs, xg, \
             a.N, static_cast<float>(a.zero), inv, a.planes ? 1 : 0)
  switch (K) {
    case 1024: return HQ_PREP32(10);
    case 2048: return HQ_PREP32(11);
    case 4096: return HQ_PREP32(12);
    case 8192: return HQ_PREP32(13);
    case 16384: return HQ_PREP32(14);
    case 32768: return HQ_PREP32(15);
    default: return cudaErrorInvalidValue;
  }
#undef HQ_PREP32
}

template <int BITS, int NB>
static cudaError_t g32_launch(const GemvArgs& a, const G32Plan& pl, G32Params& p, cudaStream_t st) {
  if (!p.fused) {
    const cudaError_t e = g32_prep<BITS, NB>(a.K, a, st);
    if (e != cudaSuccess) return e;
  }
  const dim3 grid(pl.grid), block(kWarps * 32);
  if constexpr (BITS == 2) {
    if (a.planes) return launch_pdl(gemv32_kernel<2, NB, true>, grid, block, pl.smem, st, true, p);
  }
  return launch_pdl(gemv32_kernel<BITS, NB, false>, grid, block, pl.smem, st, true, p);
}

template <int BITS>
static cudaError_t g32_launch_b(const GemvArgs& a, const G32Plan& pl, G32Params& p, cudaStream_t st) {
  return pl.NB == 1 ? g32_launch<BITS, 1>(a, pl, p, st) : g32_launch<BITS, 2>(a, pl, p, st);
}

cudaError_t launch_gemv32(const GemvArgs& a, cudaStream_t st) {
  if (a.zeros != nullptr || a.zero_frac) return cudaErrorInvalidValue;
  const G32Plan pl = g32_plan(a.bits, a.M, a.K, a.N);
  if (pl.smem == 0) return cudaErrorInvalidValue;
  const int G = a.K / kGroup;
  G32Params p{};
  {
    // the codes viewed as [G][M][16 bits bytes]: one box = one group of 32
    // rows (8-bit rows in the 128-byte swizzle, like the GEMV's)
    const uint64_t gb = 16ull * a.bits;
    const uint64_t dims[3] = {gb, static_cast<uint64_t>(a.M), static_cast<uint64_t>(G)};
    const uint64_t strides[2] = {static_cast<uint64_t>(a.K) * a.bits / 8, gb};
    const uint32_t box[3] = {static_cast<uint32_t>(gb), static_cast<uint32_t>(kTRows), 1u};
    cudaError_t e = tensor_map_3d(&p.qmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.q, dims, strides, box,
                                  a.bits == 8 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE);
    if (e != cudaSuccess) return e;
    e = tensor_map_2d(&p.smap, CU_TENSOR_MAP_DATA_TYPE_UINT16, a.scales, static_cast<uint64_t>(G),
                      static_cast<uint64_t>(a.M), static_cast<uint64_t>(G) * 2, static_cast<uint32_t>(pl.GS),
                      kTRows, CU_TENSOR_MAP_SWIZZLE_NONE);
    if (e != cudaSuccess) return e;
  }
  p.xg = static_cast<const uint8_t*>(a.xg);
  p.y = a.y;
  p.status = a.status;
  p.M = a.M;
  p.N = a.N;
  p.ldy = a.ldy;
  p.G = G;
  p.tq = pl.tq;
  p.tr = pl.tr;
  p.S = pl.S;
  p.GS = pl.GS;
  p.NS = pl.NS;
  p.slot_bytes = pl.slot_bytes;
  p.xcol = pl.xcol;
  p.xbuf_bytes = pl.xbuf_bytes;
  p.scale_off = pl.scale_off;
  p.x_off = pl.x_off;
  p.ring_off = pl.ring_off;
  p.bar_off = pl.bar_off;
  p.fused = pl.fused && a.sync != nullptr ? 1 : 0;
  p.logk = 0;
  while ((1 << p.logk) < a.K) ++p.logk;
  p.planes = a.planes ? 1 : 0;
  p.x = reinterpret_cast<const __half*>(a.x);
  p.signs = a.signs;
  p.zero = static_cast<float>(a.zero);
  p.inv_sqrt_k = static_cast<float>(1.0 / sqrt(static_cast<double>(a.K)));
  p.sync = a.sync;
  p.withhold = p.fused && take_test_fault() ? 1 : 0;
  switch (a.bits) {
    case 2: return g32_launch_b<2>(a, pl, p, st);
    case 3: return g32_launch_b<3>(a, pl, p, st);
    case 4: return g32_launch_b<4>(a, pl, p, st);
    case 8: return g32_launch_b<8>(a, pl, p, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace hq
