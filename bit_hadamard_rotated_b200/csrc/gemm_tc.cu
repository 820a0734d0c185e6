// gemm_tc.cu -- tensor-core (tcgen05) dequant GEMM for larger batches:
//   y[n][m] = sum_k scale[m][k/128] (q[m][k] - zero) x'[n][k],  N >= 9.
// At batch 16..256 the contraction is a dense one, so it runs on the
// 5th-generation tensor cores with the fp32 accumulator in tensor memory:
//   * a prep kernel rotates x (fp32 butterflies) and writes x' 2^e as fp16 in
//     the k order of the decoded code pairs (hq_layout.cuh), so that A and B
//     agree, already in the shared-memory image the MMA reads (no-swizzle
//     K-major core matrices), one contiguous block per 128-code group; 2^e is
//     a power of two per batch row that puts the row's largest |x'| just
//     below 2^14 (small activations stay out of fp16's subnormal range), and
//     the epilogue multiplies that output column by 2^-e, exactly;
//   * per CTA, an equal contiguous range of (128-row tile, 128-code group)
//     chunks (stream-K; the first and last tile may be shared with the
//     neighbouring CTA), streamed through two rings by two producer threads:
//     the code ring (up to 16 slots, as many as fit: the weights come from
//     HBM, so it runs far ahead) takes the tile's 128 code rows in one 2D TMA
//     load per chunk (swizzled so the decoders' 16-byte row reads are free of
//     bank conflicts), plus each tile's scales in one bulk copy; a slot is
//     refilled as soon as its warpgroup has the codes in registers.  The x'
//     ring (4 slots) takes the group's x' image (L2-resident) in one bulk
//     copy per chunk and is refilled when the chunk's MMAs are done.  Each
//     copy completes on its slot's mbarrier (expected bytes);
//   * two warpgroups take the chunks in turn (chunk c to warpgroup c mod 2):
//     each thread owns one weight row, decodes its 128 codes into exact fp16
//     (q - zero) (one LOP3 and one fp16 FMA per pair), multiplies by the group
//     scale (one fp16 multiply per pair: the weight's only rounding) and
//     stores the row into tensor memory as the MMA's A operand (tcgen05.st),
//     one TMEM lane per row, in A stage c mod as (4 stages, so each
//     warpgroup decodes ahead while the MMAs of its previous chunks run);
//   * two or four MMA warps take the chunks in the same turn; each issues 8
//     tcgen05.mma (M=128, N, K=16, A from TMEM, B from shared memory) per
//     chunk into its own fp32 accumulator in tensor memory and commits their
//     completion to the x' slot's and the A stage's mbarriers.  One issuing
//     thread sustains only one MMA per ~60-80 cycles whatever N is, so at
//     batch <= 128 more issuers raise the tensor-pipe rate;
//   * an epilogue warpgroup sums a tile's accumulators (tcgen05.ld) and writes
//     y, or, for a tile shared with a neighbour, leaves its part in the
//     workspace and the second CTA to count its arrival adds left + right in
//     that order (deterministic, no waiting).  With two accumulator sets
//     (batch <= 32) the next tile's MMAs run while the epilogue reads; the
//     dequant warps never stop for it.
// Every barrier's consecutive phases are waited for by one agent, in order
// (ring depths are multiples of the agent counts), so phase-parity waits are
// unambiguous.
// Waits are bounded (status word on timeout); tensor memory is freed on exit.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <mutex>

#include "fwht.cuh"
#include "hq_common.cuh"
#include "hq_internal.h"
#include "hq_io.cuh"
#include "hq_launch.cuh"
#include "hq_layout.cuh"
#include "tcgen05.cuh"

namespace hq {
namespace tc {

constexpr int kTileM = 128;
constexpr int kNCMax = 16;        // code ring slots (HBM latency): as many as fit, <= G
constexpr int kNCMin = 4;
constexpr int kNB = 4;            // x' image ring slots (L2 latency)
constexpr int kASMax = 6;         // A stages in tensor memory (64 columns each): 4 or 6
constexpr int kDeqWG = 2;         // dequant warpgroups (groups round robin)
constexpr int kDeqWarps = 4 * kDeqWG;
constexpr int kProducerWarp = kDeqWarps;  // codes and scales
constexpr int kBWarp = kDeqWarps + 1;     // x' images
constexpr int kMmaWarp0 = kDeqWarps + 2;
constexpr int kMmaWarps = 4;      // issuing threads launched: one issues an MMA per ~60-80 cycles
constexpr int kEpiWarp0 = kMmaWarp0 + kMmaWarps;
constexpr int kEpiWarps = 4;      // the epilogue warpgroup: one thread per accumulator row
constexpr int kThreads = (kDeqWarps + 2 + kMmaWarps + kEpiWarps) * 32;
// Phase-parity waits are unambiguous only if a barrier's consecutive phases
// are waited for by the same agent (it cannot wait for round r + 1 before
// round r completed): every ring depth is a multiple of the dequant
// warpgroup count, and the A-stage count a multiple of it and of the MMA
// warp count.
// The code ring is waited for by the dequant warpgroups (its depth is even);
// the x' ring and the A stages by the MMA warps in use (n_mma = 2 or 4): the
// host picks stage counts that are multiples of it, and kNB is one.
static_assert(kNCMin % kDeqWG == 0 && kNCMax % kDeqWG == 0 && kASMax % kDeqWG == 0 &&
                  kNB % kMmaWarps == 0,
              "ring depths must be multiples of the agent counts");
// CTA chunk ranges are whole quanta of kQuant chunks, so every tile portion a
// CTA computes holds a chunk of every MMA warp and dequant warpgroup.
constexpr int kQuant = 4;
static_assert(kQuant % kMmaWarps == 0 && kQuant % kDeqWG == 0, "quantum");
constexpr int kTmemCols = 512;
// Tensor memory: accumulator j at columns [j Npad, (j + 1) Npad); A stage s at
// a_base + 64 s, a_base = 2 Npad rounded up to 64; as many stages as fit,
// rounded down to even (6 for Npad <= 64, 4 for Npad <= 128).

// 16-byte unit holding unit i of code row r in a slot: the TMA swizzle for
// the row width (32 B rows: 32-byte swizzle, 64 B: 64-byte, 128 B: 128-byte;
// 48 B rows are conflict-free unswizzled).
template <int BITS>
__device__ __forceinline__ int code_unit(int i, int r) {
  if constexpr (BITS == 2) return i ^ ((r >> 2) & 1);
  else if constexpr (BITS == 4) return i ^ ((r >> 1) & 3);
  else if constexpr (BITS == 8) return i ^ (r & 7);
  else return i;
}

// ---------------------------------------------------------------- prep: rotate, permute, lay out
// Byte offset of row n, k-position i (pair order) inside a batch block's
// image: per 128-code group g a block of 256 Npad bytes holding the 8 K=16
// slices (32 Npad bytes each) of an Npad x 128 K-major no-swizzle operand:
// [slice ks][8-element half kc][row group n/8][row n%8][8 fp16].
__host__ __device__ constexpr size_t img_offset(int g, int i, int n, int npad) {
  return static_cast<size_t>(g) * 256 * npad + ((i >> 4) & 7) * 32 * npad + ((i >> 3) & 1) * 16 * npad +
         (n >> 3) * 128 + (n & 7) * 16;
}

// Grid (nb, n_blocks): CTA (j, b) builds image row j of batch block b (rows
// b*nb .. b*nb + nb - 1 of x); rows past the batch but inside the block's
// 32-row padding are written as zeros, the rest of the CTAs exit at once.
// Image of block b at byte b * K * 2 * nb of xp.  Position i of group g holds
// x'[128 g + 32 t + code(p, h)] 2^e with i = 32 t + 2 p + h; fac[b nb + j] =
// 2^-e, the row's output factor (1 for padding rows).
template <int BITS, int LOGK>
__global__ void __launch_bounds__(FwhtShape<LOGK>::THREADS)
    tc_prep_kernel(const __half* __restrict__ x, const int8_t* __restrict__ signs,
                   uint8_t* __restrict__ xp, float* __restrict__ fac, int N, int nb, float inv) {
  using S = FwhtShape<LOGK>;
  extern __shared__ float buf[];
  float* red = buf + S::SMEM_FLOATS;  // per-warp maxima of the transform
  pdl_launch_dependents();
  const int j = blockIdx.x, b = blockIdx.y, tid = threadIdx.x;
  const int rows = min(nb, N - b * nb);
  const int npad = (rows + 31) & ~31;
  if (j >= npad) return;  // whole CTA: no barrier is reached
  const auto neg = sign_bits<S::E>(signs ? signs + tid * S::E : nullptr);
  pdl_wait();
  uint8_t* img = xp + static_cast<size_t>(b) * S::K * 2 * nb;
  const int n = b * nb + j;
  float sc = 0.f;
  if (j < rows) {
    float v[S::E];
    load_chunk<__half, S::E>(x + static_cast<size_t>(n) * S::K + tid * S::E, v);
    flip_signs<S::E>(neg, v);
    fwht_block<LOGK, 5>(v, buf, red);
    const int e = row_scale_exp(red_max(red, S::W) * inv);
    sc = inv * pow2f(e);
    if (tid == 0) fac[b * nb + j] = pow2f(-e);
  } else if (tid == 0) {
    fac[b * nb + j] = 1.f;
  }
  for (int seg = tid; seg < S::K / 8; seg += S::THREADS) {
    const int g = seg >> 4, i0 = (seg * 8) & 127;
    uint32_t w[4] = {0u, 0u, 0u, 0u};
    if (j < rows) {
      const int t = i0 >> 5;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const PairDesc pd = Pairs<BITS>::get(((i0 >> 1) & 15) + q);
        const int k0 = kGroup * g + 32 * t;
        const __half lo = __float2half_rn(buf[fwht_pad(k0 + pd.c_lo)] * sc);
        const __half hi = __float2half_rn(buf[fwht_pad(k0 + pd.c_hi)] * sc);
        w[q] = static_cast<uint32_t>(__half_as_ushort(lo)) |
               (static_cast<uint32_t>(__half_as_ushort(hi)) << 16);
      }
    }
    *reinterpret_cast<uint4*>(img + img_offset(g, i0, j, npad)) = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

// ---------------------------------------------------------------- the GEMM
struct TcParams {
  CUtensorMap qmap;       // packed codes [M][K bits / 8] as bytes; box 16 bits x 128 rows
  const uint8_t* scales;  // fp16 [M][K/128]
  const uint8_t* img;     // this batch block's x' image (G blocks of 256 Npad bytes)
  const float* fac;       // this batch block's output factors 2^-e per column [Npad]
  float* y;               // this batch block's first output row
  uint32_t* status;
  int M, K, N, Npad, ldy;
  int n_tiles;
  // Chunks (tile-major, 128-code groups inner) in quanta of kQuant: CTA c
  // owns quanta [c qq + min(c, qr), +qq + (c < qr)); qq kQuant >= G, so a tile
  // is shared by at most two CTAs.
  int qq, qr;
  float* part;      // [grid][2 sides][128 rows][Npad]: shared tiles' partial sums
  uint32_t* flags;  // [grid]: arrivals at each CTA boundary, zero between calls
  int b_off;       // x' image ring (kNB slots of 256 Npad bytes), after the code ring
  int sbuf_off;    // per-tile scale buffers (two)
  int sbuf_bytes;
  int bar_off;
  int nc;       // code ring slots (kNCMin..kNCMax, even, <= G)
  int as;       // A stages in tensor memory (4 or 6; a multiple of n_mma)
  int a_base;   // tensor-memory column of A stage 0
  int n_mma;    // MMA warps (accumulators per set) in use: 4 if Npad <= 64, else 2
  int nacc;     // accumulator sets: 2 (tile ti uses set ti & 1) if they fit beside 4 A stages, else 1
  uint32_t idesc;
  uint32_t add[16];
};

// The epilogue warpgroup: for each tile portion of the CTA, waits for its
// accumulator set, sums the n_mma accumulators of its row (TMEM lane) and
// stores y, or, for a portion shared with a neighbouring CTA, leaves the part
// in the workspace and lets the second CTA to count its arrival add left +
// right; then frees the set for the MMAs two portions on (one with a single
// set).  Runs beside the dequant warps, which never stop for it.
__device__ __forceinline__ void tc_epilogue(const TcParams& p, uint32_t tmem, uint64_t* dready,
                                            uint64_t* dfree, uint64_t* epib, uint32_t* arrival,
                                            int cta, int g_start, int total, int last_ti, int tile0) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int etid = tid - kEpiWarp0 * 32;
  const int quarter = warp & 3;  // the TMEM lane quarter this warp may access
  const int r = 32 * quarter + lane;
  const uint32_t lane_base = static_cast<uint32_t>(32 * quarter) << 16;
  const int G = p.K / kGroup;
  const uint32_t acc_set = static_cast<uint32_t>(p.n_mma * p.Npad);
  bool ok = true;
  uint32_t eph = 0;
  // all epilogue threads meet here (bounded: a thread that stopped early
  // makes the others time out instead of hang)
  auto epi_sync = [&] {
    mbar_arrive(epib);
    if (!mbar_wait(epib, eph)) ok = false;
    eph ^= 1u;
  };
  for (int ti = 0; ti <= last_ti; ++ti) {
    const int buf = p.nacc == 2 ? (ti & 1) : 0, use = p.nacc == 2 ? (ti >> 1) : ti;
    const bool good = ok && mbar_wait(&dready[buf], use & 1);
    if (!good) ok = false;
    tc_fence_after();
    const uint32_t acc0 = tmem + lane_base + buf * acc_set;
    // the row's sum of the n_mma accumulators, columns [c0, c0 + 16)
    auto acc16 = [&](int c0, float (&acc)[16]) {
      uint32_t v[16];
      tc_ld16(acc0 + c0, v);
      tc_wait_ld();
      tc_tie16(v);
#pragma unroll
      for (int i = 0; i < 16; ++i) acc[i] = __uint_as_float(v[i]);
      for (int a = 1; a < p.n_mma; ++a) {
        tc_ld16(acc0 + a * p.Npad + c0, v);
        tc_wait_ld();
        tc_tie16(v);
#pragma unroll
        for (int i = 0; i < 16; ++i) acc[i] += __uint_as_float(v[i]);
      }
    };
    const int m = (tile0 + ti) * kTileM + r;
    auto store16 = [&](int c0, const float (&acc)[16]) {
      if (m < p.M) {
        float f[16];  // the columns' output factors (the same for every thread)
#pragma unroll
        for (int i = 0; i < 16; i += 4) {
          const float4 q = __ldg(reinterpret_cast<const float4*>(p.fac + c0 + i));
          f[i] = q.x;
          f[i + 1] = q.y;
          f[i + 2] = q.z;
          f[i + 3] = q.w;
        }
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int n = c0 + i;
          if (n < p.N) p.y[static_cast<size_t>(n) * p.ldy + m] = acc[i] * f[i];
        }
      }
    };
    // a portion shared with the CTA before (this CTA holds the tile's right
    // part) or after (left part)
    const bool right = ti == 0 && g_start != 0;
    const bool left = ti == last_ti && (g_start + total) % G != 0;
    if (!right && !left) {
      for (int c0 = 0; good && c0 < p.Npad; c0 += 16) {
        float acc[16];
        acc16(c0, acc);
        store16(c0, acc);
      }
    } else {
      const int bnd = right ? cta - 1 : cta;
      float* mine = p.part + ((static_cast<size_t>(bnd) * 2 + (right ? 1 : 0)) * kTileM + r) * p.Npad;
      const float* other = p.part + ((static_cast<size_t>(bnd) * 2 + (right ? 0 : 1)) * kTileM + r) * p.Npad;
      for (int c0 = 0; good && c0 < p.Npad; c0 += 16) {
        float acc[16];
        acc16(c0, acc);
#pragma unroll
        for (int i = 0; i < 16; i += 4) {
          *reinterpret_cast<float4*>(mine + c0 + i) = make_float4(acc[i], acc[i + 1], acc[i + 2], acc[i + 3]);
        }
      }
      __threadfence();
      epi_sync();
      // after a failed wait the part is not counted (the other side then
      // finds itself first and leaves; the status word has the error)
      if (etid == 0) *arrival = ok ? atomicAdd(p.flags + bnd, 1u) : 0u;
      epi_sync();
      if (ok && *reinterpret_cast<volatile uint32_t*>(arrival) != 0) {
        __threadfence();
        for (int c0 = 0; c0 < p.Npad; c0 += 16) {
          float acc[16];
          acc16(c0, acc);
#pragma unroll
          for (int i = 0; i < 16; i += 4) {
            const float4 o = __ldcg(reinterpret_cast<const float4*>(other + c0 + i));
            if (right) {
              acc[i] = o.x + acc[i];
              acc[i + 1] = o.y + acc[i + 1];
              acc[i + 2] = o.z + acc[i + 2];
              acc[i + 3] = o.w + acc[i + 3];
            } else {
              acc[i] = acc[i] + o.x;
              acc[i + 1] = acc[i + 1] + o.y;
              acc[i + 2] = acc[i + 2] + o.z;
              acc[i + 3] = acc[i + 3] + o.w;
            }
          }
          store16(c0, acc);
        }
        if (etid == 0) p.flags[bnd] = 0;  // ready for the next call
      }
    }
    tc_fence_before();
    mbar_arrive(&dfree[buf]);
  }
  if (!ok && lane == 0) record_error(p.status, HQ_DEV_TIMEOUT);
}

template <int BITS>
__global__ void __launch_bounds__(kThreads, 1) tc_gemm_kernel(const __grid_constant__ TcParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // swizzled TMA tiles need 1 KiB-aligned slots: round the base up (the
  // launch asks for 1 KiB more than the plan)
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = p.K / kGroup;
  const int CB = 16 * BITS;  // code bytes of one row in one 128-code group
  const uint32_t code_bytes = kTileM * CB;      // one code slot
  const uint32_t b_bytes = 256u * p.Npad;        // one x' image slot
  uint64_t* cfull = reinterpret_cast<uint64_t*>(smem + p.bar_off);  // code slot landed
  uint64_t* cfree = cfull + kNCMax;   // code slot read by its dequant warpgroup (may refill)
  uint64_t* bfull = cfree + kNCMax;   // x' image slot landed
  uint64_t* bfree = bfull + kNB;      // x' image slot's MMAs done (may refill)
  uint64_t* aready = bfree + kNB;     // A stage written (MMA may read)
  uint64_t* afree = aready + kASMax;  // A stage's MMAs done (dequant may rewrite)
  uint64_t* dready = afree + kASMax;  // [2]: accumulator set's MMAs done (epilogue may read)
  uint64_t* dfree = dready + 2;       // [2]: accumulator set read out (MMA may overwrite)
  uint64_t* drain = dfree + 2;
  uint64_t* sready = drain + 1;  // [2]: a tile's scales landed in buffer ti & 1
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(sready + 2);
  uint32_t* arrival = tmem_holder + 1;  // the epilogue's boundary-counter result
  // the epilogue threads' own barrier (shared-tile epilogues), 8-byte aligned
  uint64_t* epib = reinterpret_cast<uint64_t*>(tmem_holder + 2);

  if (tid == 0) {
    for (int i = 0; i < p.nc; ++i) {
      mbar_init(&cfull[i], 1);
      mbar_init(&cfree[i], 128);  // every thread of the warpgroup, after its reads
    }
    for (int i = 0; i < kNB; ++i) {
      mbar_init(&bfull[i], 1);
      mbar_init(&bfree[i], 1);
    }
    for (int i = 0; i < p.as; ++i) {
      mbar_init(&aready[i], 128);
      mbar_init(&afree[i], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&dready[b], p.n_mma);
      mbar_init(&dfree[b], kEpiWarps * 32);
    }
    mbar_init(drain, p.n_mma);
    mbar_init(&sready[0], 1);
    mbar_init(&sready[1], 1);
    mbar_init(epib, kEpiWarps * 32);
    fence_mbar_init();
  }
  if (warp == 0) tmem_alloc(tmem_holder, kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  pdl_launch_dependents();
  pdl_wait();

  // this CTA's chunks [cb, cb + total); local tile ti is tile tile0 + ti,
  // the first starting at group g_start (a multiple of kQuant)
  const int cta = static_cast<int>(blockIdx.x);
  const int cb = (cta * p.qq + min(cta, p.qr)) * kQuant;
  const int total = (p.qq + (cta < p.qr ? 1 : 0)) * kQuant;
  const int tile0 = cb / G, g_start = cb - tile0 * G;
  const int last_ti = (g_start + total - 1) / G;
  auto tile_m0 = [&](int ti) { return (tile0 + ti) * kTileM; };

  if (warp == kProducerWarp) {
    // ---------------- code producer (one thread): TMA loads of the chunks'
    // code rows into the code ring, as far ahead as the ring allows (the
    // weights come from HBM), and each tile's scales
    if (lane == 0) {
      bool ok = true;
      int issued = 0;
      // ring position kept incrementally (no divisions on the issue path)
      int sl = 0, g = g_start;
      uint32_t rph = 0;  // parity of the ring round of chunk c
      int m0 = tile_m0(0), ti = 0;
      int rows = min(kTileM, p.M - m0);
      for (int c = 0; c < total; ++c) {
        // slot reuse: chunk c - nc's dequant warpgroup has read the slot.
        // Waiting for every chunk in order also means that at a tile's first
        // chunk every chunk two tiles back has read its scales (nc <= G), so
        // the scale buffer ti & 1 is free again.
        if (c >= p.nc && !mbar_wait(&cfree[sl], rph ^ 1u)) {
          ok = false;
          break;
        }
        // the tile's scales, once per tile, on the buffer's own barrier (a
        // bulk copy's completion shows only on the barrier it signals)
        if (g == 0 || c == 0) {
          const uint32_t s_bytes = static_cast<uint32_t>(rows) * G * 2;
          mbar_arrive_expect_tx(&sready[ti & 1], s_bytes);
          bulk_g2s(smem + p.sbuf_off + (ti & 1) * p.sbuf_bytes,
                   p.scales + static_cast<size_t>(m0) * G * 2, s_bytes, &sready[ti & 1]);
        }
        // a TMA tile always delivers the whole box (rows past M read as zero)
        mbar_arrive_expect_tx(&cfull[sl], code_bytes);
        tma_load_2d(smem + sl * code_bytes, &p.qmap, g * CB, m0, &cfull[sl]);
        issued = c + 1;
        if (++sl == p.nc) {
          sl = 0;
          rph ^= 1u;
        }
        if (++g == G) {
          g = 0;
          ++ti;
          m0 += kTileM;
          rows = min(kTileM, p.M - m0);
        }
      }
      // Drain: the copies of the last slots must have landed before exit (they
      // have on the normal path, where the dequant warps consumed them).
      for (int c = max(0, issued - p.nc); c < issued; ++c) {
        if (!mbar_wait(&cfull[c % p.nc], (c / p.nc) & 1)) ok = false;
      }
      if (issued > 0) {
        const int lt = (g_start + issued - 1) / G;  // the last tile whose scales were requested
        if (!mbar_wait(&sready[lt & 1], (lt >> 1) & 1)) ok = false;
      }
      if (!ok) record_error(p.status, HQ_DEV_TIMEOUT);
    }
    __syncwarp();
  } else if (warp == kBWarp) {
    // ---------------- x' producer (one thread): the chunk's group image
    // (256 Npad bytes, L2-resident) into the x' ring, freed by the MMAs
    if (lane == 0) {
      bool ok = true;
      int issued = 0;
      int sl = 0, g = g_start;
      uint32_t rph = 0;
      const uint8_t* bsrc = p.img + static_cast<size_t>(g_start) * b_bytes;
      uint8_t* bring = smem + p.b_off;
      for (int c = 0; c < total; ++c) {
        if (c >= kNB && !mbar_wait(&bfree[sl], rph ^ 1u)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&bfull[sl], b_bytes);
        bulk_g2s(bring + sl * b_bytes, bsrc, b_bytes, &bfull[sl]);
        issued = c + 1;
        bsrc += b_bytes;
        if (++sl == kNB) {
          sl = 0;
          rph ^= 1u;
        }
        if (++g == G) {
          g = 0;
          bsrc = p.img;
        }
      }
      for (int c = max(0, issued - kNB); c < issued; ++c) {
        if (!mbar_wait(&bfull[c % kNB], (c / kNB) & 1)) ok = false;
      }
      if (!ok) record_error(p.status, HQ_DEV_TIMEOUT);
    }
    __syncwarp();
  } else if (warp >= kEpiWarp0) {
    tc_epilogue(p, tmem, dready, dfree, epib, arrival, cta, g_start, total, last_ti, tile0);
  } else if (warp >= kMmaWarp0) {
    // ---------------- MMA issue: warp j takes chunks j, j + n_mma, ...
    const int j = warp - kMmaWarp0;
    if (j < p.n_mma) {
      bool ok = true;
      // B descriptors: the slot-0, slice-0 descriptor plus start-address steps
      // (in 16-byte units; every address stays below 2^18, so the 14-bit
      // field never carries)
      const uint64_t bdesc0 = smem_desc(smem_u32(smem + p.b_off), 16 * p.Npad, 128);
      const uint32_t slot16 = b_bytes >> 4;
      const uint32_t ks16 = 2u * p.Npad;  // 32 Npad bytes
      const uint32_t acc_set = static_cast<uint32_t>(p.n_mma * p.Npad);  // columns per set
      const int step = p.n_mma;  // divides as, kNB, G and kQuant
      int sl = j, st = j, g = g_start + j, ti = 0;  // x' slot (mod kNB), A stage (mod as)
      uint32_t aph = 0, sph = 0;                    // A-stage and x' slot round parities
      bool first = true;  // the next chunk is this warp's first of its tile portion
      for (int c = j; c < total && ok; c += step) {
        // a new tile portion overwrites its accumulator set: the epilogue of
        // the portion that used the set before must be done with it
        const int buf = p.nacc == 2 ? (ti & 1) : 0, use = p.nacc == 2 ? (ti >> 1) : ti;
        if (first && use > 0) ok = mbar_wait(&dfree[buf], (use - 1) & 1);
        ok = ok && mbar_wait(&aready[st], aph);
        ok = ok && mbar_wait(&bfull[sl], sph);  // the group's x' image has landed
        if (!ok) break;
        tc_fence_after();
        if (lane == 0) {
          const uint32_t dacc = tmem + buf * acc_set + j * p.Npad;
          const uint32_t a0 = tmem + p.a_base + st * 64;
          const uint64_t d0 = bdesc0 + sl * slot16;
          tc_mma_ts(dacc, a0, d0, p.idesc, first ? 0u : 1u);
#pragma unroll
          for (int ks = 1; ks < 8; ++ks) tc_mma_ts(dacc, a0 + ks * 8, d0 + ks * ks16, p.idesc, 1u);
          tc_commit(&bfree[sl]);
          tc_commit(&afree[st]);
          // this warp's last chunk of the portion (tile end or range end)
          if (g + step >= G || c + step >= total) tc_commit(&dready[buf]);
        }
        __syncwarp();
        first = false;
        sl += step;
        if (sl >= kNB) {
          sl -= kNB;
          sph ^= 1u;
        }
        st += step;
        if (st >= p.as) {
          st -= p.as;
          aph ^= 1u;
        }
        g += step;
        if (g >= G) {
          g -= G;
          ++ti;
          first = true;
        }
      }
      // Drain: no MMA may be in flight when tensor memory is freed.
      if (lane == 0) tc_commit(drain);
      __syncwarp();
      if (!mbar_wait(drain, 0)) ok = false;
      if (!ok && lane == 0) record_error(p.status, HQ_DEV_TIMEOUT);
    }
  } else {
    // ---------------- dequant (kDeqWG warpgroups, groups round robin)
    const int wg = warp >> 2;
    const int sub = warp & 3;
    const int r = 32 * sub + lane;  // tile row = TMEM lane
    const uint32_t lane_base = static_cast<uint32_t>(32 * sub) << 16;
    uint32_t add[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) add[i] = p.add[i];
    int prev_ti = -1;
    bool ok = true;
    uint4 scache = make_uint4(0, 0, 0, 0);  // this row's scales for 8 groups
    int sblock = -1;                         // which block of 8 groups scache holds
    // this warpgroup's chunks c = wg, wg + kDeqWG, ...: code slot (mod nc), A
    // stage (mod as), their round parities, group and tile advance
    // incrementally (kDeqWG divides as and nc; kDeqWG < G).  Every round of
    // this warpgroup's slots and stages is waited for by this warpgroup alone,
    // in order, so a parity wait never meets a phase two rounds old.
    int sl = wg, st = wg, g = g_start + wg, ti = 0;
    uint32_t sph = 0, aph = 0;
    for (int c = wg; c < total && ok; c += kDeqWG) {
      if (ti != prev_ti) {
        prev_ti = ti;
        sblock = -1;  // the new tile's scales are in the other buffer
        if (!ok || !mbar_wait(&sready[ti & 1], (ti >> 1) & 1)) {
          ok = false;
          break;
        }
      }
      // the slot's codes have landed, and the A stage's previous MMAs are done
      if (!mbar_wait(&cfull[sl], sph) || (c >= p.as && !mbar_wait(&afree[st], aph ^ 1u))) {
        ok = false;
        break;
      }
      const uint4* rowp = reinterpret_cast<const uint4*>(smem + sl * code_bytes + r * CB);
      if ((g >> 3) != sblock) {  // first group of this warpgroup in a block of 8
        sblock = g >> 3;
        scache = *reinterpret_cast<const uint4*>(smem + p.sbuf_off + (ti & 1) * p.sbuf_bytes +
                                                 r * G * 2 + (g >> 3) * 16);
      }
      const int j = (g >> 1) & 3;
      const uint32_t sw = j == 0 ? scache.x : j == 1 ? scache.y : j == 2 ? scache.z : scache.w;
      const uint32_t s2 = ((g & 1) ? (sw >> 16) : (sw & 0xFFFFu)) * 0x10001u;
      const uint32_t a0 = tmem + lane_base + p.a_base + st * 64;
      uint32_t rw[4 * BITS];  // the row's 128 codes, 16-byte loads
#pragma unroll
      for (int i = 0; i < BITS; ++i) {
        const uint4 u = rowp[code_unit<BITS>(i, r)];
        rw[4 * i] = u.x;
        rw[4 * i + 1] = u.y;
        rw[4 * i + 2] = u.z;
        rw[4 * i + 3] = u.w;
      }
      // the codes (and this block's scales) are in registers: order these
      // generic-proxy reads before the TMA (async proxy) that refills the slot
      fence_proxy_async_smem();
      mbar_arrive(&cfree[sl]);
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        uint32_t w[BITS];
#pragma unroll
        for (int i = 0; i < BITS; ++i) w[i] = rw[t * BITS + i];
        uint32_t P[16];
        decode16<BITS, kMagic1024>(w, P);
#pragma unroll
        for (int i = 0; i < 16; ++i) P[i] = hmul2(hfma2(P[i], pair_mult<BITS>(i), add[i]), s2);
        tc_st16(a0 + 16 * t, P);
      }
      tc_wait_st();
      tc_fence_before();
      mbar_arrive(&aready[st]);
      sl += kDeqWG;
      if (sl >= p.nc) {
        sl -= p.nc;
        sph ^= 1u;
      }
      st += kDeqWG;
      if (st >= p.as) {
        st -= p.as;
        aph ^= 1u;
      }
      g += kDeqWG;
      if (g >= G) {
        g -= G;
        ++ti;
      }
    }
    if (!ok && lane == 0) record_error(p.status, HQ_DEV_TIMEOUT);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
    tmem_relinquish();
  }
}

// ---------------------------------------------------------------- host side
struct TcPlan {
  int nc = 0, b_off = 0, sbuf_off = 0, sbuf_bytes = 0, bar_off = 0;
  size_t smem = 0;
};

constexpr size_t kMaxSmemTc = 227 * 1024 - 1024;  // dynamic; the base is rounded up to 1 KiB
constexpr size_t kMinSmemTc = 116 * 1024;         // > half an SM's shared memory
constexpr size_t kBarBytes = 512;  // 59 mbarriers, the TMEM address and arrival words, 1 mbarrier

// Plan with nc code slots (0 smem when it does not fit): [nc code slots: 128
// rows x 16 bits bytes, swizzled, each a multiple of 1 KiB so every slot keeps
// the swizzle atom][kNB x' image slots of 256 npad bytes][two scale buffers]
// [barriers].
static TcPlan tc_plan_nc(int bits, int K, int npad, int nc) {
  TcPlan pl;
  const int G = K / kGroup;
  pl.nc = nc;
  pl.b_off = nc * kTileM * 16 * bits;
  pl.sbuf_off = pl.b_off + kNB * 256 * npad;
  pl.sbuf_bytes = kTileM * G * 2;
  pl.bar_off = pl.sbuf_off + 2 * pl.sbuf_bytes;
  pl.smem = static_cast<size_t>(pl.bar_off) + kBarBytes + 1024;
  if (pl.smem > kMaxSmemTc) pl.smem = 0;
  return pl;
}

// The deepest code ring that fits: kNCMin..kNCMax slots, even, and at most G
// (a tile's scale buffer is refilled only once every chunk two tiles back has
// read it); smem 0 if none fits.
static TcPlan tc_plan(int bits, int K, int npad) {
  const int G = K / kGroup;
  TcPlan best = tc_plan_nc(bits, K, npad, kNCMin);
  for (int nc = kNCMin + kDeqWG; nc <= std::min(kNCMax, G) && best.smem != 0; nc += kDeqWG) {
    const TcPlan pl = tc_plan_nc(bits, K, npad, nc);
    if (pl.smem == 0) break;
    best = pl;
  }
  // one CTA per SM: each holds all 512 tensor-memory columns
  if (best.smem != 0) best.smem = std::max(best.smem, kMinSmemTc);
  return best;
}

using EncodeTiled = PFN_cuTensorMapEncodeTiled_v12000;

static EncodeTiled encode_tiled() {
  static std::once_flag once;
  static EncodeTiled fn = nullptr;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &f, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess) {
      fn = reinterpret_cast<EncodeTiled>(f);
    }
  });
  return fn;
}

// Codes of W as a 2D byte tensor [M][K bits / 8]; box = one group's 16*bits
// bytes x 128 rows, swizzled for the decoders' row reads.
static cudaError_t code_map(CUtensorMap* map, const void* q, int bits, int M, int K) {
  const CUtensorMapSwizzle swz = bits == 2   ? CU_TENSOR_MAP_SWIZZLE_32B
                                 : bits == 4 ? CU_TENSOR_MAP_SWIZZLE_64B
                                 : bits == 8 ? CU_TENSOR_MAP_SWIZZLE_128B
                                             : CU_TENSOR_MAP_SWIZZLE_NONE;
  const uint64_t row_bytes = static_cast<uint64_t>(K) * bits / 8;
  return tensor_map_2d(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, q, row_bytes, static_cast<uint64_t>(M),
                       row_bytes, static_cast<uint32_t>(16 * bits), kTileM, swz);
}

}  // namespace tc

cudaError_t tensor_map_2d(CUtensorMap* map, CUtensorMapDataType dtype, const void* base, uint64_t inner,
                          uint64_t rows, uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_rows,
                          CUtensorMapSwizzle swizzle) {
  tc::EncodeTiled fn = tc::encode_tiled();
  if (fn == nullptr) return cudaErrorNotSupported;
  const cuuint64_t dims[2] = {inner, rows};
  const cuuint64_t strides[1] = {row_stride_bytes};
  const cuuint32_t box[2] = {box_inner, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = fn(map, dtype, 2, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

cudaError_t tensor_map_3d(CUtensorMap* map, CUtensorMapDataType dtype, const void* base,
                          const uint64_t (&dims)[3], const uint64_t (&strides_bytes)[2],
                          const uint32_t (&box)[3], CUtensorMapSwizzle swizzle) {
  tc::EncodeTiled fn = tc::encode_tiled();
  if (fn == nullptr) return cudaErrorNotSupported;
  const cuuint64_t d[3] = {dims[0], dims[1], dims[2]};
  const cuuint64_t st[2] = {strides_bytes[0], strides_bytes[1]};
  const cuuint32_t b[3] = {box[0], box[1], box[2]};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = fn(map, dtype, 3, const_cast<void*>(base), d, st, b, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

int tc_col_block(int bits, int K) {
  // K >= 1024: whole 16-byte scale rows, and >= 8 groups per tile (a tile's
  // scale buffer is refilled only after the MMAs two tiles back are done)
  if (K < 1024 || K > 32768) return 0;
  for (int nb = 128; nb >= 32; nb -= 32) {
    if (tc::tc_plan(bits, K, nb).smem != 0) return nb;
  }
  return 0;
}

// [images of the batch blocks][shared tiles' partial sums: kMaxTcGrid
// boundaries x 2 sides x 128 rows x nb columns fp32][output factors: nb per
// batch block, fp32]
static size_t tc_img_bytes(int nb, int K, int batch) {
  return (static_cast<size_t>((batch + nb - 1) / nb) * nb * K * 2 + 255) & ~static_cast<size_t>(255);
}
static size_t tc_part_bytes(int nb) { return static_cast<size_t>(kMaxTcGrid) * 2 * tc::kTileM * nb * 4; }
size_t tc_xp_bytes(int bits, int K, int batch) {
  const int nb = tc_col_block(bits, K);
  if (nb == 0) return 0;
  return tc_img_bytes(nb, K, batch) + tc_part_bytes(nb) +
         ((static_cast<size_t>((batch + nb - 1) / nb) * nb * 4 + 255) & ~static_cast<size_t>(255));
}

int tc_launches(int bits, int K, int batch) {
  const int nb = tc_col_block(bits, K);
  return nb == 0 ? 0 : 1 + (batch + nb - 1) / nb;
}

template <int BITS, int LOGK>
static cudaError_t tc_prep_t(const __half* x, const int8_t* s, uint8_t* xp, float* fac, int N,
                             int nb, cudaStream_t st) {
  using S = FwhtShape<LOGK>;
  const float inv = static_cast<float>(1.0 / sqrt(static_cast<double>(S::K)));
  const dim3 grid(nb, (N + nb - 1) / nb);
  return launch_pdl(tc::tc_prep_kernel<BITS, LOGK>, grid, dim3(S::THREADS),
                    (S::SMEM_FLOATS + 32) * sizeof(float), st, true, x, s, xp, fac, N, nb, inv);
}

template <int BITS>
static cudaError_t tc_prep_b(int K, const __half* x, const int8_t* s, uint8_t* xp, float* fac, int N,
                             int nb, cudaStream_t st) {
  switch (K) {
    case 1024: return tc_prep_t<BITS, 10>(x, s, xp, fac, N, nb, st);
    case 2048: return tc_prep_t<BITS, 11>(x, s, xp, fac, N, nb, st);
    case 4096: return tc_prep_t<BITS, 12>(x, s, xp, fac, N, nb, st);
    case 8192: return tc_prep_t<BITS, 13>(x, s, xp, fac, N, nb, st);
    case 16384: return tc_prep_t<BITS, 14>(x, s, xp, fac, N, nb, st);
    case 32768: return tc_prep_t<BITS, 15>(x, s, xp, fac, N, nb, st);
    default: return cudaErrorInvalidValue;
  }
}

template <int BITS>
static void tc_addends(uint32_t (&add)[16], int zero) {
  for (int i = 0; i < 16; ++i) add[i] = pair_addend<BITS>(i, zero);
}

cudaError_t launch_linear_tc(const TcArgs& a, cudaStream_t st) {
  const int nb = tc_col_block(a.bits, a.K);
  if (nb == 0) return cudaErrorInvalidValue;
  uint8_t* xp = static_cast<uint8_t*>(a.xp);
  const __half* xh = reinterpret_cast<const __half*>(a.x);
  float* fac = reinterpret_cast<float*>(xp + tc_img_bytes(nb, a.K, a.N) + tc_part_bytes(nb));
  cudaError_t e;
  switch (a.bits) {
    case 2: e = tc_prep_b<2>(a.K, xh, a.signs, xp, fac, a.N, nb, st); break;
    case 3: e = tc_prep_b<3>(a.K, xh, a.signs, xp, fac, a.N, nb, st); break;
    case 4: e = tc_prep_b<4>(a.K, xh, a.signs, xp, fac, a.N, nb, st); break;
    case 8: e = tc_prep_b<8>(a.K, xh, a.signs, xp, fac, a.N, nb, st); break;
    default: return cudaErrorInvalidValue;
  }
  if (e != cudaSuccess) return e;
  CUtensorMap qmap;
  e = tc::code_map(&qmap, a.q, a.bits, a.M, a.K);
  if (e != cudaSuccess) return e;
  const int n_tiles = (a.M + tc::kTileM - 1) / tc::kTileM;
  // one CTA per SM; the chunks (tile x group) split evenly in quanta, each CTA
  // at least a tile's worth (grid <= n_tiles)
  const int grid_i = std::min(std::min(n_tiles, sm_count()), kMaxTcGrid);
  const unsigned grid = static_cast<unsigned>(grid_i);
  const int quanta = n_tiles * (a.K / kGroup) / tc::kQuant;
  float* part = reinterpret_cast<float*>(xp + tc_img_bytes(nb, a.K, a.N));
  for (int b = 0, n0 = 0; n0 < a.N; ++b, n0 += nb) {
    const int nk = std::min(nb, a.N - n0);
    const int npad = (nk + 31) & ~31;
    const tc::TcPlan pl = tc::tc_plan(a.bits, a.K, npad);
    tc::TcParams p{};
    p.qmap = qmap;
    p.scales = reinterpret_cast<const uint8_t*>(a.scales);
    p.img = xp + static_cast<size_t>(b) * a.K * 2 * nb;
    p.fac = fac + static_cast<size_t>(b) * nb;
    p.y = a.y + static_cast<size_t>(n0) * a.ldy;
    p.status = a.status;
    p.M = a.M;
    p.K = a.K;
    p.N = nk;
    p.Npad = npad;
    p.ldy = a.ldy;
    p.n_tiles = n_tiles;
    p.qq = quanta / grid_i;
    p.qr = quanta % grid_i;
    p.part = part;
    p.flags = a.counters;
    p.b_off = pl.b_off;
    p.sbuf_off = pl.sbuf_off;
    p.sbuf_bytes = pl.sbuf_bytes;
    p.bar_off = pl.bar_off;
    // accumulators: sets of n_mma, one per MMA warp (at N <= 64 an MMA costs
    // its issuer about twice its tensor-pipe time, so four issuers), two sets
    // (so the next tile's MMAs need not wait for the epilogue) while they fit
    // in half of tensor memory, leaving 4 A stages
    p.n_mma = npad <= 64 ? 4 : 2;
    p.nacc = 2 * p.n_mma * npad <= 256 ? 2 : 1;
    p.a_base = (p.nacc * p.n_mma * npad + 63) & ~63;
    p.as = ((tc::kTmemCols - p.a_base) / 64) / p.n_mma * p.n_mma;
    if (p.as > tc::kASMax) p.as = tc::kASMax / p.n_mma * p.n_mma;
    p.nc = pl.nc;
    p.idesc = tc::idesc_f16(tc::kTileM, npad);
    const dim3 g(grid), blk(tc::kThreads);
    switch (a.bits) {
      case 2: tc_addends<2>(p.add, a.zero); e = launch_pdl(tc::tc_gemm_kernel<2>, g, blk, pl.smem, st, true, p); break;
      case 3: tc_addends<3>(p.add, a.zero); e = launch_pdl(tc::tc_gemm_kernel<3>, g, blk, pl.smem, st, true, p); break;
      case 4: tc_addends<4>(p.add, a.zero); e = launch_pdl(tc::tc_gemm_kernel<4>, g, blk, pl.smem, st, true, p); break;
      default: tc_addends<8>(p.add, a.zero); e = launch_pdl(tc::tc_gemm_kernel<8>, g, blk, pl.smem, st, true, p); break;
    }
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace hq
