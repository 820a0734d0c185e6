// gemm_tc.cu -- tensor-core (tcgen05) dequant GEMM for larger batches:
//   y[n][m] = sum_k scale[m][k/128] (q[m][k] - zero) x'[n][k],  N >= 9.
// At batch 16..256 the contraction is a dense one, so it runs on the
// 5th-generation tensor cores with the fp32 accumulator in tensor memory:
//   * a prep kernel rotates x (fp32 butterflies) and writes x' as fp16 in the
//     k order of the decoded code pairs (hq_layout.cuh), so that A and B agree;
//   * per CTA, one 128-row tile at a time: a producer warp streams each 128-code
//     group (codes, scales, and the matching N x 128 block of x') through a
//     4-slot cp.async ring, the B block landing in the canonical no-swizzle
//     K-major core-matrix layout the MMA reads from shared memory;
//   * two warpgroups alternate groups: each thread owns one weight row,
//     decodes its 128 codes into exact fp16 (q - zero) (one LOP3 and one fp16
//     FMA per pair), multiplies by the group scale (one fp16 multiply per pair:
//     the weight's only rounding) and stores the row into tensor memory as the
//     MMA's A operand (tcgen05.st), one TMEM lane per row;
//   * the same producer warp issues 8 tcgen05.mma (M=128, N, K=16, A from TMEM,
//     B from shared memory) per group and commits their completion to the
//     slot's mbarrier; the tile's last commit releases the epilogue, which reads
//     the fp32 accumulator with tcgen05.ld and writes y.
// Waits are bounded (status word on timeout); tensor memory is freed on exit.
#include <algorithm>

#include "fwht.cuh"
#include "hq_common.cuh"
#include "hq_internal.h"
#include "hq_io.cuh"
#include "hq_launch.cuh"
#include "hq_layout.cuh"

namespace hq {
namespace tc {

constexpr int kTileM = 128;
constexpr int kNS = 4;            // ring slots (and A stages in tensor memory)
constexpr int kDeqWarps = 8;      // two warpgroups
constexpr int kThreads = (kDeqWarps + 1) * 32;
constexpr int kTmemCols = 512;
constexpr int kAColBase = 256;    // A stages at columns 256 + 64 s; D at 0

// ---------------------------------------------------------------- tcgen05 wrappers
__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tc_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// Completion of every tcgen05.mma issued so far by this thread arrives once on bar.
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem desc]; M=128, N from idesc, K=16, fp16 in, fp32 out.
__device__ __forceinline__ void tc_mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, {%5, %6, %7, %8}, p;\n\t}" ::"r"(
          d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(0u), "r"(0u), "r"(0u), "r"(0u)
      : "memory");
}

// 16 consecutive 32-bit TMEM columns of this thread's lane <- registers.
__device__ __forceinline__ void tc_st16(uint32_t taddr, const uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
      "%14,%15,%16};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
      "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
      : "memory");
}

// registers <- 16 consecutive 32-bit TMEM columns of this thread's lane.
__device__ __forceinline__ void tc_ld16(uint32_t taddr, uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,"
      "%15}, [%16];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
        "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]),
        "=r"(v[14]), "=r"(v[15])
      : "r"(taddr)
      : "memory");
}

// Shared-memory matrix descriptor, no swizzle, K-major: core matrices of
// 8 rows x 16 bytes; lbo = byte distance between the two core matrices along
// K, sbo = byte distance between consecutive 8-row groups.
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
  return static_cast<uint64_t>((addr >> 4) & 0x3FFFu) |
         (static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16) |
         (static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46);
}

// Instruction descriptor: fp32 accumulate, fp16 A and B, both K-major.
__host__ __device__ constexpr uint32_t idesc_f16(int M, int N) {
  return (1u << 4) | (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}

// ---------------------------------------------------------------- prep: rotate + permute
// One CTA per batch row: x'[n] (fp16) in the k order of the decoded pairs:
// position 128 g + 32 t + 2 p + h holds x'[128 g + 32 t + code(p, h)].
template <int BITS, int LOGK>
__global__ void __launch_bounds__(FwhtShape<LOGK>::THREADS)
    tc_prep_kernel(const __half* __restrict__ x, const int8_t* __restrict__ signs,
                   __half* __restrict__ xp, float inv) {
  using S = FwhtShape<LOGK>;
  extern __shared__ float buf[];
  pdl_launch_dependents();
  pdl_wait();
  const int tid = threadIdx.x, n = blockIdx.x;
  float v[S::E];
  load_chunk<__half, S::E>(x + static_cast<size_t>(n) * S::K + tid * S::E, v);
  apply_signs<S::E>(signs ? signs + tid * S::E : nullptr, v);
  fwht_block<LOGK, 5>(v, buf);
  __half* out = xp + static_cast<size_t>(n) * S::K;
  for (int i = tid; i < S::K; i += S::THREADS) {
    const int g = i >> 7, t = (i >> 5) & 3, p = (i >> 1) & 15, h = i & 1;
    const PairDesc pd = Pairs<BITS>::get(p);
    const int k = kGroup * g + 32 * t + (h ? pd.c_hi : pd.c_lo);
    out[i] = __float2half_rn(buf[fwht_pad(k)] * inv);
  }
}


// ---------------------------------------------------------------- the GEMM
struct TcParams {
  const uint32_t* q;
  const __half* scales;
  const __half* xp;  // [N][K] rotated, pair-permuted activations
  float* y;
  uint32_t* status;
  int M, K, N, Npad, ldy;
  int n_tiles;
  int cstride;     // bytes between code rows in a slot
  int slot_bytes;  // codes + B block
  int b_off;       // B block offset inside a slot
  int sbuf_off;    // per-tile scale buffers (two)
  int sbuf_bytes;
  int sstride;     // bytes between scale rows in a scale buffer
  int bar_off;
  uint32_t idesc;
  uint32_t add[16];
};

template <int BITS>
__global__ void __launch_bounds__(kThreads, 1) tc_gemm_kernel(const __grid_constant__ TcParams p) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = p.K / kGroup;
  const int CB = 16 * BITS;  // code bytes of one row in one 128-code group
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + p.bar_off);
  uint64_t* freeb = full + kNS;
  uint64_t* aready = freeb + kNS;
  uint64_t* dready = aready + kNS;
  uint64_t* dfree = dready + 1;
  uint64_t* drain = dfree + 1;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);
  __shared__ int abort_flag;

  if (tid == 0) {
    for (int i = 0; i < kNS; ++i) {
      mbar_init(&full[i], 32);
      mbar_init(&freeb[i], 1);
      mbar_init(&aready[i], 128);
    }
    mbar_init(dready, 1);
    mbar_init(dfree, 2 * 128);
    mbar_init(drain, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) tmem_alloc(tmem_holder, kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  pdl_launch_dependents();
  pdl_wait();

  const int n_my = (p.n_tiles - static_cast<int>(blockIdx.x) + gridDim.x - 1) / gridDim.x;
  const int total = n_my * G;

  if (warp == kDeqWarps) {
    // ---------------- producer + MMA issue
    const uint8_t* qb = reinterpret_cast<const uint8_t*>(p.q);
    const size_t row_bytes = static_cast<size_t>(p.K) * BITS / 8;
    auto load = [&](int c) {
      const int sl = c % kNS, ti = c / G, g = c % G;
      const int m0 = (static_cast<int>(blockIdx.x) + ti * static_cast<int>(gridDim.x)) * kTileM;
      uint8_t* base = smem + sl * p.slot_bytes;
      if (g == 0) {  // the tile's scales: rows m0..m0+127, all groups, padded rows
        uint8_t* sb = smem + p.sbuf_off + (ti & 1) * p.sbuf_bytes;
        const int row_b = G * 2, pieces = (row_b + 15) >> 4;
        for (int i = lane; i < kTileM * pieces; i += 32) {
          const int r = i / pieces, pc = i - r * pieces;
          const int nb = (m0 + r < p.M) ? min(16, row_b - pc * 16) : 0;
          const uint8_t* src = reinterpret_cast<const uint8_t*>(p.scales) +
                               (nb ? (static_cast<size_t>(m0 + r) * G * 2 + pc * 16) : 0);
          cp_async16(sb + r * p.sstride + pc * 16, src, nb);
        }
      }
      for (int i = lane; i < kTileM * BITS; i += 32) {
        const int r = i / BITS, c16 = i - r * BITS;
        const bool ok = m0 + r < p.M;
        const uint8_t* src = ok ? qb + static_cast<size_t>(m0 + r) * row_bytes +
                                      static_cast<size_t>(g) * CB + c16 * 16
                                : qb;
        cp_async16(base + r * p.cstride + c16 * 16, src, ok ? 16 : 0);
      }
      uint8_t* bdst = base + p.b_off;
      for (int i = lane; i < 16 * p.Npad; i += 32) {
        const int n = i >> 4, ks = (i >> 1) & 7, kc = i & 1;
        const bool ok = n < p.N;
        const __half* src = ok ? p.xp + static_cast<size_t>(n) * p.K + g * kGroup + ks * 16 + kc * 8 : p.xp;
        cp_async16(bdst + ks * 32 * p.Npad + kc * 16 * p.Npad + (n >> 3) * 128 + (n & 7) * 16, src,
                   ok ? 16 : 0);
      }
      cp_async_mbar_arrive(&full[sl]);
    };
    for (int c = 0; c < kNS && c < total; ++c) load(c);
    bool ok = true;
    for (int c = 0; c < total && ok; ++c) {
      const int sl = c % kNS, ti = c / G, g = c % G;
      if (g == 0 && ti > 0) ok = mbar_wait(dfree, (ti - 1) & 1);
      ok = ok && mbar_wait(&aready[sl], (c / kNS) & 1);
      if (!ok) break;
      tc_fence_after();
      if (lane == 0) {
        const uint32_t a0 = tmem + kAColBase + sl * 64;
        const uint32_t b0 = smem_u32(smem + sl * p.slot_bytes + p.b_off);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          const uint64_t bd = smem_desc(b0 + ks * 32 * p.Npad, 16 * p.Npad, 128);
          tc_mma_ts(tmem, a0 + ks * 8, bd, p.idesc, (g > 0 || ks > 0) ? 1u : 0u);
        }
        tc_commit(&freeb[sl]);
        if (g == G - 1) tc_commit(dready);
      }
      __syncwarp();
      if (c >= 1 && c - 1 + kNS < total) {
        ok = mbar_wait(&freeb[(c - 1) % kNS], ((c - 1) / kNS) & 1);
        if (ok) load(c - 1 + kNS);
      }
    }
    if (!ok) {
      if (lane == 0) {
        record_error(p.status, HQ_DEV_TIMEOUT);
        atomicExch(&abort_flag, 1);
      }
    }
    // Drain: no copy or MMA of this CTA may be in flight when tensor memory
    // is freed (matters only after a timeout; a no-op on the normal path).
    asm volatile("cp.async.wait_all;" ::: "memory");
    if (lane == 0) tc_commit(drain);
    __syncwarp();
    if (!mbar_wait(drain, 0) && lane == 0) record_error(p.status, HQ_DEV_TIMEOUT);
  } else {
    // ---------------- dequant (two warpgroups, alternate groups) + epilogue
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
    auto epilogue = [&](int ti) {
      if (!mbar_wait(dready, ti & 1)) {
        ok = false;
        return;
      }
      tc_fence_after();
      const int m = (static_cast<int>(blockIdx.x) + ti * static_cast<int>(gridDim.x)) * kTileM + r;
      const int half = p.Npad / 2;
      for (int c0 = wg * half; c0 < (wg + 1) * half; c0 += 16) {
        uint32_t v[16];
        tc_ld16(tmem + lane_base + c0, v);
        tc_wait_ld();
        if (m < p.M) {
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int n = c0 + j;
            if (n < p.N) p.y[static_cast<size_t>(n) * p.ldy + m] = __uint_as_float(v[j]);
          }
        }
      }
      tc_fence_before();
      mbar_arrive(dfree);
    };
    for (int c = wg; c < total && ok; c += 2) {
      const int sl = c % kNS, ti = c / G, g = c % G;
      if (ti != prev_ti) {
        if (prev_ti >= 0) epilogue(prev_ti);
        prev_ti = ti;
        if (!ok) break;
      }
      if (!mbar_wait(&full[sl], (c / kNS) & 1)) {
        ok = false;
        break;
      }
      const uint8_t* rowp = smem + sl * p.slot_bytes + r * p.cstride;
      if ((g & 7) < 2) {  // first group of this warpgroup in a block of 8
        scache = *reinterpret_cast<const uint4*>(smem + p.sbuf_off + (ti & 1) * p.sbuf_bytes +
                                                 r * p.sstride + (g >> 3) * 16);
      }
      const int j = (g >> 1) & 3;
      const uint32_t sw = j == 0 ? scache.x : j == 1 ? scache.y : j == 2 ? scache.z : scache.w;
      const uint32_t s2 = ((g & 1) ? (sw >> 16) : (sw & 0xFFFFu)) * 0x10001u;
      const uint32_t a0 = tmem + lane_base + kAColBase + sl * 64;
      uint32_t rw[4 * BITS];  // the row's 128 codes, 16-byte loads
#pragma unroll
      for (int i = 0; i < BITS; ++i) {
        const uint4 u = reinterpret_cast<const uint4*>(rowp)[i];
        rw[4 * i] = u.x;
        rw[4 * i + 1] = u.y;
        rw[4 * i + 2] = u.z;
        rw[4 * i + 3] = u.w;
      }
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
      // the slot's B block arrived through cp.async (generic proxy); the MMA
      // reads it through the async proxy
      fence_proxy_async_smem();
      mbar_arrive(&aready[sl]);
    }
    if (ok && prev_ti >= 0) epilogue(prev_ti);
    if (!ok) {
      if (lane == 0) record_error(p.status, HQ_DEV_TIMEOUT);
      atomicExch(&abort_flag, 1);
    }
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
  int cstride = 0, slot = 0, b_off = 0, sbuf_off = 0, sbuf_bytes = 0, sstride = 0, bar_off = 0;
  size_t smem = 0;
};

constexpr size_t kMaxSmemTc = 226 * 1024;  // dynamic; leaves room for the static words
constexpr size_t kMinSmemTc = 116 * 1024;  // > half an SM's shared memory

static TcPlan tc_plan(int bits, int K, int npad) {
  TcPlan pl;
  const int G = K / kGroup;
  // code rows: 16*bits bytes, padded to an odd number of 16-byte units so that
  // the 16-byte row loads of 8 consecutive threads hit distinct banks
  pl.cstride = 16 * bits + ((bits & 1) ? 0 : 16);
  pl.b_off = (kTileM * pl.cstride + 127) & ~127;
  pl.slot = pl.b_off + 256 * npad;
  pl.sbuf_off = kNS * pl.slot;
  // scale rows padded to an odd number of 16-byte units (conflict-free uint4 reads)
  pl.sstride = ((G * 2 + 15) & ~15);
  if (((pl.sstride >> 4) & 1) == 0) pl.sstride += 16;
  pl.sbuf_bytes = kTileM * pl.sstride;
  pl.bar_off = (pl.sbuf_off + 2 * pl.sbuf_bytes + 15) & ~15;
  pl.smem = static_cast<size_t>(pl.bar_off) + (3 * kNS + 3) * 8 + 16;
  // one CTA per SM: each holds all 512 tensor-memory columns
  pl.smem = std::max(pl.smem, kMinSmemTc);
  return pl;
}

}  // namespace tc

int tc_col_block(int bits, int K) {
  // K >= 1024: whole 16-byte scale pieces per row, and >= 8 groups per tile
  // (a tile's scale buffer is reloaded only after the previous tile's MMAs)
  if (K < 1024) return 0;
  for (int nb = 128; nb >= 32; nb -= 32) {
    if (tc::tc_plan(bits, K, nb).smem <= tc::kMaxSmemTc) return nb;
  }
  return 0;
}

template <int BITS, int LOGK>
static cudaError_t tc_prep_t(const __half* x, const int8_t* s, __half* xp, int N, cudaStream_t st) {
  using S = FwhtShape<LOGK>;
  const float inv = static_cast<float>(1.0 / sqrt(static_cast<double>(S::K)));
  return launch_pdl(tc::tc_prep_kernel<BITS, LOGK>, dim3(N), dim3(S::THREADS),
                    S::SMEM_FLOATS * sizeof(float), st, true, x, s, xp, inv);
}

template <int BITS>
static cudaError_t tc_prep_b(int K, const __half* x, const int8_t* s, __half* xp, int N,
                             cudaStream_t st) {
  switch (K) {
    case 512: return tc_prep_t<BITS, 9>(x, s, xp, N, st);
    case 1024: return tc_prep_t<BITS, 10>(x, s, xp, N, st);
    case 2048: return tc_prep_t<BITS, 11>(x, s, xp, N, st);
    case 4096: return tc_prep_t<BITS, 12>(x, s, xp, N, st);
    case 8192: return tc_prep_t<BITS, 13>(x, s, xp, N, st);
    case 16384: return tc_prep_t<BITS, 14>(x, s, xp, N, st);
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
  __half* xp = static_cast<__half*>(a.xp);
  const __half* xh = reinterpret_cast<const __half*>(a.x);
  cudaError_t e;
  switch (a.bits) {
    case 2: e = tc_prep_b<2>(a.K, xh, a.signs, xp, a.N, st); break;
    case 3: e = tc_prep_b<3>(a.K, xh, a.signs, xp, a.N, st); break;
    case 4: e = tc_prep_b<4>(a.K, xh, a.signs, xp, a.N, st); break;
    case 8: e = tc_prep_b<8>(a.K, xh, a.signs, xp, a.N, st); break;
    default: return cudaErrorInvalidValue;
  }
  if (e != cudaSuccess) return e;
  const int n_tiles = (a.M + tc::kTileM - 1) / tc::kTileM;
  const unsigned grid = static_cast<unsigned>(std::min(n_tiles, gemv_max_warps() / 8));
  for (int n0 = 0; n0 < a.N; n0 += nb) {
    const int nk = std::min(nb, a.N - n0);
    const int npad = (nk + 31) & ~31;
    const tc::TcPlan pl = tc::tc_plan(a.bits, a.K, npad);
    tc::TcParams p{};
    p.q = a.q;
    p.scales = reinterpret_cast<const __half*>(a.scales);
    p.xp = xp + static_cast<size_t>(n0) * a.K;
    p.y = a.y + static_cast<size_t>(n0) * a.ldy;
    p.status = a.status;
    p.M = a.M;
    p.K = a.K;
    p.N = nk;
    p.Npad = npad;
    p.ldy = a.ldy;
    p.n_tiles = n_tiles;
    p.cstride = pl.cstride;
    p.slot_bytes = pl.slot;
    p.b_off = pl.b_off;
    p.sbuf_off = pl.sbuf_off;
    p.sbuf_bytes = pl.sbuf_bytes;
    p.sstride = pl.sstride;
    p.bar_off = pl.bar_off;
    p.idesc = tc::idesc_f16(tc::kTileM, npad);
    const dim3 g(grid), b(tc::kThreads);
    switch (a.bits) {
      case 2: tc_addends<2>(p.add, a.zero); e = launch_pdl(tc::tc_gemm_kernel<2>, g, b, pl.smem, st, true, p); break;
      case 3: tc_addends<3>(p.add, a.zero); e = launch_pdl(tc::tc_gemm_kernel<3>, g, b, pl.smem, st, true, p); break;
      case 4: tc_addends<4>(p.add, a.zero); e = launch_pdl(tc::tc_gemm_kernel<4>, g, b, pl.smem, st, true, p); break;
      default: tc_addends<8>(p.add, a.zero); e = launch_pdl(tc::tc_gemm_kernel<8>, g, b, pl.smem, st, true, p); break;
    }
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace hq
