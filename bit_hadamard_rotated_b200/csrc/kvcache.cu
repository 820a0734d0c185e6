// kvcache.cu -- the int4 KV cache ("Runtime int4 (keys per channel per 32-token
// block, values per token)": LLaDA2.2-mini Orin-Nano model card, Properties
// table).  hq_kv_append quantises new keys and values into the cache;
// hq_kv_attend runs softmax attention of a block of query tokens over it,
// reading the 4-bit codes straight into tensor-core operands.
//
// Quantiser (this library's reading of the card: asymmetric min/scale, 4-bit
// codes), per group of values x in IEEE single precision:
//   scale = fp16((max x - min x) / 15), mn = fp16(min x),
//   code  = clamp(rint((x - mn) / scale), 0, 15)   (0 where scale = 0),
// so x ~ scale * code + mn.  A key group is one channel of one kv head over a
// 32-token block, a value group all head_dim channels of one kv head for one
// token.
//
// Memory layout (per kv head h, 32-token block b; chosen so that both
// products below read their operand straight from the codes):
//   keys   k_codes [h][b][token 32][d/2]   token-major: channel c in byte c/2
//                                           (low nibble for even c)
//          k_scale, k_min [h][b][d]        fp16
//   values v_codes [h][b][channel d][16]   channel-major: token t in byte t/2
//                                           (low nibble for even t)
//          v_scale, v_min [h][token]       fp16
//
// Attention (split over the context, flash-decoding style): kv_attn_kernel
// takes one kv head, one group of 128 query rows (a row is one query token
// of one head of the kv head's group) and a chunk of 128-token steps per CTA,
// about one CTA per SM, on the 5th-generation tensor cores:
//   producer warps   copy each step's codes (cp.async) and write the MMA
//                    operands into shared memory: key planes s_hi code and
//                    s_lo code (the scale split so that both products with a
//                    4-bit code are exact in fp16) plus the 4 blocks' minima
//                    as extra key rows, and the value codes as exact fp16;
//   score issuer     S = Q [Khi | minima]^T + Q Klo^T (M = 128, N = 144) into
//                    one of two tensor-memory buffers;
//   softmax warps    4 threads per row read their 32 scores once, add the
//                    block's minima term, keep a reference maximum that moves
//                    (rescaling O in tensor memory) only when a row's maximum
//                    exceeds it by 2^8, and write P = 2^(S c2 - m) v_scale as
//                    fp16 hi + lo over the scores it came from;
//   P.V issuer       O += P V^T with P from tensor memory (M = 128, N = d);
// plus sum_t p v_min added to every channel at the end.  Every product of a
// score is exact; sums are fp32.  The chunk's (max, sum, O) go to the
// workspace; kv_combine_kernel merges the chunks of each row.
#include <cuda_fp16.h>

#include <algorithm>

#include "hq_common.cuh"
#include "hq_internal.h"
#include "hq_launch.cuh"
#include "tcgen05.cuh"

namespace hq {
namespace kv {

constexpr int kRows = 128;  // query rows per CTA (the MMAs' M)
constexpr int kTargetCtas = 148;    // one wave over the SMs
constexpr int kMaxRows = 4096;

// Floats per row of a chunk's partial result: D outputs, max, exp-sum, two
// pad floats so that rows start on 16-byte boundaries.
template <int D>
constexpr int kPartRow = D + 4;

struct Cache {
  int d, n_kv, cap;
  const uint8_t* kc;
  const __half* ks;
  const __half* km;
  const uint8_t* vc;
  const __half* vs;
  const __half* vm;
};

// ---------------------------------------------------------------- quantiser

// The single-precision steps of the quantiser, in the oracle's order.
struct Quant {
  float s, m;
  __half s16, m16;
  __device__ __forceinline__ Quant(float lo, float hi) {
    const float sf = __fdiv_rn(__fsub_rn(hi, lo), 15.f);
    s16 = __float2half_rn(sf);
    m16 = __float2half_rn(lo);
    s = __half2float(s16);
    m = __half2float(m16);
  }
  __device__ __forceinline__ uint32_t code(float x) const {
    if (!(s > 0.f)) return 0u;
    const float r = rintf(__fdiv_rn(__fsub_rn(x, m), s));
    return static_cast<uint32_t>(fminf(fmaxf(r, 0.f), 15.f));
  }
};

// Keys of one 32-token block of kv head blockIdx.y: d threads, thread =
// channel (its group); codes staged in shared memory, then packed token-major.
__global__ void kv_append_k_kernel(int d, int n_kv, int cap, uint8_t* __restrict__ kc, __half* __restrict__ ks,
                                   __half* __restrict__ km, const __half* __restrict__ k, int pos) {
  __shared__ uint8_t codes[32][128];
  pdl_launch_dependents();
  pdl_wait();
  const int ch = threadIdx.x, h = blockIdx.y, b = blockIdx.x;
  const size_t row = static_cast<size_t>(n_kv) * d;
  const __half* src = k + static_cast<size_t>(32) * b * row + static_cast<size_t>(h) * d + ch;
  float x[32];
  float lo = 0.f, hi = 0.f;
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    x[i] = __half2float(src[i * row]);
    lo = i == 0 ? x[i] : fminf(lo, x[i]);
    hi = i == 0 ? x[i] : fmaxf(hi, x[i]);
  }
  const Quant q(lo, hi);
#pragma unroll
  for (int i = 0; i < 32; ++i) codes[i][ch] = static_cast<uint8_t>(q.code(x[i]));
  const size_t blk = static_cast<size_t>(h) * (cap / 32) + pos / 32 + b;
  ks[blk * d + ch] = q.s16;
  km[blk * d + ch] = q.m16;
  __syncthreads();
  // 32 tokens x d/2 bytes, one 32-bit word (8 channels) per step
  uint32_t* dst = reinterpret_cast<uint32_t*>(kc + blk * 32 * (d / 2));
  const int words = 32 * d / 8;
  for (int w = ch; w < words; w += d) {
    const int t = w / (d / 8), c0 = (w % (d / 8)) * 8;
    uint32_t v = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) v |= static_cast<uint32_t>(codes[t][c0 + j]) << (4 * j);
    dst[w] = v;
  }
}

// Values of one 32-token block of kv head blockIdx.y: d threads, thread =
// channel; each token's group is the d channels (min and max through warp
// shuffles and shared memory); each thread packs its channel's 32 codes.
__global__ void kv_append_v_kernel(int d, int n_kv, int cap, uint8_t* __restrict__ vc, __half* __restrict__ vs,
                                   __half* __restrict__ vm, const __half* __restrict__ v, int pos) {
  __shared__ float red[2][32][4];
  pdl_launch_dependents();
  pdl_wait();
  const int ch = threadIdx.x, lane = ch & 31, warp = ch >> 5, nw = d / 32;
  const int h = blockIdx.y, b = blockIdx.x;
  const size_t row = static_cast<size_t>(n_kv) * d;
  const __half* src = v + static_cast<size_t>(32) * b * row + static_cast<size_t>(h) * d + ch;
  float x[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    x[i] = __half2float(src[i * row]);
    float lo = x[i], hi = x[i];
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) {
      lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
      hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
    }
    if (lane == 0) {
      red[0][i][warp] = lo;
      red[1][i][warp] = hi;
    }
  }
  __syncthreads();
  uint32_t w[4] = {0u, 0u, 0u, 0u};
  const size_t tok0 = static_cast<size_t>(h) * cap + pos + 32 * b;
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    float lo = red[0][i][0], hi = red[1][i][0];
    for (int j = 1; j < nw; ++j) {
      lo = fminf(lo, red[0][i][j]);
      hi = fmaxf(hi, red[1][i][j]);
    }
    const Quant q(lo, hi);
    w[i >> 3] |= q.code(x[i]) << (4 * (i & 7));
    if (ch == i) {
      vs[tok0 + i] = q.s16;
      vm[tok0 + i] = q.m16;
    }
  }
  const size_t blk = static_cast<size_t>(h) * (cap / 32) + pos / 32 + b;
  *reinterpret_cast<uint4*>(vc + (blk * d + ch) * 16) = make_uint4(w[0], w[1], w[2], w[3]);
}

// ---------------------------------------------------------------- attention

__device__ __forceinline__ uint32_t h2u(__half2 h) { return *reinterpret_cast<uint32_t*>(&h); }

// Byte j of w (two 4-bit codes) as the exact fp16 pair (low nibble, high
// nibble): the byte is copied to bits 0-7 and 16-23, the nibbles are masked
// into the mantissas of 1024 and 1024 + 16 n_hi, and one fused multiply-add
// takes (1024 + n_lo, 1024 + 16 n_hi) to (n_lo, n_hi), every step exact.
__device__ __forceinline__ __half2 nibble_pair(uint32_t w, int j) {
  const uint32_t sel = static_cast<uint32_t>(j) | 0x40u | (static_cast<uint32_t>(j) << 8) | 0x4000u;
  const uint32_t x = and_or(prmt(w, 0u, sel), 0x00F0000Fu, 0x64006400u);
  const __half2 scale = __halves2half2(__float2half_rn(1.f), __float2half_rn(0.0625f));
  const __half2 bias = __halves2half2(__float2half_rn(-1024.f), __float2half_rn(-64.f));
  return __hfma2(*reinterpret_cast<const __half2*>(&x), scale, bias);
}

__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// 2^x (PTX ex2.approx, relative error about 2^-22); exp(s) is taken as
// 2^(s log2 e) with log2 e folded into the score scale.
__device__ __forceinline__ float exp2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Roles of the 832 threads of an attention CTA.
constexpr int kAttThreads = 832;
constexpr int kSoftWarps = 16;   // warps 0-15: warp w takes rows 32 (w % 4) + lane (its tensor-memory
                                 // lane quarter) and column quarter w / 4
constexpr int kProdWarp0 = 16;   // warps 16-23: copies and dequantisation
constexpr int kQkWarp = 24;      // warp 24, lane 0: score MMAs
constexpr int kPvWarp = 25;      // warp 25, lane 0: P.V MMAs (a second issuer: the two run concurrently)
constexpr int kProdThreads = 256, kSoftThreads = 512;
constexpr int kStep = 128;       // tokens per step (4 key blocks): the MMAs' N and K extents
constexpr int kKRows = 144;      // key tile rows: 128 tokens, then the 4 blocks' minima, 12 zero rows
constexpr int kSCols = 160;      // tensor-memory columns of one score buffer (144 used)
constexpr int kOCol = 2 * kSCols;  // O at columns 320 .. 320 + D
constexpr int kTmemCols = 512;

// Named barriers (id 0 is __syncthreads'): 1 the producer threads, 2 the
// softmax threads.  *_all returns the AND of v over them, so that they leave
// a loop together when any bounded wait ran out.
template <int N>
__device__ __forceinline__ void named_sync(int id) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "n"(N) : "memory");
}
template <int N>
__device__ __forceinline__ bool named_all(int id, bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %2, 0;\n\t"
      "bar.red.and.pred q, %1, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(id), "r"(v ? 1u : 0u), "n"(N)
      : "memory");
  return r != 0;
}

// Operand tiles in shared memory, fp16, K-major without swizzle: core
// matrices of 8 rows x 8 elements (128 contiguous bytes), element (row, k) at
// (k / 8) rows 16 + (row / 8) 128 + (row % 8) 16 + (k % 8) 2 for a tile of
// `rows` rows: an MMA's K = 16 slice starting at element k0 is the descriptor
// (base + k0 rows 2, LBO = rows 16, SBO = 128).
__device__ __forceinline__ uint32_t tile_off(int rows, int row, int k8) {
  return k8 * rows * 16 + (row >> 3) * 128 + (row & 7) * 16;
}

template <int D>
struct AttLayout {
  static constexpr int kQ = 0;                      // Q [128 rows][D]
  static constexpr int kKhi = kQ + 256 * D;          // key planes [144 rows][D]: s_hi code (tokens), then
  static constexpr int kKlo = kKhi + 288 * D;        //   the minima (hi plane) / zeros; s_lo code (lo plane)
  static constexpr int kV = kKlo + 288 * D;          // value codes [2 steps][D channels][128 tokens]
  static constexpr int kRawK = kV + 512 * D;         // the step's key codes (4 blocks x 32 tokens x D/2),
  static constexpr int kRawKs = kRawK + 64 * D;      //   scales (4 blocks x D fp16),
  static constexpr int kRawKm = kRawKs + 8 * D;      //   minima
  static constexpr int kRawV = kRawKm + 8 * D;       // the step's value codes (4 blocks x D x 16 bytes),
  static constexpr int kRawVs = kRawV + 64 * D;      //   scales (128 fp16),
  static constexpr int kRawVm = kRawVs + 256;        //   minima
  static constexpr int kKsh = kRawVm + 256;          // key scales split s = s_hi + s_lo, fp16 [2][4 blocks][D]
  static constexpr int kVsf = kKsh + 16 * D;         // value scales and minima as floats [2 steps][2][128]
  static constexpr int kVmx = kVsf + 2 * 2 * 128 * 4;  // largest value scale of a step [2 steps][4 warps]
  static constexpr int kXch = kVmx + 32;             // softmax exchange [4 parts][3][128] floats
  static constexpr int kBars = kXch + 4 * 3 * 128 * 4;
  static constexpr int kNumBars = 14;
  static constexpr int kHolder = kBars + 8 * kNumBars;
  static constexpr int kBytes = kHolder + 16;
};

// Barriers, each waited for in phase order by its agents (no agent can fall
// two phases behind: every next phase needs work that follows the wait):
//   k_full     256 producer arrivals: the step's key planes           (QK issuer)
//   k_empty    commit: the step's score MMAs have read them            (producer)
//   v_full b   256 producer arrivals: value codes and scales in buffer b
//                                                           (PV issuer, softmax)
//   v_empty b  commit: the P.V MMAs have read buffer b                 (producer)
//   s_full b   commit: a step's scores in tensor-memory buffer b       (softmax)
//   s_free b   commit: the P.V MMAs have read P from buffer b          (QK issuer)
//   p_full     256 softmax arrivals: P written over the scores         (PV issuer)
//   o_done     commit: a step's P.V done (O stable)                    (softmax)
//   qk_end, pv_end  commit: every MMA of that issuer complete       (the issuer)
enum {
  kBarKFull = 0, kBarKEmpty, kBarVFull0, kBarVFull1, kBarVEmpty0, kBarVEmpty1, kBarSFull0, kBarSFull1,
  kBarSFree0, kBarSFree1, kBarPFull, kBarODone, kBarQkEnd, kBarPvEnd
};

// The copies of step i's raw cache bytes (blocks b0 .. b0 + 3 that exist),
// by the 256 producer threads; keys and values separately so that each part
// can be reloaded as soon as its last reader is done.  A key token row is
// written with its 16-byte pieces XOR-swizzled so that 8 consecutive tokens'
// pieces fall in distinct bank groups.
template <int D>
__device__ __forceinline__ int key_swz(int t) {
  return (t / (256 / D)) & (D / 32 - 1);
}

template <int D>
__device__ __forceinline__ void raw_keys_issue(uint8_t* smem, const Cache& c, int h, int b0, int nbT, int pt) {
  using L = AttLayout<D>;
  constexpr int kPieces = D / 32;  // 16-byte pieces of a token's codes
  const int nbk = min(4, nbT - b0);
  const size_t blk = static_cast<size_t>(h) * (c.cap / 32) + b0;
  const uint8_t* kc = c.kc + blk * 16 * D;
  for (int i = pt; i < nbk * 32 * kPieces; i += kProdThreads) {
    const int t = i / kPieces, q = i % kPieces;
    cp_async16(smem + L::kRawK + t * (D / 2) + 16 * (q ^ key_swz<D>(t)), kc + 16 * i, 16u);
  }
  const uint8_t* ks = reinterpret_cast<const uint8_t*>(c.ks + blk * D);
  const uint8_t* km = reinterpret_cast<const uint8_t*>(c.km + blk * D);
  for (int i = pt; i < nbk * D / 8; i += kProdThreads) {
    cp_async16(smem + L::kRawKs + 16 * i, ks + 16 * i, 16u);
    cp_async16(smem + L::kRawKm + 16 * i, km + 16 * i, 16u);
  }
}

template <int D>
__device__ __forceinline__ void raw_values_issue(uint8_t* smem, const Cache& c, int h, int b0, int nbT, int pt) {
  using L = AttLayout<D>;
  const int nbk = min(4, nbT - b0);
  const size_t blk = static_cast<size_t>(h) * (c.cap / 32) + b0;
  const uint8_t* vc = c.vc + blk * 16 * D;
  for (int i = pt; i < nbk * D; i += kProdThreads) cp_async16(smem + L::kRawV + 16 * i, vc + 16 * i, 16u);
  const uint8_t* vs = reinterpret_cast<const uint8_t*>(c.vs + static_cast<size_t>(h) * c.cap + 32 * b0);
  const uint8_t* vm = reinterpret_cast<const uint8_t*>(c.vm + static_cast<size_t>(h) * c.cap + 32 * b0);
  for (int i = pt; i < nbk * 4; i += kProdThreads) {
    cp_async16(smem + L::kRawVs + 16 * i, vs + 16 * i, 16u);
    cp_async16(smem + L::kRawVm + 16 * i, vm + 16 * i, 16u);
  }
}

// The step's key scales split as s = s_hi + s_lo, s_hi keeping 7 significant
// bits (the fp16 pattern with its 4 low mantissa bits cleared), so that
// s_hi code (<= 11 bits) and s_lo code (<= 8 bits) are exact fp16 products;
// and the blocks' minima as rows 128 .. 131 of the hi key plane (zero for
// blocks past the context), so that the score MMA also yields sum_c q_c min_c
// per block in score columns 128 .. 131.
template <int D>
__device__ __forceinline__ void key_scales_store(uint8_t* smem, int pt, int nbk) {
  using L = AttLayout<D>;
  const uint16_t* ks = reinterpret_cast<const uint16_t*>(smem + L::kRawKs);
  uint16_t* sh = reinterpret_cast<uint16_t*>(smem + L::kKsh);
  for (int i = pt; i < nbk * D; i += kProdThreads) {
    const uint16_t sb = ks[i];
    const uint16_t hb = sb & 0xFFF0u;
    sh[i] = hb;
    sh[4 * D + i] = __half_as_ushort(__hsub(__ushort_as_half(sb), __ushort_as_half(hb)));
  }
  if (pt < 4 * (D / 8)) {
    const int blk = pt / (D / 8), c8 = pt % (D / 8);
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (blk < nbk) v = reinterpret_cast<const uint4*>(smem + L::kRawKm)[blk * (D / 8) + c8];
    *reinterpret_cast<uint4*>(smem + L::kKhi + tile_off(kKRows, kStep + blk, c8)) = v;
  }
}

// Zero rows of the key planes that no step writes: hi rows 132 .. 143, lo
// rows 128 .. 143.
template <int D>
__device__ __forceinline__ void key_pad_rows(uint8_t* smem, int pt) {
  using L = AttLayout<D>;
  for (int i = pt; i < 28 * (D / 8); i += kProdThreads) {
    const int lo = i >= 12 * (D / 8);
    const int j = lo ? i - 12 * (D / 8) : i;
    const int row = lo ? kStep + j / (D / 8) : kStep + 4 + j / (D / 8), c8 = j % (D / 8);
    *reinterpret_cast<uint4*>(smem + (lo ? L::kKlo : L::kKhi) + tile_off(kKRows, row, c8)) = make_uint4(0u, 0u, 0u, 0u);
  }
}

// Key planes of one step: hi = s_hi code, lo = s_lo code, both exact (one
// fp16 multiply per pair each).  Producer thread pt takes channel group
// cg = (pt / 8) % (D / 8) (8 channels) and tokens pt % 8 + 8 m for its range
// of m: consecutive lanes hold consecutive tokens of one 8-row core matrix
// (conflict-free 16-byte stores), and a thread loads a block's scales once
// for all its tokens of that block.  Tokens past the blocks that exist keep
// stale planes (their scores are masked).
template <int D>
__device__ __forceinline__ void keys_store(uint8_t* smem, int pt, int nbk) {
  using L = AttLayout<D>;
  constexpr int kCG = D / 8;            // channel groups
  constexpr int kTpt = 16 * kCG / 32;   // tokens per thread (8 for D = 128, 4 for D = 64)
  const int tlo = pt & 7, cg = (pt >> 3) % kCG, m0 = (pt / (8 * kCG)) * kTpt;
  const int q = cg >> 2;                // 16-byte piece of the token's codes
#pragma unroll
  for (int bb = 0; bb < kTpt / 4; ++bb) {  // the thread's blocks: 4 tokens each
    const int blk = (m0 + 4 * bb) / 4;
    if (blk >= nbk) break;
    const uint4 h16 = reinterpret_cast<const uint4*>(smem + L::kKsh)[blk * (D / 8) + cg];
    const uint4 l16 = reinterpret_cast<const uint4*>(smem + L::kKsh + 8 * D)[blk * (D / 8) + cg];
    const uint32_t shw[4] = {h16.x, h16.y, h16.z, h16.w}, slw[4] = {l16.x, l16.y, l16.z, l16.w};
#pragma unroll
    for (int mm = 0; mm < 4; ++mm) {
      const int tok = tlo + 8 * (m0 + 4 * bb + mm);
      const uint32_t w = *reinterpret_cast<const uint32_t*>(smem + L::kRawK + tok * (D / 2) +
                                                            16 * (q ^ key_swz<D>(tok)) + 4 * (cg & 3));
      uint32_t hw[4], lw[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const __half2 n2 = nibble_pair(w, j);
        hw[j] = h2u(__hmul2(*reinterpret_cast<const __half2*>(&shw[j]), n2));
        lw[j] = h2u(__hmul2(*reinterpret_cast<const __half2*>(&slw[j]), n2));
      }
      const uint32_t off = tile_off(kKRows, tok, cg);
      *reinterpret_cast<uint4*>(smem + L::kKhi + off) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
      *reinterpret_cast<uint4*>(smem + L::kKlo + off) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
    }
  }
}

// Value codes of one step as exact fp16 integers, tile [D channels][128
// tokens]: producer thread pt takes channel pt % D and blocks pt / D,
// pt / D + 256 / D, ...; threads pt < 128 also token pt's value scale and
// minimum as floats (0 past T), and each of their warps the largest scale.
template <int D>
__device__ __forceinline__ void values_store(uint8_t* smem, int pt, int nbk, int t0, int T, int vbuf) {
  using L = AttLayout<D>;
  if (pt < 128) {
    const bool ok = t0 + pt < T;
    float* vsf = reinterpret_cast<float*>(smem + L::kVsf) + vbuf * 256;
    const float vs = ok ? __half2float(reinterpret_cast<const __half*>(smem + L::kRawVs)[pt]) : 0.f;
    vsf[pt] = vs;
    vsf[128 + pt] = ok ? __half2float(reinterpret_cast<const __half*>(smem + L::kRawVm)[pt]) : 0.f;
    float mx = fabsf(vs);
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    if ((pt & 31) == 0) reinterpret_cast<float*>(smem + L::kVmx)[4 * vbuf + pt / 32] = mx;
  }
  const int ch = pt % D;
  for (int blk = pt / D; blk < nbk; blk += kProdThreads / D) {
    const uint4 w4 = *reinterpret_cast<const uint4*>(smem + L::kRawV + (blk * D + ch) * 16);
    const uint32_t w[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
    for (int u = 0; u < 4; ++u) {  // tokens 32 blk + 8 u ..
      *reinterpret_cast<uint4*>(smem + L::kV + 256 * D * vbuf + tile_off(D, ch, 4 * blk + u)) =
          make_uint4(h2u(nibble_pair(w[u], 0)), h2u(nibble_pair(w[u], 1)), h2u(nibble_pair(w[u], 2)),
                     h2u(nibble_pair(w[u], 3)));
    }
  }
}

// Partial attention of steps [chunk * spc, ...) of kv head blockIdx.y for
// query rows 128 blockIdx.z + (0..127).  part: [n_kv][n_chunks][R][D + 4]:
// the chunk's unnormalised P.V of each row, then its max (natural log units)
// and exp-sum.  Per step (128 tokens):
//   producer:  key planes -> k_full; value codes and scales -> v_full
//   QK issuer: S[i % 2] = Q Khi^T + Q Klo^T (2 D/16 MMAs, N = 128)
//   softmax:   row max of S (the two threads of a row exchange halves); if it
//              rose, O and the running sums are rescaled (after the previous
//              P.V is done); p = 2^(S c2 - m), P = p v_scale as fp16 hi + lo
//              into shared memory; sums of p and p v_min
//   PV issuer: O (+)= Phi V^T + Plo V^T (16 MMAs, N = D)
template <int D>
__global__ void __launch_bounds__(kAttThreads, 1)
    kv_attn_kernel(Cache c, int T, const __half* __restrict__ q, int n_heads, int R, int spc, float c2,
                   float* __restrict__ part, uint32_t* __restrict__ status) {
  using L = AttLayout<D>;
  extern __shared__ __align__(128) uint8_t smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int h = blockIdx.y, chunk = blockIdx.x, n_chunks = gridDim.x;
  const int G = n_heads / c.n_kv;
  const int nbT = (T + 31) / 32;
  const int n_steps_all = (nbT + 3) / 4;
  const int s0 = chunk * spc, s1 = min(n_steps_all, s0 + spc);
  const int ns = s1 - s0;
  const int r0 = kRows * blockIdx.z;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBars);
  uint32_t* holder = reinterpret_cast<uint32_t*>(smem + L::kHolder);
  const bool producer = warp >= kProdWarp0 && warp < kQkWarp;
  const int pt = tid - 32 * kProdWarp0;

  if (tid == 0) {
    for (int i = 0; i < L::kNumBars; ++i) {
      const uint32_t cnt = (i == kBarKFull || i == kBarVFull0 || i == kBarVFull1) ? kProdThreads
                           : i == kBarPFull                                        ? kSoftThreads
                                                                                   : 1u;
      mbar_init(&bars[i], cnt);
    }
    fence_mbar_init();
  }
  if (warp == 0) tc::tmem_alloc(holder, kTmemCols);
  pdl_launch_dependents();
  pdl_wait();
  if (producer) {
    // commit groups in order K(s0), V(s0), K(s0 + 1), V(s0 + 1), ...: a part
    // is waited for with at most its successor still in flight
    raw_keys_issue<D>(smem, c, h, 4 * s0, nbT, pt);
    cp_async_commit();
    raw_values_issue<D>(smem, c, h, 4 * s0, nbT, pt);
    cp_async_commit();
  } else {
    // queries of rows r0 .. r0 + 127 (zero past R) into the Q tile
    const int qt = warp < kProdWarp0 ? tid : tid - kProdThreads;  // 0 .. 575
    for (int i = qt; i < kRows * (D / 8); i += kAttThreads - kProdThreads) {
      const int row = i / (D / 8), k8 = i % (D / 8), r = r0 + row;
      uint4 v = make_uint4(0u, 0u, 0u, 0u);
      if (r < R) {
        v = *reinterpret_cast<const uint4*>(q + (static_cast<size_t>(r / G) * n_heads + h * G + r % G) * D +
                                            8 * k8);
      }
      *reinterpret_cast<uint4*>(smem + L::kQ + tile_off(kRows, row, k8)) = v;
    }
    fence_proxy_async_smem();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = *holder;
  bool ok = true;
  const uint32_t sb = smem_u32(smem);

  if (producer) {
    // ------------------------------------------------------------ producer
    key_pad_rows<D>(smem, pt);
    for (int i = 0; i < ns && ok; ++i) {
      const int b0 = 4 * (s0 + i), nbk = min(4, nbT - b0);
      cp_async_wait<1>();
      // the step's raw keys are in, from every producer thread; the key planes are free
      if (!named_all<kProdThreads>(1, i == 0 || mbar_wait(&bars[kBarKEmpty], (i - 1) & 1))) { ok = false; break; }
      key_scales_store<D>(smem, pt, nbk);
      named_sync<kProdThreads>(1);
      keys_store<D>(smem, pt, nbk);
      fence_proxy_async_smem();
      mbar_arrive(&bars[kBarKFull]);
      named_sync<kProdThreads>(1);  // raw keys consumed: reload them for the next step
      if (i + 1 < ns) raw_keys_issue<D>(smem, c, h, b0 + 4, nbT, pt);
      cp_async_commit();
      cp_async_wait<1>();
      // the step's raw values are in; value buffer i % 2 is free (read by
      // the P.V of step i - 2)
      if (!named_all<kProdThreads>(1, i < 2 || mbar_wait(&bars[kBarVEmpty0 + (i & 1)], ((i >> 1) - 1) & 1))) { ok = false; break; }
      values_store<D>(smem, pt, nbk, 32 * b0, T, i & 1);
      fence_proxy_async_smem();
      mbar_arrive(&bars[kBarVFull0 + (i & 1)]);
      named_sync<kProdThreads>(1);
      if (i + 1 < ns) raw_values_issue<D>(smem, c, h, b0 + 4, nbT, pt);
      cp_async_commit();
    }
    cp_async_wait_all();
  } else if (warp == kQkWarp) {
    // ------------------------------------------------------------ score MMAs
    if (lane == 0) {
      const uint32_t id_s = tc::idesc_f16(128, kKRows);
      for (int i = 0; i < ns; ++i) {
        if (!mbar_wait(&bars[kBarKFull], i & 1)) { ok = false; break; }
        if (i >= 2 && !mbar_wait(&bars[kBarSFree0 + (i & 1)], ((i >> 1) - 1) & 1)) { ok = false; break; }
        tc::tc_fence_after();
        const uint32_t s_tm = tmem + kSCols * (i & 1);
#pragma unroll
        for (int s = 0; s < D / 16; ++s) {
          const uint64_t qd = tc::smem_desc(sb + L::kQ + 2 * s * kRows * 16, kRows * 16, 128);
          const uint64_t kh = tc::smem_desc(sb + L::kKhi + 2 * s * kKRows * 16, kKRows * 16, 128);
          const uint64_t kl = tc::smem_desc(sb + L::kKlo + 2 * s * kKRows * 16, kKRows * 16, 128);
          tc::tc_mma_ss(s_tm, qd, kh, id_s, s > 0 ? 1u : 0u);
          tc::tc_mma_ss(s_tm, qd, kl, id_s, 1u);
        }
        tc::tc_commit(&bars[kBarSFull0 + (i & 1)]);
        tc::tc_commit(&bars[kBarKEmpty]);
      }
      tc::tc_commit(&bars[kBarQkEnd]);
      (void)mbar_wait(&bars[kBarQkEnd], 0);  // none of its MMAs still runs
    }
    __syncwarp();
  } else if (warp == kPvWarp) {
    // ------------------------------------------------------------ P.V MMAs
    if (lane == 0) {
      const uint32_t id_o = tc::idesc_f16(128, D);
      const uint32_t o_tm = tmem + kOCol;
      for (int j = 0; j < ns; ++j) {
        if (!mbar_wait(&bars[kBarPFull], j & 1) || !mbar_wait(&bars[kBarVFull0 + (j & 1)], (j >> 1) & 1)) {
          ok = false;
          break;
        }
        tc::tc_fence_after();
        // A = P from tensor memory: tokens 16 u .. 16 u + 15 of buffer j % 2
        // hold the hi plane in columns 16 u .. + 7 and the lo plane in + 8 .. + 15
        const uint32_t p_tm = tmem + kSCols * (j & 1);
        const uint32_t vb = sb + L::kV + 256 * D * (j & 1);
#pragma unroll
        for (int u = 0; u < kStep / 16; ++u) {
          const uint64_t vd = tc::smem_desc(vb + 2 * u * D * 16, D * 16, 128);
          tc::tc_mma_ts(o_tm, p_tm + 16 * u, vd, id_o, (j > 0 || u > 0) ? 1u : 0u);
          tc::tc_mma_ts(o_tm, p_tm + 16 * u + 8, vd, id_o, 1u);
        }
        tc::tc_commit(&bars[kBarODone]);
        tc::tc_commit(&bars[kBarVEmpty0 + (j & 1)]);
        tc::tc_commit(&bars[kBarSFree0 + (j & 1)]);
      }
      tc::tc_commit(&bars[kBarPvEnd]);
      (void)mbar_wait(&bars[kBarPvEnd], 0);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax (warps 0-15)
    // Each thread reads its 32 scores of a step from tensor memory once.  The
    // reference maximum m2 (log2 units) moves only when a row's maximum
    // exceeds it by more than tau (2^8, or 0 when a value scale is so large
    // that 2^8 scale might not fit fp16), so O is rarely rescaled; p <= 2^tau.
    const int quarter = warp & 3, part4 = warp >> 2;
    const int r = 32 * quarter + lane;  // row of the tile = tensor-memory lane
    const uint32_t lane_base = static_cast<uint32_t>(32 * quarter) << 16;
    const uint32_t o_tm = tmem + lane_base + kOCol + part4 * (D / 4);
    float* xch = reinterpret_cast<float*>(smem + L::kXch);  // [part][3][128]
    float m2 = -INFINITY, l = 0.f, vms = 0.f;  // reference max (log2 units), this part's sums
    for (int i = 0; i < ns; ++i) {
      const int t0 = kStep * (s0 + i);
      const int valid = T - t0 - 32 * part4;  // this part's columns >= valid are masked
      const uint32_t s_tm = tmem + lane_base + kSCols * (i & 1) + 32 * part4;
      // this part's 32 tokens are key block part4: its minima term sits in
      // score column 128 + part4
      const uint32_t m_tm = tmem + lane_base + kSCols * (i & 1) + kStep;
      if (!named_all<kSoftThreads>(2, ok && mbar_wait(&bars[kBarSFull0 + (i & 1)], (i >> 1) & 1))) {
        ok = false;
        break;
      }
      tc::tc_fence_after();
      uint32_t sv[2][16], mv[16];
      tc::tc_ld16(s_tm, sv[0]);
      tc::tc_ld16(s_tm + 16, sv[1]);
      tc::tc_ld16(m_tm, mv);
      tc::tc_wait_ld();
      tc::tc_tie16(sv[0]);
      tc::tc_tie16(sv[1]);
      tc::tc_tie16(mv);
      const float mterm = __uint_as_float(part4 == 0 ? mv[0] : part4 == 1 ? mv[1] : part4 == 2 ? mv[2] : mv[3]);
      float mx = -INFINITY;
#pragma unroll
      for (int c16 = 0; c16 < 2; ++c16)
#pragma unroll
        for (int j = 0; j < 16; ++j)
          if (valid >= 32 || 16 * c16 + j < valid) mx = fmaxf(mx, __uint_as_float(sv[c16][j]));
      xch[part4 * 384 + r] = mx + mterm;
      // the step's value scales must be in; the barrier also publishes the
      // other parts' maxima
      if (!named_all<kSoftThreads>(2, mbar_wait(&bars[kBarVFull0 + (i & 1)], (i >> 1) & 1))) {
        ok = false;
        break;
      }
      const float cand = fmaxf(fmaxf(xch[r], xch[384 + r]), fmaxf(xch[768 + r], xch[1152 + r])) * c2;
      const float* vmx = reinterpret_cast<const float*>(smem + L::kVmx) + 4 * (i & 1);
      const float tau = fmaxf(fmaxf(vmx[0], vmx[1]), fmaxf(vmx[2], vmx[3])) <= 255.f ? 8.f : 0.f;
      if (i == 0) {
        m2 = cand;
      } else {
        const bool need = cand > m2 + tau;
        if (__any_sync(0xffffffffu, need)) {
          // O is rescaled once the previous step's P.V is done
          if (!__all_sync(0xffffffffu, mbar_wait(&bars[kBarODone], (i - 1) & 1))) ok = false;
          tc::tc_fence_after();
          const float a = need ? exp2_approx(m2 - cand) : 1.f;
          l *= a;
          vms *= a;
#pragma unroll
          for (int c16 = 0; c16 < D / 64; ++c16) {
            uint32_t v[16];
            tc::tc_ld16(o_tm + 16 * c16, v);
            tc::tc_wait_ld();
            tc::tc_tie16(v);
#pragma unroll
            for (int j = 0; j < 16; ++j) v[j] = __float_as_uint(__uint_as_float(v[j]) * a);
            tc::tc_st16(o_tm + 16 * c16, v);
          }
          if (need) m2 = cand;
        }
      }
      const float bias = fmaf(mterm, c2, -m2);  // p = 2^(S c2 + bias)
      const float4* vs4 = reinterpret_cast<const float4*>(smem + L::kVsf + (i & 1) * 1024 + 128 * part4);
      const float4* vm4 = vs4 + 32;
#pragma unroll
      for (int c16 = 0; c16 < 2; ++c16) {
        float lp = 0.f, vp = 0.f;
        uint32_t pw[16];
#pragma unroll
        for (int j4 = 0; j4 < 4; ++j4) {
          const float4 s4 = vs4[4 * c16 + j4], m4 = vm4[4 * c16 + j4];
          const float scv[4] = {s4.x, s4.y, s4.z, s4.w}, mnv[4] = {m4.x, m4.y, m4.z, m4.w};
#pragma unroll
          for (int j = 0; j < 4; j += 2) {
            const int tk = 16 * c16 + 4 * j4 + j;
            float p0 = exp2_approx(fmaf(__uint_as_float(sv[c16][4 * j4 + j]), c2, bias));
            float p1 = exp2_approx(fmaf(__uint_as_float(sv[c16][4 * j4 + j + 1]), c2, bias));
            if (valid < 32) {
              p0 = tk < valid ? p0 : 0.f;
              p1 = tk + 1 < valid ? p1 : 0.f;
            }
            lp += p0 + p1;
            vp = fmaf(p0, mnv[j], fmaf(p1, mnv[j + 1], vp));
            const float w0 = p0 * scv[j], w1 = p1 * scv[j + 1];
            const __half2 hi = __floats2half2_rn(w0, w1);
            const float2 hf = __half22float2(hi);
            // P over the 16 score columns it came from: hi pairs in the
            // first 8, lo pairs in the last 8
            pw[2 * j4 + j / 2] = h2u(hi);
            pw[8 + 2 * j4 + j / 2] = h2u(__floats2half2_rn(w0 - hf.x, w1 - hf.y));
          }
        }
        l += lp;
        vms += vp;
        tc::tc_st16(s_tm + 16 * c16, pw);
      }
      tc::tc_wait_st();
      tc::tc_fence_before();
      mbar_arrive(&bars[kBarPFull]);
    }
    // the chunk's partial: O + sum p v_min (all parts' sums), max in
    // natural-log units, sum p
    const bool fin = named_all<kSoftThreads>(2, ok && mbar_wait(&bars[kBarODone], (ns - 1) & 1));
    xch[part4 * 384 + 128 + r] = l;
    xch[part4 * 384 + 256 + r] = vms;
    named_sync<kSoftThreads>(2);
    tc::tc_fence_after();
    if (!fin) {
      ok = false;
    } else {
      float lt = 0.f, vt = 0.f;
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) {
        lt += xch[q4 * 384 + 128 + r];
        vt += xch[q4 * 384 + 256 + r];
      }
      const bool mine = r0 + r < R;
      float* dst = part + ((static_cast<size_t>(h) * n_chunks + chunk) * R + r0 + r) * kPartRow<D>;
#pragma unroll
      for (int c16 = 0; c16 < D / 64; ++c16) {
        uint32_t v[16];
        tc::tc_ld16(o_tm + 16 * c16, v);
        tc::tc_wait_ld();
        tc::tc_tie16(v);
        if (mine) {
#pragma unroll
          for (int j = 0; j < 16; j += 4) {
            *reinterpret_cast<float4*>(dst + part4 * (D / 4) + 16 * c16 + j) =
                make_float4(__uint_as_float(v[j]) + vt, __uint_as_float(v[j + 1]) + vt,
                            __uint_as_float(v[j + 2]) + vt, __uint_as_float(v[j + 3]) + vt);
          }
        }
      }
      if (mine && part4 == 0) *reinterpret_cast<float2*>(dst + D) = make_float2(m2 * 0.69314718055994531f, lt);
    }
  }
  if (!ok) record_error(status, HQ_DEV_TIMEOUT);
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  if (warp == 0) {
    tc::tmem_dealloc(tmem, kTmemCols);
    tc::tmem_relinquish();
  }
}

// Merge the chunks' partials of one row: grid (R, n_kv), 4 warps; warp w
// takes chunks w, w + 4, ... (at most kCombinePer), lane j chunk w + 4 j's
// maximum and sum, and every lane its D/32 channels of all the warp's
// chunks, loaded up front (the loads are independent of the maxima), so the
// merge costs about one round trip to L2.
constexpr int kCombineWarps = 4;
constexpr int kCombinePer = (kTargetCtas + kCombineWarps - 1) / kCombineWarps;  // 37

template <int D>
__global__ void __launch_bounds__(32 * kCombineWarps)
    kv_combine_kernel(const float* __restrict__ part, int n_chunks, int R, int n_heads, int n_kv,
                      float* __restrict__ out) {
  constexpr int kC = D / 32;  // channels per lane
  __shared__ float wm[kCombineWarps], wl[kCombineWarps];
  __shared__ __align__(16) float wo[kCombineWarps][D];
  pdl_launch_dependents();
  pdl_wait();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r = blockIdx.x, h = blockIdx.y;
  const int G = n_heads / n_kv;
  const size_t stride = static_cast<size_t>(R) * kPartRow<D>;
  const float* base = part + (static_cast<size_t>(h) * n_chunks * R + r) * kPartRow<D>;
  const int cnt = n_chunks > warp ? (n_chunks - warp + kCombineWarps - 1) / kCombineWarps : 0;
  // lane j: chunk warp + 4 j's maximum and sum (j < cnt <= 37: lanes and a second pass)
  float mj[2], lj[2];
#pragma unroll
  for (int u = 0; u < 2; ++u) {
    const int j = lane + 32 * u;
    const bool in = j < cnt;
    const float* pk = base + static_cast<size_t>(warp + kCombineWarps * j) * stride;
    mj[u] = in ? pk[D] : -INFINITY;
    lj[u] = in ? pk[D + 1] : 0.f;
  }
  // every chunk's values for this lane's channels
  float v[kCombinePer][kC];
#pragma unroll
  for (int j = 0; j < kCombinePer; ++j) {
    const float* pk = base + static_cast<size_t>(warp + kCombineWarps * j) * stride + kC * lane;
#pragma unroll
    for (int c = 0; c < kC; ++c) v[j][c] = j < cnt ? pk[c] : 0.f;
  }
  float M = fmaxf(mj[0], mj[1]);
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  if (lane == 0) wm[warp] = M;
  __syncthreads();
  M = fmaxf(fmaxf(wm[0], wm[1]), fmaxf(wm[2], wm[3]));
  // chunk factors exp(m - M), through 2^x
  float f[2];
  float L = 0.f;
#pragma unroll
  for (int u = 0; u < 2; ++u) {
    f[u] = mj[u] > -INFINITY ? exp2_approx((mj[u] - M) * 1.4426950408889634f) : 0.f;
    L = fmaf(lj[u], f[u], L);
  }
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) L += __shfl_xor_sync(0xffffffffu, L, o);
  float acc[kC];
#pragma unroll
  for (int c = 0; c < kC; ++c) acc[c] = 0.f;
#pragma unroll
  for (int j = 0; j < kCombinePer; ++j) {
    const float fj = __shfl_sync(0xffffffffu, j < 32 ? f[0] : f[1], j & 31);
#pragma unroll
    for (int c = 0; c < kC; ++c) acc[c] = fmaf(v[j][c], fj, acc[c]);
  }
#pragma unroll
  for (int c = 0; c < kC; ++c) wo[warp][kC * lane + c] = acc[c];
  if (lane == 0) wl[warp] = L;
  __syncthreads();
  if (warp == 0) {
    const float lt = wl[0] + wl[1] + wl[2] + wl[3];
    float* dst = out + (static_cast<size_t>(r / G) * n_heads + h * G + r % G) * D + kC * lane;
#pragma unroll
    for (int c = 0; c < kC; ++c) dst[c] = (wo[0][kC * lane + c] + wo[1][kC * lane + c] + wo[2][kC * lane + c] +
                                           wo[3][kC * lane + c]) / lt;
  }
}

// ---------------------------------------------------------------- host side

static bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

static hq_status check_cache(const hq_kv_cache* c) {
  if (c == nullptr) return HQ_ERR_INVALID_ARG;
  if (c->head_dim != 64 && c->head_dim != 128) return HQ_ERR_UNSUPPORTED;
  if (c->n_kv_heads < 1 || c->n_kv_heads > 65535 || c->capacity < 32 || c->capacity % 32 != 0 ||
      c->capacity > (1 << 24)) {
    return HQ_ERR_INVALID_ARG;
  }
  if (!c->k_codes || !c->k_scale || !c->k_min || !c->v_codes || !c->v_scale || !c->v_min) {
    return HQ_ERR_INVALID_ARG;
  }
  if (!aligned(c->k_codes, 16) || !aligned(c->k_scale, 16) || !aligned(c->k_min, 16) ||
      !aligned(c->v_codes, 16) || !aligned(c->v_scale, 16) || !aligned(c->v_min, 16)) {
    return HQ_ERR_INVALID_ARG;
  }
  return HQ_OK;
}

static Cache cache_of(const hq_kv_cache* c) {
  Cache k;
  k.d = c->head_dim;
  k.n_kv = c->n_kv_heads;
  k.cap = c->capacity;
  k.kc = c->k_codes;
  k.ks = reinterpret_cast<const __half*>(c->k_scale);
  k.km = reinterpret_cast<const __half*>(c->k_min);
  k.vc = c->v_codes;
  k.vs = reinterpret_cast<const __half*>(c->v_scale);
  k.vm = reinterpret_cast<const __half*>(c->v_min);
  return k;
}

struct Plan {
  int n_rg, spc, n_chunks;
};

// Steps (128 tokens) per chunk such that the grid is about one CTA per SM.
static Plan plan_of(int n_kv, int T, int R) {
  Plan p;
  const int n_steps = ((T + 31) / 32 + 3) / 4;
  p.n_rg = (R + kRows - 1) / kRows;
  const long units = static_cast<long>(n_kv) * p.n_rg;
  const int want = static_cast<int>(std::max<long>(1, (kTargetCtas + units - 1) / units));
  p.spc = std::max(1, (n_steps + want - 1) / want);
  p.n_chunks = (n_steps + p.spc - 1) / p.spc;
  return p;
}

// Workspace: [status word, 256 bytes][partials [n_kv][n_chunks][R][D + 4] fp32].
constexpr size_t kStatusBytes = 256;

}  // namespace kv
}  // namespace hq

using namespace hq;

extern "C" {

hq_status hq_kv_append(const hq_kv_cache* cache, const uint16_t* k, const uint16_t* v, int pos, int n_new,
                       hq_stream_t stream) {
  const hq_status cs = kv::check_cache(cache);
  if (cs != HQ_OK) return cs;
  if (pos < 0 || n_new < 0 || pos % 32 != 0 || n_new % 32 != 0 || n_new > cache->capacity - pos) {
    return HQ_ERR_INVALID_ARG;
  }
  if (n_new == 0) return HQ_OK;
  if (!k || !v || !kv::aligned(k, 2) || !kv::aligned(v, 2)) return HQ_ERR_INVALID_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int d = cache->head_dim;
  const dim3 grid(n_new / 32, cache->n_kv_heads);
  cudaError_t e = launch_pdl(kv::kv_append_k_kernel, grid, dim3(d), 0, st, true, d, cache->n_kv_heads,
                             cache->capacity, cache->k_codes, reinterpret_cast<__half*>(cache->k_scale),
                             reinterpret_cast<__half*>(cache->k_min), reinterpret_cast<const __half*>(k), pos);
  if (e == cudaSuccess) {
    e = launch_pdl(kv::kv_append_v_kernel, grid, dim3(d), 0, st, true, d, cache->n_kv_heads, cache->capacity,
                   cache->v_codes, reinterpret_cast<__half*>(cache->v_scale),
                   reinterpret_cast<__half*>(cache->v_min), reinterpret_cast<const __half*>(v), pos);
  }
  if (e != cudaSuccess) {
    (void)cudaGetLastError();
    return HQ_ERR_CUDA;
  }
  return HQ_OK;
}

size_t hq_kv_attend_workspace_size(const hq_kv_cache* cache, int n_tokens, int n_q, int n_heads) {
  if (kv::check_cache(cache) != HQ_OK || n_tokens < 1 || n_tokens > cache->capacity || n_q < 1 ||
      n_heads < 1 || n_heads % cache->n_kv_heads != 0) {
    return 0;
  }
  const long R = static_cast<long>(n_q) * (n_heads / cache->n_kv_heads);
  if (R > kv::kMaxRows) return 0;
  const kv::Plan p = kv::plan_of(cache->n_kv_heads, n_tokens, static_cast<int>(R));
  return kv::kStatusBytes + 4 * static_cast<size_t>(cache->n_kv_heads) * p.n_chunks * R * (cache->head_dim + 4);
}

int hq_kv_attend_launches(void) { return 2; }

hq_status hq_kv_attend(const hq_kv_cache* cache, int n_tokens, const uint16_t* q, int n_q, int n_heads,
                       float* out, void* workspace, size_t ws_bytes, hq_stream_t stream) {
  const hq_status cs = kv::check_cache(cache);
  if (cs != HQ_OK) return cs;
  if (n_q < 0 || n_heads < 1 || n_heads % cache->n_kv_heads != 0) return HQ_ERR_INVALID_ARG;
  if (n_tokens < 1 || n_tokens > cache->capacity) return HQ_ERR_INVALID_ARG;
  if (n_q == 0) return HQ_OK;
  const long Rl = static_cast<long>(n_q) * (n_heads / cache->n_kv_heads);
  if (Rl > kv::kMaxRows) return HQ_ERR_UNSUPPORTED;
  const int R = static_cast<int>(Rl);
  if (!q || !out || !kv::aligned(q, 16) || !kv::aligned(out, 16)) return HQ_ERR_INVALID_ARG;
  const size_t need = hq_kv_attend_workspace_size(cache, n_tokens, n_q, n_heads);
  if (!workspace || !kv::aligned(workspace, 256) || ws_bytes < need) return HQ_ERR_WORKSPACE;
  const kv::Cache c = kv::cache_of(cache);
  const kv::Plan p = kv::plan_of(c.n_kv, n_tokens, R);
  uint32_t* status = static_cast<uint32_t*>(workspace);
  float* part = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + kv::kStatusBytes);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  // scores enter the softmax as 2^(S c2 - m): c2 = log2(e) / sqrt(d)
  const float c2 = static_cast<float>(1.4426950408889634 / sqrt(static_cast<double>(c.d)));
  const __half* qh = reinterpret_cast<const __half*>(q);
  const dim3 grid(p.n_chunks, c.n_kv, p.n_rg);
  cudaError_t e;
  if (c.d == 128) {
    e = launch_pdl(kv::kv_attn_kernel<128>, grid, dim3(kv::kAttThreads), kv::AttLayout<128>::kBytes, st, true, c,
                   n_tokens, qh, n_heads, R, p.spc, c2, part, status);
    if (e == cudaSuccess) {
      e = launch_pdl(kv::kv_combine_kernel<128>, dim3(R, c.n_kv), dim3(32 * kv::kCombineWarps), 0, st, true,
                     static_cast<const float*>(part), p.n_chunks, R, n_heads, c.n_kv, out);
    }
  } else {
    e = launch_pdl(kv::kv_attn_kernel<64>, grid, dim3(kv::kAttThreads), kv::AttLayout<64>::kBytes, st, true, c,
                   n_tokens, qh, n_heads, R, p.spc, c2, part, status);
    if (e == cudaSuccess) {
      e = launch_pdl(kv::kv_combine_kernel<64>, dim3(R, c.n_kv), dim3(32 * kv::kCombineWarps), 0, st, true,
                     static_cast<const float*>(part), p.n_chunks, R, n_heads, c.n_kv, out);
    }
  }
  if (e != cudaSuccess) {
    (void)cudaGetLastError();
    return HQ_ERR_CUDA;
  }
  return HQ_OK;
}

}  // extern "C"
