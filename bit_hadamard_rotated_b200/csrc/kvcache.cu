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
// Attention (split over the context, flash-decoding style; one CTA per kv
// head, chunk of 32-token blocks and group of 128 query rows; a row is one
// query token of one head of the kv head's group).  Per block the CTA
// dequantises the keys into two fp16 planes hi + lo (hi = fp16(k), lo =
// fp16(k - hi): k to about 2^-22 relative) and the value codes into exact fp16
// integers, in shared memory; each warp owns 16 rows, keeps its queries as
// mma.sync A fragments and its running softmax state in registers:
//   S  = Q K^T          one m16n8k16 MMA per tile and plane (hi, lo), fp32
//   p  = exp(S/sqrt(d) - running max), rescaling the previous partials
//   O += (p vs) N_v     p * v_scale split into fp16 hi + lo, N_v the value
//                       codes, plus sum_t p v_min added to every channel
// The chunk's (max, sum, O) go to the workspace; kv_combine_kernel merges
// the chunks of each row.
#include <cuda_fp16.h>

#include <algorithm>

#include "hq_common.cuh"
#include "hq_internal.h"
#include "hq_launch.cuh"

namespace hq {
namespace kv {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kRows = 16 * kWarps;  // query rows per CTA
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

__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

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

// Shared memory of one block buffer: key planes [32 tokens][D] (hi, lo),
// value codes [D channels][32 tokens], all fp16 with 16-byte chunks swizzled
// so that each ldmatrix phase touches eight distinct bank groups; then the
// block's value scales and minima as floats.
template <int D>
struct Buf {
  static constexpr int kKPlane = 32 * D * 2;
  static constexpr int kV = D * 32 * 2;
  static constexpr int kBytes = 2 * kKPlane + kV + 2 * 32 * 4;
};

template <int D>
__device__ __forceinline__ uint32_t koff(int tok, int chunk) {
  return tok * (2 * D) + ((chunk ^ (tok & 7)) << 4);
}
__device__ __forceinline__ uint32_t voff(int ch, int chunk) { return ch * 64 + ((chunk ^ ((ch >> 1) & 3)) << 4); }

// The cache bytes of one block as they arrive (cp.async, 16 bytes a copy):
// key codes, key scales, key minima, value codes, value scales, value minima.
template <int D>
struct Raw {
  static constexpr int kKc = 0, kKs = 16 * D, kKm = 18 * D, kVc = 20 * D, kVs = 36 * D, kVm = 36 * D + 64;
  static constexpr int kBytes = 36 * D + 128;
  static constexpr int kPieces = kBytes / 16;
};
constexpr int kRing = 4;  // blocks in flight

__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Issue the copies of block b into a raw slot (every thread a share).
template <int D>
__device__ __forceinline__ void raw_issue(uint8_t* raw, const Cache& c, int h, int b, int tid) {
  const size_t blk = static_cast<size_t>(h) * (c.cap / 32) + b;
  const uint8_t* kc = c.kc + blk * 16 * D;
  const uint8_t* ks = reinterpret_cast<const uint8_t*>(c.ks + blk * D);
  const uint8_t* km = reinterpret_cast<const uint8_t*>(c.km + blk * D);
  const uint8_t* vc = c.vc + blk * 16 * D;
  const uint8_t* vs = reinterpret_cast<const uint8_t*>(c.vs + static_cast<size_t>(h) * c.cap + 32 * b);
  const uint8_t* vm = reinterpret_cast<const uint8_t*>(c.vm + static_cast<size_t>(h) * c.cap + 32 * b);
  for (int i = tid; i < Raw<D>::kPieces; i += kThreads) {
    const int o = 16 * i;
    const uint8_t* src;
    if (o < Raw<D>::kKs) src = kc + o;
    else if (o < Raw<D>::kKm) src = ks + (o - Raw<D>::kKs);
    else if (o < Raw<D>::kVc) src = km + (o - Raw<D>::kKm);
    else if (o < Raw<D>::kVs) src = vc + (o - Raw<D>::kVc);
    else if (o < Raw<D>::kVm) src = vs + (o - Raw<D>::kVs);
    else src = vm + (o - Raw<D>::kVm);
    cp_async16(raw + o, src, 16u);
  }
}

// Dequantise the raw block into a compute buffer: each thread kE = D/8 key
// channels of one token (hi and lo planes) and kE value tokens of one channel;
// threads 0..31 one token's value scale and minimum (zero past T).
template <int D>
__device__ __forceinline__ void stage_store(const uint8_t* raw, uint8_t* buf, int b, int T, int tid) {
  constexpr int kE = D / 8;
  constexpr int kTpc = kThreads / D;  // threads per value channel
  uint8_t* khi = buf;
  uint8_t* klo = buf + Buf<D>::kKPlane;
  uint8_t* vb = buf + 2 * Buf<D>::kKPlane;
  float* vsv = reinterpret_cast<float*>(buf + 2 * Buf<D>::kKPlane + Buf<D>::kV);
  const int tok = tid >> 3, kpart = tid & 7;
  const int vch = tid / kTpc, vpart = tid % kTpc;
  const uint32_t* kn = reinterpret_cast<const uint32_t*>(raw + Raw<D>::kKc + tok * (D / 2) + kpart * (kE / 2));
  const uint4* ks = reinterpret_cast<const uint4*>(raw + Raw<D>::kKs + 2 * kpart * kE);
  const uint4* km = reinterpret_cast<const uint4*>(raw + Raw<D>::kKm + 2 * kpart * kE);
  const uint32_t* vn = reinterpret_cast<const uint32_t*>(raw + Raw<D>::kVc + vch * 16 + vpart * (kE / 2));
#pragma unroll
  for (int i = 0; i < kE / 8; ++i) {
    const uint32_t kw = kn[i];
    const uint4 s4 = ks[i], m4 = km[i];
    const uint32_t sw[4] = {s4.x, s4.y, s4.z, s4.w}, mw[4] = {m4.x, m4.y, m4.z, m4.w};
    uint32_t hw[4], lw[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 n = __half22float2(nibble_pair(kw, j));
      const float2 sc = __half22float2(*reinterpret_cast<const __half2*>(&sw[j]));
      const float2 mn = __half22float2(*reinterpret_cast<const __half2*>(&mw[j]));
      const float k0 = fmaf(sc.x, n.x, mn.x), k1 = fmaf(sc.y, n.y, mn.y);
      const __half2 hi = __floats2half2_rn(k0, k1);
      const float2 hf = __half22float2(hi);
      hw[j] = h2u(hi);
      lw[j] = h2u(__floats2half2_rn(k0 - hf.x, k1 - hf.y));
    }
    const int chunk = kpart * (kE / 8) + i;
    *reinterpret_cast<uint4*>(khi + koff<D>(tok, chunk)) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
    *reinterpret_cast<uint4*>(klo + koff<D>(tok, chunk)) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
    const uint32_t vw = vn[i];
    *reinterpret_cast<uint4*>(vb + voff(vch, vpart * (kE / 8) + i)) =
        make_uint4(h2u(nibble_pair(vw, 0)), h2u(nibble_pair(vw, 1)), h2u(nibble_pair(vw, 2)),
                   h2u(nibble_pair(vw, 3)));
  }
  if (tid < 32) {
    const bool ok = 32 * b + tid < T;
    const __half* vs = reinterpret_cast<const __half*>(raw + Raw<D>::kVs);
    const __half* vm = reinterpret_cast<const __half*>(raw + Raw<D>::kVm);
    vsv[tid] = ok ? __half2float(vs[tid]) : 0.f;
    vsv[32 + tid] = ok ? __half2float(vm[tid]) : 0.f;
  }
}

// Partial attention of blocks [chunk * bpc, ...) of kv head blockIdx.y for
// query rows 128 blockIdx.z + (0..127).  part: [n_kv][n_chunks][R][D + 4]:
// the chunk's unnormalised P.V of each row, then its max and exp-sum.
template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    kv_partial_kernel(Cache c, int T, const __half* __restrict__ q, int n_heads, int R, int bpc,
                      float inv_sqrt_d, float* __restrict__ part) {
  extern __shared__ __align__(128) uint8_t smem[];
  constexpr int kKS = D / 16;  // k-steps of the score product
  constexpr int kNT = D / 8;   // channel tiles of the value product
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, t4 = lane & 3;
  const int h = blockIdx.y, chunk = blockIdx.x, n_chunks = gridDim.x;
  const int G = n_heads / c.n_kv;
  const int nbT = (T + 31) / 32;
  const int b0 = chunk * bpc, b1 = min(nbT, b0 + bpc);
  const int r_lo = kRows * blockIdx.z + 16 * warp + g, r_hi = r_lo + 8;
  const bool active = kRows * blockIdx.z + 16 * warp < R;

  pdl_launch_dependents();
  pdl_wait();

  // queries of rows r_lo, r_hi as A fragments (zero for rows >= R)
  uint32_t qa[kKS][4];
  {
    const uint32_t* ql = r_lo < R ? reinterpret_cast<const uint32_t*>(
                                        q + (static_cast<size_t>(r_lo / G) * n_heads + h * G + r_lo % G) * D)
                                  : nullptr;
    const uint32_t* qh = r_hi < R ? reinterpret_cast<const uint32_t*>(
                                        q + (static_cast<size_t>(r_hi / G) * n_heads + h * G + r_hi % G) * D)
                                  : nullptr;
#pragma unroll
    for (int s = 0; s < kKS; ++s) {
      qa[s][0] = ql ? __ldg(ql + 8 * s + t4) : 0u;
      qa[s][1] = qh ? __ldg(qh + 8 * s + t4) : 0u;
      qa[s][2] = ql ? __ldg(ql + 8 * s + 4 + t4) : 0u;
      qa[s][3] = qh ? __ldg(qh + 8 * s + 4 + t4) : 0u;
    }
  }

  float O[kNT][4];
#pragma unroll
  for (int j = 0; j < kNT; ++j) O[j][0] = O[j][1] = O[j][2] = O[j][3] = 0.f;
  float m_lo = -INFINITY, m_hi = -INFINITY, l_lo = 0.f, l_hi = 0.f, vm_lo = 0.f, vm_hi = 0.f;

  // raw ring after the two compute buffers; blocks b0 .. b0 + kRing - 2 in flight
  uint8_t* ring = smem + 2 * Buf<D>::kBytes;
#pragma unroll
  for (int i = 0; i < kRing - 1; ++i) {
    if (b0 + i < b1) raw_issue<D>(ring + i * Raw<D>::kBytes, c, h, b0 + i, tid);
    cp_async_commit();
  }
  const uint32_t sbase = smem_u32(smem);
  for (int b = b0; b < b1; ++b) {
    const int slot = (b - b0) & 1;
    uint8_t* buf = smem + slot * Buf<D>::kBytes;
    cp_async_wait<kRing - 2>();  // this thread's copies of block b have landed
    __syncthreads();             // everyone's have; iteration b - 1 is over everywhere
    if (b + kRing - 1 < b1) raw_issue<D>(ring + ((b - b0 + kRing - 1) % kRing) * Raw<D>::kBytes, c, h, b + kRing - 1, tid);
    cp_async_commit();
    stage_store<D>(ring + ((b - b0) % kRing) * Raw<D>::kBytes, buf, b, T, tid);
    __syncthreads();
    if (!active) continue;
    const uint32_t khi = sbase + slot * Buf<D>::kBytes;
    const uint32_t klo = khi + Buf<D>::kKPlane;
    const uint32_t vb = khi + 2 * Buf<D>::kKPlane;
    const float* vsv = reinterpret_cast<const float*>(buf + 2 * Buf<D>::kKPlane + Buf<D>::kV);

    // ---- scores: 4 token tiles of 8, hi and lo planes in separate chains
    float Sh[4][4], Sl[4][4];
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) Sh[j][e] = Sl[j][e] = 0.f;
#pragma unroll
    for (int s = 0; s < kKS; s += 2) {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint32_t off = koff<D>(8 * j + (lane & 7), 2 * s + (lane >> 3));
        uint32_t bh[4], bl[4];
        ldsm_x4(bh, khi + off);
        ldsm_x4(bl, klo + off);
        mma_16816_acc(Sh[j], qa[s], bh[0], bh[1]);
        mma_16816_acc(Sl[j], qa[s], bl[0], bl[1]);
        mma_16816_acc(Sh[j], qa[s + 1], bh[2], bh[3]);
        mma_16816_acc(Sl[j], qa[s + 1], bl[2], bl[3]);
      }
    }
    // ---- online softmax of rows r_lo (elements 0, 1) and r_hi (2, 3)
    float mx_lo = -INFINITY, mx_hi = -INFINITY;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int tk = 32 * b + 8 * j + 2 * t4 + (e & 1);
        Sh[j][e] = tk < T ? (Sh[j][e] + Sl[j][e]) * inv_sqrt_d : -INFINITY;
      }
      mx_lo = fmaxf(mx_lo, fmaxf(Sh[j][0], Sh[j][1]));
      mx_hi = fmaxf(mx_hi, fmaxf(Sh[j][2], Sh[j][3]));
    }
#pragma unroll
    for (int o = 1; o <= 2; o <<= 1) {
      mx_lo = fmaxf(mx_lo, __shfl_xor_sync(0xffffffffu, mx_lo, o));
      mx_hi = fmaxf(mx_hi, __shfl_xor_sync(0xffffffffu, mx_hi, o));
    }
    const float mn_lo = fmaxf(m_lo, mx_lo), mn_hi = fmaxf(m_hi, mx_hi);
    const float a_lo = expf(m_lo - mn_lo), a_hi = expf(m_hi - mn_hi);
    m_lo = mn_lo;
    m_hi = mn_hi;
    l_lo *= a_lo;
    l_hi *= a_hi;
    vm_lo *= a_lo;
    vm_hi *= a_hi;
#pragma unroll
    for (int j = 0; j < kNT; ++j) {
      O[j][0] *= a_lo;
      O[j][1] *= a_lo;
      O[j][2] *= a_hi;
      O[j][3] *= a_hi;
    }
    uint32_t ph[2][4], pl[2][4];  // A fragments of p * v_scale, k-steps of 16 tokens
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int tl = 8 * j + 2 * t4;
      const float vs0 = vsv[tl], vs1 = vsv[tl + 1], vm0 = vsv[32 + tl], vm1 = vsv[32 + tl + 1];
      const float p0 = expf(Sh[j][0] - mn_lo), p1 = expf(Sh[j][1] - mn_lo);
      const float p2 = expf(Sh[j][2] - mn_hi), p3 = expf(Sh[j][3] - mn_hi);
      l_lo += p0 + p1;
      l_hi += p2 + p3;
      vm_lo = fmaf(p0, vm0, fmaf(p1, vm1, vm_lo));
      vm_hi = fmaf(p2, vm0, fmaf(p3, vm1, vm_hi));
      const float w0 = p0 * vs0, w1 = p1 * vs1, w2 = p2 * vs0, w3 = p3 * vs1;
      const __half2 h01 = __floats2half2_rn(w0, w1), h23 = __floats2half2_rn(w2, w3);
      const float2 f01 = __half22float2(h01), f23 = __half22float2(h23);
      // tile j is k-step j/2, columns 0-7 (j even: a0, a1) or 8-15 (j odd: a2, a3)
      ph[j >> 1][(j & 1) * 2 + 0] = h2u(h01);
      ph[j >> 1][(j & 1) * 2 + 1] = h2u(h23);
      pl[j >> 1][(j & 1) * 2 + 0] = h2u(__floats2half2_rn(w0 - f01.x, w1 - f01.y));
      pl[j >> 1][(j & 1) * 2 + 1] = h2u(__floats2half2_rn(w2 - f23.x, w3 - f23.y));
    }
    // ---- O += (p v_scale) N_v over the block's two k-steps
#pragma unroll
    for (int j = 0; j < kNT; ++j) {
      uint32_t bv[4];
      ldsm_x4(bv, vb + voff(8 * j + (lane & 7), lane >> 3));
      mma_16816_acc(O[j], ph[0], bv[0], bv[1]);
      mma_16816_acc(O[j], pl[0], bv[0], bv[1]);
      mma_16816_acc(O[j], ph[1], bv[2], bv[3]);
      mma_16816_acc(O[j], pl[1], bv[2], bv[3]);
    }
  }
  if (!active) return;
#pragma unroll
  for (int o = 1; o <= 2; o <<= 1) {
    l_lo += __shfl_xor_sync(0xffffffffu, l_lo, o);
    l_hi += __shfl_xor_sync(0xffffffffu, l_hi, o);
    vm_lo += __shfl_xor_sync(0xffffffffu, vm_lo, o);
    vm_hi += __shfl_xor_sync(0xffffffffu, vm_hi, o);
  }
  const size_t base = (static_cast<size_t>(h) * n_chunks + chunk) * R;
  if (r_lo < R) {
    float* dst = part + (base + r_lo) * kPartRow<D>;
#pragma unroll
    for (int j = 0; j < kNT; ++j) {
      *reinterpret_cast<float2*>(dst + 8 * j + 2 * t4) = make_float2(O[j][0] + vm_lo, O[j][1] + vm_lo);
    }
    if (t4 == 0) *reinterpret_cast<float2*>(dst + D) = make_float2(m_lo, l_lo);
  }
  if (r_hi < R) {
    float* dst = part + (base + r_hi) * kPartRow<D>;
#pragma unroll
    for (int j = 0; j < kNT; ++j) {
      *reinterpret_cast<float2*>(dst + 8 * j + 2 * t4) = make_float2(O[j][2] + vm_hi, O[j][3] + vm_hi);
    }
    if (t4 == 0) *reinterpret_cast<float2*>(dst + D) = make_float2(m_hi, l_hi);
  }
}

// Merge the chunks' partials: one warp per row (8 rows a CTA, grid
// (ceil(R / 8), n_kv)); lanes first take the chunks' maxima and sums (lane k
// chunk k, k + 32, ...), then each lane its D/32 channels over all chunks.
template <int D>
__global__ void __launch_bounds__(256)
    kv_combine_kernel(const float* __restrict__ part, int n_chunks, int R, int n_heads, int n_kv,
                      float* __restrict__ out) {
  constexpr int kC = D / 32;  // channels per lane
  __shared__ float fs[8][kTargetCtas];
  pdl_launch_dependents();
  pdl_wait();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r = 8 * blockIdx.x + warp, h = blockIdx.y;
  if (r >= R) return;
  const int G = n_heads / n_kv;
  const size_t stride = static_cast<size_t>(R) * kPartRow<D>;
  const float* base = part + (static_cast<size_t>(h) * n_chunks * R + r) * kPartRow<D>;
  float M = -INFINITY;
  for (int k = lane; k < n_chunks; k += 32) M = fmaxf(M, base[k * stride + D]);
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  float L = 0.f;
  for (int k = lane; k < n_chunks; k += 32) {
    const float f = expf(base[k * stride + D] - M);
    fs[warp][k] = f;
    L = fmaf(base[k * stride + D + 1], f, L);
  }
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) L += __shfl_xor_sync(0xffffffffu, L, o);
  __syncwarp();
  float acc[kC];
#pragma unroll
  for (int i = 0; i < kC; ++i) acc[i] = 0.f;
  const float* col = base + kC * lane;
#pragma unroll 8
  for (int k = 0; k < n_chunks; ++k) {
    const float f = fs[warp][k];
    if constexpr (kC == 4) {
      const float4 v = *reinterpret_cast<const float4*>(col + k * stride);
      acc[0] = fmaf(v.x, f, acc[0]);
      acc[1] = fmaf(v.y, f, acc[1]);
      acc[2] = fmaf(v.z, f, acc[2]);
      acc[3] = fmaf(v.w, f, acc[3]);
    } else {
      const float2 v = *reinterpret_cast<const float2*>(col + k * stride);
      acc[0] = fmaf(v.x, f, acc[0]);
      acc[1] = fmaf(v.y, f, acc[1]);
    }
  }
  float* dst = out + (static_cast<size_t>(r / G) * n_heads + h * G + r % G) * D + kC * lane;
  if constexpr (kC == 4) {
    *reinterpret_cast<float4*>(dst) = make_float4(acc[0] / L, acc[1] / L, acc[2] / L, acc[3] / L);
  } else {
    *reinterpret_cast<float2*>(dst) = make_float2(acc[0] / L, acc[1] / L);
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

template <int D>
constexpr size_t smem_bytes() {
  return 2 * Buf<D>::kBytes + kRing * Raw<D>::kBytes;
}

struct Plan {
  int n_rg, bpc, n_chunks;
};

// Blocks per chunk such that the grid is about one CTA per SM.
static Plan plan_of(int n_kv, int T, int R) {
  Plan p;
  const int nbT = (T + 31) / 32;
  p.n_rg = (R + kRows - 1) / kRows;
  const long units = static_cast<long>(n_kv) * p.n_rg;
  const int want = static_cast<int>(std::max<long>(1, (kTargetCtas + units - 1) / units));
  p.bpc = std::max(1, (nbT + want - 1) / want);
  p.n_chunks = (nbT + p.bpc - 1) / p.bpc;
  return p;
}

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
  return 4 * static_cast<size_t>(cache->n_kv_heads) * p.n_chunks * R * (cache->head_dim + 4);
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
  float* part = static_cast<float*>(workspace);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const float inv = static_cast<float>(1.0 / sqrt(static_cast<double>(c.d)));
  const __half* qh = reinterpret_cast<const __half*>(q);
  const dim3 grid(p.n_chunks, c.n_kv, p.n_rg);
  cudaError_t e;
  if (c.d == 128) {
    e = launch_pdl(kv::kv_partial_kernel<128>, grid, dim3(kv::kThreads), kv::smem_bytes<128>(), st, true, c,
                   n_tokens, qh, n_heads, R, p.bpc, inv, part);
    if (e == cudaSuccess) {
      e = launch_pdl(kv::kv_combine_kernel<128>, dim3((R + 7) / 8, c.n_kv), dim3(256), 0, st, true,
                     static_cast<const float*>(part), p.n_chunks, R, n_heads, c.n_kv, out);
    }
  } else {
    e = launch_pdl(kv::kv_partial_kernel<64>, grid, dim3(kv::kThreads), kv::smem_bytes<64>(), st, true, c,
                   n_tokens, qh, n_heads, R, p.bpc, inv, part);
    if (e == cudaSuccess) {
      e = launch_pdl(kv::kv_combine_kernel<64>, dim3((R + 7) / 8, c.n_kv), dim3(256), 0, st, true,
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
