// gemv_frag.cuh -- the rotated activations in mma.sync B-fragment order, shared
// by the GEMV kernels (gemv.cu: batch blocks of up to 8 columns; gemv32.cu:
// 32-row tiles, up to 16 columns): the fragment layout, the rotation (prep)
// kernel that writes it, and the register views that turn packed codes into
// A fragments (hq_layout.cuh).
#pragma once

#include "fwht.cuh"
#include "hq_common.cuh"
#include "hq_internal.h"
#include "hq_io.cuh"
#include "hq_layout.cuh"

namespace hq {

constexpr int kWarps = 16;
// Warps of the prep kernel: its FWHT uses at most 8 for K <= 16384 (64 values
// per thread at K = 16384), and 32 for K = 32768 (32 values per thread).
__host__ __device__ constexpr int prep_warps(int logk) { return logk >= 15 ? 32 : 8; }
__host__ __device__ constexpr int prep_logw(int logk) { return logk >= 15 ? 5 : 3; }
constexpr int kRows = 16;
// B fragments of one column: per 128-code group 4 blocks (one per k-quad t)
// of 64 bytes = 8 MMA steps x 4 fp16 activations; inside block t the four
// 16-byte pieces are rotated by t (piece i at position (i + t) & 3), and
// columns are kXsCol bytes apart (an odd multiple of 64 past G * 256), so that
// the 16-byte loads of a quarter warp (two columns x four k-quads) hit eight
// different bank groups.
constexpr int kXsBlock = 64;
__host__ __device__ constexpr size_t gemv_xs_col(int G) { return static_cast<size_t>(G) * 4 * kXsBlock + 64; }
// Shared memory after a batch block's zero-point terms: the per-column output
// factors 2^(24 - e) (8 floats) and the FWHT's per-warp maxima (16 floats).
// The zero-point terms themselves, zq [G][4][4] fp32: for group g and lane
// quad t, {z(2t), z(2t+1), z(2t), z(2t+1)} with z(n) = -zero sum_k x'_k
// 2^(e-24) of column n (0 for absent columns), the initial value of the
// lane's MMA accumulator fragment (rows g and g + 8).  With per-group zero
// points the factor zero is left out (1) and applied per row and group.
constexpr int kZcTail = 32 + 64;

// Bytes of the prep output for a batch block of nb columns (16-byte multiple):
// the fragments, the zero-point fragments zq [G][blocks][16] and the output
// factors [8 blocks], where blocks = ceil(nb / 8) column blocks of the MMA.
__host__ __device__ constexpr int gemv_blocks(int nb) { return (nb + 7) / 8; }
__host__ __device__ constexpr size_t gemv_xs_bytes(int G, int nb) {
  return static_cast<size_t>(nb) * gemv_xs_col(G);
}
__host__ __device__ constexpr size_t gemv_zq_bytes(int G, int blocks = 1) {
  return static_cast<size_t>(G) * 16 * 4 * blocks;
}
__host__ __device__ constexpr size_t gemv_xg_bytes(int G, int nb) {
  return gemv_xs_bytes(G, nb) + gemv_zq_bytes(G, gemv_blocks(nb)) + 8 * 4 * gemv_blocks(nb);
}

// ---------------------------------------------------------------- rotation -> B fragments
// Lane (s, t) of a warp writes the B-fragment quad of step s for k-quad t:
// the code fields (columns kc, exponent offsets ka) of its four values.
// With bit-plane 2-bit codes (planes) the bundle's two words are rebuilt as
// the packed words of its even and of its odd codes (plane_bundle), so bundle
// code c is code 2c (c < 16) or 2 (c - 16) + 1 of the 32.
template <int BITS>
struct FragLane {
  int kc[4], ka[4];
  __device__ __forceinline__ FragLane(int lane, bool planes) {
    const int s = lane >> 2, t = lane & 3;
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const PairDesc pd = Pairs<BITS>::get(2 * s + (r >> 1));
      const int c = (r & 1) ? pd.c_hi : pd.c_lo;
      kc[r] = 32 * t + (planes ? (c < 16 ? 2 * c : 2 * (c - 16) + 1) : c);
      ka[r] = (r & 1) ? pd.a_hi : pd.a_lo;
    }
  }
};

// A 32-code bundle in the bit-plane layout (w[0]: bit 0 of codes 0..31, w[1]:
// bit 1) as two packed 2-bit words: the even codes 0, 2, .., 30, then the odd
// ones.  Bit 2m of the first word is b0 of code 2m, bit 2m + 1 its b1 (from
// bit 2m of w[1]); likewise for the odd codes one bit further up.
__device__ __forceinline__ void plane_bundle(uint32_t (&w)[2]) {
  const uint32_t p0 = w[0], p1 = w[1];
  w[0] = (p0 & 0x55555555u) | ((p1 << 1) & 0xAAAAAAAAu);
  w[1] = ((p0 >> 1) & 0x55555555u) | (p1 & 0xAAAAAAAAu);
}

// Index in zq of value j (0..3) of lane quad t for group gg (one column block).
__host__ __device__ constexpr int zq_index(int gg, int t, int j) { return (gg * 4 + t) * 4 + j; }
// With NBLK column blocks of 8, zq is [G][NBLK][4][4]: the place (0 or 1) of
// column n's term in its quad's fragment.
template <int NBLK>
__host__ __device__ constexpr int zq_index_n(int gg, int n, int place) {
  return ((gg * NBLK + (n >> 3)) * 4 + ((n & 7) >> 1)) * 4 + (n & 1) + 2 * place;
}

// The groups gg = warp + nw i (i < GPW, gg < G) of one warp: of a rotated row
// (buf: unnormalised fwht_block output), x' 2^e rounded to fp16 (sc = 2^e /
// sqrt(K)), each value scaled by the 2^-a of its code field, written as
// column n of the fragment blocks (xs, kXsBlock layout); each group's
// zero-point term -zero * sum_k x'_k * 2^(e-24) goes to both places of
// column n in zq.  Unrolled over the warp's groups so that their loads and
// zero-point reductions overlap.
template <int BITS, int GPW, int NBLK = 1>
__device__ __forceinline__ void put_groups(const FragLane<BITS>& fl, const float* buf, int warp, int nw,
                                           int n, int G, float sc, float zero, uint16_t* xs, float* zq,
                                           int lane) {
  const int s = lane >> 2, t = lane & 3;
  uint16_t hv[GPW][4];
  float part[GPW];
#pragma unroll
  for (int i = 0; i < GPW; ++i) {
    const int gg = warp + nw * i;
    part[i] = 0.f;
    if (gg < G) {
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const float xv = __half2float(__float2half_rn(buf[fwht_pad(kGroup * gg + fl.kc[r])] * sc));
        const __half b = __float2half_rn(xv * __int_as_float((127 - fl.ka[r]) << 23));
        hv[i][r] = __half_as_ushort(b);
        part[i] += __half2float(b) * __int_as_float((127 + fl.ka[r]) << 23);
      }
    }
  }
#pragma unroll
  for (int m = 16; m >= 1; m >>= 1) {
#pragma unroll
    for (int i = 0; i < GPW; ++i) part[i] += __shfl_xor_sync(0xffffffffu, part[i], m);
  }
#pragma unroll
  for (int i = 0; i < GPW; ++i) {
    const int gg = warp + nw * i;
    if (gg < G) {
      uint2 pk;
      pk.x = hv[i][0] | (static_cast<uint32_t>(hv[i][1]) << 16);
      pk.y = hv[i][2] | (static_cast<uint32_t>(hv[i][3]) << 16);
      *reinterpret_cast<uint2*>(reinterpret_cast<uint8_t*>(xs) + n * gemv_xs_col(G) + (gg * 4 + t) * kXsBlock +
                                ((((s >> 1) + t) & 3) << 4) + (s & 1) * 8) = pk;
      if (lane < 2) {
        zq[zq_index_n<NBLK>(gg, n, lane)] =
            -zero * part[i] * 5.9604644775390625e-8f;
      }
    }
  }
}

// Zero the zero-point terms of the absent columns (N .. 8 NBLK - 1) of zq
// [G][NBLK][16].
template <int NBLK = 1>
__device__ __forceinline__ void zq_clear_absent(float* zq, int G, int N, int tid, int nthreads) {
  for (int i = tid; i < G * 16 * NBLK; i += nthreads) {
    const int n = 8 * ((i >> 4) % NBLK) + 2 * ((i >> 2) & 3) + (i & 1);
    if (n >= N) zq[i] = 0.f;
  }
}

// Prep kernel (batches the GEMV CTAs do not rotate themselves): CTA n rotates
// activation row n in fp32 and writes its fragments, zero-point terms and
// output factor to global memory; CTA 0 also zeroes the zero-point terms of
// the absent columns (N .. 8 NBLK - 1).  NBLK column blocks of 8: 1 for the
// GEMV (batch blocks of at most 8), 2 for the 32-row GEMV (up to 16).
template <int BITS, int LOGK, int NBLK = 1>
__global__ void __launch_bounds__(prep_warps(LOGK) * 32) gemv_prep_kernel(const __half* __restrict__ x,
                                                                 const int8_t* __restrict__ signs,
                                                                 uint8_t* __restrict__ xg, int N,
                                                                 float zero, float inv_sqrt_k, int planes) {
  using FS = FwhtShape<LOGK, prep_logw(LOGK)>;
  constexpr int kPrepWarps = prep_warps(LOGK);
  constexpr int K = 1 << LOGK;
  constexpr int G = K / kGroup;
  extern __shared__ __align__(128) float buf[];
  pdl_launch_dependents();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int n = blockIdx.x;
  uint16_t* xs = reinterpret_cast<uint16_t*>(xg);
  float* zq = reinterpret_cast<float*>(xg + gemv_xs_bytes(G, N));
  float* fac = zq + G * 16 * NBLK;
  float* red = buf + FS::SMEM_FLOATS;  // per-warp maxima of the transform
  const FragLane<BITS> fl(lane, planes != 0);
  const SignMask<FS::E> neg =
      tid < FS::THREADS ? sign_bits<FS::E>(signs ? signs + tid * FS::E : nullptr) : 0u;
  pdl_wait();  // x is the previous kernel's output; xg may still be read by it
  if (n == 0) zq_clear_absent<NBLK>(zq, G, N, tid, kPrepWarps * 32);
  float v[FS::E];
  if (tid < FS::THREADS) {
    load_chunk<__half, FS::E>(x + static_cast<size_t>(n) * K + tid * FS::E, v);
    flip_signs<FS::E>(neg, v);
  }
  fwht_block<LOGK, prep_logw(LOGK)>(v, buf, red);
  const int e = row_scale_exp(red_max(red, FS::W) * inv_sqrt_k);
  if (tid == 0) fac[n] = pow2f(24 - e);
  const float sc = inv_sqrt_k * pow2f(e);
  put_groups<BITS, (G + kPrepWarps - 1) / kPrepWarps, NBLK>(fl, buf, warp, kPrepWarps, n, G, sc, zero, xs, zq,
                                                           lane);
}

// Bytes of B fragments of one group of one column.
constexpr int kXsGroup = 4 * kXsBlock;

// Shifted views of a lane's code bundle from which each fp16 pair of the A
// fragment is one mask (LOP3) or byte permute away; pair(p) is that last step.
template <int BITS> struct DecodeViews;
template <> struct DecodeViews<2> {
  uint32_t x[2], h[2];
  __device__ __forceinline__ void init(const uint32_t (&w)[2]) { x[0] = w[0]; x[1] = w[1]; h[0] = w[0] >> 10; h[1] = w[1] >> 10; }
  __device__ __forceinline__ uint32_t pair(int p) const {
    const int u = p >> 3, i = p & 7;
    return i < 5 ? (x[u] & (0x00030003u << (2 * i))) : (h[u] & (0x00030003u << (2 * (i - 5))));
  }
};
template <> struct DecodeViews<4> {
  uint32_t x[4], h[4];
  __device__ __forceinline__ void init(const uint32_t (&w)[4]) {
#pragma unroll
    for (int u = 0; u < 4; ++u) { x[u] = w[u]; h[u] = w[u] >> 8; }
  }
  __device__ __forceinline__ uint32_t pair(int p) const {
    const int u = p >> 2, i = p & 3;
    const uint32_t v = i < 2 ? x[u] : h[u];
    return v & ((i & 1) ? 0x00F000F0u : 0x000F000Fu);
  }
};
template <> struct DecodeViews<8> {
  uint32_t x[8];
  __device__ __forceinline__ void init(const uint32_t (&w)[8]) {
#pragma unroll
    for (int u = 0; u < 8; ++u) x[u] = w[u];
  }
  __device__ __forceinline__ uint32_t pair(int p) const { return prmt(x[p >> 1], 0u, (p & 1) ? 0x4341u : 0x4240u); }
};
template <> struct DecodeViews<3> {
  uint32_t P[16];
  __device__ __forceinline__ void init(const uint32_t (&w)[3]) { decode16<3>(w, P); }
  __device__ __forceinline__ uint32_t pair(int p) const { return P[p]; }
};

}  // namespace hq
