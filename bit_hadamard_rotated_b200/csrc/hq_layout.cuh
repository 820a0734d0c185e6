// hq_layout.cuh -- register-level decode of packed codes into fp16 MMA operands.
//
// A lane of the GEMV owns a "bundle" of 32 consecutive codes of one weight row
// inside a 128-code group: BITS words (2-bit: 2 words, 3-bit: one 96-bit
// triplet, 4-bit: 4 words, 8-bit: 8 words).  decode16<BITS> turns the bundle
// into 16 half2 registers P[p], each holding two codes (lo, hi).  A code's
// bits are masked straight into the mantissa field of an fp16 whose exponent
// field is zero, i.e. the subnormal value code * 2^(a - 24), where a is the
// field's bit offset inside its 16-bit half: one LOP3 (or PRMT for bytes)
// yields two codes, with no shift when the field already lies in the low 10
// bits of its half, and the value is exact.  The activation operand carries
// the compensating 2^-a (so every product is q x' 2^-24 exactly), the group
// scale carries 2^24, and the zero point enters as zero * sum_k x'_k per group,
// folded into the accumulator's initial value: w = scale (q - zero) is applied
// inside the matmul without a per-weight instruction.
//
// Pairs<BITS>::get(p) names, for each half of pair p, the code index inside
// the bundle and its shift a.  Step s (0..7) of a 128-code group feeds the
// m16n8k16 MMA with P[2s] as A-fragment columns (2t, 2t+1) and P[2s+1] as
// columns (2t+8, 2t+9), t = lane & 3; the B fragment of lane (n, t) at that
// step holds the four activations with those code indices, in that order.
#pragma once

#include <stdint.h>

#include "hq_common.cuh"

namespace hq {

struct PairDesc {
  uint8_t c_lo, a_lo, c_hi, a_hi;
};

template <int BITS>
struct Pairs;

template <>
struct Pairs<2> {
  // word u (codes 16u..16u+15), pair i = codes (i, i+8): fields at 2i for
  // i < 5, then at 2(i-5) after >> 10.
  static __host__ __device__ constexpr PairDesc get(int p) {
    return PairDesc{static_cast<uint8_t>(16 * (p >> 3) + (p & 7)),
                    static_cast<uint8_t>((p & 7) < 5 ? 2 * (p & 7) : 2 * ((p & 7) - 5)),
                    static_cast<uint8_t>(16 * (p >> 3) + (p & 7) + 8),
                    static_cast<uint8_t>((p & 7) < 5 ? 2 * (p & 7) : 2 * ((p & 7) - 5))};
  }
};

template <>
struct Pairs<4> {
  // word u (codes 8u..8u+7), pair i = codes (i, i+4): fields at 0, 4, then
  // 0, 4 after >> 8.
  static __host__ __device__ constexpr PairDesc get(int p) {
    return PairDesc{static_cast<uint8_t>(8 * (p >> 2) + (p & 3)),
                    static_cast<uint8_t>(4 * (p & 1)),
                    static_cast<uint8_t>(8 * (p >> 2) + (p & 3) + 4),
                    static_cast<uint8_t>(4 * (p & 1))};
  }
};

template <>
struct Pairs<8> {
  // word u (codes 4u..4u+3), pair i = bytes (i, i+2) placed by PRMT.
  static __host__ __device__ constexpr PairDesc get(int p) {
    return PairDesc{static_cast<uint8_t>(4 * (p >> 1) + (p & 1)), 0,
                    static_cast<uint8_t>(4 * (p >> 1) + (p & 1) + 2), 0};
  }
};

template <>
struct Pairs<3> {
  // 96-bit triplet, code c at stream bits [3c, 3c+3).  Seven shifted views
  // of the triplet each expose two or three (lo, hi) pairs whose fields lie
  // in mantissa slots: lo within bits 0..9, hi within bits 16..25.
  // (c_lo, a_lo, c_hi, a_hi) of the 16 pairs:
  //   (0,1,5,0) (1,4,6,3) (2,7,7,6) (3,1,8,0) (4,4,9,3) (10,0,16,2) (11,3,17,5)
  //   (12,0,18,2) (13,3,19,5) (14,0,20,2) (15,3,21,5) (22,1,27,0) (23,4,28,3)
  //   (24,7,29,6) (25,1,30,0) (26,4,31,3)
  // packed 16 bits each (c_lo | a_lo << 5 | c_hi << 8 | a_hi << 13), four per
  // word and selected without an array, so that a lookup at a run-time index
  // stays in registers.
  static __host__ __device__ constexpr PairDesc get(int p) {
    const uint64_t w = (p >> 2) == 0   ? 0x0823c7e266810520ull
                       : (p >> 2) == 1 ? 0x520cb16b500a6984ull
                       : (p >> 2) == 2 ? 0x1b36b56f540eb36dull
                                       : 0x7f9a1e39ddf87c97ull;
    const uint32_t e = static_cast<uint32_t>(w >> (16 * (p & 3))) & 0xffffu;
    return PairDesc{static_cast<uint8_t>(e & 31u), static_cast<uint8_t>((e >> 5) & 7u),
                    static_cast<uint8_t>((e >> 8) & 31u), static_cast<uint8_t>((e >> 13) & 7u)};
  }
};

constexpr uint32_t kMagic = 0u;  // exponent field 0: the masked code is a subnormal

// (x & m) | e: the code field(s) of x with exponent bits e (0: subnormal).
__device__ __forceinline__ uint32_t mask_field(uint32_t x, uint32_t m, uint32_t e) {
  return e ? and_or(x, m, e) : (x & m);
}

template <int B>
struct int_tag {};

template <int BITS, uint32_t MAGIC = kMagic>
__device__ __forceinline__ void decode16(const uint32_t (&w)[BITS], uint32_t (&P)[16]);

template <int BITS, uint32_t MAGIC>
__device__ __forceinline__ void decode16_impl(const uint32_t (&w)[2], uint32_t (&P)[16], int_tag<2>) {
#pragma unroll
  for (int u = 0; u < 2; ++u) {
    const uint32_t x = w[u];
    const uint32_t x2 = x >> 10;
#pragma unroll
    for (int i = 0; i < 5; ++i) P[8 * u + i] = mask_field(x, 0x00030003u << (2 * i), MAGIC);
#pragma unroll
    for (int i = 0; i < 3; ++i) P[8 * u + 5 + i] = mask_field(x2, 0x00030003u << (2 * i), MAGIC);
  }
}

template <int BITS, uint32_t MAGIC>
__device__ __forceinline__ void decode16_impl(const uint32_t (&w)[4], uint32_t (&P)[16], int_tag<4>) {
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const uint32_t x = w[u];
    const uint32_t x2 = x >> 8;
    P[4 * u + 0] = mask_field(x, 0x000F000Fu, MAGIC);
    P[4 * u + 1] = mask_field(x, 0x00F000F0u, MAGIC);
    P[4 * u + 2] = mask_field(x2, 0x000F000Fu, MAGIC);
    P[4 * u + 3] = mask_field(x2, 0x00F000F0u, MAGIC);
  }
}

template <int BITS, uint32_t MAGIC>
__device__ __forceinline__ void decode16_impl(const uint32_t (&w)[8], uint32_t (&P)[16], int_tag<8>) {
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    P[2 * u + 0] = prmt(w[u], MAGIC ? 0x64646464u : 0u, 0x4240u);
    P[2 * u + 1] = prmt(w[u], MAGIC ? 0x64646464u : 0u, 0x4341u);
  }
}

__device__ __forceinline__ constexpr uint32_t m3(int a_lo, int a_hi) {
  return (7u << a_lo) | (7u << (16 + a_hi));
}

template <int BITS, uint32_t MAGIC>
__device__ __forceinline__ void decode16_impl(const uint32_t (&w)[3], uint32_t (&P)[16], int_tag<3>) {
  const uint32_t v1 = w[0] << 1;
  const uint32_t v2 = w[0] >> 8;
  const uint32_t v3 = funnel_r(w[0], w[1], 30);
  const uint32_t v4 = w[1] >> 4;
  const uint32_t v5 = funnel_r(w[1], w[2], 10);
  const uint32_t v6 = w[2] >> 1;
  const uint32_t v7 = w[2] >> 10;
  P[0] = mask_field(v1, m3(1, 0), MAGIC);
  P[1] = mask_field(v1, m3(4, 3), MAGIC);
  P[2] = mask_field(v1, m3(7, 6), MAGIC);
  P[3] = mask_field(v2, m3(1, 0), MAGIC);
  P[4] = mask_field(v2, m3(4, 3), MAGIC);
  P[5] = mask_field(v3, m3(0, 2), MAGIC);
  P[6] = mask_field(v3, m3(3, 5), MAGIC);
  P[7] = mask_field(v4, m3(0, 2), MAGIC);
  P[8] = mask_field(v4, m3(3, 5), MAGIC);
  P[9] = mask_field(v5, m3(0, 2), MAGIC);
  P[10] = mask_field(v5, m3(3, 5), MAGIC);
  P[11] = mask_field(v6, m3(1, 0), MAGIC);
  P[12] = mask_field(v6, m3(4, 3), MAGIC);
  P[13] = mask_field(v6, m3(7, 6), MAGIC);
  P[14] = mask_field(v7, m3(1, 0), MAGIC);
  P[15] = mask_field(v7, m3(4, 3), MAGIC);
}

template <int BITS, uint32_t MAGIC>
__device__ __forceinline__ void decode16(const uint32_t (&w)[BITS], uint32_t (&P)[16]) {
  decode16_impl<BITS, MAGIC>(w, P, int_tag<BITS>{});
}

// ---- normal-range variant (tensor-core GEMM): with exponent field 0x6400
// the pair holds 1024 + (code << a); one exact fp16 FMA per pair turns it
// into q - zero: (1024 + 2^a q) * 2^-a - (1024 * 2^-a + zero).
constexpr uint32_t kMagic1024 = 0x64006400u;

__host__ __device__ constexpr uint32_t half_pow2_neg(int a) {
  return static_cast<uint32_t>(15 - a) << 10;
}

template <int BITS>
__host__ __device__ constexpr uint32_t pair_mult(int p) {
  return half_pow2_neg(Pairs<BITS>::get(p).a_lo) | (half_pow2_neg(Pairs<BITS>::get(p).a_hi) << 16);
}

// fp16 bit pattern of -v for an integer 1 <= v < 2048 (exact).
__host__ __device__ constexpr uint32_t half_neg_int(int v) {
  int e = 0;
  while ((v >> (e + 1)) != 0) ++e;
  return 0x8000u | (static_cast<uint32_t>(e + 15) << 10) |
         ((static_cast<uint32_t>(v) << (10 - e)) & 0x3FFu);
}

template <int BITS>
__host__ __device__ inline uint32_t pair_addend(int p, int zero) {
  return half_neg_int((1024 >> Pairs<BITS>::get(p).a_lo) + zero) |
         (half_neg_int((1024 >> Pairs<BITS>::get(p).a_hi) + zero) << 16);
}

__device__ __forceinline__ uint32_t hfma2(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

__device__ __forceinline__ uint32_t hmul2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// Load a lane's BITS-word bundle from shared memory (16-byte aligned for
// BITS 4 and 8, 8-byte for BITS 2, 4-byte for BITS 3).
template <int BITS>
__device__ __forceinline__ void load_bundle(const uint8_t* p, uint32_t (&w)[BITS]);

template <>
__device__ __forceinline__ void load_bundle<2>(const uint8_t* p, uint32_t (&w)[2]) {
  const uint2 v = *reinterpret_cast<const uint2*>(p);
  w[0] = v.x;
  w[1] = v.y;
}
template <>
__device__ __forceinline__ void load_bundle<3>(const uint8_t* p, uint32_t (&w)[3]) {
  const uint32_t* q = reinterpret_cast<const uint32_t*>(p);
  w[0] = q[0];
  w[1] = q[1];
  w[2] = q[2];
}
template <>
__device__ __forceinline__ void load_bundle<4>(const uint8_t* p, uint32_t (&w)[4]) {
  const uint4 v = *reinterpret_cast<const uint4*>(p);
  w[0] = v.x;
  w[1] = v.y;
  w[2] = v.z;
  w[3] = v.w;
}
template <>
__device__ __forceinline__ void load_bundle<8>(const uint8_t* p, uint32_t (&w)[8]) {
  const uint4 v = *reinterpret_cast<const uint4*>(p);
  const uint4 u = *reinterpret_cast<const uint4*>(p + 16);
  w[0] = v.x;
  w[1] = v.y;
  w[2] = v.z;
  w[3] = v.w;
  w[4] = u.x;
  w[5] = u.y;
  w[6] = u.z;
  w[7] = u.w;
}

// Shared-memory row stride (in 32-bit words, mod 32) that keeps the lanes'
// bundle loads free of bank conflicts (8 rows x 4 lanes per warp).
__host__ __device__ constexpr int bank_target_words(int bits) {
  return bits == 2 ? 8 : bits == 3 ? 4 : bits == 4 ? 16 : 4;
}

}  // namespace hq
