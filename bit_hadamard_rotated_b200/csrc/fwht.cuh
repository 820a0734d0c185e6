// fwht.cuh -- block-wide fast Walsh-Hadamard transform in fp32 (sm_100a).
//
// H_K in Sylvester natural order factors over the bits of the index: with
// K = 32 * E * W and i = w*(32E) + l*E + e (warp w, lane l, register e),
// H_K = H_W (x) H_32 (x) H_E.  So 32*W threads transform one row:
//   1. butterflies over e inside each thread's E registers,
//   2. butterflies over l with warp shuffles (xor 1..16),
//   3. butterflies over w after one transpose through shared memory, where each
//      thread gathers the W values of E/W (l, e) columns.
// log2(K) butterfly stages in total, two __syncthreads.  The butterfly
// (a, b) -> (a + b, a - b) is the Sylvester matrix applied one index bit at a
// time.  W is capped at 2^LOGW_MAX so that the transform fits the CTA that
// calls it; threads beyond 32*W skip the arithmetic but still reach every
// barrier.
#pragma once

#include <stdint.h>

namespace hq {

template <int LOGK, int LOGW_MAX = 5>
struct FwhtShape {
  static constexpr int K = 1 << LOGK;
  static constexpr int LOGW_NAT = (LOGK - 5) / 2;
  static constexpr int LOGW = LOGW_NAT < LOGW_MAX ? LOGW_NAT : LOGW_MAX;
  static constexpr int LOGE = LOGK - 5 - LOGW;
  static constexpr int E = 1 << LOGE;
  static constexpr int W = 1 << LOGW;
  static constexpr int THREADS = 32 * W;
  static constexpr int C = E / W;                  // columns per thread in stage 3
  static constexpr int SMEM_FLOATS = K + K / 32;  // one pad word per 32
  static_assert(LOGK >= 5 && LOGK <= 15, "K must be in [32, 32768]");
  static_assert(E >= W, "shape");
};

__device__ __forceinline__ int fwht_pad(int i) { return i + (i >> 5); }

// Largest |value| held by the lanes of a warp (every lane gets it).
__device__ __forceinline__ float warp_absmax(float m) {
#pragma unroll
  for (int s = 16; s >= 1; s >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, s));
  return m;
}

// On entry thread tid = 32*w + l < THREADS holds v[e] = u[tid*E + e].  On exit
// the transformed (unnormalised) row is in buf[fwht_pad(i)], i in [0, K), and
// the block has synchronised.  With red != nullptr, red[w] (w < W) also holds
// the largest |value| of the part of the row warp w wrote last, so the row's
// largest |value| is the max of red[0..W).  Every thread of the block must
// call this.
template <int LOGK, int LOGW_MAX>
__device__ __forceinline__ void fwht_block(float (&v)[FwhtShape<LOGK, LOGW_MAX>::E], float* buf,
                                           float* red = nullptr) {
  using S = FwhtShape<LOGK, LOGW_MAX>;
  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const bool active = tid < S::THREADS;
  if (active) {
#pragma unroll
    for (int h = 1; h < S::E; h <<= 1) {
#pragma unroll
      for (int e = 0; e < S::E; ++e) {
        if ((e & h) == 0) {
          const float a = v[e], b = v[e + h];
          v[e] = a + b;
          v[e + h] = a - b;
        }
      }
    }
#pragma unroll
    for (int m = 1; m < 32; m <<= 1) {
      // lower lane: a + b; upper lane: a - b = partner - own
      const float sgn = (lane & m) ? -1.f : 1.f;
#pragma unroll
      for (int e = 0; e < S::E; ++e) {
        const float p = __shfl_xor_sync(0xffffffffu, v[e], m);
        v[e] = fmaf(sgn, v[e], p);
      }
    }
#pragma unroll
    for (int e = 0; e < S::E; ++e) buf[fwht_pad(tid * S::E + e)] = v[e];
    if constexpr (S::W == 1) {
      if (red != nullptr) {
        float m = 0.f;
#pragma unroll
        for (int e = 0; e < S::E; ++e) m = fmaxf(m, fabsf(v[e]));
        m = warp_absmax(m);
        if (lane == 0) red[tid >> 5] = m;
      }
    }
  }
  __syncthreads();
  if constexpr (S::W > 1) {
    if (active) {
      float r[S::C][S::W];
#pragma unroll
      for (int j = 0; j < S::C; ++j)
#pragma unroll
        for (int w = 0; w < S::W; ++w) r[j][w] = buf[fwht_pad(w * 32 * S::E + tid * S::C + j)];
#pragma unroll
      for (int j = 0; j < S::C; ++j) {
#pragma unroll
        for (int h = 1; h < S::W; h <<= 1) {
#pragma unroll
          for (int w = 0; w < S::W; ++w) {
            if ((w & h) == 0) {
              const float a = r[j][w], b = r[j][w + h];
              r[j][w] = a + b;
              r[j][w + h] = a - b;
            }
          }
        }
      }
#pragma unroll
      for (int j = 0; j < S::C; ++j)
#pragma unroll
        for (int w = 0; w < S::W; ++w) buf[fwht_pad(w * 32 * S::E + tid * S::C + j)] = r[j][w];
      if (red != nullptr) {
        float m = 0.f;
#pragma unroll
        for (int j = 0; j < S::C; ++j)
#pragma unroll
          for (int w = 0; w < S::W; ++w) m = fmaxf(m, fabsf(r[j][w]));
        m = warp_absmax(m);
        if (lane == 0) red[tid >> 5] = m;
      }
    }
    __syncthreads();
  }
}

// The same transform for a 512-thread CTA (16 warps) and 512 <= K <= 8192:
// K = 16 (warps) x 32 (lanes) x E (registers), E = K / 512.  Stages 1 and 2
// as above; for the 16 warps (stage 3) thread t takes column p = t / T of the
// shared-memory image (T = 16 / E threads per column) and the E warps h E ..
// h E + E - 1 of it (h = t % T): butterflies over those E in registers, then
// over the T threads of the column with shuffles.  Twice the threads of the
// 8-warp shape at K = 4096, so half the work per thread on the critical path.
template <int LOGK>
struct Fwht512 {
  static constexpr int K = 1 << LOGK;
  static constexpr int E = K / 512;
  static constexpr int T = 16 / E;
  static constexpr int SMEM_FLOATS = K + K / 32;
  static_assert(LOGK >= 9 && LOGK <= 13, "K must be in [512, 8192]");
};

// On entry thread tid (of 512) holds v[e] = u[tid*E + e]; on exit the
// transformed (unnormalised) row is in buf[fwht_pad(i)] and the block has
// synchronised; with red != nullptr, red[w] (w < 16) holds the largest
// |value| written by warp w.  Every thread of the block must call this.
template <int LOGK>
__device__ __forceinline__ void fwht_block512(float (&v)[Fwht512<LOGK>::E], float* buf,
                                              float* red = nullptr) {
  using S = Fwht512<LOGK>;
  constexpr int E = S::E, T = S::T;
  const int tid = threadIdx.x, lane = tid & 31;
#pragma unroll
  for (int h = 1; h < E; h <<= 1) {
#pragma unroll
    for (int e = 0; e < E; ++e) {
      if ((e & h) == 0) {
        const float a = v[e], b = v[e + h];
        v[e] = a + b;
        v[e + h] = a - b;
      }
    }
  }
#pragma unroll
  for (int m = 1; m < 32; m <<= 1) {
    const float sgn = (lane & m) ? -1.f : 1.f;
#pragma unroll
    for (int e = 0; e < E; ++e) {
      const float p = __shfl_xor_sync(0xffffffffu, v[e], m);
      v[e] = fmaf(sgn, v[e], p);
    }
  }
#pragma unroll
  for (int e = 0; e < E; ++e) buf[fwht_pad(tid * E + e)] = v[e];
  __syncthreads();
  const int col = tid / T, h = tid % T;
  float r[E];
#pragma unroll
  for (int i = 0; i < E; ++i) r[i] = buf[fwht_pad((h * E + i) * 32 * E + col)];
#pragma unroll
  for (int hb = 1; hb < E; hb <<= 1) {
#pragma unroll
    for (int i = 0; i < E; ++i) {
      if ((i & hb) == 0) {
        const float a = r[i], b = r[i + hb];
        r[i] = a + b;
        r[i + hb] = a - b;
      }
    }
  }
#pragma unroll
  for (int j = 1; j < T; j <<= 1) {
    const float sgn = (h & j) ? -1.f : 1.f;
#pragma unroll
    for (int i = 0; i < E; ++i) {
      const float q = __shfl_xor_sync(0xffffffffu, r[i], j);
      r[i] = fmaf(sgn, r[i], q);
    }
  }
#pragma unroll
  for (int i = 0; i < E; ++i) buf[fwht_pad((h * E + i) * 32 * E + col)] = r[i];
  if (red != nullptr) {
    float m = 0.f;
#pragma unroll
    for (int i = 0; i < E; ++i) m = fmaxf(m, fabsf(r[i]));
    m = warp_absmax(m);
    if (lane == 0) red[tid >> 5] = m;
  }
  __syncthreads();
}

// Largest of red[0..n) (the per-warp maxima the transforms above leave).
__device__ __forceinline__ float red_max(const float* red, int n) {
  float m = 0.f;
  for (int i = 0; i < n; ++i) m = fmaxf(m, red[i]);
  return m;
}

// Power-of-two exponent e for a row whose largest |x'| is m: x' * 2^e has its
// largest magnitude in (2^13, 2^14], so when x' is rounded to fp16 (and, in
// the GEMV, scaled down by up to 2^-8 more) every element within 2^-20 of the
// largest stays in fp16's normal range, whatever the scale of the input.  The
// product is undone exactly at the output (times 2^-e).  Rows of zeros (or
// with an inf or NaN) keep e = 0; e is clamped to [-30, 60].
__device__ __forceinline__ int row_scale_exp(float m) {
  if (!(m > 0.f) || !(m < 3.0e38f)) return 0;
  const int be = (__float_as_int(m) >> 23) & 0xff;  // m < 2^(be - 126)
  const int e = be == 0 ? 60 : 140 - be;
  return e < -30 ? -30 : (e > 60 ? 60 : e);
}

// 2^n as a float, -126 <= n <= 127.
__device__ __forceinline__ float pow2f(int n) { return __int_as_float((127 + n) << 23); }

}  // namespace hq
