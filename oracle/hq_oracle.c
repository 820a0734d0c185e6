/*
 * hq_oracle.c -- plain fp64 CPU oracle (TEST INFRASTRUCTURE ONLY).
 *
 * Only tests/, the smoke check and the benchmark's CPU-baseline leg may load
 * this code.  It includes nothing from the CUDA library and the library
 * includes nothing from here.  Every function follows its definition with
 * scalar loops in the definition's own order; see hq_oracle.h for the
 * formulas and the readings of the pages they rest on.
 */
#include "hq_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

/* binary16: 1 sign bit, 5 exponent bits (bias 15), 10 mantissa bits. */
double hqo_f16_to_f64(uint16_t h) {
  int sign = (h >> 15) & 1;
  int e = (h >> 10) & 0x1f;
  int m = h & 0x3ff;
  double v;
  if (e == 0) {
    v = ldexp((double)m, -24); /* subnormal or zero: m * 2^-14 * 2^-10 */
  } else if (e == 31) {
    v = (m == 0) ? INFINITY : NAN;
  } else {
    v = ldexp((double)(1024 + m), e - 25); /* (1.m) * 2^(e-15) */
  }
  return sign ? -v : v;
}

/* Bit i of the little-endian stream formed by the words. */
static int stream_bit(const uint32_t* words, size_t i) {
  return (int)((words[i / 32] >> (i % 32)) & 1u);
}

void hqo_unpack(const uint32_t* words, int bits, size_t n_codes,
                uint8_t* codes) {
  for (size_t j = 0; j < n_codes; ++j) {
    int c = 0;
    for (int t = 0; t < bits; ++t) {
      c |= stream_bit(words, (size_t)bits * j + (size_t)t) << t;
    }
    codes[j] = (uint8_t)c;
  }
}

void hqo_pack(const uint8_t* codes, int bits, size_t n_codes,
              uint32_t* words) {
  size_t n_words = ((size_t)bits * n_codes + 31) / 32;
  memset(words, 0, n_words * sizeof(uint32_t));
  for (size_t j = 0; j < n_codes; ++j) {
    for (int t = 0; t < bits; ++t) {
      size_t i = (size_t)bits * j + (size_t)t;
      uint32_t b = (uint32_t)((codes[j] >> t) & 1);
      words[i / 32] |= b << (i % 32);
    }
  }
}

void hqo_unpack_planes2(const uint32_t* words, size_t n_codes, uint8_t* codes) {
  for (size_t j = 0; j < n_codes; ++j) {
    const uint32_t lo = (words[2 * (j / 32)] >> (j % 32)) & 1u;     /* plane 0 */
    const uint32_t hi = (words[2 * (j / 32) + 1] >> (j % 32)) & 1u; /* plane 1 */
    codes[j] = (uint8_t)(lo | (hi << 1));
  }
}

void hqo_pack_planes2(const uint8_t* codes, size_t n_codes, uint32_t* words) {
  memset(words, 0, (n_codes / 32) * 2 * sizeof(uint32_t));
  for (size_t j = 0; j < n_codes; ++j) {
    words[2 * (j / 32)] |= (uint32_t)(codes[j] & 1u) << (j % 32);
    words[2 * (j / 32) + 1] |= (uint32_t)((codes[j] >> 1) & 1u) << (j % 32);
  }
}

/* Sylvester-order butterflies: at stride h, (a, b) -> (a + b, a - b). */
void hqo_fwht(double* v, int n) {
  for (int h = 1; h < n; h *= 2) {
    for (int i = 0; i < n; i += 2 * h) {
      for (int j = i; j < i + h; ++j) {
        double a = v[j];
        double b = v[j + h];
        v[j] = a + b;
        v[j + h] = a - b;
      }
    }
  }
}

static double sign_of(const int8_t* signs, int i) {
  if (signs == NULL) return 1.0;
  return signs[i] < 0 ? -1.0 : 1.0;
}

void hqo_rotate(const double* x, const int8_t* signs, int K, double* out) {
  for (int i = 0; i < K; ++i) out[i] = sign_of(signs, i) * x[i];
  hqo_fwht(out, K);
  double inv = 1.0 / sqrt((double)K);
  for (int i = 0; i < K; ++i) out[i] *= inv;
}

void hqo_rotate_f16(const uint16_t* x, const int8_t* signs, int K,
                    double* out) {
  double* xd = (double*)malloc(sizeof(double) * (size_t)K);
  for (int i = 0; i < K; ++i) xd[i] = hqo_f16_to_f64(x[i]);
  hqo_rotate(xd, signs, K, out);
  free(xd);
}

void hqo_dequant_dot(int bits, int M, int K, int zero, const uint8_t* zeros,
                     const uint32_t* q, const uint16_t* scales, const double* xr,
                     int N, int m_begin, int m_end, double* y, double* bound) {
  const int G = K / 128;
  const size_t words_per_row = (size_t)K * (size_t)bits / 32;
  uint8_t* codes = (uint8_t*)malloc((size_t)K);
  double* w = (double*)malloc(sizeof(double) * (size_t)K);
  for (int m = m_begin; m < m_end; ++m) {
    hqo_unpack(q + (size_t)m * words_per_row, bits, (size_t)K, codes);
    for (int k = 0; k < K; ++k) {
      double s = hqo_f16_to_f64(scales[(size_t)m * G + k / 128]);
      int z = zeros ? (int)zeros[(size_t)m * G + k / 128] : zero;
      w[k] = s * (double)((int)codes[k] - z);
    }
    for (int n = 0; n < N; ++n) {
      const double* xn = xr + (size_t)n * K;
      double acc = 0.0, abs_acc = 0.0;
      for (int k = 0; k < K; ++k) {
        double p = w[k] * xn[k];
        acc += p;
        abs_acc += fabs(p);
      }
      y[(size_t)n * M + m] = acc;
      if (bound) bound[(size_t)n * M + m] = abs_acc;
    }
  }
  free(w);
  free(codes);
}

void hqo_linear(int bits, int M, int K, int zero, const uint8_t* zeros,
                const uint32_t* q, const uint16_t* scales, const int8_t* signs,
                const uint16_t* x, int N, int m_begin, int m_end, double* y,
                double* bound) {
  double* xr = (double*)malloc(sizeof(double) * (size_t)N * (size_t)K);
  for (int n = 0; n < N; ++n) {
    hqo_rotate_f16(x + (size_t)n * K, signs, K, xr + (size_t)n * K);
  }
  hqo_dequant_dot(bits, M, K, zero, zeros, q, scales, xr, N, m_begin, m_end, y,
                  bound);
  free(xr);
}

void hqo_moe(const hqo_expert* experts, int n_experts, int hidden, int inter,
             const uint16_t* x, int T, const int32_t* topk_ids,
             const float* topk_w, int k, const int8_t* s_in,
             const int8_t* s_mid, int t_begin, int t_end, double* y,
             double* bound, double* h_out) {
  (void)n_experts;
  double* xr = (double*)malloc(sizeof(double) * (size_t)hidden);
  double* g = (double*)malloc(sizeof(double) * (size_t)inter);
  double* u = (double*)malloc(sizeof(double) * (size_t)inter);
  double* h = (double*)malloc(sizeof(double) * (size_t)inter);
  double* hr = (double*)malloc(sizeof(double) * (size_t)inter);
  double* d = (double*)malloc(sizeof(double) * (size_t)hidden);
  double* db = (double*)malloc(sizeof(double) * (size_t)hidden);
  double* xe = (double*)malloc(sizeof(double) * (size_t)hidden);
  for (int t = t_begin; t < t_end; ++t) {
    hqo_rotate_f16(x + (size_t)t * hidden, s_in, hidden, xr);
    double* yt = y + (size_t)t * hidden;
    double* bt = bound ? bound + (size_t)t * hidden : NULL;
    for (int i = 0; i < hidden; ++i) {
      yt[i] = 0.0;
      if (bt) bt[i] = 0.0;
    }
    for (int j = 0; j < k; ++j) {
      const hqo_expert* e = &experts[topk_ids[(size_t)t * k + j]];
      /* the expert's own input signs rotate the token again */
      const double* xin = xr;
      if (e->signs_in) {
        hqo_rotate_f16(x + (size_t)t * hidden, e->signs_in, hidden, xe);
        xin = xe;
      }
      hqo_dequant_dot(e->bits, inter, hidden, e->zero, NULL, e->q_gate,
                      e->s_gate, xin, 1, 0, inter, g, NULL);
      hqo_dequant_dot(e->bits, inter, hidden, e->zero, NULL, e->q_up, e->s_up,
                      xin, 1, 0, inter, u, NULL);
      for (int i = 0; i < inter; ++i) {
        h[i] = g[i] / (1.0 + exp(-g[i])) * u[i];
      }
      if (h_out) {
        memcpy(h_out + ((size_t)t * k + j) * inter, h,
               sizeof(double) * (size_t)inter);
      }
      hqo_rotate(h, e->signs_mid ? e->signs_mid : s_mid, inter, hr);
      hqo_dequant_dot(e->bits, hidden, inter, e->zero, NULL, e->q_down,
                      e->s_down, hr, 1, 0, hidden, d, db);
      double wj = (double)topk_w[(size_t)t * k + j];
      for (int i = 0; i < hidden; ++i) {
        yt[i] += wj * d[i];
        if (bt) bt[i] += fabs(wj) * db[i];
      }
    }
  }
  free(xe);
  free(db);
  free(d);
  free(hr);
  free(h);
  free(u);
  free(g);
  free(xr);
}

/* binary16 from the definition: 1 sign bit, 5 exponent bits (bias 15), 10
 * fraction bits; values below 2^-14 are subnormal multiples of 2^-24. */
uint16_t hqo_f64_to_f16(double v) {
  uint16_t sign = signbit(v) ? 0x8000u : 0u;
  double a = fabs(v);
  if (isnan(v)) return (uint16_t)(sign | 0x7e00u);
  /* 65520 is halfway between 65504 (odd fraction) and 65536: ties go to 65536 = inf */
  if (a >= 65520.0) return (uint16_t)(sign | 0x7c00u);
  if (a < ldexp(1.0, -14)) {
    /* subnormal (or zero): a = m 2^-24; m = 1024 is the smallest normal */
    long m = lrint(ldexp(a, 24));
    return (uint16_t)(sign | (uint16_t)m);
  }
  int e2 = 0;
  frexp(a, &e2); /* a = f 2^e2, f in [0.5, 1): a in [2^(e2-1), 2^e2) */
  int E = e2 - 1;
  long mant = lrint(ldexp(a, 10 - E)); /* in [1024, 2048] */
  if (mant == 2048) {
    mant = 1024;
    E += 1;
  }
  if (E > 15) return (uint16_t)(sign | 0x7c00u);
  return (uint16_t)(sign | (uint16_t)((E + 15) << 10) | (uint16_t)(mant - 1024));
}

void hqo_quantize(const double* W, int M, int K, int bits, const int8_t* signs,
                  int m_begin, int m_end, uint32_t* qweight, uint16_t* scales,
                  double* rotated) {
  (void)M;
  const int G = K / 128;
  const int zero = 1 << (bits - 1);
  const int qmax = (1 << bits) - 1;
  const size_t words_per_row = (size_t)K * (size_t)bits / 32;
  double* r = (double*)malloc(sizeof(double) * (size_t)K);
  uint8_t* q = (uint8_t*)malloc((size_t)K);
  for (int m = m_begin; m < m_end; ++m) {
    hqo_rotate(W + (size_t)m * K, signs, K, r);
    if (rotated) memcpy(rotated + (size_t)m * K, r, sizeof(double) * (size_t)K);
    for (int g = 0; g < G; ++g) {
      double amax = 0.0;
      for (int k = 128 * g; k < 128 * g + 128; ++k) {
        if (fabs(r[k]) > amax) amax = fabs(r[k]);
      }
      double want = 2.0 * amax / (double)qmax;
      if (want > 65504.0) want = 65504.0;
      uint16_t s16 = hqo_f64_to_f16(want);
      double s = hqo_f16_to_f64(s16);
      scales[(size_t)m * G + g] = s16;
      for (int k = 128 * g; k < 128 * g + 128; ++k) {
        long c = zero;
        if (s > 0.0) {
          c = lrint(r[k] / s) + zero;
          if (c < 0) c = 0;
          if (c > qmax) c = qmax;
        }
        q[k] = (uint8_t)c;
      }
    }
    hqo_pack(q, bits, (size_t)K, qweight + (size_t)m * words_per_row);
  }
  free(q);
  free(r);
}

void hqo_readout(const uint32_t* hi, const uint32_t* lo, const uint16_t* scales,
                 const int8_t* signs, int V, int K, int zero, const uint16_t* x, int N,
                 int topk, double beta, int32_t* ids, double* out, uint8_t* cand,
                 double* y_all, double* e_out) {
  const int G = K / 128;
  const size_t wpr = (size_t)K * 4 / 32; /* words per row of a 4-bit plane */
  double* xr = (double*)malloc(sizeof(double) * (size_t)K);
  uint8_t* ch = (uint8_t*)malloc((size_t)K);
  uint8_t* cl = (uint8_t*)malloc((size_t)K);
  double* y = (double*)malloc(sizeof(double) * (size_t)V);
  double* L = (double*)malloc(sizeof(double) * (size_t)V);
  double* U = (double*)malloc(sizeof(double) * (size_t)V);
  for (int n = 0; n < N; ++n) {
    hqo_rotate_f16(x + (size_t)n * K, signs, K, xr);
    for (int m = 0; m < V; ++m) {
      hqo_unpack(hi + (size_t)m * wpr, 4, (size_t)K, ch);
      hqo_unpack(lo + (size_t)m * wpr, 4, (size_t)K, cl);
      double ye = 0.0, ys = 0.0, var = 0.0;
      for (int k = 0; k < K; ++k) {
        double s = hqo_f16_to_f64(scales[(size_t)m * G + k / 128]);
        ye += s * (double)(16 * (int)ch[k] + (int)cl[k] - zero) * xr[k];
        ys += s * (16.0 * (double)ch[k] + 7.5 - (double)zero) * xr[k];
        var += s * s * xr[k] * xr[k];
      }
      double sd = sqrt(21.25 * var);
      y[m] = ye;
      L[m] = ys - beta * sd;
      U[m] = ys + beta * sd;
      if (y_all) y_all[(size_t)n * V + m] = ye;
      if (e_out) e_out[(size_t)n * V + m] = ys;
    }
    /* tau: the topk-th largest L (selection by repeated maximum: O(topk V)) */
    double tau = INFINITY;
    {
      uint8_t* taken = (uint8_t*)calloc((size_t)V, 1);
      for (int r = 0; r < topk; ++r) {
        int best = -1;
        for (int m = 0; m < V; ++m) {
          if (!taken[m] && (best < 0 || L[m] > L[best])) best = m;
        }
        taken[best] = 1;
        tau = L[best];
      }
      free(taken);
    }
    /* the topk candidates of largest exact y, ties to the lower index */
    uint8_t* used = (uint8_t*)calloc((size_t)V, 1);
    for (int r = 0; r < topk; ++r) {
      int best = -1;
      for (int m = 0; m < V; ++m) {
        if (used[m] || U[m] < tau) continue;
        if (best < 0 || y[m] > y[best]) best = m;
      }
      used[best] = 1;
      ids[(size_t)n * topk + r] = best;
      out[(size_t)n * topk + r] = y[best];
    }
    free(used);
    if (cand) {
      for (int m = 0; m < V; ++m) cand[(size_t)n * V + m] = U[m] >= tau ? 1 : 0;
    }
  }
  free(U);
  free(L);
  free(y);
  free(cl);
  free(ch);
  free(xr);
}

void hqo_kv_quant_group(const uint16_t* x, int n, int stride, uint8_t* codes,
                        uint16_t* scale, uint16_t* mn) {
  float lo = (float)hqo_f16_to_f64(x[0]), hi = lo;
  for (int i = 1; i < n; ++i) {
    float v = (float)hqo_f16_to_f64(x[(size_t)i * stride]);
    if (v < lo) lo = v;
    if (v > hi) hi = v;
  }
  volatile float span = hi - lo; /* single-precision steps, in this order */
  volatile float sf = span / 15.0f;
  uint16_t s16 = hqo_f64_to_f16((double)sf);
  uint16_t m16 = hqo_f64_to_f16((double)lo);
  float s = (float)hqo_f16_to_f64(s16), m = (float)hqo_f16_to_f64(m16);
  for (int i = 0; i < n; ++i) {
    int c = 0;
    if (s > 0.0f) {
      volatile float diff = (float)hqo_f16_to_f64(x[(size_t)i * stride]) - m;
      volatile float r = diff / s;
      c = (int)rintf(r);
      if (c < 0) c = 0;
      if (c > 15) c = 15;
    }
    codes[i] = (uint8_t)c;
  }
  *scale = s16;
  *mn = m16;
}

void hqo_kv_quantize(const uint16_t* k, const uint16_t* v, int T, int n_kv, int d, uint8_t* kc,
                     uint16_t* ks, uint16_t* km, uint8_t* vc, uint16_t* vs, uint16_t* vm) {
  const int nb = T / 32;
  for (int h = 0; h < n_kv; ++h) {
    for (int b = 0; b < nb; ++b) {
      for (int c = 0; c < d; ++c) { /* channel c over the block's 32 tokens */
        const size_t g = ((size_t)h * nb + b) * d + c;
        hqo_kv_quant_group(k + ((size_t)32 * b * n_kv + h) * d + c, 32, n_kv * d, kc + g * 32, ks + g,
                           km + g);
      }
    }
    for (int t = 0; t < T; ++t) { /* all channels of token t */
      const size_t g = (size_t)h * T + t;
      hqo_kv_quant_group(v + ((size_t)t * n_kv + h) * d, d, 1, vc + g * d, vs + g, vm + g);
    }
  }
}

void hqo_kv_attend(const uint8_t* kc, const uint16_t* ks, const uint16_t* km,
                   const uint8_t* vc, const uint16_t* vs, const uint16_t* vm,
                   int n_kv, int d, int T, const uint16_t* q, int n_q, int n_heads,
                   double* out, double* base) {
  const int G = n_heads / n_kv;
  const int nb = (T + 31) / 32; /* key blocks that tokens 0 .. T-1 fall in */
  double* sc = (double*)malloc(sizeof(double) * (size_t)T);
  double* qd = (double*)malloc(sizeof(double) * (size_t)d);
  for (int i = 0; i < n_q; ++i) {
    for (int j = 0; j < n_heads; ++j) {
      const int h = j / G;
      for (int c = 0; c < d; ++c) qd[c] = hqo_f16_to_f64(q[((size_t)i * n_heads + j) * d + c]);
      double mx = -INFINITY;
      for (int t = 0; t < T; ++t) {
        const int b = t / 32;
        double acc = 0.0;
        for (int c = 0; c < d; ++c) {
          size_t kb = ((size_t)h * nb + b) * d + c;
          double kv = hqo_f16_to_f64(ks[kb]) * (double)kc[kb * 32 + (t % 32)] + hqo_f16_to_f64(km[kb]);
          acc += qd[c] * kv;
        }
        sc[t] = acc / sqrt((double)d);
        if (sc[t] > mx) mx = sc[t];
      }
      double l = 0.0;
      for (int t = 0; t < T; ++t) {
        sc[t] = exp(sc[t] - mx);
        l += sc[t];
      }
      for (int c = 0; c < d; ++c) {
        double o = 0.0, bs = 0.0;
        for (int t = 0; t < T; ++t) {
          size_t vt = (size_t)h * T + t;
          double v = hqo_f16_to_f64(vs[vt]) * (double)vc[vt * d + c] + hqo_f16_to_f64(vm[vt]);
          o += sc[t] / l * v;
          bs += sc[t] / l * fabs(v);
        }
        out[((size_t)i * n_heads + j) * d + c] = o;
        if (base) base[((size_t)i * n_heads + j) * d + c] = bs;
      }
    }
  }
  free(qd);
  free(sc);
}
