/*
 * hq_oracle.h -- plain fp64 CPU oracle for the rotated low-bit linear.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product library links, includes
 * or calls this code; only the tests, the smoke check and the benchmark's
 * CPU-baseline leg do.  It shares no header, helper or constant with the CUDA
 * path.
 *
 * What it computes (all in double precision, scalar loops, no blocking):
 *   - the random-sign Hadamard rotation  x' = H_K . diag(s) . x / sqrt(K)
 *     ("group-128 GPTQ in a Hadamard-rotated basis", rotation signs kept in
 *     small.bin: LLaDA2.2-mini Orin-Nano model card, Properties table and the
 *     file-list paragraph; "behind a random Hadamard rotation": Qwen3.8-27B
 *     Pingala-8 2-bit card, "What this is"),
 *   - the group-128 dequantisation  w[m][k] = scale[m][k/128] * (q[m][k] - z),
 *   - the contraction  y[n][m] = sum_k w[m][k] * x'[n][k],
 *   - the MoE expert composition (gate/up, SwiGLU, down, weighted combine),
 *   - the rotated round-to-nearest quantiser that produces packed weights.
 *
 * Readings where the pages are silent (the plainest reading in each case):
 *   - H_K is the Sylvester Hadamard matrix in natural order,
 *     H[i][j] = (-1)^popcount(i & j); the 1/sqrt(K) factor is applied once.
 *   - sign s_i = -1 where signs[i] < 0, else +1; a NULL sign vector means s = 1.
 *   - packed codes: code j of a row occupies bits [b*j, b*j+b) of the row's
 *     little-endian bit stream (word w holds stream bits [32w, 32w+32)).
 *     For b = 3 this makes three words carry 32 codes, codes 10 and 21
 *     straddling a word boundary.
 *   - zero point z is one integer per tensor (2^(b-1) in every workload).
 *
 * Parity pins (tests/test_oracle_pins.py): dense brute-force Hadamard,
 * H.H^T = K.I, norm preservation, involution, closed forms, numpy bit
 * unpacking, an explicit dense W_eff = dequant(Q).H.diag(s)/sqrt(K) product,
 * and MoE reductions to single-expert chains.
 */
#ifndef HQ_ORACLE_H
#define HQ_ORACLE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* IEEE binary16 bit pattern -> double (normals, subnormals, zeros, inf, nan). */
double hqo_f16_to_f64(uint16_t h);

/* Decode n_codes codes of width bits (1..8) from the packed little-endian bit
 * stream in words.  codes[j] = stream bits [bits*j, bits*j+bits). */
void hqo_unpack(const uint32_t* words, int bits, size_t n_codes, uint8_t* codes);

/* 2-bit codes kept as two bit-planes ("2-bit bit-planes ... kept that way for
 * the whole run": Qwen3-8B BPDQ 2-bit card, introduction; the page gives no
 * layout, this is the library's): per span of 32 codes j = 32 s + i, word 2s
 * holds bit 0 of each code (bit i), word 2s + 1 bit 1; code = b0 + 2 b1.
 * n_codes a multiple of 32. */
void hqo_unpack_planes2(const uint32_t* words, size_t n_codes, uint8_t* codes);
/* Inverse of hqo_unpack_planes2 (n_codes / 16 words, fully overwritten). */
void hqo_pack_planes2(const uint8_t* codes, size_t n_codes, uint32_t* words);

/* Inverse of hqo_unpack.  Words must have room for ceil(bits*n_codes/32)
 * entries; they are fully overwritten (unused high bits are zero). */
void hqo_pack(const uint8_t* codes, int bits, size_t n_codes, uint32_t* words);

/* In-place unnormalised fast Walsh-Hadamard transform, v <- H_n v, n a power
 * of two, Sylvester natural order. */
void hqo_fwht(double* v, int n);

/* out = H_K diag(s) x / sqrt(K) for one row.  x in double. */
void hqo_rotate(const double* x, const int8_t* signs, int K, double* out);

/* Same, input row given as fp16 bit patterns. */
void hqo_rotate_f16(const uint16_t* x, const int8_t* signs, int K, double* out);

/* Dequantise-and-dot for output rows [m_begin, m_end):
 *   y[n][m]     = sum_k scale[m][k/128] * (q[m][k] - z[m][k/128]) * xr[n][k]
 *   bound[n][m] = sum_k |scale[m][k/128] * (q[m][k] - z[m][k/128]) * xr[n][k]|
 * z[m][g] = zeros[m][g] (uint8 [M][K/128], per-group zero points, the GPTQ
 * form) when zeros is not NULL, else the per-tensor integer `zero`.
 * q: row-major packed codes, K*bits/32 words per row.
 * scales: fp16 bit patterns [M][K/128].  xr: already-rotated inputs [N][K].
 * y, bound: [N][M] (only columns m_begin..m_end-1 are written; bound may be
 * NULL). */
void hqo_dequant_dot(int bits, int M, int K, int zero, const uint8_t* zeros,
                     const uint32_t* q, const uint16_t* scales, const double* xr,
                     int N, int m_begin, int m_end, double* y, double* bound);

/* The whole rotated linear for rows [m_begin, m_end): rotate each of the N
 * fp16 input rows with signs, then hqo_dequant_dot (zeros as there). */
void hqo_linear(int bits, int M, int K, int zero, const uint8_t* zeros,
                const uint32_t* q, const uint16_t* scales, const int8_t* signs,
                const uint16_t* x, int N, int m_begin, int m_end, double* y,
                double* bound);

/* One routed expert: three packed linears with a shared bit width. */
typedef struct {
  int bits;
  int zero;
  const uint32_t* q_gate; /* [inter][hidden*bits/32] */
  const uint32_t* q_up;   /* [inter][hidden*bits/32] */
  const uint32_t* q_down; /* [hidden][inter*bits/32] */
  const uint16_t* s_gate; /* [inter][hidden/128] */
  const uint16_t* s_up;   /* [inter][hidden/128] */
  const uint16_t* s_down; /* [hidden][inter/128] */
  const int8_t* signs_in;  /* [hidden] this expert's own rotation signs, or NULL */
  const int8_t* signs_mid; /* [inter] likewise for its down projection, or NULL */
} hqo_expert;

/* MoE expert layer for tokens [t_begin, t_end) (s_in, s_mid: the expert's
 * own signs_in / signs_mid where it has them, else the shared vectors):
 *   x'_t   = rot(x_t, s_in)                        (hidden)
 *   g, u   = W_gate^e x'_t, W_up^e x'_t            (inter)
 *   h      = g / (1 + exp(-g)) * u                 (SwiGLU)
 *   h'     = rot(h, s_mid)                         (inter)
 *   d      = W_down^e h'                           (hidden)
 *   y_t    = sum_{j=0..k-1} topk_w[t][j] * d_{t,j}  (j ascending)
 *   bound_t = sum_j |topk_w[t][j]| * sum_k |w_down * h'|
 * h_out (optional, [T*k][inter]) receives h for pair (t, j) at row t*k+j. */
void hqo_moe(const hqo_expert* experts, int n_experts, int hidden, int inter,
             const uint16_t* x, int T, const int32_t* topk_ids,
             const float* topk_w, int k, const int8_t* s_in,
             const int8_t* s_mid, int t_begin, int t_end, double* y,
             double* bound, double* h_out);

/* IEEE binary16 bit pattern nearest to v (round to nearest, ties to even;
 * overflow to infinity, NaN to a quiet NaN). */
uint16_t hqo_f64_to_f16(double v);

/* Rotated round-to-nearest quantiser, the step that produces the packed
 * weights ("group-128 GPTQ in a Hadamard-rotated basis": LLaDA2.2-mini
 * Orin-Nano model card, Properties table; weights "behind a random Hadamard
 * rotation": Qwen3.8-27B Pingala-8 2-bit card, "What this is"), without
 * GPTQ's calibration-driven rounding, for rows [m_begin, m_end):
 *   r        = H_K diag(s) W[m] / sqrt(K)        (fp64; = (W diag(s) H_K)[m] / sqrt(K))
 *   a_g      = max_{k in group g} |r_k|          (groups of 128 along K)
 *   scale_g  = fp16(min(2 a_g / (2^b - 1), 65504))   (round to nearest even)
 *   q_k      = clamp(rint(r_k / scale_g) + 2^(b-1), 0, 2^b - 1), or 2^(b-1)
 *              where scale_g = 0                  (rint: ties to even)
 * so that dequant(q) = scale (q - 2^(b-1)) with the library's zero point.
 * W: [M][K] doubles.  qweight: [M][K*bits/32] words (hqo_pack layout per
 * row); scales: [M][K/128] fp16 bit patterns; rotated (optional, [M][K]):
 * r.  Only rows m_begin..m_end-1 are written. */
void hqo_quantize(const double* W, int M, int K, int bits, const int8_t* signs,
                  int m_begin, int m_end, uint32_t* qweight, uint16_t* scales,
                  double* rotated);

/* Nibble-split screened readout over an 8-bit lm_head (the "high/low nibble
 * split planes ... for screened readout" of the LLaDA2.2-mini Orin-Nano model
 * card, file list and Properties table; the pages give no rule, this is the
 * library's).  W has 8-bit codes q = 16 hi + lo (zero point `zero`, group-128
 * fp16 scales), stored as two 4-bit planes hi[V][K/8], lo[V][K/8] (hqo_pack
 * layout).  For each batch row n, with x' = H diag(s) x_n / sqrt(K):
 *   exact     y[m]  = sum_k scale (16 hi + lo - zero) x'_k
 *   screen    e[m]  = sum_k scale (16 hi + 7.5 - zero) x'_k   (low nibble at
 *                     its mean; reads only the high plane)
 *   spread    sd[m] = sqrt(21.25 sum_k scale^2 x'_k^2)   (standard deviation
 *                     of the low-nibble term if the low nibbles were
 *                     independent and uniform on 0..15: variance 255/12)
 *   bounds    L[m] = e[m] - beta sd[m],  U[m] = e[m] + beta sd[m]
 *   tau       = the topk-th largest L
 *   cand[m]   = U[m] >= tau
 *   result    the topk rows of largest exact y among the candidates (ties to
 *             the lower row index), ids and y, descending.
 * cand (optional, [N][V] bytes), y_all (optional, [N][V] exact logits of
 * every row), e_out (optional, [N][V]).  ids [N][topk] int32, out [N][topk]. */
void hqo_readout(const uint32_t* hi, const uint32_t* lo, const uint16_t* scales,
                 const int8_t* signs, int V, int K, int zero, const uint16_t* x, int N,
                 int topk, double beta, int32_t* ids, double* out, uint8_t* cand,
                 double* y_all, double* e_out);

/* int4 KV cache ("Runtime int4 (keys per channel per 32-token block, values
 * per token)": LLaDA2.2-mini Orin-Nano model card, Properties table; the
 * quantiser is this library's reading, asymmetric min/scale with 4-bit codes).
 * One group of n values x (fp16 bit patterns, stride `stride` elements):
 *   lo = min x, hi = max x                     (in float)
 *   scale = fp16(float(hi - lo) / 15), mn = fp16(lo)      (round to nearest even)
 *   code_i = clamp(rintf((x_i - mn) / scale), 0, 15), 0 where scale = 0
 * computed in IEEE single precision (the decision's precision).  Keys: a group
 * is one channel of one head over a 32-token block; values: all head_dim
 * channels of one head for one token.  codes receives n bytes. */
void hqo_kv_quant_group(const uint16_t* x, int n, int stride, uint8_t* codes,
                        uint16_t* scale, uint16_t* mn);

/* The whole cache of T tokens (T a multiple of 32): k, v fp16
 * [T][n_kv][d]; kc [n_kv][T/32][d][32], ks, km [n_kv][T/32][d], vc
 * [n_kv][T][d], vs, vm [n_kv][T], each group through hqo_kv_quant_group. */
void hqo_kv_quantize(const uint16_t* k, const uint16_t* v, int T, int n_kv, int d, uint8_t* kc,
                     uint16_t* ks, uint16_t* km, uint8_t* vc, uint16_t* vs, uint16_t* vm);

/* Attention over a dequantised cache, fp64: for each query row r (query
 * token i, head j; kv head j / (n_heads / n_kv)):
 *   s_t = (q_r . k_t) / sqrt(d),  p = softmax over t < T,  out_r = sum_t p_t v_t
 * with k_t[c] = k_scale[c of t's block] code + k_min, v_t[c] = v_scale[t] code
 * + v_min[t].  T >= 1 need not be a multiple of 32: the key arrays hold
 * the nb = ceil(T/32) blocks that tokens 0 .. T-1 fall in, and only those
 * tokens are attended.  kc: [n_kv][nb][d][32] key codes (one byte each), ks,
 * km: [n_kv][nb][d] fp16; vc: [n_kv][T][d] value codes, vs, vm: [n_kv][T].
 * q: [n_q][n_heads][d] fp16; out, base: [n_q][n_heads][d] (base = sum_t p_t
 * |v_t[c]|, the tolerance base; may be NULL). */
void hqo_kv_attend(const uint8_t* kc, const uint16_t* ks, const uint16_t* km,
                   const uint8_t* vc, const uint16_t* vs, const uint16_t* vm,
                   int n_kv, int d, int T, const uint16_t* q, int n_q, int n_heads,
                   double* out, double* base);

#ifdef __cplusplus
}
#endif
#endif /* HQ_ORACLE_H */
