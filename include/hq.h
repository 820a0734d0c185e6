/*
 * hq.h -- C ABI of libhq: matmuls over packed low-bit, Hadamard-rotated
 * weights on NVIDIA B200 (sm_100a).
 *
 * The method (LLaDA2.2-mini Orin-Nano model card, Properties table and the
 * file-list paragraph): routed-expert weights are "group-128 GPTQ in a
 * Hadamard-rotated basis", 2/3/4 bits per expert, non-expert layers 8-bit,
 * with the rotation signs stored beside them.  The weights stay packed for
 * the whole run and are dequantised inside the matmul (Qwen3-8B BPDQ 2-bit
 * card, introduction: "kept that way for the whole run"; decode time follows
 * the weight bytes: Laguna-S-2.1 gridbook card, "Reading it honestly").
 *
 * Definitions used by every entry point (this library's reading of the pages,
 * which give no formulas):
 *   rotation     x' = H_K . diag(s) . x / sqrt(K)
 *                H_K: Sylvester Hadamard matrix, natural order,
 *                H[i][j] = (-1)^popcount(i & j); s_i = -1 if signs[i] < 0,
 *                else +1; signs == NULL means s = 1.
 *   codes        row m of a packed matrix is K*bits/32 uint32 words; code k of
 *                the row occupies bits [bits*k, bits*k + bits) of the row's
 *                little-endian bit stream (word w holds stream bits
 *                [32w, 32w+32)).  For bits = 3, three words carry 32 codes and
 *                codes 10 and 21 of each triplet straddle a word boundary.
 *   dequant      w[m][k] = scale[m][k/128] * (q[m][k] - zero), group size 128
 *                along K, scale an IEEE fp16 bit pattern, zero an integer
 *                (one per tensor, or one per row and group: hq_weight.zeros).
 *   linear       y[n][m] = sum_k w[m][k] * x'[n][k], fp32 output.
 *
 * Conventions:
 *   - Every pointer argument is a DEVICE pointer owned by the caller unless
 *     stated otherwise.  The library allocates and frees nothing.
 *   - Every call is asynchronous on `stream` (a cudaStream_t; NULL is the
 *     legacy default stream) and returns before the work finishes, except
 *     hq_check_status, which synchronises the stream.
 *   - Argument errors are detected on the host before anything is launched;
 *     the call then returns the status and writes nothing.  A launch failure
 *     returns HQ_ERR_CUDA.  Errors found by device code (a bounded wait that
 *     ran out, an expert id or bit width out of range in device data) are
 *     OR-ed into the status word at the start of the caller's workspace and
 *     read back by hq_check_status; device code never traps.
 *   - A workspace must be at least the queried size, 256-byte aligned, and
 *     zero-filled before its first use.  Calls leave it ready for the next
 *     call (counters back at zero) unless a device error was recorded; after
 *     HQ_ERR_TIMEOUT, zero it again.  One workspace serves one stream at a
 *     time: calls that overlap on the GPU must not share it.
 *   - Outputs are overwritten, never accumulated into.  Inputs and outputs
 *     must not alias.
 *   - Kernels are launched with programmatic dependent launch: a call's
 *     kernels may start while the library kernel before them on the stream is
 *     finishing, and read the weights (packed codes, scales, signs, the
 *     expert table) before waiting for it; activations, routing inputs and
 *     the workspace are read only after it has finished.  Weights must
 *     therefore not be rewritten by the library call just before on the same
 *     stream (no library call writes them), and any other kernel or copy that
 *     writes them must complete, in stream order, before the call.
 *   - Alignment: packed weights, scales, activations and outputs must be
 *     16-byte aligned; the library checks this and returns
 *     HQ_ERR_INVALID_ARG otherwise.
 */
#ifndef HQ_H
#define HQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

struct CUstream_st;
/* The same handle as cudaStream_t. */
typedef struct CUstream_st* hq_stream_t;

typedef enum {
  HQ_OK = 0,
  HQ_ERR_INVALID_ARG = 1, /* bad pointer, size, alignment or value */
  HQ_ERR_UNSUPPORTED = 2, /* valid but not implemented (e.g. K not a power of two) */
  HQ_ERR_WORKSPACE = 3,   /* workspace NULL, misaligned or smaller than queried */
  HQ_ERR_CUDA = 4,        /* a CUDA launch or runtime call failed */
  HQ_ERR_DATA = 5,        /* device data out of range (expert id, bits, zero) */
  HQ_ERR_TIMEOUT = 6      /* a bounded device-side wait ran out */
} hq_status;

typedef enum { HQ_F16 = 0, HQ_BF16 = 1, HQ_F32 = 2 } hq_dtype;

/* Storage of the codes of a weight row.  HQ_LAYOUT_PACKED: the little-endian
 * bit stream above.  HQ_LAYOUT_BITPLANES (2-bit codes only): the codes as two
 * bit-planes ("2-bit bit-planes ... kept that way for the whole run": Qwen3-8B
 * BPDQ 2-bit card, introduction; the page gives no layout, this is the
 * library's): per span of 32 codes k = 32 s + i, word 2s holds bit 0 of each
 * code (at bit i), word 2s + 1 bit 1, so q = b0 + 2 b1.  Same size as the
 * packed stream (K/16 words a row).  hq_to_bitplanes converts. */
typedef enum { HQ_LAYOUT_PACKED = 0, HQ_LAYOUT_BITPLANES = 1 } hq_layout;

/* One packed, rotated weight matrix W [M][K]. */
typedef struct {
  int bits;                /* 2, 3, 4 or 8 */
  int M;                   /* output features, >= 1 */
  int K;                   /* input features: power of two, 128 <= K <= 32768 */
  int zero;                /* integer zero point, 0 <= zero < 2^bits (2^(bits-1) usual) */
  const uint32_t* qweight; /* [M][K*bits/32] packed codes, 16-byte aligned */
  const uint16_t* scales;  /* [M][K/128] fp16 bit patterns, 16-byte aligned */
  const int8_t* signs;     /* [K] rotation signs, or NULL for s = 1 */
  const uint8_t* zeros;    /* [M][K/128] per-group zero points (each < 2^bits), or
                              NULL: `zero` for every group.  16-byte aligned.  The
                              per-group form is GPTQ's usual one; with it, every
                              batch runs the small-batch kernel in blocks of up to
                              8 columns (the tensor-core path takes the scalar
                              zero only). */
  int layout;              /* hq_layout of qweight (HQ_LAYOUT_PACKED = 0 when the
                              struct is zero-initialised).  HQ_LAYOUT_BITPLANES
                              needs bits = 2 (HQ_ERR_UNSUPPORTED otherwise) and,
                              like per-group zeros, runs every batch on the
                              small-batch kernel in blocks of up to 8 columns. */
} hq_weight;

/*
 * hq_rotate -- the random-sign Hadamard rotation alone, row by row.
 *   x_rot[r][:] = H_K diag(s) x[r][:] / sqrt(K),   r < n_rows.
 * x: [n_rows][K] of x_dtype (HQ_F16, HQ_BF16 or HQ_F32), row-major.
 * x_rot: [n_rows][K] of out_dtype (HQ_F16, HQ_BF16 or HQ_F32).
 * K: power of two, 32 <= K <= 32768.  n_rows >= 0 (0 launches nothing).
 * Computed in fp32 (butterflies), rounded once to out_dtype.
 * Cites: "Hadamard-rotated basis" and "rotation signs" (LLaDA2.2-mini
 * Orin-Nano model card, Properties table, file list); "behind a random
 * Hadamard rotation" (Qwen3.8-27B Pingala-8 2-bit card, "What this is").
 */
hq_status hq_rotate(const void* x, hq_dtype x_dtype, void* x_rot, hq_dtype out_dtype,
                    int n_rows, int K, const int8_t* signs, hq_stream_t stream);

/* Bytes of workspace hq_linear needs for this weight and batch (0 on a bad
 * argument).  Constant for a given (bits, M, K, batch). */
size_t hq_linear_workspace_size(const hq_weight* w, int batch);

/*
 * hq_linear -- y = dequant(Q) . x' with x' the rotated activations:
 *   y[n][m] = sum_k scale[m][k/128] (q[m][k] - zero) (H_K diag(s) x[n] / sqrt(K))[k]
 * w: host pointer to the weight descriptor (device pointers inside).
 * x: [batch][K] fp16 activations.  batch >= 0 (0 launches nothing).
 * y: [batch][M] fp32 output.
 * workspace: >= hq_linear_workspace_size(w, batch) bytes.
 * Small batches run a fused unpack-dequant GEMV that streams the packed
 * codes; batches up to 16 a 32-row variant of it (activations staged in K
 * slices); larger batches a tensor-core GEMM (hq_linear_path tells which).
 * All accumulate in fp32.
 * Cites: group-128 codes, 2/3/4-bit experts and 8-bit non-expert layers
 * (LLaDA2.2-mini Orin-Nano model card, Properties table).
 */
hq_status hq_linear(const hq_weight* w, const uint16_t* x, int batch, float* y,
                    void* workspace, size_t ws_bytes, hq_stream_t stream);

/* One routed expert: SwiGLU FFN with packed gate/up [inter][hidden] and
 * down [hidden][inter], all at one bit width.  Device-side table entry. */
typedef struct {
  int bits;               /* 2, 3 or 4 (8 also accepted) */
  int zero;               /* 0 <= zero < 2^bits */
  const uint32_t* q_gate; /* [inter][hidden*bits/32] */
  const uint32_t* q_up;   /* [inter][hidden*bits/32] */
  const uint32_t* q_down; /* [hidden][inter*bits/32] */
  const uint16_t* s_gate; /* [inter][hidden/128] fp16 */
  const uint16_t* s_up;   /* [inter][hidden/128] fp16 */
  const uint16_t* s_down; /* [hidden][inter/128] fp16 */
  const int8_t* signs_in;  /* [hidden] this expert's own rotation signs for gate/up,
                              or NULL: the call's signs_in (16-byte aligned) */
  const int8_t* signs_mid; /* [inter] its own signs for down, or NULL: the call's */
} hq_expert;

size_t hq_moe_workspace_size(int n_experts, int hidden, int inter, int T, int k);

/*
 * hq_moe_experts -- the routed-expert part of an MoE layer, all experts and
 * bit widths in one pass per phase, no host synchronisation:
 *   x'_t  = H_hidden diag(s_in) x_t / sqrt(hidden)   (s_in, s_mid: the expert's
 *                                                    own signs where it has them)
 *   g, u  = W_gate^e x'_t,  W_up^e x'_t           for e = topk_ids[t][j]
 *   h     = g / (1 + exp(-g)) * u                  (SwiGLU)
 *   h'    = H_inter diag(s_mid) h / sqrt(inter)
 *   d     = W_down^e h'
 *   y_t   = sum_{j=0..k-1} topk_w[t][j] * d_{t,j}  (j ascending, fixed order)
 * experts: DEVICE array [n_experts] of hq_expert.  x: [T][hidden] fp16.
 * topk_ids: [T][k] int32, topk_w: [T][k] fp32.  signs_in [hidden], signs_mid
 * [inter] (NULL = no sign flip).  y: [T][hidden] fp32.
 * hidden, inter: powers of two in [128, 32768].  1 <= k <= 32.
 * 1 <= n_experts <= 16384 (HQ_ERR_UNSUPPORTED above).
 * An expert id outside [0, n_experts), or an expert whose bits or zero is out
 * of range, is skipped (its contribution is zero) and sets HQ_ERR_DATA in the
 * workspace status word.
 * Cites: mixed 2/3/4-bit routed experts with per-expert widths in a manifest
 * and the 32-token denoising block (LLaDA2.2-mini Orin-Nano model card,
 * Properties table and "Measured Throughput").
 */
hq_status hq_moe_experts(const hq_expert* experts, int n_experts, int hidden, int inter,
                         const uint16_t* x, int T, const int32_t* topk_ids,
                         const float* topk_w, int k, const int8_t* signs_in,
                         const int8_t* signs_mid, float* y, void* workspace,
                         size_t ws_bytes, hq_stream_t stream);

/*
 * hq_linear_noalloc -- hq_linear without a workspace, for callers that cannot
 * allocate device memory (a plug-in whose host program owns the device heap, a
 * latency-critical loop that must not call cudaMalloc, a binding with device
 * pointers but no allocator).  The pages have no counterpart: this is a
 * packaging variant of hq_linear, same arguments minus the workspace, results
 * within the same tolerance: every batch runs the GEMV kernels in blocks of up
 * to 8 columns (the 32-row GEMV and tensor-core paths that hq_linear uses for
 * larger batches need a workspace for their activation images).
 * Its scratch is a 512 KiB array in the library's device memory, held on every
 * GPU that loads the library until the process exits: the status word and the
 * rotated activations of one batch block (at most 332 KiB).  Limits:
 * as hq_linear (HQ_ERR_WORKSPACE if a block's activations did not fit, which
 * no supported K reaches).
 * The array's device address is looked up on every call (a runtime query that
 * allocates nothing); the first call in a CUDA context also loads the
 * library's device code there, so make that first call before any stream
 * capture.  All calls share the array: calls that overlap on the GPU race and
 * must be serialised by the caller.  Each call clears the array's status word
 * before its kernels run; hq_linear_noalloc_check_status reads it back.
 */
hq_status hq_linear_noalloc(const hq_weight* w, const uint16_t* x, int batch, float* y,
                            hq_stream_t stream);

/*
 * hq_quantize -- packs real-valued weights W [M][K] into the format above: a
 * rotated round-to-nearest quantiser (the pages quantise with GPTQ, whose
 * rounding needs calibration data; this is its data-free counterpart).
 *   r       = H_K diag(s) W[m] / sqrt(K)                  (computed in fp64)
 *   scale_g = fp16(min(2 max_{k in g} |r_k| / (2^bits - 1), 65504)),
 *             g a group of 128 consecutive k (round to nearest even)
 *   q_k     = clamp(rint(r_k / scale_g) + 2^(bits-1), 0, 2^bits - 1),
 *             2^(bits-1) where scale_g = 0                 (rint: ties to even)
 * The result is used as an hq_weight with zero = 2^(bits-1) and the same
 * signs: then y = dequant(Q) x' approximates W x (the rotation cancels), each
 * rotated weight within about half a grid step, scale_g / 2.
 * W: [M][K] of w_dtype (HQ_F16, HQ_BF16 or HQ_F32), row-major, finite values.
 * qweight: [M][K*bits/32] words, scales: [M][K/128] fp16 bit patterns, both
 * written whole.  All pointers 16-byte aligned device pointers.  bits 2, 3, 4
 * or 8; K a power of two in [128, 32768]; M >= 0 (0 launches nothing).
 * Cites: "group-128 GPTQ in a Hadamard-rotated basis" (LLaDA2.2-mini
 * Orin-Nano model card, Properties table); weights "behind a random Hadamard
 * rotation" (Qwen3.8-27B Pingala-8 2-bit card, "What this is").
 */
hq_status hq_quantize(const void* W, hq_dtype w_dtype, int M, int K, int bits,
                      const int8_t* signs, uint32_t* qweight, uint16_t* scales,
                      hq_stream_t stream);

/* An 8-bit lm_head kept as high and low nibble planes: codes q = 16 hi + lo,
 * w[m][k] = scale[m][k/128] (q - zero), in the rotated basis. */
typedef struct {
  int V;                  /* rows (vocabulary), >= 1 */
  int K;                  /* input features: power of two, 128 <= K <= 32768 */
  int zero;               /* integer zero point of the 8-bit codes, 0..255 (128 usual) */
  const uint32_t* hi;     /* [V][K/8] high nibbles, 4-bit layout (as a 4-bit hq_weight) */
  const uint32_t* lo;     /* [V][K/8] low nibbles, likewise */
  const uint16_t* scales; /* [V][K/128] fp16 */
  const int8_t* signs;    /* [K] rotation signs, or NULL */
} hq_readout_weight;

/* Bytes of workspace hq_readout_topk needs (0 on a bad argument). */
size_t hq_readout_workspace_size(const hq_readout_weight* r, int batch);

/*
 * hq_readout_topk -- the topk rows of largest logit y[n][m] = sum_k w[m][k]
 * x'[n][k] (x' = H_K diag(s) x[n] / sqrt(K)), reading the high-nibble plane
 * of every row but the low-nibble plane of screened candidates only.
 * Screening rule (the pages give none; this library's): the screen
 * e[m] = sum_k scale (16 hi + 7.5 - zero) x'_k puts each low nibble at its
 * mean; the low nibbles' term has standard deviation sd[m] = sqrt(21.25
 * sum_k scale^2 x'_k^2) were they independent and uniform on 0..15; rows with
 * e + beta sd at or above the topk-th largest e - beta sd (taken, on the GPU,
 * at the lower edge of its bin in a histogram of the top 11 bits, which only
 * widens the set) get their exact logit from both planes; the topk largest
 * exact logits are returned, descending, ties to the lower row.  The result
 * is exact whenever no candidate's low-nibble term strays beyond beta
 * standard deviations (beta = 6 in tests).
 * x: [batch][K] fp16, 1 <= batch <= 8.  ids: [batch][topk] int32, logits:
 * [batch][topk] fp32.  1 <= topk <= 256, topk <= V.  beta >= 0.
 * workspace: >= hq_readout_workspace_size bytes, zero-filled before first
 * use; calls leave it ready for the next call.
 * Cites: "8-bit lm_head.bin + nibble-split lm_head_split.bin (screened
 * readout)" (LLaDA2.2-mini Orin-Nano model card, Properties table and file
 * list).
 */
hq_status hq_readout_topk(const hq_readout_weight* r, const uint16_t* x, int batch, int topk,
                          float beta, int32_t* ids, float* logits, void* workspace,
                          size_t ws_bytes, hq_stream_t stream);

/* Splits 8-bit packed codes q8 [rows][K/4] into high and low nibble planes
 * hi, lo [rows][K/8] (4-bit layout): the "same codes split into high/low
 * nibble planes" of the model card's file list.  K a multiple of 8. */
hq_status hq_split_nibbles(const uint32_t* q8, int rows, int K, uint32_t* hi, uint32_t* lo,
                           hq_stream_t stream);

/*
 * The int4 KV cache of one attention layer: keys quantised per channel per
 * 32-token block, values per token ("KV Cache Format: Runtime int4 (keys per
 * channel per 32-token block, values per token)": LLaDA2.2-mini Orin-Nano
 * model card, Properties table).  Each group of values x gets, in IEEE single
 * precision, scale = fp16((max x - min x) / 15), mn = fp16(min x) and codes
 * clamp(rint((x - mn) / scale), 0, 15) (0 where scale = 0); x ~ scale * code
 * + mn.  The caller allocates the six arrays (device memory; the library
 * keeps no pointer past a call); with nb = capacity / 32 and d = head_dim:
 *   k_codes [n_kv][nb][32 tokens][d/2] bytes  channel c of a token in byte
 *                                             c/2, low nibble for even c
 *   k_scale, k_min [n_kv][nb][d]   fp16       one group per (block, channel)
 *   v_codes [n_kv][nb][d][16] bytes           token t of a block in byte t/2
 *                                             of its channel's line, low
 *                                             nibble for even t
 *   v_scale, v_min [n_kv][capacity] fp16      one group per token
 * head_dim 64 or 128 (HQ_ERR_UNSUPPORTED otherwise); capacity a multiple of
 * 32, <= 2^24; all six arrays 16-byte aligned.
 */
typedef struct {
  int head_dim;
  int n_kv_heads;
  int capacity;
  uint8_t* k_codes;
  uint16_t* k_scale;
  uint16_t* k_min;
  uint8_t* v_codes;
  uint16_t* v_scale;
  uint16_t* v_min;
} hq_kv_cache;

/* Quantises n_new new tokens into cache positions pos .. pos + n_new - 1.
 * k, v: fp16 [n_new][n_kv_heads][head_dim] (device).  pos and n_new are
 * multiples of 32 (whole key blocks), pos + n_new <= capacity; n_new = 0
 * launches nothing.  Bit-exact with the quantiser above. */
hq_status hq_kv_append(const hq_kv_cache* cache, const uint16_t* k, const uint16_t* v, int pos,
                       int n_new, hq_stream_t stream);

/* Bytes of workspace hq_kv_attend needs (0 on a bad argument). */
size_t hq_kv_attend_workspace_size(const hq_kv_cache* cache, int n_tokens, int n_q, int n_heads);

/* Kernels one hq_kv_attend call enqueues. */
int hq_kv_attend_launches(void);

/*
 * hq_kv_attend -- softmax attention of n_q query tokens over the first
 * n_tokens tokens of the cache, grouped-query: head j reads kv head
 * j / (n_heads / n_kv_heads).  For query token i, head j, kv head h:
 *   s_t = q[i][j] . k_h(t) / sqrt(head_dim),  p = softmax_t(s),
 *   out[i][j] = sum_t p_t v_h(t),
 * k_h(t), v_h(t) the dequantised cached key and value; no causal mask (every
 * query sees all n_tokens, as a block of tokens being denoised together
 * does).  q: fp16 [n_q][n_heads][head_dim], 16-byte aligned; out: fp32
 * [n_q][n_heads][head_dim], 16-byte aligned.  1 <= n_tokens <= capacity,
 * and every 32-token block that n_tokens reaches must have been appended.
 * n_q * n_heads / n_kv_heads <= 4096 (HQ_ERR_UNSUPPORTED above); n_q = 0
 * launches nothing.  workspace: >= hq_kv_attend_workspace_size bytes,
 * 256-byte aligned (HQ_ERR_WORKSPACE otherwise), zero-filled before its
 * first use: its first word is a status word that a bounded device-side wait
 * which ran out sets (read and cleared by hq_check_status).
 * Numerics: a score is sum_c q_c s_c code + sum_c q_c min_c with every
 * product exact in the tensor cores (the key scale split into two fp16
 * halves whose products with a 4-bit code are exact), sums in fp32; p *
 * v_scale enters as fp16 hi + lo (about 2^-22 relative); exp through the
 * hardware 2^x (about 2^-22 relative).  Key groups whose scale times 15
 * exceeds 65504 (a group spanning more than the fp16 range, keys beyond
 * about +-32752 of both signs) are outside this exactness and overflow.
 */
hq_status hq_kv_attend(const hq_kv_cache* cache, int n_tokens, const uint16_t* q, int n_q,
                       int n_heads, float* out, void* workspace, size_t ws_bytes,
                       hq_stream_t stream);

/* Converts 2-bit codes from the packed stream (n_codes / 16 words) to the
 * bit-plane layout of HQ_LAYOUT_BITPLANES (as many words).  n_codes a
 * multiple of 32; both arrays 8-byte aligned; 0 launches nothing.
 * Bit-exact. */
hq_status hq_to_bitplanes(const uint32_t* packed, size_t n_codes, uint32_t* planes,
                          hq_stream_t stream);

/* Intermediates an hq_moe_experts call leaves in its workspace, for checking
 * the layer stage by stage:
 *   HQ_MOE_POS  int32 [T*k]: row of pair (t, j) (index t*k + j) in the two
 *               arrays below, or -1 if the pair was skipped (bad id or
 *               descriptor);
 *   HQ_MOE_H    fp32 [rows][inter]: h = silu(W_gate x') * (W_up x') of each pair;
 *   HQ_MOE_D    fp32 [rows][hidden]: d = W_down h' of each pair.
 * The rows are grouped by expert (the order of the stable sort by expert id). */
typedef enum { HQ_MOE_POS = 0, HQ_MOE_H = 1, HQ_MOE_D = 2 } hq_moe_part;

/* Byte offset of `part` inside an hq_moe_experts workspace of these sizes,
 * valid after the call has completed (SIZE_MAX on a bad argument). */
size_t hq_moe_workspace_offset(int n_experts, int hidden, int inter, int T, int k,
                               hq_moe_part part);

/* Synchronises `stream`, then reads and clears the status word that the last
 * hq_linear_noalloc call left in the library's scratch array: HQ_OK, or
 * HQ_ERR_TIMEOUT if a bounded device-side wait of that call ran out (its
 * output is then incomplete).  No counterpart on the pages, like
 * hq_linear_noalloc.  HQ_ERR_CUDA if a CUDA call fails. */
hq_status hq_linear_noalloc_check_status(hq_stream_t stream);

/* Synchronises `stream`, reads the status word of a workspace used by
 * hq_linear or hq_moe_experts, clears it, and returns HQ_OK or the first
 * recorded device error (HQ_ERR_TIMEOUT before HQ_ERR_DATA). */
hq_status hq_check_status(void* workspace, hq_stream_t stream);

/*
 * hq_unpack_codes -- decode n_codes codes of width bits (1..8) from a packed
 * little-endian bit stream into one byte each: codes_out[j] = stream bits
 * [bits*j, bits*j + bits), the layout every packed weight of this library
 * uses.  Bit-exact; test-facing (it checks the layout on its own, apart from
 * the matmuls that decode it in registers).
 * packed: 4-byte aligned, ceil(bits*n_codes/32) words; codes_out: n_codes
 * bytes.  n_codes = 0 launches nothing.
 * Cites: the per-expert 2/3/4-bit and 8-bit group-128 integer codes that stay
 * packed through the run (LLaDA2.2-mini Orin-Nano model card, Properties
 * table; Qwen3-8B BPDQ 2-bit card, introduction).
 */
hq_status hq_unpack_codes(const uint32_t* packed, int bits, size_t n_codes,
                          uint8_t* codes_out, hq_stream_t stream);

/* Static string for a status code. */
const char* hq_status_string(hq_status s);

/* Total number of kernels this process has enqueued through libhq. */
uint64_t hq_launch_count(void);

/* Kernels one hq_linear call enqueues for this weight and batch. */
int hq_linear_launches(const hq_weight* w, int batch);

/* Kernels one hq_moe_experts call enqueues (route + rotate x, gate/up,
 * rotate h, down, combine). */
int hq_moe_launches(void);

/* 1 if hq_linear runs this weight and batch on the tensor-core GEMM, 0 if on
 * the GEMV, -1 for an invalid weight or batch < 1 (nothing is launched). */
int hq_linear_uses_tensor_cores(const hq_weight* w, int batch);

/* Batch size from which hq_linear uses the tensor-core GEMM (when K >= 1024).
 * 0 (the default) selects it automatically: from batch 17 where the 32-row
 * GEMV takes batches up to 16 (hq_linear_path), else from batch 5 for
 * 3/4/8-bit codes with K >= 8192 and from batch 9 otherwise.  A value >= 1
 * applies to every weight and takes precedence over the 32-row GEMV.
 * Returns the previous value; negative values change nothing. */
int hq_set_tc_min_batch(int n);

/* The kernel family hq_linear runs a weight and batch on. */
typedef enum {
  HQ_PATH_GEMV = 0,    /* register-decode GEMV, batch blocks of up to 8 */
  HQ_PATH_TENSOR = 1,  /* tcgen05 GEMM (codes dequantised into tensor memory) */
  HQ_PATH_GEMV32 = 2   /* register-decode GEMV over 32-row tiles, up to 16 columns */
} hq_path;

/* The hq_path of hq_linear for this weight and batch; -1 for an invalid
 * weight or batch < 1 (nothing is launched).  The 32-row GEMV applies to the
 * packed and bit-plane layouts with the scalar zero point, K >= 1024 and at
 * most 16 x 148 32-row tiles' worth of rows per streaming multiprocessor
 * count (M <= 75,776 on a B200). */
int hq_linear_path(const hq_weight* w, int batch);

/* Batch size from which hq_linear uses the 32-row GEMV (batches up to 16,
 * where it applies).  0 (the default) selects it automatically: from batch 4
 * for 8-bit codes, 5 for 3/4-bit codes, 6 for 2-bit codes (9 above 16384
 * rows), from batch sweeps on B200.  n >= 1 applies to
 * every weight (n = 1: every batch up to 16); an explicit
 * hq_set_tc_min_batch still takes precedence.  Returns the previous value;
 * negative values change nothing. */
int hq_set_gemv32_min_batch(int n);

/* For tests of the device error path (no counterpart on the pages): the next
 * n launches of the small-batch GEMV kernel each leave one shared-memory copy
 * of CTA 0's last warp unrequested (its second chunk: a launch where that warp
 * has fewer than two chunks withholds nothing), so that warp's bounded wait runs out
 * (after about one second) and records HQ_ERR_TIMEOUT in the status word
 * (hq_check_status, hq_linear_noalloc_check_status); that call's outputs are
 * then incomplete.  A 32-row GEMV launch that rotates its batch itself takes
 * one of the n instead: its CTA 0 does not publish its rotated row, so every
 * CTA's bounded wait at the rotation gate runs out the same way (the
 * workspace must then be zeroed again).  Nothing faults and the context stays
 * usable.  Returns the previous count; n < 0 only reads it. */
int hq_set_test_fault(int n);

#ifdef __cplusplus
}
#endif
#endif /* HQ_H */
