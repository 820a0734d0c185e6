// moe.cu -- hq_moe_experts: the routed-expert part of an MoE layer with
// per-expert bit widths (mixed 2/3/4-bit experts, widths from a per-expert
// manifest: LLaDA2.2-mini Orin-Nano model card, Properties table; one
// 32-token denoising block per call: same card, "Measured Throughput").
//
// Six kernels, one stream, no host synchronisation:
//   1. moe_route_kernel   validate ids and descriptors, stable counting sort
//                         of the (token, slot) pairs by expert, work lists;
//   2. moe_rot_x_kernel   x'_t = H diag(s_in) x_t / sqrt(hidden), written in
//                         the MMA B-fragment layout of every bit width;
//   3. moe_phase_kernel<A>  gate and up of every touched expert in one launch,
//                         SwiGLU in the epilogue -> h [pairs][inter];
//   4. moe_rot_h_kernel   h' = H diag(s_mid) h / sqrt(inter) per pair, in the
//                         layout of the pair's expert;
//   5. moe_phase_kernel<B>  down of every touched expert -> d [pairs][hidden];
//   6. moe_combine_kernel y_t = sum_j topk_w[t][j] d_{t,j}, j ascending.
// Every output element is written by exactly one thread and every sum runs in
// a fixed order, so results are deterministic.
#include <algorithm>

#include "fwht.cuh"
#include "hq_common.cuh"
#include "hq_internal.h"
#include "hq_io.cuh"
#include "hq_launch.cuh"
#include "hq_layout.cuh"

namespace hq {

namespace moe {

constexpr int kRows = 16;
constexpr int kXq = 40;             // halves per (row, group, k-quad) B block (64 B + pad)
constexpr float kUnit = 16777216.f;  // 2^24, the subnormal code unit
constexpr int kWarps = 16;

__host__ __device__ inline int layout_index(int bits) {
  return bits == 2 ? 0 : bits == 3 ? 1 : bits == 4 ? 2 : 3;
}

// Views into the caller's workspace (carved on the host; see hq_moe_ws).
struct Ws {
  uint32_t* status;
  int* counts;     // [E] valid pairs per expert
  int* offsets;    // [E + 1] first sorted position of each expert
  int* pos;        // [P] sorted position of pair i = t*k + j, or -1 if skipped
  int* sorted;     // [P] pair index at each sorted position
  int* n_items;    // [2] work items of phase A, phase B
  uint2* items_a;  // [cap_a] (expert, tile << 16 | column block)
  uint2* items_b;  // [cap_b]
  uint16_t* xl;    // [4][T][G_h][4][kXq] rotated tokens, per bit-width layout
  float* xsum;     // [4][T][G_h] sum over each group of the effective x'
  float* h;        // [P][inter]
  uint16_t* hl;    // [P][G_i][4][kXq] rotated h, in its expert's layout
  float* hsum;     // [P][G_i]
  float* d;        // [P][hidden]
};

struct Dims {
  int E, hidden, inter, T, k, P;
  int cap_a, cap_b;
};

}  // namespace moe

// Workspace carve-up (host side; also sizes hq_moe_workspace_size).
static size_t a256(size_t v) { return (v + 255) & ~static_cast<size_t>(255); }

struct MoePlan {
  moe::Dims d;
  size_t off[16];
  size_t bytes;
};

static MoePlan moe_plan(int E, int hidden, int inter, int T, int k) {
  MoePlan pl{};
  moe::Dims& d = pl.d;
  d.E = E;
  d.hidden = hidden;
  d.inter = inter;
  d.T = T;
  d.k = k;
  d.P = T * k;
  const int nb_max = std::min(E, d.P) + (d.P + 7) / 8;  // bound on sum_e ceil(cnt_e / 8)
  d.cap_a = (inter / moe::kRows) * nb_max;
  d.cap_b = (hidden / moe::kRows) * nb_max;
  const size_t Gh = hidden / kGroup, Gi = inter / kGroup;
  const size_t sizes[14] = {
      256,                                             // status
      sizeof(int) * E,                                 // counts
      sizeof(int) * (E + 1),                           // offsets
      sizeof(int) * d.P,                               // pos
      sizeof(int) * d.P,                               // sorted
      sizeof(int) * 2,                                 // n_items
      sizeof(uint2) * d.cap_a,                         // items_a
      sizeof(uint2) * d.cap_b,                         // items_b
      2 * 4 * static_cast<size_t>(T) * Gh * 4 * moe::kXq,  // xl
      4 * 4 * static_cast<size_t>(T) * Gh,                 // xsum
      4 * static_cast<size_t>(d.P) * inter,                // h
      2 * static_cast<size_t>(d.P) * Gi * 4 * moe::kXq,    // hl
      4 * static_cast<size_t>(d.P) * Gi,                   // hsum
      4 * static_cast<size_t>(d.P) * hidden,               // d
  };
  size_t o = 0;
  for (int i = 0; i < 14; ++i) {
    pl.off[i] = o;
    o += a256(sizes[i]);
  }
  pl.bytes = o + 256;  // 256 bytes of zeros: the B block of lanes without a column
  pl.off[14] = o;
  return pl;
}

static moe::Ws moe_ws(void* base, const MoePlan& pl) {
  uint8_t* b = static_cast<uint8_t*>(base);
  moe::Ws w;
  w.status = reinterpret_cast<uint32_t*>(b + pl.off[0]);
  w.counts = reinterpret_cast<int*>(b + pl.off[1]);
  w.offsets = reinterpret_cast<int*>(b + pl.off[2]);
  w.pos = reinterpret_cast<int*>(b + pl.off[3]);
  w.sorted = reinterpret_cast<int*>(b + pl.off[4]);
  w.n_items = reinterpret_cast<int*>(b + pl.off[5]);
  w.items_a = reinterpret_cast<uint2*>(b + pl.off[6]);
  w.items_b = reinterpret_cast<uint2*>(b + pl.off[7]);
  w.xl = reinterpret_cast<uint16_t*>(b + pl.off[8]);
  w.xsum = reinterpret_cast<float*>(b + pl.off[9]);
  w.h = reinterpret_cast<float*>(b + pl.off[10]);
  w.hl = reinterpret_cast<uint16_t*>(b + pl.off[11]);
  w.hsum = reinterpret_cast<float*>(b + pl.off[12]);
  w.d = reinterpret_cast<float*>(b + pl.off[13]);
  return w;
}

namespace moe {

__device__ __forceinline__ bool valid_desc(const hq_expert& e) {
  const bool bits_ok = e.bits == 2 || e.bits == 3 || e.bits == 4 || e.bits == 8;
  return bits_ok && e.zero >= 0 && e.zero < (1 << e.bits) && e.q_gate && e.q_up && e.q_down &&
         e.s_gate && e.s_up && e.s_down;
}

// Single CTA.  Stable counting sort of the pairs by expert: pair i = t*k + j
// is ranked among the pairs of its expert in increasing i, so the sorted
// order, and every sum taken over it, is independent of thread timing.
__global__ void __launch_bounds__(1024) moe_route_kernel(const hq_expert* __restrict__ ex,
                                                        const int32_t* __restrict__ ids, Ws w,
                                                        Dims d, uint32_t* zero_block) {
  pdl_launch_dependents();
  pdl_wait();
  // first column block of each expert; [E] = total (s_nb0[e+1] - s_nb0[e] = blocks of e)
  extern __shared__ int s_nb0[];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid < 64) zero_block[tid] = 0u;  // B block of lanes without a column
  for (int e = tid; e < d.E; e += blockDim.x) w.counts[e] = 0;
  // validity of every pair (its expert id and that expert's descriptor)
  for (int i = tid; i < d.P; i += blockDim.x) {
    const int e = ids[i];
    int ok = 0;
    if (e < 0 || e >= d.E) {
      record_error(w.status, HQ_DEV_BAD_EXPERT);
    } else {
      const hq_expert de = ex[e];
      ok = valid_desc(de);
      if (!ok) record_error(w.status, HQ_DEV_BAD_BITS);
    }
    w.pos[i] = ok ? e : -1;  // expert id of a valid pair, for the ranking pass
  }
  __syncthreads();
  if (warp == 0) {
    // ranks in pair order, 32 pairs at a time
    for (int c = 0; c < d.P; c += 32) {
      const int i = c + lane;
      const int e = i < d.P ? w.pos[i] : -1;
      const unsigned mask = __match_any_sync(0xffffffffu, e);
      const int before = __popc(mask & ((1u << lane) - 1u));
      const int base = e >= 0 ? w.counts[e] : 0;
      __syncwarp();
      if (e >= 0) w.pos[i] = -2 - (base + before);  // rank, encoded below -1
      const int leader = 31 - __clz(mask);          // highest lane of the group
      if (e >= 0 && lane == leader) w.counts[e] = base + __popc(mask);
      __syncwarp();
    }
  }
  __syncthreads();
  if (warp == 0) {
    // exclusive scan of counts; item counts per expert
    int run = 0, run_a = 0, run_b = 0;
    const int ta = d.inter / kRows, tb = d.hidden / kRows;
    for (int c = 0; c < d.E; c += 32) {
      const int e = c + lane;
      const int cnt = e < d.E ? w.counts[e] : 0;
      const int nb = (cnt + 7) / 8;
      int x = cnt, xa = nb;
#pragma unroll
      for (int m = 1; m < 32; m <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, m);
        const int ya = __shfl_up_sync(0xffffffffu, xa, m);
        if (lane >= m) {
          x += y;
          xa += ya;
        }
      }
      if (e < d.E) {
        w.offsets[e] = run + x - cnt;
        // first column block of this expert (the items are written below by
        // all warps: column blocks x row tiles, block-major)
        s_nb0[e] = run_a + xa - nb;
      }
      run += __shfl_sync(0xffffffffu, x, 31);
      const int tot_nb = __shfl_sync(0xffffffffu, xa, 31);
      run_a += tot_nb;
      run_b += tot_nb;
    }
    if (lane == 0) {
      w.offsets[d.E] = run;
      w.n_items[0] = run_a * ta;
      w.n_items[1] = run_b * tb;
      s_nb0[d.E] = run_a;
    }
  }
  __syncthreads();
  {
    // work items, one warp per expert, lanes over the expert's items
    const int ta = d.inter / kRows, tb = d.hidden / kRows;
    const int nw = blockDim.x >> 5;
    for (int e = warp; e < d.E; e += nw) {
      const int nb0 = s_nb0[e], nb = s_nb0[e + 1] - nb0;
      for (int i = lane; i < nb * ta; i += 32) {
        w.items_a[nb0 * ta + i] = make_uint2(e, ((i % ta) << 16) | (i / ta));
      }
      for (int i = lane; i < nb * tb; i += 32) {
        w.items_b[nb0 * tb + i] = make_uint2(e, ((i % tb) << 16) | (i / tb));
      }
    }
  }
  for (int i = tid; i < d.P; i += blockDim.x) {
    const int r = w.pos[i];
    if (r <= -2) {
      const int p = w.offsets[ids[i]] + (-2 - r);
      w.pos[i] = p;
      w.sorted[p] = i;
    }
  }
}


// Write one rotated row (fwht_block output in buf, unnormalised) as fp16 B
// blocks for the code decode of BITS: block (group gg, k-quad t) holds the
// 8 steps x 4 activations, each scaled by 2^-a of its code field; sums[gg] =
// sum over the group of the effective activations (B * 2^a), for the
// zero-point term.  Warp-per-group; nw warps of the block take part.
template <int BITS>
__device__ __forceinline__ void write_layout(const float* buf, float inv, int G, uint16_t* out,
                                             float* sums, int warp, int nw, int lane) {
  const int s = lane >> 2, t = lane & 3;
  int kc[4], ka[4];
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const PairDesc pd = Pairs<BITS>::get(2 * s + (r >> 1));
    kc[r] = 32 * t + ((r & 1) ? pd.c_hi : pd.c_lo);
    ka[r] = (r & 1) ? pd.a_hi : pd.a_lo;
  }
  for (int gg = warp; gg < G; gg += nw) {
    uint16_t hv[4];
    float part = 0.f;
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const float xv = __half2float(__float2half_rn(buf[fwht_pad(kGroup * gg + kc[r])] * inv));
      const __half b = __float2half_rn(xv * __int_as_float((127 - ka[r]) << 23));
      hv[r] = __half_as_ushort(b);
      part += __half2float(b) * __int_as_float((127 + ka[r]) << 23);
    }
#pragma unroll
    for (int m = 16; m >= 1; m >>= 1) part += __shfl_xor_sync(0xffffffffu, part, m);
    uint2 pk;
    pk.x = hv[0] | (static_cast<uint32_t>(hv[1]) << 16);
    pk.y = hv[2] | (static_cast<uint32_t>(hv[3]) << 16);
    *reinterpret_cast<uint2*>(out + (gg * 4 + t) * kXq + s * 4) = pk;
    if (lane == 0) sums[gg] = part;
  }
}

__device__ __forceinline__ void write_layout_bits(int bits, const float* buf, float inv, int G,
                                                  uint16_t* out, float* sums, int warp, int nw,
                                                  int lane) {
  switch (bits) {
    case 2: write_layout<2>(buf, inv, G, out, sums, warp, nw, lane); break;
    case 3: write_layout<3>(buf, inv, G, out, sums, warp, nw, lane); break;
    case 4: write_layout<4>(buf, inv, G, out, sums, warp, nw, lane); break;
    default: write_layout<8>(buf, inv, G, out, sums, warp, nw, lane); break;
  }
}

// One CTA per token: rotate x_t and write it in the layout of every width.
template <int LOGK>
__global__ void __launch_bounds__(FwhtShape<LOGK>::THREADS)
    moe_rot_x_kernel(const __half* __restrict__ x, const int8_t* __restrict__ signs, Ws w,
                     Dims d, float inv) {
  using S = FwhtShape<LOGK>;
  extern __shared__ float buf[];
  pdl_launch_dependents();
  pdl_wait();
  const int tid = threadIdx.x, t = blockIdx.x;
  float v[S::E];
  load_chunk<__half, S::E>(x + static_cast<size_t>(t) * S::K + tid * S::E, v);
  apply_signs<S::E>(signs ? signs + tid * S::E : nullptr, v);
  fwht_block<LOGK, 5>(v, buf);
  const int G = S::K / kGroup;
  const int bits_of[4] = {2, 3, 4, 8};
  for (int L = 0; L < 4; ++L) {
    const size_t row = static_cast<size_t>(L) * d.T + t;
    write_layout_bits(bits_of[L], buf, inv, G, w.xl + row * G * 4 * kXq, w.xsum + row * G,
                      tid >> 5, S::THREADS / 32, tid & 31);
  }
}

// One CTA per sorted pair position: rotate h and write it in the layout of
// the pair's expert.
template <int LOGK>
__global__ void __launch_bounds__(FwhtShape<LOGK>::THREADS)
    moe_rot_h_kernel(const hq_expert* __restrict__ ex, const int32_t* __restrict__ ids,
                     const int8_t* __restrict__ signs, Ws w, Dims d, float inv) {
  using S = FwhtShape<LOGK>;
  extern __shared__ float buf[];
  pdl_launch_dependents();
  pdl_wait();
  const int tid = threadIdx.x, p = blockIdx.x;
  if (p >= w.offsets[d.E]) return;  // block-uniform: no barrier is skipped by part of it
  const int e = ids[w.sorted[p]];
  const int bits = ex[e].bits;
  float v[S::E];
  load_chunk<float, S::E>(w.h + static_cast<size_t>(p) * S::K + tid * S::E, v);
  apply_signs<S::E>(signs ? signs + tid * S::E : nullptr, v);
  fwht_block<LOGK, 5>(v, buf);
  const int G = S::K / kGroup;
  write_layout_bits(bits, buf, inv, G, w.hl + static_cast<size_t>(p) * G * 4 * kXq,
                    w.hsum + static_cast<size_t>(p) * G, tid >> 5, S::THREADS / 32, tid & 31);
}

// y[t][c] = sum_{j=0..k-1} topk_w[t][j] d[pos(t,j)][c]; skipped pairs add 0.
__global__ void moe_combine_kernel(const float* __restrict__ topk_w, Ws w, Dims d,
                                   float* __restrict__ y) {
  pdl_launch_dependents();
  pdl_wait();
  const size_t n = static_cast<size_t>(d.T) * d.hidden;
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const int t = static_cast<int>(i / d.hidden), c = static_cast<int>(i % d.hidden);
    float acc = 0.f;
    for (int j = 0; j < d.k; ++j) {
      const int p = w.pos[t * d.k + j];
      if (p >= 0) acc = fmaf(topk_w[t * d.k + j], w.d[static_cast<size_t>(p) * d.hidden + c], acc);
    }
    y[i] = acc;
  }
}


// ---------------------------------------------------------------- expert phases
// Chunk geometry, shared by producer and consumer: a chunk is `len` groups of
// one item's 16 rows in each of its NMAT matrices, rows at a bank-conflict-
// free stride, then each matrix's scales.
__host__ __device__ inline int chunk_stride(int bits, int len) {
  const int row = len * 16 * bits;
  const int pad_w = ((bank_target_words(bits) - row / 4) % 32 + 32) % 32;
  return row + 4 * pad_w;
}
__host__ __device__ inline int chunk_scale_bytes(int G) {
  return G >= 8 ? kRows * 32 : ((kRows * G * 2 + 15) & ~15);
}
constexpr int kChunkBytes = 6 * 1024;
constexpr int kRing = 2;  // slots per warp
__host__ __device__ inline int chunk_len(int bits, int G, int nmat) {
  for (int len = 8; len > 1; len >>= 1) {
    if (len <= G && nmat * (kRows * chunk_stride(bits, len) + chunk_scale_bytes(G)) <= kChunkBytes)
      return len;
  }
  return 1;
}

template <int BITS>
__device__ __forceinline__ void group_mma(const uint8_t* ra, const uint8_t* rb, const uint4 (&bq)[4],
                                          float2 z, float sa, float sb, float (&acc)[4]) {
  uint32_t wa[BITS], wb[BITS];
  load_bundle<BITS>(ra, wa);
  load_bundle<BITS>(rb, wb);
  uint32_t Pa[16], Pb[16];
  decode16<BITS>(wa, Pa);
  decode16<BITS>(wb, Pb);
  float c0[4] = {z.x, z.y, z.x, z.y}, c1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int s = 0; s < 8; ++s) {
    const uint32_t b0 = (s & 1) ? bq[s >> 1].z : bq[s >> 1].x;
    const uint32_t b1 = (s & 1) ? bq[s >> 1].w : bq[s >> 1].y;
    const uint32_t a[4] = {Pa[2 * s], Pb[2 * s], Pa[2 * s + 1], Pb[2 * s + 1]};
    if (s & 1) {
      mma_16816(c1, a, b0, b1, c1);
    } else {
      mma_16816(c0, a, b0, b1, c0);
    }
  }
  acc[0] = fmaf(sa, c0[0] + c1[0], acc[0]);
  acc[1] = fmaf(sa, c0[1] + c1[1], acc[1]);
  acc[2] = fmaf(sb, c0[2] + c1[2], acc[2]);
  acc[3] = fmaf(sb, c0[3] + c1[3], acc[3]);
}

// Phase A (PHASE 0): gate and up, SwiGLU -> h.  Phase B (PHASE 1): down -> d.
// Warp gw takes items gw, gw + GW, ...  Its ring runs up to kRing chunks
// ahead, across item boundaries.
template <int PHASE>
__global__ void __launch_bounds__(kWarps * 32, 1)
    moe_phase_kernel(const hq_expert* __restrict__ ex, const int32_t* __restrict__ ids, Ws w,
                     Dims d, const uint4* __restrict__ zero_block) {
  constexpr int NMAT = PHASE == 0 ? 2 : 1;
  extern __shared__ __align__(128) uint8_t smem[];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, t = lane & 3;
  const int K = PHASE == 0 ? d.hidden : d.inter;
  const int M = PHASE == 0 ? d.inter : d.hidden;
  const int G = K / kGroup;
  uint8_t* ring = smem + warp * kRing * kChunkBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kWarps * kRing * kChunkBytes) + warp * kRing;
  if (lane == 0) {
    for (int i = 0; i < kRing; ++i) mbar_init(&bars[i], 32);
    fence_mbar_init();
  }
  __syncthreads();
  pdl_launch_dependents();
  pdl_wait();  // routing lists and activations come from the previous kernels
  const int n_items = w.n_items[PHASE];
  const uint2* items = PHASE == 0 ? w.items_a : w.items_b;
  const int GW = gridDim.x * kWarps;
  const int gw = blockIdx.x * kWarps + warp;

  // ---- producer
  int pi = gw, pg = 0;  // next item and group to copy
  int issued = 0;
  auto issue = [&](int slot) {
    const uint2 it = items[pi];
    const hq_expert ed = ex[it.x];
    const int bits = ed.bits;
    const int len = min(chunk_len(bits, G, NMAT), G - pg);
    const int stride = chunk_stride(bits, chunk_len(bits, G, NMAT));
    const int GB = 16 * bits;
    const int m0 = static_cast<int>(it.y >> 16) * kRows;
    const size_t row_bytes = static_cast<size_t>(K) * bits / 8;
    uint8_t* base = ring + slot * kChunkBytes;
    const int pr = len * bits;  // 16-byte pieces per row
#pragma unroll
    for (int mi = 0; mi < NMAT; ++mi) {
      const uint32_t* q = PHASE == 0 ? (mi == 0 ? ed.q_gate : ed.q_up) : ed.q_down;
      const uint16_t* sc = PHASE == 0 ? (mi == 0 ? ed.s_gate : ed.s_up) : ed.s_down;
      const uint8_t* src = reinterpret_cast<const uint8_t*>(q) + m0 * row_bytes +
                           static_cast<size_t>(pg) * GB;
      uint8_t* cdst = base + mi * kRows * stride;
      for (int i = lane; i < kRows * pr; i += 32) {
        const int r = i / pr, c = i - r * pr;
        cp_async16(cdst + r * stride + c * 16, src + r * row_bytes + c * 16, 16);
      }
      uint8_t* sdst = base + NMAT * kRows * stride + mi * chunk_scale_bytes(G);
      if (G >= 8) {
        const int sg0 = pg & ~7;
        const int nblk = (((pg + len + 7) & ~7) - sg0) / 8;
        const int r = lane & 15, blk = lane >> 4;
        if (blk < nblk) cp_async16(sdst + r * 32 + blk * 16, sc + static_cast<size_t>(m0 + r) * G + sg0 + 8 * blk, 16);
      } else {
        if (lane < 2 * G) cp_async16(sdst + lane * 16, reinterpret_cast<const uint8_t*>(sc + static_cast<size_t>(m0) * G) + lane * 16, 16);
      }
    }
    cp_async_mbar_arrive(&bars[slot]);
    pg += len;
    if (pg >= G) {
      pg = 0;
      pi += GW;
    }
    ++issued;
  };
  for (int s = 0; s < kRing && pi < n_items; ++s) issue(s);

  // ---- consumer
  int consumed = 0;
  bool ok = true;
  for (int item = gw; item < n_items && ok; item += GW) {
    const uint2 it = items[item];
    const int e = static_cast<int>(it.x);
    const hq_expert ed = ex[e];
    const int bits = ed.bits;
    const int L = layout_index(bits);
    const float zneg = -static_cast<float>(ed.zero) * 5.9604644775390625e-8f;  // -zero * 2^-24
    const int m0 = static_cast<int>(it.y >> 16) * kRows;
    const int cb = static_cast<int>(it.y & 0xffff);
    const int off = w.offsets[e] + 8 * cb;
    const int ncol = min(8, w.counts[e] - 8 * cb);
    // B-operand rows of this lane's column and the two columns it accumulates
    auto brow = [&](int col) -> int {
      const int p = off + col;
      return PHASE == 0 ? L * d.T + w.sorted[p] / d.k : p;
    };
    const uint16_t* blk_base = PHASE == 0 ? w.xl : w.hl;
    const float* sum_base = PHASE == 0 ? w.xsum : w.hsum;
    const bool has_b = g < ncol;
    const uint4* bp = has_b ? reinterpret_cast<const uint4*>(blk_base + (static_cast<size_t>(brow(g)) * G * 4 + t) * kXq)
                            : zero_block;
    const int bstep = has_b ? 4 * kXq / 8 : 0;  // uint4 per group
    const float* s0p = 2 * t < ncol ? sum_base + static_cast<size_t>(brow(2 * t)) * G : nullptr;
    const float* s1p = 2 * t + 1 < ncol ? sum_base + static_cast<size_t>(brow(2 * t + 1)) * G : nullptr;
    const int len_max = chunk_len(bits, G, NMAT);
    const int stride = chunk_stride(bits, len_max);
    const int GB = 16 * bits;
    float acc[NMAT][4] = {};
    uint4 bq[4];
    float2 z;
#pragma unroll
    for (int i = 0; i < 4; ++i) bq[i] = bp[i];
    z = make_float2(s0p ? zneg * s0p[0] : 0.f, s1p ? zneg * s1p[0] : 0.f);
    for (int g0 = 0; g0 < G && ok; g0 += len_max) {
      const int len = min(len_max, G - g0);
      const int slot = consumed % kRing;
      if (!mbar_wait(&bars[slot], (consumed / kRing) & 1)) {
        ok = false;
        break;
      }
      __syncwarp();
      const uint8_t* base = ring + slot * kChunkBytes;
      for (int j = 0; j < len; ++j) {
        const int gi = g0 + j;
        // prefetch the next group's B blocks and zero-point sums
        uint4 bn[4];
        float2 zn = make_float2(0.f, 0.f);
        if (gi + 1 < G) {
#pragma unroll
          for (int i = 0; i < 4; ++i) bn[i] = bp[(gi + 1) * bstep + i];
          zn = make_float2(s0p ? zneg * s0p[gi + 1] : 0.f, s1p ? zneg * s1p[gi + 1] : 0.f);
        }
#pragma unroll
        for (int mi = 0; mi < NMAT; ++mi) {
          const uint8_t* ra = base + mi * kRows * stride + g * stride + j * GB + t * 4 * bits;
          const uint8_t* rb = ra + 8 * stride;
          const __half* sc = reinterpret_cast<const __half*>(base + NMAT * kRows * stride + mi * chunk_scale_bytes(G));
          const int sidx = G >= 8 ? (gi - (g0 & ~7)) : gi;
          const int sstr = G >= 8 ? 16 : G;
          const float sa = __half2float(sc[g * sstr + sidx]);
          const float sb = __half2float(sc[(g + 8) * sstr + sidx]);
          switch (bits) {
            case 2: group_mma<2>(ra, rb, bq, z, sa, sb, acc[mi]); break;
            case 3: group_mma<3>(ra, rb, bq, z, sa, sb, acc[mi]); break;
            case 4: group_mma<4>(ra, rb, bq, z, sa, sb, acc[mi]); break;
            default: group_mma<8>(ra, rb, bq, z, sa, sb, acc[mi]); break;
          }
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) bq[i] = bn[i];
        z = zn;
      }
      __syncwarp();
      if (pi < n_items) issue(slot);
      ++consumed;
    }
    if (!ok) break;
    // ---- epilogue: rows g, g+8; columns 2t, 2t+1
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int col = 2 * t + (q & 1);
      const int m = m0 + g + 8 * (q >> 1);
      if (col < ncol && m < M) {
        const size_t prow = static_cast<size_t>(off + col);
        if (PHASE == 0) {
          const float gv = acc[0][q] * kUnit, uv = acc[NMAT - 1][q] * kUnit;
          w.h[prow * d.inter + m] = gv / (1.f + expf(-gv)) * uv;
        } else {
          w.d[prow * d.hidden + m] = acc[0][q] * kUnit;
        }
      }
    }
  }
  if (!ok) {
    if (lane == 0) record_error(w.status, HQ_DEV_TIMEOUT);
    for (int k2 = consumed; k2 < issued; ++k2) (void)mbar_wait(&bars[k2 % kRing], (k2 / kRing) & 1);
  }
}

}  // namespace moe

// ---------------------------------------------------------------- host side
static cudaError_t moe_launch_rot_x(int hidden, const __half* x, const int8_t* s, const moe::Ws& w,
                                    const moe::Dims& d, cudaStream_t st) {
  const float inv = static_cast<float>(1.0 / sqrt(static_cast<double>(hidden)));
#define HQ_ROTX(LK)                                                                           \
  case (1 << LK):                                                                             \
    return launch_pdl(moe::moe_rot_x_kernel<LK>, dim3(d.T), dim3(FwhtShape<LK>::THREADS),       \
                      FwhtShape<LK>::SMEM_FLOATS * sizeof(float), st, true, x, s, w, d, inv);
  switch (hidden) {
    HQ_ROTX(7) HQ_ROTX(8) HQ_ROTX(9) HQ_ROTX(10) HQ_ROTX(11) HQ_ROTX(12) HQ_ROTX(13) HQ_ROTX(14)
    default: return cudaErrorInvalidValue;
  }
#undef HQ_ROTX
}

static cudaError_t moe_launch_rot_h(int inter, const hq_expert* ex, const int32_t* ids,
                                    const int8_t* s, const moe::Ws& w, const moe::Dims& d,
                                    cudaStream_t st) {
  const float inv = static_cast<float>(1.0 / sqrt(static_cast<double>(inter)));
#define HQ_ROTH(LK)                                                                           \
  case (1 << LK):                                                                             \
    return launch_pdl(moe::moe_rot_h_kernel<LK>, dim3(d.P), dim3(FwhtShape<LK>::THREADS),       \
                      FwhtShape<LK>::SMEM_FLOATS * sizeof(float), st, true, ex, ids, s, w, d, inv);
  switch (inter) {
    HQ_ROTH(7) HQ_ROTH(8) HQ_ROTH(9) HQ_ROTH(10) HQ_ROTH(11) HQ_ROTH(12) HQ_ROTH(13) HQ_ROTH(14)
    default: return cudaErrorInvalidValue;
  }
#undef HQ_ROTH
}

static int moe_grid() { return sm_count(); }  // one CTA per SM

}  // namespace hq

using namespace hq;

// The route kernel keeps one int per expert in shared memory.
constexpr int kMaxExperts = 32768;

extern "C" {

size_t hq_moe_workspace_size(int n_experts, int hidden, int inter, int T, int k) {
  auto pow2 = [](int v) { return v > 0 && (v & (v - 1)) == 0; };
  if (n_experts < 1 || n_experts > kMaxExperts || T < 0 || k < 1 || k > 32 || !pow2(hidden) ||
      !pow2(inter) || hidden < 128 || inter < 128 || hidden > 16384 || inter > 16384 ||
      static_cast<long>(T) * k > (1L << 24)) {
    return 0;
  }
  return moe_plan(n_experts, hidden, inter, T, k).bytes;
}

int hq_moe_launches(void) { return 6; }

hq_status hq_moe_experts(const hq_expert* experts, int n_experts, int hidden, int inter,
                         const uint16_t* x, int T, const int32_t* topk_ids, const float* topk_w,
                         int k, const int8_t* signs_in, const int8_t* signs_mid, float* y,
                         void* workspace, size_t ws_bytes, hq_stream_t stream) {
  auto pow2 = [](int v) { return v > 0 && (v & (v - 1)) == 0; };
  auto al = [](const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; };
  if (n_experts < 1 || T < 0 || k < 1 || k > 32 || hidden <= 0 || inter <= 0) {
    return HQ_ERR_INVALID_ARG;
  }
  if (!pow2(hidden) || !pow2(inter) || hidden < 128 || inter < 128 || hidden > 16384 ||
      inter > 16384 || n_experts > kMaxExperts) {
    return HQ_ERR_UNSUPPORTED;
  }
  if (static_cast<long>(T) * k > (1L << 24)) return HQ_ERR_INVALID_ARG;
  if (T == 0) return HQ_OK;
  if (!experts || !x || !topk_ids || !topk_w || !y) return HQ_ERR_INVALID_ARG;
  if (!al(experts, 8) || !al(x, 16) || !al(y, 16) || !al(topk_ids, 4) || !al(topk_w, 4) ||
      (signs_in && !al(signs_in, 16)) || (signs_mid && !al(signs_mid, 16))) {
    return HQ_ERR_INVALID_ARG;
  }
  const MoePlan pl = moe_plan(n_experts, hidden, inter, T, k);
  if (!workspace || !al(workspace, 256) || ws_bytes < pl.bytes) return HQ_ERR_WORKSPACE;
  const moe::Ws w = moe_ws(workspace, pl);
  const moe::Dims& d = pl.d;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  uint32_t* zb = reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(workspace) + pl.off[14]);
  const uint4* zb4 = reinterpret_cast<const uint4*>(zb);
  const __half* xh = reinterpret_cast<const __half*>(x);
  cudaError_t e = launch_pdl(moe::moe_route_kernel, dim3(1), dim3(1024),
                             static_cast<size_t>(n_experts + 1) * sizeof(int), st, true, experts,
                             topk_ids, w, d, zb);
  if (e == cudaSuccess) e = moe_launch_rot_x(hidden, xh, signs_in, w, d, st);
  const size_t psmem = moe::kWarps * moe::kRing * moe::kChunkBytes + moe::kWarps * moe::kRing * 8;
  if (e == cudaSuccess) {
    e = launch_pdl(moe::moe_phase_kernel<0>, dim3(moe_grid()), dim3(moe::kWarps * 32), psmem, st,
                   true, experts, topk_ids, w, d, zb4);
  }
  if (e == cudaSuccess) e = moe_launch_rot_h(inter, experts, topk_ids, signs_mid, w, d, st);
  if (e == cudaSuccess) {
    e = launch_pdl(moe::moe_phase_kernel<1>, dim3(moe_grid()), dim3(moe::kWarps * 32), psmem, st,
                   true, experts, topk_ids, w, d, zb4);
  }
  if (e == cudaSuccess) {
    const size_t n = static_cast<size_t>(T) * hidden;
    const unsigned blocks = static_cast<unsigned>(std::min<size_t>((n + 255) / 256, 148 * 8));
    e = launch_pdl(moe::moe_combine_kernel, dim3(blocks), dim3(256), 0, st, true, topk_w, w, d, y);
  }
  if (e != cudaSuccess) {
    (void)cudaGetLastError();
    return HQ_ERR_CUDA;
  }
  return HQ_OK;
}

}  // extern "C"
