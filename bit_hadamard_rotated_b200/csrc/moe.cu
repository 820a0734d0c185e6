// moe.cu -- hq_moe_experts: the routed-expert part of an MoE layer with
// per-expert bit widths (mixed 2/3/4-bit experts, widths from a per-expert
// manifest: LLaDA2.2-mini Orin-Nano model card, Properties table; one
// 32-token denoising block per call: same card, "Measured Throughput").
//
// Five kernels, one stream, no host synchronisation:
//   1. moe_front_kernel   block 0: validate ids and descriptors, stable
//                         counting sort of the (token, slot) pairs by expert,
//                         the block list and each phase's per-CTA work split;
//                         blocks 1..T: x'_t = H diag(s_in) x_t / sqrt(hidden),
//                         written in the MMA B-fragment layout of every width;
//   2. moe_phase_kernel<A>  gate and up of every touched expert in one launch,
//                         SwiGLU in the epilogue -> h [pairs][inter];
//   3. moe_rot_h_kernel   h' = H diag(s_mid) h / sqrt(inter) per pair, in the
//                         layout of the pair's expert;
//   4. moe_phase_kernel<B>  down of every touched expert -> d [pairs][hidden];
//   5. moe_combine_kernel y_t = sum_j topk_w[t][j] d_{t,j}, j ascending.
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
  uint2* blk;      // [nb_max] (expert, column block) of each block, expert-major
  int* bounds;     // [2][kMaxGrid + 1] first work item of each CTA, phase A then B
  uint16_t* xl;    // [4][T][G_h][4][kXq] rotated tokens, per bit-width layout
  float* xsum;     // [4][T][G_h] sum over each group of the effective x'
  float* h;        // [P][inter]
  uint16_t* hl;    // [P][G_i][4][kXq] rotated h, in its expert's layout
  float* hsum;     // [P][G_i]
  float* d;        // [P][hidden]
};

struct Dims {
  int E, hidden, inter, T, k, P;
  int nb_max;  // bound on the number of (expert, column block) blocks
  int grid;    // CTAs of each expert phase
};

constexpr int kMaxGrid = 1024;

// Relative cost of one 16-row tile of a width, for splitting the phases'
// work between CTAs: the code bytes (proportional to the width) plus a fixed
// part for the per-group instructions that do not depend on it.
__host__ __device__ constexpr int tile_weight(int bits) { return bits + 2; }

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
  d.nb_max = std::min(E, d.P) + (d.P + 7) / 8;  // bound on sum_e ceil(cnt_e / 8)
  d.grid = std::min(sm_count(), moe::kMaxGrid);
  const size_t Gh = hidden / kGroup, Gi = inter / kGroup;
  const size_t sizes[14] = {
      256,                                             // status
      sizeof(int) * E,                                 // counts
      sizeof(int) * (E + 1),                           // offsets
      sizeof(int) * d.P,                               // pos
      sizeof(int) * d.P,                               // sorted
      sizeof(uint2) * d.nb_max,                        // blk
      sizeof(int) * 2 * (moe::kMaxGrid + 1),           // bounds
      0,                                               // (unused)
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
  pl.bytes = o;
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
  w.blk = reinterpret_cast<uint2*>(b + pl.off[5]);
  w.bounds = reinterpret_cast<int*>(b + pl.off[6]);
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

// The routing CTA (block 0 of the first launch).  Stable counting sort of the
// pairs by expert: pair i = t*k + j is ranked among the pairs of its expert in
// increasing i, so the sorted order, and every sum taken over it, is
// independent of thread timing.  Then the block list and, for each expert
// phase, the first work item of every CTA, splitting the summed tile weights
// evenly.  Shared memory: 3 E + 2 ints.
__device__ void route_cta(const hq_expert* __restrict__ ex, const int32_t* __restrict__ ids,
                          const Ws& w, const Dims& d, int* sm) {
  int* s_cnt = sm;              // [E] valid pairs per expert
  int* s_nb0 = sm + d.E;        // [E + 1] first block of each expert; [E] = blocks in all
  int* s_sw = s_nb0 + d.E + 1;  // [E + 1] tile weight, then the block-weight prefix
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nt = blockDim.x;
  for (int e = tid; e < d.E; e += nt) {
    s_cnt[e] = 0;
    s_sw[e] = 0;
  }
  __syncthreads();
  // validity of every pair (its expert id and that expert's descriptor)
  for (int i = tid; i < d.P; i += nt) {
    const int e = ids[i];
    int ok = 0;
    if (e < 0 || e >= d.E) {
      record_error(w.status, HQ_DEV_BAD_EXPERT);
    } else {
      const hq_expert de = ex[e];
      ok = valid_desc(de);
      if (ok) {
        s_sw[e] = tile_weight(de.bits);  // same value from every pair of e
      } else {
        record_error(w.status, HQ_DEV_BAD_BITS);
      }
    }
    w.pos[i] = ok ? e : -1;  // expert id of a valid pair, for the ranking pass
  }
  __syncthreads();
  if (warp == 0) {
    // ranks in pair order, 32 pairs at a time; the next 32 ids are loaded ahead
    int e_next = lane < d.P ? w.pos[lane] : -1;
    for (int c = 0; c < d.P; c += 32) {
      const int i = c + lane;
      const int e = e_next;
      e_next = i + 32 < d.P ? w.pos[i + 32] : -1;
      const unsigned mask = __match_any_sync(0xffffffffu, e);
      const int before = __popc(mask & ((1u << lane) - 1u));
      const int base = e >= 0 ? s_cnt[e] : 0;
      __syncwarp();
      if (e >= 0) w.pos[i] = -2 - (base + before);  // rank, encoded below -1
      const int leader = 31 - __clz(mask);          // highest lane of the group
      if (e >= 0 && lane == leader) s_cnt[e] = base + __popc(mask);
      __syncwarp();
    }
    // exclusive scans over experts: pairs, blocks, block weights
    int run = 0, run_b = 0, run_w = 0;
    for (int c = 0; c < d.E; c += 32) {
      const int e = c + lane;
      const int cnt = e < d.E ? s_cnt[e] : 0;
      const int nb = (cnt + 7) / 8;
      const int wt = nb * (e < d.E ? s_sw[e] : 0);
      int x = cnt, xb = nb, xw = wt;
#pragma unroll
      for (int m = 1; m < 32; m <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, m);
        const int yb = __shfl_up_sync(0xffffffffu, xb, m);
        const int yw = __shfl_up_sync(0xffffffffu, xw, m);
        if (lane >= m) {
          x += y;
          xb += yb;
          xw += yw;
        }
      }
      if (e < d.E) {
        w.offsets[e] = run + x - cnt;
        w.counts[e] = cnt;
        s_nb0[e] = run_b + xb - nb;
        s_sw[e] = run_w + xw - wt;
      }
      run += __shfl_sync(0xffffffffu, x, 31);
      run_b += __shfl_sync(0xffffffffu, xb, 31);
      run_w += __shfl_sync(0xffffffffu, xw, 31);
    }
    if (lane == 0) {
      w.offsets[d.E] = run;
      s_nb0[d.E] = run_b;
      s_sw[d.E] = run_w;
    }
  }
  __syncthreads();
  // the block list: block nb0_e + i is column block i of expert e
  for (int e = tid; e < d.E; e += nt) {
    const int nb0 = s_nb0[e], nb = s_nb0[e + 1] - nb0;
    for (int i = 0; i < nb; ++i) w.blk[nb0 + i] = make_uint2(e, i);
  }
  {
    // CTA bounds.  Work item i of a phase is tile i % TPB of block i / TPB
    // and weighs its expert's tile weight; CTA c starts at the first item
    // whose weight prefix reaches c / grid of the total.  Thread c finds the
    // expert whose block-weight range [s_sw[e], s_sw[e + 1]) holds that point
    // (s_sw[e] grid <= c tot < s_sw[e + 1] grid) by bisection.
    const int tpb[2] = {d.inter / kRows, d.hidden / kRows};
    const long long tot = s_sw[d.E];
    const int gc = d.grid;
    for (int c = tid; c <= gc; c += nt) {
      if (tot == 0 || c == gc) {
        w.bounds[c] = tot == 0 ? 0 : s_nb0[d.E] * tpb[0];
        w.bounds[kMaxGrid + 1 + c] = tot == 0 ? 0 : s_nb0[d.E] * tpb[1];
        continue;
      }
      const long long pt = static_cast<long long>(c) * tot;
      int lo = 0, hi = d.E - 1;  // largest e with s_sw[e] * gc <= pt
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (static_cast<long long>(s_sw[mid]) * gc <= pt) {
          lo = mid;
        } else {
          hi = mid - 1;
        }
      }
      const int e = lo;
      const int nb0 = s_nb0[e], nb = s_nb0[e + 1] - nb0;
      const long long X = s_sw[e], we = (s_sw[e + 1] - X) / nb;
#pragma unroll
      for (int ph = 0; ph < 2; ++ph) {
        const long long T = tpb[ph];
        const long long local = (pt * T) / gc - T * X;
        const long long bo = local / (T * we);
        const long long tau = (local - bo * T * we + we - 1) / we;
        w.bounds[ph * (kMaxGrid + 1) + c] = static_cast<int>((nb0 + bo) * T + tau);
      }
    }
  }
  __syncthreads();
  // sorted positions (w.offsets is complete after the barrier)
  for (int i = tid; i < d.P; i += nt) {
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

// Block 0 routes (route_cta); block 1 + t rotates x_t and writes it in the
// layout of every width.  The two parts are independent, so they share one
// launch.
template <int LOGK>
__global__ void __launch_bounds__(FwhtShape<LOGK>::THREADS)
    moe_front_kernel(const hq_expert* __restrict__ ex, const int32_t* __restrict__ ids,
                     const __half* __restrict__ x, const int8_t* __restrict__ signs, Ws w, Dims d,
                     float inv) {
  using S = FwhtShape<LOGK>;
  extern __shared__ float buf[];
  pdl_launch_dependents();
  pdl_wait();  // the workspace is free once the previous call's kernels are done
  if (blockIdx.x == 0) {
    route_cta(ex, ids, w, d, reinterpret_cast<int*>(buf));
    return;
  }
  const int tid = threadIdx.x, t = blockIdx.x - 1;
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
// The loads of 8 pairs are issued before their sum, which runs in j order.
__global__ void moe_combine_kernel(const float* __restrict__ topk_w, Ws w, Dims d,
                                   float* __restrict__ y) {
  pdl_launch_dependents();
  pdl_wait();
  const size_t n = static_cast<size_t>(d.T) * d.hidden;
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const int t = static_cast<int>(i / d.hidden), c = static_cast<int>(i % d.hidden);
    float acc = 0.f;
    for (int j0 = 0; j0 < d.k; j0 += 8) {
      float dv[8], wv[8];
      unsigned live = 0;
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int j = j0 + u;
        const int p = j < d.k ? w.pos[t * d.k + j] : -1;
        dv[u] = p >= 0 ? w.d[static_cast<size_t>(p) * d.hidden + c] : 0.f;
        wv[u] = p >= 0 ? topk_w[t * d.k + j] : 0.f;
        live |= p >= 0 ? 1u << u : 0u;
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        if (live >> u & 1u) acc = fmaf(wv[u], dv[u], acc);
      }
    }
    y[i] = acc;
  }
}


// ---------------------------------------------------------------- expert phases
// Chunk geometry, shared by producer and consumer: a chunk is `len` groups of
// one item's 16 rows in each of its NMAT matrices, rows at a bank-conflict-
// free stride, then each matrix's scales.  len is a power of two and chunks
// start at multiples of it, so with G >= 8 (G a power of two) a chunk's
// groups lie in one aligned run of 8 and one 16-byte piece per row holds
// their scales; with G < 8 the tile's whole [16][G] scale block is copied.
__host__ __device__ inline int chunk_stride(int bits, int len) {
  const int row = len * 16 * bits;
  const int pad_w = ((bank_target_words(bits) - row / 4) % 32 + 32) % 32;
  return row + 4 * pad_w;
}
__host__ __device__ inline int chunk_scale_bytes(int G) {
  return G >= 8 ? kRows * 16 : kRows * G * 2;
}
constexpr int kRing = 2;               // slots per warp
constexpr int kChunkMax = 6 * 1024;    // slot bytes when the B fragments stay in global memory
constexpr int kSmemMax = 227 * 1024;
__host__ __device__ inline int chunk_bytes(int bits, int G, int nmat, int len) {
  return nmat * (kRows * chunk_stride(bits, len) + chunk_scale_bytes(G));
}
// Longest chunk (8, 4, 2 or 1 groups) that fits `cbytes`; 0 if none does.
__host__ __device__ inline int chunk_len(int bits, int G, int nmat, int cbytes) {
  for (int len = 8; len >= 1; len >>= 1) {
    if (len <= G && chunk_bytes(bits, G, nmat, len) <= cbytes) return len;
  }
  return 0;
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

// Shared-memory plan of one phase launch (host and device agree on it).
struct PhaseSmem {
  int bsmem;     // 1: the segment's B fragments are staged in shared memory
  int cbytes;    // ring slot bytes
  int xs_off, ring_off, bar_off, total;
};

__host__ __device__ inline int round128(int v) { return (v + 127) & ~127; }

__host__ __device__ inline PhaseSmem phase_smem(int G, int nmat) {
  PhaseSmem p{};
  // the largest len-1 chunk of any width must fit a slot
  int need = 0;
  for (int b = 2; b <= 8; b = b == 4 ? 8 : b + 1) need = max(need, chunk_bytes(b, G, nmat, 1));
  p.xs_off = round128(G * 8 * 4 + 64);  // zero-point terms [G][8], zero B block
  const int xs_bytes = G * 8 * 4 * 64;  // [G][8 columns][4 k-quads][64 B]
  const int ring_off = round128(p.xs_off + xs_bytes);
  const int fit = ((kSmemMax - ring_off - kWarps * kRing * 8) / (kWarps * kRing)) & ~127;
  p.bsmem = fit >= max(need, 4096) ? 1 : 0;  // else the rings would be too shallow
  p.cbytes = p.bsmem ? min(fit, kChunkMax) : kChunkMax;
  p.ring_off = p.bsmem ? ring_off : p.xs_off;
  p.bar_off = p.ring_off + kWarps * kRing * p.cbytes;
  p.total = p.bar_off + kWarps * kRing * 8;
  return p;
}

// The 16-byte piece pc of the B block (column col, k-quad q) sits at pc ^
// bswz(col, q) in shared memory, so that the 8 lanes of a quarter warp
// (two columns x four k-quads) read 8 different bank groups.
__device__ __forceinline__ int bswz(int col, int q) { return ((col & 1) << 1) | (q >> 1); }

// One warp's copy ring: kRing slots of ps.cbytes, one mbarrier each (32
// arrivals: every lane's cp.async group), counters over the whole kernel.
struct RingState {
  uint8_t* ring;
  uint64_t* bars;
  int consumed, issued;
  bool ok;  // false once a wait has timed out; the warp then stops
};

// The part of a segment one warp computes: items [w0, w1) of one block.
struct SegArgs {
  int w0, w1, tile0;  // tile of item j is tile0 + j
  int off, ncol;      // first sorted pair of the block, its columns (<= 8)
  int G, K, M;
  size_t brow_g;      // B row of this lane's column g (when g < ncol)
};

template <int PHASE, bool BSMEM, int BITS>
__device__ __forceinline__ void phase_tiles(const hq_expert& ed, Ws& w, const Dims& d,
                                            const PhaseSmem& ps, const SegArgs& sa, RingState& rs,
                                            const float* zc, const uint4* xs,
                                            const uint16_t* bsrc, int lane) {
  constexpr int NMAT = PHASE == 0 ? 2 : 1;
  constexpr int GB = 16 * BITS;  // code bytes of one row in one group
  const int g = lane >> 2, t = lane & 3;
  const int G = sa.G;
  const int len = chunk_len(BITS, G, NMAT, ps.cbytes);  // divides G (both powers of two)
  const int stride = chunk_stride(BITS, len);
  const int row_bytes = sa.K * BITS / 8;
  const int sbytes = chunk_scale_bytes(G);
  // producer geometry: pr 16-byte pieces per row, 16 rows; lane's first piece
  // (r0, c0) and the step of 32 pieces (dr rows + dc pieces)
  const int pr = len * BITS;
  const int npc = kRows * pr;
  const int r0 = lane / pr, c0 = lane - r0 * pr;
  const int dr = 32 / pr, dc = 32 - dr * pr;
  const uint8_t* qbase[NMAT];
  const uint16_t* sbase[NMAT];
  if (PHASE == 0) {
    qbase[0] = reinterpret_cast<const uint8_t*>(ed.q_gate);
    qbase[NMAT - 1] = reinterpret_cast<const uint8_t*>(ed.q_up);
    sbase[0] = ed.s_gate;
    sbase[NMAT - 1] = ed.s_up;
  } else {
    qbase[0] = reinterpret_cast<const uint8_t*>(ed.q_down);
    sbase[0] = ed.s_down;
  }
  int pj = sa.w0, pg = 0;  // next (item, group) to copy
  auto issue = [&](int slot) {
    const int m0 = (sa.tile0 + pj) * kRows;
    uint8_t* base = rs.ring + slot * ps.cbytes;
#pragma unroll
    for (int mi = 0; mi < NMAT; ++mi) {
      const uint8_t* src = qbase[mi] + static_cast<size_t>(m0) * row_bytes + pg * GB;
      uint8_t* cdst = base + mi * kRows * stride;
      int r = r0, c = c0;
      for (int i = lane; i < npc; i += 32) {
        cp_async16(cdst + r * stride + c * 16, src + r * row_bytes + c * 16, 16);
        c += dc;
        r += dr;
        if (c >= pr) {
          c -= pr;
          ++r;
        }
      }
      uint8_t* sdst = base + NMAT * kRows * stride + mi * sbytes;
      if (G >= 8) {
        if (lane < kRows) cp_async16(sdst + lane * 16, sbase[mi] + static_cast<size_t>(m0 + lane) * G + (pg & ~7), 16);
      } else if (lane < 2 * G) {
        cp_async16(sdst + lane * 16, reinterpret_cast<const uint8_t*>(sbase[mi] + static_cast<size_t>(m0) * G) + lane * 16, 16);
      }
    }
    cp_async_mbar_arrive(&rs.bars[slot]);
    pg += len;
    if (pg >= G) {
      pg = 0;
      ++pj;
    }
    ++rs.issued;
  };
  if (!rs.ok) return;
  for (int k2 = 0; k2 < kRing && pj < sa.w1; ++k2) issue(rs.issued % kRing);

  // consumer: this lane's B blocks (column g, k-quad t), or the zero block
  const bool has_b = g < sa.ncol;
  const uint4* zero_blk = reinterpret_cast<const uint4*>(zc + G * 8);
  const uint4* bl;
  int bstep;  // uint4 per group
  int bo[4];  // uint4 offset of piece i within a block
  if constexpr (BSMEM) {
    bl = has_b ? xs + (g * 4 + t) * 4 : zero_blk;
    bstep = has_b ? sa.ncol * 16 : 0;
    const int sw = has_b ? bswz(g, t) : 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) bo[i] = i ^ sw;
  } else {
    bl = has_b ? reinterpret_cast<const uint4*>(bsrc + (sa.brow_g * G * 4 + t) * kXq) : zero_blk;
    bstep = has_b ? 4 * kXq / 8 : 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) bo[i] = i;
  }
  for (int j = sa.w0; j < sa.w1; ++j) {
    const int m0 = (sa.tile0 + j) * kRows;
    float acc[NMAT][4] = {};
    uint4 bq[4];
    if constexpr (!BSMEM) {
#pragma unroll
      for (int i = 0; i < 4; ++i) bq[i] = bl[bo[i]];
    }
    for (int g0 = 0; g0 < G; g0 += len) {
      const int slot = rs.consumed % kRing;
      if (!mbar_wait(&rs.bars[slot], (rs.consumed / kRing) & 1)) {
        rs.ok = false;
        return;
      }
      __syncwarp();
      const uint8_t* base = rs.ring + slot * ps.cbytes;
      const __half* scb = reinterpret_cast<const __half*>(base + NMAT * kRows * stride);
      for (int jj = 0; jj < len; ++jj) {
        const int gi = g0 + jj;
        uint4 bn[4];
        if constexpr (BSMEM) {
#pragma unroll
          for (int i = 0; i < 4; ++i) bq[i] = bl[gi * bstep + bo[i]];
        } else {
          // the next group's blocks, one group ahead of their use
          const int gn = gi + 1 < G ? gi + 1 : gi;
#pragma unroll
          for (int i = 0; i < 4; ++i) bn[i] = bl[gn * bstep + bo[i]];
        }
        const float2 z = *reinterpret_cast<const float2*>(zc + gi * 8 + 2 * t);
        const int sa_idx = G >= 8 ? g * 8 + (gi & 7) : g * G + gi;
        const int sb_idx = G >= 8 ? (g + 8) * 8 + (gi & 7) : (g + 8) * G + gi;
#pragma unroll
        for (int mi = 0; mi < NMAT; ++mi) {
          const uint8_t* ra = base + mi * kRows * stride + g * stride + jj * GB + t * 4 * BITS;
          const __half* scp = scb + mi * (sbytes / 2);
          group_mma<BITS>(ra, ra + 8 * stride, bq, z, __half2float(scp[sa_idx]),
                          __half2float(scp[sb_idx]), acc[mi]);
        }
        if constexpr (!BSMEM) {
#pragma unroll
          for (int i = 0; i < 4; ++i) bq[i] = bn[i];
        }
      }
      __syncwarp();
      if (pj < sa.w1) issue(slot);
      ++rs.consumed;
    }
    // epilogue: rows g, g+8; columns 2t, 2t+1
#pragma unroll
    for (int q4 = 0; q4 < 4; ++q4) {
      const int col = 2 * t + (q4 & 1);
      const int m = m0 + g + 8 * (q4 >> 1);
      if (col < sa.ncol && m < sa.M) {
        const size_t prow = static_cast<size_t>(sa.off + col);
        if (PHASE == 0) {
          const float gv = acc[0][q4] * kUnit, uv = acc[NMAT - 1][q4] * kUnit;
          w.h[prow * d.inter + m] = gv / (1.f + expf(-gv)) * uv;
        } else {
          w.d[prow * d.hidden + m] = acc[0][q4] * kUnit;
        }
      }
    }
  }
}

// Phase A (PHASE 0): gate and up, SwiGLU -> h.  Phase B (PHASE 1): down -> d.
//
// Work item i is 16-row tile i % TPB of block i / TPB, a block being one
// expert's <= 8-token column block (w.blk); CTA c owns items [bounds[c],
// bounds[c + 1]), split by tile weight, and walks them one segment (the part
// of one block) at a time.  Per segment the CTA writes the zero-point terms of the
// block's <= 8 columns to shared memory and, when BSMEM, stages the block's
// B fragments (the rotated activations, every group) there too; then its
// warps split the segment's tiles and stream each tile's codes and scales
// through a private cp.async ring.  Without BSMEM (K too large for the B
// fragments to fit beside the rings) each lane reads its B blocks from
// global memory, one group ahead.
template <int PHASE, bool BSMEM>
__global__ void __launch_bounds__(kWarps * 32, 1)
    moe_phase_kernel(const hq_expert* __restrict__ ex, Ws w, Dims d, PhaseSmem ps) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2;
  const int K = PHASE == 0 ? d.hidden : d.inter;
  const int M = PHASE == 0 ? d.inter : d.hidden;
  const int G = K / kGroup;
  const int TPB = M / kRows;  // tiles per block
  float* zc = reinterpret_cast<float*>(smem);  // [G][8], then a zero B block (64 B)
  uint4* xs = reinterpret_cast<uint4*>(smem + ps.xs_off);  // [G][ncol][4][4 pieces], swizzled
  uint8_t* ring = smem + ps.ring_off + warp * kRing * ps.cbytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + ps.bar_off) + warp * kRing;
  if (lane == 0) {
    for (int i = 0; i < kRing; ++i) mbar_init(&bars[i], 32);
    fence_mbar_init();
  }
  if (tid < 16) (zc + G * 8)[tid] = 0.f;
  __syncthreads();
  pdl_launch_dependents();
  pdl_wait();  // routing lists and activations come from the previous kernels
  const int* bounds = w.bounds + PHASE * (kMaxGrid + 1);
  const uint16_t* bsrc = PHASE == 0 ? w.xl : w.hl;
  const float* sums = PHASE == 0 ? w.xsum : w.hsum;
  const int ib = bounds[blockIdx.x], ie = bounds[blockIdx.x + 1];
  RingState rs{ring, bars, 0, 0, true};  // this warp's ring, over the whole kernel

  for (int it = ib; it < ie;) {
    // ---- the segment: items [it, se) of one (expert, column block)
    const int b = it / TPB;
    const uint2 bk = w.blk[b];
    const int e = static_cast<int>(bk.x);
    const int cb = static_cast<int>(bk.y);
    const int tile_first = it - b * TPB;
    const int se = min(ie, (b + 1) * TPB);
    const hq_expert ed = ex[e];
    const int bits = ed.bits;
    const int L = layout_index(bits);
    const int off = w.offsets[e] + 8 * cb;
    const int ncol = min(8, w.counts[e] - 8 * cb);
    // B-operand row of column col of this block
    auto brow = [&](int col) -> size_t {
      const int p = off + col;
      return PHASE == 0 ? static_cast<size_t>(L) * d.T + w.sorted[p] / d.k : static_cast<size_t>(p);
    };
    __syncthreads();  // every warp is done with the previous segment's B and zc
    {
      if constexpr (BSMEM) {
        // 64 bytes of each 80-byte block (the rest is padding), 16-byte pieces
        const int per_col = G * 16;
        for (int i = tid; i < ncol * per_col; i += kWarps * 32) {
          const int col = i / per_col, r = i - col * per_col;
          const int gg = r >> 4, q = (r >> 2) & 3, pc = r & 3;
          cp_async16(xs + ((gg * ncol + col) * 4 + q) * 4 + (pc ^ bswz(col, q)),
                     bsrc + ((brow(col) * G + gg) * 4 + q) * kXq + pc * 8, 16);
        }
      }
      // zero-point terms -zero * sum_k x' * 2^-24 (0 for absent columns)
      const float zneg = -static_cast<float>(ed.zero) * 5.9604644775390625e-8f;
      for (int i = tid; i < G * 8; i += kWarps * 32) {
        const int gg = i >> 3, col = i & 7;
        zc[i] = col < ncol ? zneg * sums[brow(col) * G + gg] : 0.f;
      }
      if constexpr (BSMEM) asm volatile("cp.async.wait_all;" ::: "memory");
    }
    __syncthreads();

    // ---- this warp's tiles of the segment: items [w0, w1)
    const int n = se - it;
    SegArgs sa;
    sa.w0 = it + (n * warp) / kWarps;
    sa.w1 = it + (n * (warp + 1)) / kWarps;
    sa.tile0 = tile_first - it;  // tile of item j is tile0 + j
    sa.off = off;
    sa.ncol = ncol;
    sa.G = G;
    sa.K = K;
    sa.M = M;
    sa.brow_g = g < ncol ? brow(g) : 0;
    switch (bits) {
      case 2: phase_tiles<PHASE, BSMEM, 2>(ed, w, d, ps, sa, rs, zc, xs, bsrc, lane); break;
      case 3: phase_tiles<PHASE, BSMEM, 3>(ed, w, d, ps, sa, rs, zc, xs, bsrc, lane); break;
      case 4: phase_tiles<PHASE, BSMEM, 4>(ed, w, d, ps, sa, rs, zc, xs, bsrc, lane); break;
      default: phase_tiles<PHASE, BSMEM, 8>(ed, w, d, ps, sa, rs, zc, xs, bsrc, lane); break;
    }
    it = se;
  }
  if (!rs.ok) {
    // a ring wait timed out: report it and let the copies still in flight land
    if (lane == 0) record_error(w.status, HQ_DEV_TIMEOUT);
    for (int k2 = rs.consumed; k2 < rs.issued; ++k2) {
      (void)mbar_wait(&rs.bars[k2 % kRing], (k2 / kRing) & 1);
    }
  }
}

}  // namespace moe

// ---------------------------------------------------------------- host side
static cudaError_t moe_launch_front(int hidden, const hq_expert* ex, const int32_t* ids,
                                    const __half* x, const int8_t* s, const moe::Ws& w,
                                    const moe::Dims& d, cudaStream_t st) {
  const float inv = static_cast<float>(1.0 / sqrt(static_cast<double>(hidden)));
  const size_t route_smem = (3 * static_cast<size_t>(d.E) + 2) * sizeof(int);
#define HQ_FRONT(LK)                                                                          \
  case (1 << LK):                                                                             \
    return launch_pdl(moe::moe_front_kernel<LK>, dim3(d.T + 1), dim3(FwhtShape<LK>::THREADS),   \
                      std::max(FwhtShape<LK>::SMEM_FLOATS * sizeof(float), route_smem), st, true, \
                      ex, ids, x, s, w, d, inv);
  switch (hidden) {
    HQ_FRONT(7) HQ_FRONT(8) HQ_FRONT(9) HQ_FRONT(10) HQ_FRONT(11) HQ_FRONT(12) HQ_FRONT(13)
    HQ_FRONT(14)
    default: return cudaErrorInvalidValue;
  }
#undef HQ_FRONT
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

template <int PHASE>
static cudaError_t moe_launch_phase(const hq_expert* ex, const moe::Ws& w, const moe::Dims& d,
                                    cudaStream_t st) {
  constexpr int nmat = PHASE == 0 ? 2 : 1;
  const int G = (PHASE == 0 ? d.hidden : d.inter) / kGroup;
  const moe::PhaseSmem ps = moe::phase_smem(G, nmat);
  for (int b : {2, 3, 4, 8}) {
    if (moe::chunk_len(b, G, nmat, ps.cbytes) == 0) return cudaErrorInvalidConfiguration;
  }
  if (ps.total > moe::kSmemMax) return cudaErrorInvalidConfiguration;
  const dim3 grid(d.grid), block(moe::kWarps * 32);  // one CTA per SM; the routing CTA split
                                                     // the work for exactly d.grid CTAs
  return ps.bsmem ? launch_pdl(moe::moe_phase_kernel<PHASE, true>, grid, block, ps.total, st, true,
                               ex, w, d, ps)
                  : launch_pdl(moe::moe_phase_kernel<PHASE, false>, grid, block, ps.total, st, true,
                               ex, w, d, ps);
}

}  // namespace hq

using namespace hq;

// The routing CTA keeps three ints per expert in shared memory.
constexpr int kMaxExperts = 16384;

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

int hq_moe_launches(void) { return 5; }

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
  const __half* xh = reinterpret_cast<const __half*>(x);
  cudaError_t e = moe_launch_front(hidden, experts, topk_ids, xh, signs_in, w, d, st);
  if (e == cudaSuccess) e = moe_launch_phase<0>(experts, w, d, st);
  if (e == cudaSuccess) e = moe_launch_rot_h(inter, experts, topk_ids, signs_mid, w, d, st);
  if (e == cudaSuccess) e = moe_launch_phase<1>(experts, w, d, st);
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
