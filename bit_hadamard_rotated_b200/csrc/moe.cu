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
//                         written in the MMA B-fragment layout of every width
//                         (scaled by a power of two 2^e per token that puts
//                         its largest |x'| just below 2^14, undone exactly in
//                         the phase epilogue, as is the same scale of h');
//                         and, for each of the token's pairs whose expert has
//                         its own input signs, x_t rotated with those signs,
//                         in that expert's layout;
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
  float* xfac;     // [T] output factor 2^(24 - e) of each token's scaled x'
  float* h;        // [P][inter]
  uint16_t* hl;    // [P][G_i][4][kXq] rotated h, in its expert's layout
  float* hsum;     // [P][G_i]
  float* hfac;     // [P] output factor 2^(24 - e) of each pair's scaled h'
  float* d;        // [P][hidden]
  uint16_t* xpl;   // [P][G_h][4][kXq] x rotated with the pair's expert's own signs (pair index t k + j)
  float* xpsum;    // [P][G_h]
  float* xpfac;    // [P]
};

struct Dims {
  int E, hidden, inter, T, k, P;
  int nb_max;  // bound on the number of (expert, column block) blocks
  int grid;    // CTAs of each expert phase
};

constexpr int kMaxGrid = 1024;

// Relative cost of one work item of a width in each phase, for splitting
// the phases' work between CTAs and warps: a part proportional to the width
// (code bytes and decode) plus a fixed part (per-tile and per-group overhead).
// On the 256-expert layer, per-CTA times put a 4-bit gate/up tile (K = 2048)
// at ~1.7x a 2-bit one (bits + 1: 59.7 -> 57.2 us for the phase); for down
// (K = 512) bits + 2 measured best (bits + 11, the per-CTA fit, was 12 %
// slower: the down phase's cost follows its segments, not only its tiles).
__host__ __device__ constexpr int tile_weight(int phase, int bits) {
  return phase == 0 ? bits + 1 : bits + 2;
}

// Rows of one work item: a phase-A item is a 16-row tile of gate and of up;
// a phase-B item is a 32-row tile of down, taken as two 16-row halves.  Either
// way a group's activation fragments and zero-point terms are loaded once
// for two 16-row code tiles.
__host__ __device__ constexpr int item_rows(int phase) { return phase == 0 ? 16 : 32; }

}  // namespace moe

// Workspace carve-up (host side; also sizes hq_moe_workspace_size).
static size_t a256(size_t v) { return (v + 255) & ~static_cast<size_t>(255); }

struct MoePlan {
  moe::Dims d;
  size_t off[18];
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
  const size_t sizes[18] = {
      256,                                             // status
      sizeof(int) * E,                                 // counts
      sizeof(int) * (E + 1),                           // offsets
      sizeof(int) * d.P,                               // pos
      sizeof(int) * d.P,                               // sorted
      sizeof(uint2) * d.nb_max,                        // blk
      sizeof(int) * 2 * (moe::kMaxGrid + 1),           // bounds
      4 * static_cast<size_t>(T),                      // xfac
      2 * 4 * static_cast<size_t>(T) * Gh * 4 * moe::kXq,  // xl
      4 * 4 * static_cast<size_t>(T) * Gh,                 // xsum
      4 * static_cast<size_t>(d.P) * inter,                // h
      2 * static_cast<size_t>(d.P) * Gi * 4 * moe::kXq,    // hl
      4 * static_cast<size_t>(d.P) * Gi,                   // hsum
      4 * static_cast<size_t>(d.P) * hidden,               // d
      4 * static_cast<size_t>(d.P),                        // hfac
      2 * static_cast<size_t>(d.P) * Gh * 4 * moe::kXq,    // xpl
      4 * static_cast<size_t>(d.P) * Gh,                   // xpsum
      4 * static_cast<size_t>(d.P),                        // xpfac
  };
  size_t o = 0;
  for (int i = 0; i < 18; ++i) {
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
  w.xfac = reinterpret_cast<float*>(b + pl.off[7]);
  w.xl = reinterpret_cast<uint16_t*>(b + pl.off[8]);
  w.xsum = reinterpret_cast<float*>(b + pl.off[9]);
  w.h = reinterpret_cast<float*>(b + pl.off[10]);
  w.hl = reinterpret_cast<uint16_t*>(b + pl.off[11]);
  w.hsum = reinterpret_cast<float*>(b + pl.off[12]);
  w.d = reinterpret_cast<float*>(b + pl.off[13]);
  w.hfac = reinterpret_cast<float*>(b + pl.off[14]);
  w.xpl = reinterpret_cast<uint16_t*>(b + pl.off[15]);
  w.xpsum = reinterpret_cast<float*>(b + pl.off[16]);
  w.xpfac = reinterpret_cast<float*>(b + pl.off[17]);
  return w;
}

namespace moe {

__device__ __forceinline__ bool valid_desc(const hq_expert& e) {
  const bool bits_ok = e.bits == 2 || e.bits == 3 || e.bits == 4 || e.bits == 8;
  // the kernels read sign vectors in 16-byte pieces: a misaligned one is a bad descriptor
  const bool signs_ok = (reinterpret_cast<uintptr_t>(e.signs_in) & 15u) == 0 &&
                        (reinterpret_cast<uintptr_t>(e.signs_mid) & 15u) == 0;
  return bits_ok && signs_ok && e.zero >= 0 && e.zero < (1 << e.bits) && e.q_gate && e.q_up &&
         e.q_down && e.s_gate && e.s_up && e.s_down;
}

// The routing CTA (block 0 of the first launch).  Stable counting sort of the
// pairs by expert: pair i = t*k + j is ranked among the pairs of its expert in
// increasing i, so the sorted order, and every sum taken over it, is
// independent of thread timing.  Then the block list and, for each expert
// phase, the first work item of every CTA, splitting the summed tile weights
// evenly.  Shared memory: 3 E + 3 ints.
__device__ void route_cta(const hq_expert* __restrict__ ex, const int32_t* __restrict__ ids,
                          const Ws& w, const Dims& d, int* sm) {
  int* s_cnt = sm;                  // [E + 1] valid pairs per expert, then phase B's weight prefix
  int* s_nb0 = sm + d.E + 1;        // [E + 1] first block of each expert; [E] = blocks in all
  int* s_sw = s_nb0 + d.E + 1;      // [E + 1] width, then phase A's block-weight prefix
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nt = blockDim.x;
  // s_sw[e]: the width of expert e if its descriptor is valid, else -1 (or 0
  // while unknown).  With a few descriptors per thread, all of them are
  // checked before the wait (the expert table is a weight: no earlier kernel
  // of the library writes it); with more, only those the pairs name, after it.
  const bool all_desc = d.E <= 4 * nt;
  for (int e = tid; e < d.E; e += nt) {
    s_cnt[e] = 0;
    int sw = 0;
    if (all_desc) {
      const hq_expert de = ex[e];
      sw = valid_desc(de) ? de.bits : -1;
    }
    s_sw[e] = sw;
  }
  __syncthreads();
  pdl_wait();  // ids may be the previous kernel's output; the workspace is free once it is done
  // validity of every pair (its expert id and that expert's descriptor)
  for (int i = tid; i < d.P; i += nt) {
    const int e = ids[i];
    bool ok = e >= 0 && e < d.E;
    if (!ok) {
      record_error(w.status, HQ_DEV_BAD_EXPERT);
    } else if (all_desc) {
      ok = s_sw[e] > 0;
    } else {
      const hq_expert de = ex[e];
      ok = valid_desc(de);
      if (ok) s_sw[e] = de.bits;  // the same value from every pair of e
    }
    if (!ok) {
      if (e >= 0 && e < d.E) record_error(w.status, HQ_DEV_BAD_BITS);
      w.pos[i] = -1;
    }
  }
  __syncthreads();
  if (warp == 0) {
    // ranks in pair order, 32 pairs at a time; the ids (cached on chip since
    // the pass above) are loaded one round ahead, validity comes from s_sw
    auto key = [&](int i) {
      const int e = i < d.P ? ids[i] : -1;
      return e >= 0 && e < d.E && s_sw[e] > 0 ? e : -1;
    };
    int e_next = key(lane);
    for (int c = 0; c < d.P; c += 32) {
      const int i = c + lane;
      const int e = e_next;
      e_next = key(i + 32);
      const unsigned mask = __match_any_sync(0xffffffffu, e);
      const int before = __popc(mask & ((1u << lane) - 1u));
      const int base = e >= 0 ? s_cnt[e] : 0;
      __syncwarp();
      if (e >= 0) w.pos[i] = -2 - (base + before);  // rank, encoded below -1
      const int leader = 31 - __clz(mask);          // highest lane of the group
      if (e >= 0 && lane == leader) s_cnt[e] = base + __popc(mask);
      __syncwarp();
    }
    // exclusive scans over experts: pairs, blocks, block weights of each phase
    int run = 0, run_b = 0, run_w = 0, run_v = 0;
    for (int c = 0; c < d.E; c += 32) {
      const int e = c + lane;
      const int cnt = e < d.E ? s_cnt[e] : 0;
      const int nb = (cnt + 7) / 8;
      const int bits = nb > 0 ? s_sw[e] : 0;
      const int wt = nb * tile_weight(0, bits), wv = nb * tile_weight(1, bits);
      int x = cnt, xb = nb, xw = wt, xv = wv;
#pragma unroll
      for (int m = 1; m < 32; m <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, m);
        const int yb = __shfl_up_sync(0xffffffffu, xb, m);
        const int yw = __shfl_up_sync(0xffffffffu, xw, m);
        const int yv = __shfl_up_sync(0xffffffffu, xv, m);
        if (lane >= m) {
          x += y;
          xb += yb;
          xw += yw;
          xv += yv;
        }
      }
      if (e < d.E) {
        w.offsets[e] = run + x - cnt;
        w.counts[e] = cnt;
        s_nb0[e] = run_b + xb - nb;
        s_sw[e] = run_w + xw - wt;
        s_cnt[e] = run_v + xv - wv;
      }
      run += __shfl_sync(0xffffffffu, x, 31);
      run_b += __shfl_sync(0xffffffffu, xb, 31);
      run_w += __shfl_sync(0xffffffffu, xw, 31);
      run_v += __shfl_sync(0xffffffffu, xv, 31);
    }
    if (lane == 0) {
      w.offsets[d.E] = run;
      s_nb0[d.E] = run_b;
      s_sw[d.E] = run_w;
      s_cnt[d.E] = run_v;
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
    // and weighs its expert's tile weight in that phase; CTA c starts at the
    // first item whose weight prefix reaches c / grid of the total.  Thread
    // (c, phase) finds the expert whose block-weight range [pre[e],
    // pre[e + 1]) holds that point (pre[e] grid <= c tot < pre[e + 1] grid)
    // by bisection.
    const int tpb[2] = {d.inter / item_rows(0), d.hidden / item_rows(1)};
    const int gc = d.grid;
    for (int job = tid; job < 2 * (gc + 1); job += nt) {
      const int ph = job / (gc + 1), c = job - ph * (gc + 1);
      const int* pre = ph == 0 ? s_sw : s_cnt;
      const long long tot = pre[d.E];
      int* out = w.bounds + ph * (kMaxGrid + 1);
      if (tot == 0 || c == gc) {
        out[c] = tot == 0 ? 0 : s_nb0[d.E] * tpb[ph];
        continue;
      }
      const long long pt = static_cast<long long>(c) * tot;
      int lo = 0, hi = d.E - 1;  // largest e with pre[e] * gc <= pt
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (static_cast<long long>(pre[mid]) * gc <= pt) {
          lo = mid;
        } else {
          hi = mid - 1;
        }
      }
      const int e = lo;
      const int nb0 = s_nb0[e], nb = s_nb0[e + 1] - nb0;
      const long long X = pre[e], we = (pre[e + 1] - X) / nb;
      const long long T = tpb[ph];
      const long long local = (pt * T) / gc - T * X;
      const long long bo = local / (T * we);
      const long long tau = (local - bo * T * we + we - 1) / we;
      out[c] = static_cast<int>((nb0 + bo) * T + tau);
    }
  }
  __syncthreads();
  // sorted positions (w.offsets is complete after the barrier); the rank and
  // the expert's offset are loaded together
  for (int i = tid; i < d.P; i += nt) {
    const int e = ids[i];
    const int off = w.offsets[e >= 0 && e < d.E ? e : 0];
    const int r = w.pos[i];
    if (r <= -2) {
      const int p = off + (-2 - r);
      w.pos[i] = p;
      w.sorted[p] = i;
    }
  }
}


// Write one rotated row (fwht_block output in buf, unnormalised; sc = 2^e /
// sqrt(K)) as fp16 B blocks for the code decode of BITS: block (group gg,
// k-quad t) holds the 8 steps x 4 activations x' 2^e, each scaled by 2^-a of
// its code field; sums[gg] = sum over the group of the effective activations
// (B * 2^a), for the zero-point term.  Warp-per-group; nw warps of the block
// take part.
template <int BITS>
__device__ __forceinline__ void write_layout(const float* buf, float sc, int G, uint16_t* out,
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
      const float xv = __half2float(__float2half_rn(buf[fwht_pad(kGroup * gg + kc[r])] * sc));
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

__device__ __forceinline__ void write_layout_bits(int bits, const float* buf, float sc, int G,
                                                  uint16_t* out, float* sums, int warp, int nw,
                                                  int lane) {
  switch (bits) {
    case 2: write_layout<2>(buf, sc, G, out, sums, warp, nw, lane); break;
    case 3: write_layout<3>(buf, sc, G, out, sums, warp, nw, lane); break;
    case 4: write_layout<4>(buf, sc, G, out, sums, warp, nw, lane); break;
    default: write_layout<8>(buf, sc, G, out, sums, warp, nw, lane); break;
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
  if (blockIdx.x == 0) {
    route_cta(ex, ids, w, d, reinterpret_cast<int*>(buf));  // waits inside
    return;
  }
  const int tid = threadIdx.x, t = blockIdx.x - 1;
  const auto neg = sign_bits<S::E>(signs ? signs + tid * S::E : nullptr);
  pdl_wait();  // x may be the previous kernel's output
  float v[S::E];
  float* red = buf + S::SMEM_FLOATS;
  load_chunk<__half, S::E>(x + static_cast<size_t>(t) * S::K + tid * S::E, v);
  flip_signs<S::E>(neg, v);
  fwht_block<LOGK, 5>(v, buf, red);
  const int e = row_scale_exp(red_max(red, S::W) * inv);
  if (tid == 0) w.xfac[t] = pow2f(24 - e);
  const float sc = inv * pow2f(e);
  const int G = S::K / kGroup;
  const int bits_of[4] = {2, 3, 4, 8};
  for (int L = 0; L < 4; ++L) {
    const size_t row = static_cast<size_t>(L) * d.T + t;
    write_layout_bits(bits_of[L], buf, sc, G, w.xl + row * G * 4 * kXq, w.xsum + row * G,
                      tid >> 5, S::THREADS / 32, tid & 31);
  }
  // pairs of this token whose expert brings its own input signs: x_t rotated
  // with them, in that expert's layout (rows of bad ids or descriptors are
  // never read: their pairs are skipped)
  for (int j = 0; j < d.k; ++j) {
    const int i = t * d.k + j;
    const int e = ids[i];
    if (e < 0 || e >= d.E) continue;  // uniform over the block
    const hq_expert de = ex[e];
    if (de.signs_in == nullptr || !valid_desc(de)) continue;
    __syncthreads();  // buf and red are free again
    const auto own = sign_bits<S::E>(de.signs_in + tid * S::E);
    load_chunk<__half, S::E>(x + static_cast<size_t>(t) * S::K + tid * S::E, v);
    flip_signs<S::E>(own, v);
    fwht_block<LOGK, 5>(v, buf, red);
    const int ej = row_scale_exp(red_max(red, S::W) * inv);
    if (tid == 0) w.xpfac[i] = pow2f(24 - ej);
    write_layout_bits(de.bits, buf, inv * pow2f(ej), G, w.xpl + static_cast<size_t>(i) * G * 4 * kXq,
                      w.xpsum + static_cast<size_t>(i) * G, tid >> 5, S::THREADS / 32, tid & 31);
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
  const int tid = threadIdx.x, p = blockIdx.x;
  const auto neg = sign_bits<S::E>(signs ? signs + tid * S::E : nullptr);
  pdl_wait();
  if (p >= w.offsets[d.E]) return;  // block-uniform: no barrier is skipped by part of it
  const int e = ids[w.sorted[p]];
  const hq_expert de = ex[e];
  const int bits = de.bits;
  float v[S::E];
  float* red = buf + S::SMEM_FLOATS;
  load_chunk<float, S::E>(w.h + static_cast<size_t>(p) * S::K + tid * S::E, v);
  // the expert's own signs for its down projection, where it has them
  flip_signs<S::E>(de.signs_mid != nullptr ? sign_bits<S::E>(de.signs_mid + tid * S::E) : neg, v);
  fwht_block<LOGK, 5>(v, buf, red);
  const int ex_ = row_scale_exp(red_max(red, S::W) * inv);
  if (tid == 0) w.hfac[p] = pow2f(24 - ex_);
  const float sc = inv * pow2f(ex_);
  const int G = S::K / kGroup;
  write_layout_bits(bits, buf, sc, G, w.hl + static_cast<size_t>(p) * G * 4 * kXq,
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
// one item's two 16-row code tiles (gate and up, or the halves of a 32-row
// down tile), rows at a bank-conflict-free stride, then each tile's scales.
// len is a power of two and chunks start at multiples of it, so with G >= 8
// (G a power of two) a chunk's groups lie in one aligned run of 8 and one
// 16-byte piece per row holds their scales; with G < 8 each tile's whole
// [16][G] scale block is copied.
__host__ __device__ constexpr int chunk_stride(int bits, int len) {
  const int row = len * 16 * bits;
  const int pad_w = ((bank_target_words(bits) - row / 4) % 32 + 32) % 32;
  return row + 4 * pad_w;
}
__host__ __device__ constexpr int chunk_scale_bytes(int G) {
  return G >= 8 ? kRows * 16 : kRows * G * 2;
}
constexpr int kRing = 2;               // slots per warp
constexpr int kChunkMax = 6 * 1024;    // slot bytes when the B fragments stay in global memory
constexpr int kSmemMax = 227 * 1024;
__host__ __device__ constexpr int chunk_bytes(int bits, int G, int nmat, int len) {
  return nmat * (kRows * chunk_stride(bits, len) + chunk_scale_bytes(G));
}
// Longest chunk (8, 4, 2 or 1 groups) that fits `cbytes`; 0 if none does.
__host__ __device__ constexpr int chunk_len(int bits, int G, int nmat, int cbytes) {
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

// A pass of a phase CTA: up to kMaxSeg consecutive segments (the parts of
// (expert, column block) blocks in the CTA's item range) with at most 8
// columns in all, whose activation fragments are staged together.
constexpr int kMaxSeg = 4;

struct SegInfo {
  hq_expert ed;
  int item0, item1;  // items [item0, item1)
  int tile0;         // row tile of item0 within the expert
  int unit0;         // first (item, group) unit of the segment within the pass
  int wt0;           // weight of the pass's units before the segment (tile weight per unit)
  int off, ncol;     // first sorted pair of the block, its columns (<= 8)
  int col0;          // column offset of the block in the staged fragments
  int L;             // activation layout (bit width) of phase A
  float fac[8];      // output factor 2^(24 - e) of each column (token or pair)
  int own;           // phase A: the expert rotates its tokens with its own signs
};

struct PassMeta {
  SegInfo seg[kMaxSeg];
  int nseg, cols, units, wtot;
};
static_assert(sizeof(PassMeta) <= 1024, "pass metadata");

// Shared-memory plan of one phase launch (host and device agree on it):
// [pass metadata 1 KiB][zero-point terms [kMaxSeg][G][8] fp32, zero B block]
// [staged B fragments [G][8 columns][4 k-quads][64 B] (BSMEM)][rings][barriers]
struct PhaseSmem {
  int bsmem;     // 1: the pass's B fragments are staged in shared memory
  int cbytes;    // ring slot bytes
  int zc_off, xs_off, ring_off, bar_off, total;
};

__host__ __device__ constexpr int round128(int v) { return (v + 127) & ~127; }

__host__ __device__ constexpr PhaseSmem phase_smem(int G, int nmat) {
  PhaseSmem p{};
  // the largest len-1 chunk of any width must fit a slot
  int need = 0;
  for (int b = 2; b <= 8; b = b == 4 ? 8 : b + 1) {
    const int c = chunk_bytes(b, G, nmat, 1);
    need = need > c ? need : c;
  }
  p.zc_off = 1024;
  p.xs_off = round128(p.zc_off + kMaxSeg * G * 8 * 4 + 64);
  const int xs_bytes = G * 8 * 4 * 64;
  const int ring_off = round128(p.xs_off + xs_bytes);
  const int fit = ((kSmemMax - ring_off - kWarps * kRing * 8) / (kWarps * kRing)) & ~127;
  p.bsmem = fit >= (need > 4096 ? need : 4096) ? 1 : 0;  // else the rings would be too shallow
  p.cbytes = p.bsmem ? (fit < kChunkMax ? fit : kChunkMax) : kChunkMax;
  p.ring_off = p.bsmem ? ring_off : p.xs_off;
  p.bar_off = p.ring_off + kWarps * kRing * p.cbytes;
  p.total = p.bar_off + kWarps * kRing * 8;
  return p;
}

// The 16-byte piece pc of the B block (column col, k-quad q) sits at pc ^
// bswz(col, q) in shared memory, so that the 8 lanes of a quarter warp
// (two columns x four k-quads) read 8 different bank groups.
__device__ __forceinline__ int bswz(int col, int q) { return ((col & 1) << 1) | (q >> 1); }

// One warp's copy ring: kRing slots of the plan's cbytes, one mbarrier each (32
// arrivals: every lane's cp.async group), counters over the whole kernel.
struct RingState {
  uint8_t* ring;
  uint64_t* bars;
  int consumed, issued;
  bool ok;  // false once a wait has timed out; the warp then stops
};

// B-operand row of column col of a segment (the token's rotated activations
// in phase A -- per pair when the expert has its own signs --, the pair's
// rotated h in phase B), in the buffers seg_bsrc and seg_sums name.
template <int PHASE>
__device__ __forceinline__ size_t seg_brow(const Ws& w, const Dims& d, const SegInfo& sg, int col) {
  const int p = sg.off + col;
  if (PHASE != 0) return static_cast<size_t>(p);
  return sg.own ? static_cast<size_t>(w.sorted[p]) : static_cast<size_t>(sg.L) * d.T + w.sorted[p] / d.k;
}
template <int PHASE>
__device__ __forceinline__ const uint16_t* seg_bsrc(const Ws& w, const SegInfo& sg) {
  return PHASE == 0 ? (sg.own ? w.xpl : w.xl) : w.hl;
}
template <int PHASE>
__device__ __forceinline__ const float* seg_sums(const Ws& w, const SegInfo& sg) {
  return PHASE == 0 ? (sg.own ? w.xpsum : w.xsum) : w.hsum;
}

// Epilogue of one item: rows g, g+8 of the lane's fragments, columns 2t,
// 2t+1; o[0] and o[1] are gate and up (A) or the item's two 16-row halves (B).
template <int PHASE>
__device__ __forceinline__ void seg_store(const Ws& w, const Dims& d, const SegInfo& sg, int m0,
                                          const float4 (&o)[2], int lane) {
  const int g = lane >> 2, t = lane & 3;
  const int M = PHASE == 0 ? d.inter : d.hidden;
  const float* og = reinterpret_cast<const float*>(&o[0]);
  const float* ou = reinterpret_cast<const float*>(&o[1]);
#pragma unroll
  for (int q4 = 0; q4 < 4; ++q4) {
    const int col = 2 * t + (q4 & 1);
    const int m = m0 + g + 8 * (q4 >> 1);
    if (col < sg.ncol && m < M) {
      const size_t prow = static_cast<size_t>(sg.off + col);
      const float f = sg.fac[col];
      if (PHASE == 0) {
        const float gv = og[q4] * f, uv = ou[q4] * f;
        w.h[prow * d.inter + m] = gv / (1.f + expf(-gv)) * uv;
      } else {
        w.d[prow * d.hidden + m] = og[q4] * f;
        w.d[prow * d.hidden + m + kRows] = ou[q4] * f;  // M is a multiple of 32
      }
    }
  }
}

// Units [ua, ub) (pass-relative (item, group) units, all in segment k) of one
// warp: codes and scales stream through the warp's ring in chunks of up to
// len groups of one tile (never crossing an aligned run of 8 groups, whose
// scales are one 16-byte piece per row); B comes from the staged fragments
// (BSMEM) or from global memory one group ahead.  A tile the warp covers
// whole is stored here; a tile it covers in part (only at its range ends u0,
// u1) is kept in `part` (0: the tile holding u0, 1: the last) for the
// pass's reduction.
template <int PHASE, int LOGK, int BITS>
__device__ __forceinline__ void phase_piece(const SegInfo& sg, int k, int ua, int ub, const Ws& w,
                                            const Dims& d, RingState& rs,
                                            const float* zc, const uint4* xs, int cols,
                                            int u0, float4 (&part)[2][2],
                                            int (&ptile)[2], int lane) {
  constexpr int NMAT = 2;  // gate and up, or the two halves of a down tile
  constexpr int GB = 16 * BITS;  // code bytes of one row in one group
  const int g = lane >> 2, t = lane & 3;
  // the chunk and slot layout is fixed by K (this phase's input width)
  constexpr int K = 1 << LOGK;
  constexpr int G = K / kGroup;
  constexpr int lgG = LOGK - 7;
  constexpr PhaseSmem PS = phase_smem(G, NMAT);
  constexpr bool BSMEM = PS.bsmem != 0;
  constexpr int len_max = chunk_len(BITS, G, NMAT, PS.cbytes);
  static_assert(len_max > 0, "a one-group chunk fits a slot");
  constexpr int stride = chunk_stride(BITS, len_max);
  constexpr int row_bytes = K * BITS / 8;
  constexpr int sbytes = chunk_scale_bytes(G);
  const uint8_t* qbase[NMAT];
  const uint16_t* sbase[NMAT];
  if (PHASE == 0) {
    qbase[0] = reinterpret_cast<const uint8_t*>(sg.ed.q_gate);
    qbase[NMAT - 1] = reinterpret_cast<const uint8_t*>(sg.ed.q_up);
    sbase[0] = sg.ed.s_gate;
    sbase[NMAT - 1] = sg.ed.s_up;
  } else {
    qbase[0] = reinterpret_cast<const uint8_t*>(sg.ed.q_down);
    qbase[1] = qbase[0] + static_cast<size_t>(kRows) * row_bytes;
    sbase[0] = sg.ed.s_down;
    sbase[1] = sbase[0] + kRows * G;
  }
  auto chunk_of = [&](int u, int& j, int& g0, int& len) {
    const int r = u - sg.unit0;
    j = r >> lgG;
    g0 = r & (G - 1);
    len = min(min(len_max, G - g0), min(ub - u, 8 - (g0 & 7)));
  };
  // producer: the warp's lanes split each chunk's 16-byte pieces; every lane
  // arrives on the slot's barrier
  int pu = ua;
  // the lane's walk over a full-length chunk's 16-byte pieces (pr per row):
  // first piece (r0, c0), then steps of 32 pieces (dr rows + dc pieces)
  const int prf = len_max * BITS;
  const int r0f = lane / prf, c0f = lane - r0f * prf, drf = 32 / prf, dcf = 32 - drf * prf;
  auto issue = [&](int slot) {
    int j, g0, len;
    chunk_of(pu, j, g0, len);
    const int m0 = (sg.tile0 + j) * item_rows(PHASE);
    uint8_t* base = rs.ring + slot * PS.cbytes;
    int pr = prf, r0 = r0f, c0 = c0f, dr = drf, dc = dcf;
    if (len != len_max) {  // a shorter chunk (tile or range end)
      pr = len * BITS;
      r0 = lane / pr;
      c0 = lane - r0 * pr;
      dr = 32 / pr;
      dc = 32 - dr * pr;
    }
#pragma unroll
    for (int mi = 0; mi < NMAT; ++mi) {
      const uint8_t* src = qbase[mi] + static_cast<size_t>(m0) * row_bytes + g0 * GB;
      uint8_t* cdst = base + mi * kRows * stride;
      int r = r0, c = c0;
      for (int i = lane; i < kRows * pr; i += 32) {
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
        if (lane < kRows) cp_async16(sdst + lane * 16, sbase[mi] + static_cast<size_t>(m0 + lane) * G + (g0 & ~7), 16);
      } else if (lane < 2 * G) {
        cp_async16(sdst + lane * 16, reinterpret_cast<const uint8_t*>(sbase[mi] + static_cast<size_t>(m0) * G) + lane * 16, 16);
      }
    }
    cp_async_mbar_arrive(&rs.bars[slot]);
    pu += len;
    ++rs.issued;
  };
  if (!rs.ok) return;
  for (int k2 = 0; k2 < kRing && pu < ub; ++k2) issue(rs.issued % kRing);

  // consumer: this lane's B blocks (column g of the segment, k-quad t), or the zero block
  const bool has_b = g < sg.ncol;
  const uint4* zero_blk = reinterpret_cast<const uint4*>(zc + kMaxSeg * G * 8);
  const float* zck = zc + k * G * 8;
  const uint4* bl;
  int bstep;  // uint4 per group
  int bo[4];  // uint4 offset of piece i within a block
  if constexpr (BSMEM) {
    bl = has_b ? xs + ((sg.col0 + g) * 4 + t) * 4 : zero_blk;
    bstep = has_b ? cols * 16 : 0;
    const int sw = has_b ? bswz(sg.col0 + g, t) : 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) bo[i] = i ^ sw;
  } else {
    bl = has_b ? reinterpret_cast<const uint4*>(seg_bsrc<PHASE>(w, sg) + (seg_brow<PHASE>(w, d, sg, g) * G * 4 + t) * kXq)
               : zero_blk;
    bstep = has_b ? 4 * kXq / 8 : 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) bo[i] = i;
  }
  float acc[NMAT][4] = {};
  int tile_g0 = -1;  // first group of the current tile this warp computes
  uint4 bq[4];
  for (int u = ua; u < ub;) {
    int j, g0, len;
    chunk_of(u, j, g0, len);
    if (tile_g0 < 0) {
      tile_g0 = g0;
      if constexpr (!BSMEM) {
#pragma unroll
        for (int i = 0; i < 4; ++i) bq[i] = bl[g0 * bstep + bo[i]];
      }
    }
    const int slot = rs.consumed % kRing;
    if (!mbar_wait(&rs.bars[slot], (rs.consumed / kRing) & 1)) {
      rs.ok = false;
      return;
    }
    __syncwarp();
    const uint8_t* base = rs.ring + slot * PS.cbytes;
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
      const float2 z = *reinterpret_cast<const float2*>(zck + gi * 8 + 2 * t);
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
    if (pu < ub) issue(slot);
    ++rs.consumed;
    u += len;
    if (g0 + len == G || u == ub) {
      // this warp's part of tile j is done
      float4 o[2];
#pragma unroll
      for (int mi = 0; mi < 2; ++mi) {
        const int mm = mi < NMAT ? mi : 0;
        o[mi] = make_float4(acc[mm][0], acc[mm][1], acc[mm][2], acc[mm][3]);
      }
      if (tile_g0 == 0 && g0 + len == G) {
        seg_store<PHASE>(w, d, sg, (sg.tile0 + j) * item_rows(PHASE), o, lane);
      } else {
        const int tf = sg.unit0 + (j << lgG);  // the tile's first unit
        if (tf <= u0 && u0 < tf + G) {  // the tile holding u0 (constant indices: registers)
          part[0][0] = o[0];
          part[0][1] = o[1];
          ptile[0] = sg.item0 + j;
        } else {
          part[1][0] = o[0];
          part[1][1] = o[1];
          ptile[1] = sg.item0 + j;
        }
      }
#pragma unroll
      for (int mi = 0; mi < NMAT; ++mi) acc[mi][0] = acc[mi][1] = acc[mi][2] = acc[mi][3] = 0.f;
      tile_g0 = -1;
    }
  }
}

// Phase A (PHASE 0): gate and up, SwiGLU -> h.  Phase B (PHASE 1): down -> d.
//
// Work item i is row tile i % TPB (item_rows) of block i / TPB, a block being one
// expert's <= 8-token column block (w.blk); CTA c owns items [bounds[c],
// bounds[c + 1]) (split by tile weight) and walks them in passes.  A pass
// takes up to kMaxSeg consecutive blocks' parts (segments) with at most 8
// columns in all; the CTA stages their zero-point terms and, when BSMEM,
// their B fragments (the rotated activations) in shared memory, then its 16
// warps split the pass's (item, group) units evenly, each streaming codes and
// scales through a private cp.async ring.  Tiles split between warps are
// summed in warp order through shared memory after one barrier.  Without
// BSMEM (K too large for the fragments beside the rings) lanes read their B
// blocks from global memory, one group ahead.
template <int PHASE, int LOGK>
__global__ void __launch_bounds__(kWarps * 32, 1)
    moe_phase_kernel(const hq_expert* __restrict__ ex, Ws w, Dims d) {
  constexpr int NMAT = 2;
  constexpr int G = (1 << LOGK) / kGroup;  // K = hidden (phase A) or inter (phase B)
  constexpr PhaseSmem ps = phase_smem(G, NMAT);
  constexpr bool BSMEM = ps.bsmem != 0;
  extern __shared__ __align__(128) uint8_t smem[];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int M = PHASE == 0 ? d.inter : d.hidden;
  const int TPB = M / item_rows(PHASE);  // items per block
  PassMeta& pm = *reinterpret_cast<PassMeta*>(smem);
  float* zc = reinterpret_cast<float*>(smem + ps.zc_off);  // [kMaxSeg][G][8], then a zero B block
  uint4* xs = reinterpret_cast<uint4*>(smem + ps.xs_off);  // [G][cols][4][4 pieces], swizzled
  uint8_t* ring = smem + ps.ring_off + warp * kRing * ps.cbytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + ps.bar_off) + warp * kRing;
  if (lane == 0) {
    for (int i = 0; i < kRing; ++i) mbar_init(&bars[i], 32);
    fence_mbar_init();
  }
  if (tid < 16) (zc + kMaxSeg * G * 8)[tid] = 0.f;
  __syncthreads();
  pdl_launch_dependents();
  pdl_wait();  // routing lists and activations come from the previous kernels
  const int* bounds = w.bounds + PHASE * (kMaxGrid + 1);
  const int ib = bounds[blockIdx.x], ie = bounds[blockIdx.x + 1];
  RingState rs{ring, bars, 0, 0, true};  // this warp's ring, over the whole kernel

  for (int it = ib; it < ie;) {
    __syncthreads();  // the previous pass is done with the metadata, B, zc and rings
    // ---- plan the pass (warp 0): lane k looks at block b0 + k
    if (warp == 0) {
      const int b = it / TPB + lane;
      const bool valid = lane < kMaxSeg && b * TPB < ie;
      int e = 0, cb = 0, ncol = 0, off = 0;
      if (valid) {
        const uint2 bk = w.blk[b];
        e = static_cast<int>(bk.x);
        cb = static_cast<int>(bk.y);
        off = w.offsets[e] + 8 * cb;
        ncol = min(8, w.counts[e] - 8 * cb);
      }
      const int item0 = max(it, b * TPB), item1 = min(ie, (b + 1) * TPB);
      const int ni = valid ? item1 - item0 : 0;
      const hq_expert ede = valid ? ex[e] : hq_expert{};
      const int wt = valid ? ni * G * tile_weight(PHASE, ede.bits) : 0;
      int pc = ncol, pn = ni, pw = wt;  // inclusive prefix sums of columns, items, weights
#pragma unroll
      for (int m = 1; m < 32; m <<= 1) {
        const int yc = __shfl_up_sync(0xffffffffu, pc, m);
        const int yn = __shfl_up_sync(0xffffffffu, pn, m);
        const int yw = __shfl_up_sync(0xffffffffu, pw, m);
        if (lane >= m) {
          pc += yc;
          pn += yn;
          pw += yw;
        }
      }
      const bool take = valid && (lane == 0 || pc <= 8);
      const int nseg = __popc(__ballot_sync(0xffffffffu, take));
      if (take) {
        SegInfo& sg = pm.seg[lane];
        sg.ed = ede;
        sg.wt0 = pw - wt;
        sg.item0 = item0;
        sg.item1 = item1;
        sg.tile0 = item0 - b * TPB;
        sg.unit0 = (pn - ni) * G;
        sg.off = off;
        sg.ncol = ncol;
        sg.col0 = pc - ncol;
        sg.L = layout_index(sg.ed.bits);
        sg.own = sg.ed.signs_in != nullptr ? 1 : 0;
      }
      if (lane == nseg - 1) {
        pm.nseg = nseg;
        pm.cols = pc;
        pm.units = pn * G;
        pm.wtot = pw;
      }
    }
    __syncthreads();
    const int nseg = pm.nseg, cols = pm.cols, U = pm.units;
    // ---- stage the pass's zero-point terms and (BSMEM) B fragments
    for (int k = 0; k < nseg; ++k) {
      const SegInfo& sg = pm.seg[k];
      if constexpr (BSMEM) {
        // 64 bytes of each 80-byte block (the rest is padding), 16-byte pieces
        const int per_col = G * 16;
        for (int i = tid; i < sg.ncol * per_col; i += kWarps * 32) {
          const int cl = i / per_col, r = i - cl * per_col;
          const int gg = r >> 4, q = (r >> 2) & 3, pc = r & 3;
          const int col = sg.col0 + cl;
          cp_async16(xs + ((gg * cols + col) * 4 + q) * 4 + (pc ^ bswz(col, q)),
                     seg_bsrc<PHASE>(w, sg) + ((seg_brow<PHASE>(w, d, sg, cl) * G + gg) * 4 + q) * kXq + pc * 8, 16);
        }
      }
      // output factors of the segment's columns (written before the barrier
      // below, read by the epilogue after it)
      if (tid < sg.ncol) {
        pm.seg[k].fac[tid] = PHASE == 0 ? (sg.own ? w.xpfac[w.sorted[sg.off + tid]] : w.xfac[w.sorted[sg.off + tid] / d.k])
                                        : w.hfac[sg.off + tid];
      }
      // -zero * sum_k x' * 2^-24 per group and column (0 for absent columns)
      const float zneg = -static_cast<float>(sg.ed.zero) * 5.9604644775390625e-8f;
      for (int i = tid; i < G * 8; i += kWarps * 32) {
        const int gg = i >> 3, cl = i & 7;
        zc[k * G * 8 + i] = cl < sg.ncol ? zneg * seg_sums<PHASE>(w, sg)[seg_brow<PHASE>(w, d, sg, cl) * G + gg] : 0.f;
      }
    }
    if constexpr (BSMEM) asm volatile("cp.async.wait_all;" ::: "memory");
    __syncthreads();

    // ---- this warp's units [u0, u1) of the pass (equal shares of the
    // weight: unit u of segment k weighs its tile weight), one piece per segment
    auto unit_at = [&](int wi) {  // first unit whose weight prefix reaches wi / kWarps of the total
      const int target = static_cast<int>((static_cast<long long>(pm.wtot) * wi) / kWarps);
      int k = 0;
      while (k + 1 < nseg && pm.seg[k + 1].wt0 <= target) ++k;
      const SegInfo& sg = pm.seg[k];
      const int tw = tile_weight(PHASE, sg.ed.bits);
      const int u = sg.unit0 + (target - sg.wt0 + tw - 1) / tw;
      return min(u, sg.unit0 + (sg.item1 - sg.item0) * G);
    };
    const int u0 = warp == 0 ? 0 : unit_at(warp);
    const int u1 = warp == kWarps - 1 ? U : unit_at(warp + 1);
    float4 part[2][2];
    int ptile[2] = {-1, -1};
    for (int k = 0; k < nseg && rs.ok; ++k) {
      const SegInfo& sg = pm.seg[k];
      const int sa = max(u0, sg.unit0), sb = min(u1, sg.unit0 + (sg.item1 - sg.item0) * G);
      if (sa >= sb) continue;
      switch (sg.ed.bits) {
        case 2: phase_piece<PHASE, LOGK, 2>(sg, k, sa, sb, w, d, rs, zc, xs, cols, u0, part, ptile, lane); break;
        case 3: phase_piece<PHASE, LOGK, 3>(sg, k, sa, sb, w, d, rs, zc, xs, cols, u0, part, ptile, lane); break;
        case 4: phase_piece<PHASE, LOGK, 4>(sg, k, sa, sb, w, d, rs, zc, xs, cols, u0, part, ptile, lane); break;
        default: phase_piece<PHASE, LOGK, 8>(sg, k, sa, sb, w, d, rs, zc, xs, cols, u0, part, ptile, lane); break;
      }
    }
    // ---- tiles split between warps: each warp leaves its partial sums in
    // its (drained) ring; the warp whose range holds a tile's first unit adds
    // the later contributors' parts in warp order and runs the epilogue
    float4* mine = reinterpret_cast<float4*>(ring);  // [2 which][2 mat][32 lanes]
    if (rs.ok) {
#pragma unroll
      for (int wh = 0; wh < 2; ++wh) {
#pragma unroll
        for (int mi = 0; mi < NMAT; ++mi) mine[(wh * 2 + mi) * 32 + lane] = part[wh][mi];
      }
    }
    __syncthreads();
    if (rs.ok) {
#pragma unroll
      for (int wh = 0; wh < 2; ++wh) {
        const int item = ptile[wh];
        if (item < 0 || (wh == 1 && item == ptile[0])) continue;
        int k = 0;
        while (k + 1 < nseg && item >= pm.seg[k].item1) ++k;
        const SegInfo& sg = pm.seg[k];
        const int tf = sg.unit0 + (item - sg.item0) * G, tz = tf + G - 1;
        if (tf < u0) continue;  // an earlier warp holds the tile's first unit
        float4 o[2] = {part[wh][0], part[wh][1]};
        for (int w2 = warp + 1; w2 < kWarps; ++w2) {
          const int wb = unit_at(w2);
          if (wb > tz) break;
          if (wb == (w2 == kWarps - 1 ? U : unit_at(w2 + 1))) continue;  // empty range
          const float4* other = reinterpret_cast<const float4*>(smem + ps.ring_off + w2 * kRing * ps.cbytes);
#pragma unroll
          for (int mi = 0; mi < NMAT; ++mi) {
            const float4 q4 = other[(0 * 2 + mi) * 32 + lane];  // the tile is that warp's first
            o[mi].x += q4.x;
            o[mi].y += q4.y;
            o[mi].z += q4.z;
            o[mi].w += q4.w;
          }
        }
        seg_store<PHASE>(w, d, sg, (sg.tile0 + item - sg.item0) * item_rows(PHASE), o, lane);
      }
    }
    it += U / G;
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
  const size_t route_smem = (3 * static_cast<size_t>(d.E) + 3) * sizeof(int);
#define HQ_FRONT(LK)                                                                          \
  case (1 << LK):                                                                             \
    return launch_pdl(moe::moe_front_kernel<LK>, dim3(d.T + 1), dim3(FwhtShape<LK>::THREADS),   \
                      std::max((FwhtShape<LK>::SMEM_FLOATS + 32) * sizeof(float), route_smem), st, true, \
                      ex, ids, x, s, w, d, inv);
  switch (hidden) {
    HQ_FRONT(7) HQ_FRONT(8) HQ_FRONT(9) HQ_FRONT(10) HQ_FRONT(11) HQ_FRONT(12) HQ_FRONT(13)
    HQ_FRONT(14) HQ_FRONT(15)
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
                      (FwhtShape<LK>::SMEM_FLOATS + 32) * sizeof(float), st, true, ex, ids, s, w, d, inv);
  switch (inter) {
    HQ_ROTH(7) HQ_ROTH(8) HQ_ROTH(9) HQ_ROTH(10) HQ_ROTH(11) HQ_ROTH(12) HQ_ROTH(13) HQ_ROTH(14)
    HQ_ROTH(15)
    default: return cudaErrorInvalidValue;
  }
#undef HQ_ROTH
}

template <int PHASE>
static cudaError_t moe_launch_phase(const hq_expert* ex, const moe::Ws& w, const moe::Dims& d,
                                    cudaStream_t st) {
  constexpr int nmat = 2;
  const int K = PHASE == 0 ? d.hidden : d.inter;
  const moe::PhaseSmem ps = moe::phase_smem(K / kGroup, nmat);
  for (int b : {2, 3, 4, 8}) {
    if (moe::chunk_len(b, K / kGroup, nmat, ps.cbytes) == 0) return cudaErrorInvalidConfiguration;
  }
  if (ps.total > moe::kSmemMax) return cudaErrorInvalidConfiguration;
  const dim3 grid(d.grid), block(moe::kWarps * 32);  // one CTA per SM; the routing CTA split
                                                     // the work for exactly d.grid CTAs
#define HQ_PHASE(LK) \
  case (1 << LK): \
    return launch_pdl(moe::moe_phase_kernel<PHASE, LK>, grid, block, ps.total, st, true, ex, w, d);
  switch (K) {
    HQ_PHASE(7) HQ_PHASE(8) HQ_PHASE(9) HQ_PHASE(10) HQ_PHASE(11) HQ_PHASE(12) HQ_PHASE(13)
    HQ_PHASE(14) HQ_PHASE(15)
    default: return cudaErrorInvalidValue;
  }
#undef HQ_PHASE
}

}  // namespace hq

using namespace hq;

// The routing CTA keeps three ints per expert in shared memory.
constexpr int kMaxExperts = 16384;

extern "C" {

size_t hq_moe_workspace_size(int n_experts, int hidden, int inter, int T, int k) {
  auto pow2 = [](int v) { return v > 0 && (v & (v - 1)) == 0; };
  if (n_experts < 1 || n_experts > kMaxExperts || T < 0 || k < 1 || k > 32 || !pow2(hidden) ||
      !pow2(inter) || hidden < 128 || inter < 128 || hidden > 32768 || inter > 32768 ||
      static_cast<long>(T) * k > (1L << 24)) {
    return 0;
  }
  return moe_plan(n_experts, hidden, inter, T, k).bytes;
}

int hq_moe_launches(void) { return 5; }

size_t hq_moe_workspace_offset(int n_experts, int hidden, int inter, int T, int k,
                               hq_moe_part part) {
  if (hq_moe_workspace_size(n_experts, hidden, inter, T, k) == 0) return static_cast<size_t>(-1);
  const MoePlan pl = moe_plan(n_experts, hidden, inter, T, k);
  switch (part) {
    case HQ_MOE_POS: return pl.off[3];
    case HQ_MOE_H: return pl.off[10];
    case HQ_MOE_D: return pl.off[13];
  }
  return static_cast<size_t>(-1);
}

hq_status hq_moe_experts(const hq_expert* experts, int n_experts, int hidden, int inter,
                         const uint16_t* x, int T, const int32_t* topk_ids, const float* topk_w,
                         int k, const int8_t* signs_in, const int8_t* signs_mid, float* y,
                         void* workspace, size_t ws_bytes, hq_stream_t stream) {
  auto pow2 = [](int v) { return v > 0 && (v & (v - 1)) == 0; };
  auto al = [](const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; };
  if (n_experts < 1 || T < 0 || k < 1 || k > 32 || hidden <= 0 || inter <= 0) {
    return HQ_ERR_INVALID_ARG;
  }
  if (!pow2(hidden) || !pow2(inter) || hidden < 128 || inter < 128 || hidden > 32768 ||
      inter > 32768 || n_experts > kMaxExperts) {
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
