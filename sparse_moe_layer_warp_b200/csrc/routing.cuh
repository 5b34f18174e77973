// routing.cuh -- router logits, bias-adjusted top-k with renormalised gates, and the
// deterministic expert-sorted permutation.
//
// Follows "Step 3.5 Flash: Open Frontier-Level Intelligence with 11B Active Parameters",
// section 2.2.2 (S_t = top-K experts of token t, routing probabilities p_{t,e}) and the
// note under the parameter table of "Step 3.5 Flash 技术论文深度解读" (architecture item 1:
// loss-free balancing by a bias that only adjusts the selection), and section 3.2.4 of the
// first page (fused MoE gather/scatter: tokens grouped by expert before the grouped GEMM).
#pragma once
#include <cuda_bf16.h>
#include <stdint.h>

#include "ptx_sm100.cuh"

namespace moe {

// Work counters of the expert kernels that follow a routing launch, zeroed by that launch
// (block 0) so every forward starts from zero: the grouped GEMMs' unit and row-gather
// counters (DevStatus::sched) and the per-group completion counts of the h hand-over.
struct CounterReset {
  int *sched;  // [8] or null
  int *done;   // [n_done] or null
  int n_done;
  __device__ __forceinline__ void apply() const {
    if (blockIdx.x == 0) run();
  }
  __device__ __forceinline__ void run() const {  // by the whole of one CTA
    if (sched && threadIdx.x < 8) sched[threadIdx.x] = 0;
    if (done)
      for (int i = threadIdx.x; i < n_done; i += blockDim.x) done[i] = 0;
  }
};

constexpr int kMaxExperts = 1024;   // E limit of the routing kernels
constexpr int kMaxTopK = 32;        // one slot per lane
constexpr int kChunk = 64;          // tokens per routing chunk (one CTA)
constexpr int kRouteWarps = 16;    // top-k: one warp per token, 4 tokens per warp at most
constexpr int kSplitKTokens = 64;   // largest T of the split-K router
constexpr int kSplitKSlice = 256;   // d elements per split (32 lanes x 8)

__device__ __forceinline__ float to_f32(float v) { return v; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 v) { return __bfloat162float(v); }

// 16-byte vector of inputs -> floats.
template <typename Tin>
struct Vec16;
template <>
struct Vec16<__nv_bfloat16> {
  static constexpr int N = 8;
  __device__ __forceinline__ static void load(const __nv_bfloat16 *p, float (&o)[8]) {
    uint4 u = __ldg(reinterpret_cast<const uint4 *>(p));
    const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float2 f = __bfloat1622float2(h[i]);
      o[2 * i] = f.x;
      o[2 * i + 1] = f.y;
    }
  }
};
template <>
struct Vec16<float> {
  static constexpr int N = 4;
  __device__ __forceinline__ static void load(const float *p, float (&o)[4]) {
    float4 u = __ldg(reinterpret_cast<const float4 *>(p));
    o[0] = u.x;
    o[1] = u.y;
    o[2] = u.z;
    o[3] = u.w;
  }
};

// ------------------------------------------------------------------ router logits (small T)
// Split-K over d: CTA (b, s) computes, for experts [32b, 32b + 32) and every token, the dot
// product over d-slice s (kSplitKSlice elements: 8 per lane, 16-byte loads) and writes it to
// part[s][t][e].  The last CTA of block b to finish (ticket counter) adds the splits in
// increasing s and writes logits[t][e]; the order of the sum never depends on which CTA is
// last, so the logits are deterministic.  No CTA waits for another.  Decode streams the
// E x d router matrix from HBM across ~E/32 x d/256 CTAs instead of a handful.
template <typename Tin>
__global__ void __launch_bounds__(256) router_logits_splitk_kernel(
    const Tin *__restrict__ x, const Tin *__restrict__ wr, int T, int d, int E,
    float *__restrict__ part, float *__restrict__ logits, int *__restrict__ tickets) {
  griddep_launch_dependents();
  constexpr int V = Vec16<Tin>::N;      // elements per 16-byte load
  constexpr int PER_LANE = 8;           // elements per lane per split
  constexpr int TG = 16;                // tokens per register group
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int e0 = blockIdx.x * 32 + warp * 4;
  const int s = blockIdx.y;
  const int S = gridDim.y;
  const int k0 = s * kSplitKSlice + lane * PER_LANE;
  const bool kin = k0 < d;
  float w[4][PER_LANE];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int e = e0 + i;
#pragma unroll
    for (int v0 = 0; v0 < PER_LANE; v0 += V) {
      float tmp[V];
      if (kin && e < E) Vec16<Tin>::load(wr + (size_t)e * d + k0 + v0, tmp);
      else
#pragma unroll
        for (int v = 0; v < V; ++v) tmp[v] = 0.f;
#pragma unroll
      for (int v = 0; v < V; ++v) w[i][v0 + v] = tmp[v];
    }
  }
  // the router weights above never depend on earlier kernels; x and the workspace do
  griddep_wait();
  for (int tg = 0; tg < T; tg += TG) {
    float acc[4][TG];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int t = 0; t < TG; ++t) acc[i][t] = 0.f;
#pragma unroll
    for (int t = 0; t < TG; ++t) {
      if (tg + t < T && kin) {
#pragma unroll
        for (int v0 = 0; v0 < PER_LANE; v0 += V) {
          float xv[V];
          Vec16<Tin>::load(x + (size_t)(tg + t) * d + k0 + v0, xv);
#pragma unroll
          for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int v = 0; v < V; ++v) acc[i][t] = fmaf(xv[v], w[i][v0 + v], acc[i][t]);
        }
      }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int t = 0; t < TG; ++t) {
        float v = acc[i][t];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        acc[i][t] = v;
      }
    // spread the 64 results of the warp over its lanes for the stores
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int t = 0; t < TG; ++t) {
        const int e = e0 + i;
        if (lane == ((i * TG + t) & 31) && tg + t < T && e < E)
          part[((size_t)s * T + tg + t) * E + e] = acc[i][t];
      }
  }
  // last arriver of this expert block reduces the splits in order
  __shared__ int s_last;
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) s_last = (atomicAdd(&tickets[blockIdx.x], 1) == S - 1);
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  const int eb = blockIdx.x * 32;
  const int ne = min(32, E - eb);
  for (int i = threadIdx.x; i < T * 32; i += blockDim.x) {
    const int t = i >> 5, e = eb + (i & 31);
    if ((i & 31) >= ne) continue;
    float acc = 0.f;
    for (int sp = 0; sp < S; ++sp) acc += __ldcg(part + ((size_t)sp * T + t) * E + e);
    logits[(size_t)t * E + e] = acc;
  }
  if (threadIdx.x == 0) tickets[blockIdx.x] = 0;  // ready for the next call
}

// ------------------------------------------------------------------ router logits (tiled)
// 64 tokens x 64 experts per CTA, K in steps of 32, 4 x 4 outputs per thread, fp32 FMA.
template <typename Tin>
__global__ void __launch_bounds__(256) router_logits_tiled_kernel(const Tin *__restrict__ x,
                                                                  const Tin *__restrict__ wr,
                                                                  int T, int d, int E,
                                                                  float *__restrict__ logits) {
  griddep_wait();
  griddep_launch_dependents();
  constexpr int BT = 64, BE = 64, BK = 32;
  __shared__ float xs[BK][BT + 4];
  __shared__ float ws[BK][BE + 4];
  const int t0 = blockIdx.x * BT, e0 = blockIdx.y * BE;
  const int tid = threadIdx.x;
  const int tr = (tid / 16) * 4, ec = (tid % 16) * 4;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < d; k0 += BK) {
    // 64 rows x 32 k for each operand: 2048 elements, 8 per thread
    for (int i = tid; i < BT * BK; i += 256) {
      const int row = i / BK, kk = i % BK;
      const int t = t0 + row, e = e0 + row;
      xs[kk][row] = (t < T && k0 + kk < d) ? to_f32(x[(size_t)t * d + k0 + kk]) : 0.f;
      ws[kk][row] = (e < E && k0 + kk < d) ? to_f32(wr[(size_t)e * d + k0 + kk]) : 0.f;
    }
    __syncthreads();
#pragma unroll 8
    for (int kk = 0; kk < BK; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        a[i] = xs[kk][tr + i];
        b[i] = ws[kk][ec + i];
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int t = t0 + tr + i, e = e0 + ec + j;
      if (t < T && e < E) logits[(size_t)t * E + e] = acc[i][j];
    }
}

// ------------------------------------------------------------------ top-k + chunk histogram
// Ranking: a before b iff a's fp32 score is larger, or equal with the lower expert id;
// -0.0 == +0.0; NaN below every number.  score_key maps a score to an unsigned integer with
// the same order (NaN -> 0, every number >= 0x007FFFFF), so the warp can pick the winner
// with two single-instruction reductions: the largest key, then the lowest id holding it.
__device__ __forceinline__ uint32_t score_key(float s) {
  if (s != s) return 0u;
  const uint32_t b = __float_as_uint(s == 0.f ? 0.f : s);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

// One warp per token; CTA c handles tokens [c*kChunk, (c+1)*kChunk).  Lane l holds the
// scores of experts l, l+32, ...  k rounds of warp arg-max pick S_t in rank order; lane j
// keeps slot j.  Gates: softmax over the selected UNBIASED logits (max-shifted, expf).
// The CTA's per-expert selection counts go to chunk_hist[c][e] (integer, order-free).
// logits_out (optional) receives a copy of the logits read.
// Selection and gates of token t by one warp.  Returns, in lane j < k, slot j's expert id
// and gate; other lanes return (0, 0).  logits_out (optional) receives a copy of the row.
template <int MAXV>
__device__ __forceinline__ void topk_token(const float *__restrict__ lrow,
                                           const float *__restrict__ bias, int E, int k,
                                           float *__restrict__ lout, int lane, int &my_e,
                                           float &my_gate) {
  uint32_t key[MAXV];
  float l[MAXV], b[MAXV];
  // all loads first (clamped addresses, no branches), so they are in flight together;
  // L2-coherent logits loads: they may be this kernel's own output
#pragma unroll
  for (int v = 0; v < MAXV; ++v) {
    const int e = min(lane + 32 * v, E - 1);
    l[v] = __ldcg(lrow + e);
    b[v] = bias ? __ldg(bias + e) : 0.f;
  }
#pragma unroll
  for (int v = 0; v < MAXV; ++v) {
    const int e = lane + 32 * v;
    if (e < E) {
      if (lout) lout[e] = l[v];
      key[v] = score_key(l[v] + b[v]);
    } else {
      l[v] = 0.f;
      key[v] = 0u;  // ties with NaN scores and loses on id (all ids here are >= E)
    }
  }
  my_e = 0;
  float my_l = 0.f;
  uint32_t used = 0;
  for (int r = 0; r < k; ++r) {
    // lane-local best among unused entries; ids grow with v, so '>' keeps the lower id
    uint32_t bk = 0;
    int bv = -1;
    float bl = 0.f;
#pragma unroll
    for (int v = 0; v < MAXV; ++v) {
      const bool ok = !((used >> v) & 1u);
      if (ok && (bv < 0 || key[v] > bk)) {
        bk = key[v];
        bv = v;
        bl = l[v];
      }
    }
    const uint32_t wkey = __reduce_max_sync(0xffffffffu, bk);
    const uint32_t cand = (bv >= 0 && bk == wkey) ? (uint32_t)(lane + 32 * bv) : 0xffffffffu;
    const uint32_t wid = __reduce_min_sync(0xffffffffu, cand);
    const int owner = (int)(wid & 31u);
    if (owner == lane) used |= 1u << (wid >> 5);
    const float wl = __shfl_sync(0xffffffffu, bl, owner);
    if (lane == r) {
      my_e = (int)wid;
      my_l = wl;
    }
  }
  // gates over lanes 0..k-1: softmax of the selected unbiased logits
  float m = (lane < k) ? my_l : -INFINITY;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  const float ex = (lane < k) ? expf(my_l - m) : 0.f;
  float z = ex;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
  my_gate = (lane < k) ? ex / z : 0.f;
  if (lane >= k) my_e = 0;
}

// Exclusive scan of cnt[0..E) into off[0..E) by the whole CTA (each thread a contiguous
// run, warp and block scans of the run totals).  Contains __syncthreads.
__device__ __forceinline__ void block_exclusive_scan(const int *cnt, int *off, int E,
                                                     int *warp_sum) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int per = (E + blockDim.x - 1) / blockDim.x;
  const int lo = min(E, tid * per), hi = min(E, lo + per);
  int run = 0;
  for (int e = lo; e < hi; ++e) run += cnt[e];
  int incl = run;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) warp_sum[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const int nw = blockDim.x >> 5;
    int v = (lane < nw) ? warp_sum[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, v, o);
      if (lane >= o) v += y;
    }
    if (lane < nw) warp_sum[lane] = v;  // inclusive warp totals
  }
  __syncthreads();
  int excl = incl - run + (warp > 0 ? warp_sum[warp - 1] : 0);
  for (int e = lo; e < hi; ++e) {
    off[e] = excl;
    excl += cnt[e];
  }
  __syncthreads();
}

// One warp per token; CTA c handles tokens [c*kChunk, (c+1)*kChunk).  Lane l holds the
// scores of experts l, l+32, ...  k rounds of warp arg-max pick S_t in rank order; lane j
// keeps slot j.  The CTA's per-expert selection counts go to chunk_hist[c][e] (integer,
// order-free).
template <int MAXV>
__global__ void __launch_bounds__(kRouteWarps * 32) topk_hist_kernel(
    const float *__restrict__ logits, const float *__restrict__ bias, int T, int E, int k,
    float *__restrict__ logits_out, int *__restrict__ topk_idx, float *__restrict__ topk_gate,
    int *__restrict__ chunk_hist) {
  griddep_wait();
  griddep_launch_dependents();
  __shared__ int hist[kMaxExperts];
  const int c = blockIdx.x;
  for (int e = threadIdx.x; e < E; e += blockDim.x) hist[e] = 0;
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tbeg = c * kChunk, tend = min(T, tbeg + kChunk);
  for (int t = tbeg + warp; t < tend; t += kRouteWarps) {
    int my_e;
    float my_gate;
    topk_token<MAXV>(logits + (size_t)t * E, bias, E, k,
                     logits_out ? logits_out + (size_t)t * E : nullptr, lane, my_e, my_gate);
    if (lane < k) {
      topk_idx[(size_t)t * k + lane] = my_e;
      topk_gate[(size_t)t * k + lane] = my_gate;
      atomicAdd(&hist[my_e], 1);
    }
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) chunk_hist[(size_t)c * E + e] = hist[e];
}

// ------------------------------------------------------------------ small-T fused routing
// T <= kChunk (decode): selection, gates, histogram, scan and permutation of all T tokens by
// one CTA (any multiple of 32 threads; one warp per token).
template <int MAXV>
__device__ __forceinline__ void route_small_block(
    const float *__restrict__ logits, const float *__restrict__ bias, int T, int E, int k,
    float *__restrict__ logits_out, int *__restrict__ topk_idx, float *__restrict__ topk_gate,
    int *__restrict__ counts, int *__restrict__ offsets, int *__restrict__ perm,
    int *__restrict__ slot_row) {
  __shared__ int hist[kMaxExperts];
  __shared__ int off[kMaxExperts];
  __shared__ uint32_t bits[kMaxExperts][kChunk / 32];
  __shared__ int s_idx[kChunk * kMaxTopK];
  __shared__ int warp_sum[32];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_warps = blockDim.x >> 5;
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    hist[e] = 0;
#pragma unroll
    for (int w = 0; w < kChunk / 32; ++w) bits[e][w] = 0u;
  }
  __syncthreads();
  for (int t = warp; t < T; t += n_warps) {
    int my_e;
    float my_gate;
    topk_token<MAXV>(logits + (size_t)t * E, bias, E, k,
                     logits_out ? logits_out + (size_t)t * E : nullptr, lane, my_e, my_gate);
    if (lane < k) {
      s_idx[t * k + lane] = my_e;
      atomicAdd(&hist[my_e], 1);
      atomicOr(&bits[my_e][t >> 5], 1u << (t & 31));
      topk_idx[(size_t)t * k + lane] = my_e;
      topk_gate[(size_t)t * k + lane] = my_gate;
    }
  }
  __syncthreads();
  block_exclusive_scan(hist, off, E, warp_sum);
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    counts[e] = hist[e];
    offsets[e] = off[e];
  }
  if (threadIdx.x == 0) offsets[E] = T * k;
  const int npair = T * k;
  for (int q = threadIdx.x; q < npair; q += blockDim.x) {
    const int t = q / k;
    const int e = s_idx[q];
    int rank = 0;
#pragma unroll
    for (int w = 0; w < kChunk / 32; ++w) {
      const uint32_t word = bits[e][w];
      if (w < (t >> 5)) rank += __popc(word);
      else if (w == (t >> 5)) rank += __popc(word & ((1u << (t & 31)) - 1u));
    }
    const int p = off[e] + rank;
    perm[p] = q;
    slot_row[q] = p;
  }
}

template <int MAXV>
__global__ void __launch_bounds__(kRouteWarps * 32) route_small_kernel(
    const float *__restrict__ logits, const float *__restrict__ bias, int T, int E, int k,
    float *__restrict__ logits_out, int *__restrict__ topk_idx, float *__restrict__ topk_gate,
    int *__restrict__ counts, int *__restrict__ offsets, int *__restrict__ perm,
    int *__restrict__ slot_row, CounterReset reset) {
  griddep_wait();
  griddep_launch_dependents();
  reset.apply();
  route_small_block<MAXV>(logits, bias, T, E, k, logits_out, topk_idx, topk_gate, counts,
                          offsets, perm, slot_row);
}

// ------------------------------------------------------------ decode: router + routing
// T <= kChunk tokens, bf16, E <= kDecodeMaxExperts, d a multiple of 128 and at most
// kDecodeMaxD: the router logits and the routing in ONE launch.  CTA c (kDecodeWarps warps)
// computes experts e0 = kDecodeEPC*c .. +kDecodeEPC over the full reduction: warp w takes
// the K slice [w*d/16, (w+1)*d/16), each lane 16-byte chunks of it (the CTA's router rows are loaded
// before the grid-dependency wait: they never depend on earlier kernels); per group of 16
// tokens the 32 (expert, token) partial sums of a lane are summed across the warp by a
// butterfly that leaves sum j in lane j (31 shuffles), then across the warps in a fixed
// order -- fp32 throughout, deterministic.  The CTA that finishes last (a ticket, reset by
// that CTA) then runs route_small_block on all logits, one token per warp.
constexpr int kDecodeEPC = 2;          // experts per CTA
constexpr int kDecodeMaxExperts = 288; // MAXV = 9 top-k and at most 144 CTAs
constexpr int kDecodeMaxD = 8192;      // at most 2 chunks of 8 per lane
constexpr int kDecodeWarps = 16;

__device__ __forceinline__ float dot8_bf16(const uint4 a, const uint4 b) {
  const __nv_bfloat162 *pa = reinterpret_cast<const __nv_bfloat162 *>(&a);
  const __nv_bfloat162 *pb = reinterpret_cast<const __nv_bfloat162 *>(&b);
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 fa = __bfloat1622float2(pa[i]);
    const float2 fb = __bfloat1622float2(pb[i]);
    s = fmaf(fa.x, fb.x, s);
    s = fmaf(fa.y, fb.y, s);
  }
  return s;
}

__global__ void __launch_bounds__(kDecodeWarps * 32) route_decode_kernel(
    const __nv_bfloat16 *__restrict__ x, const __nv_bfloat16 *__restrict__ wr,
    const float *__restrict__ bias, int T, int d, int E, int k, float *__restrict__ logits,
    int *__restrict__ topk_idx, float *__restrict__ topk_gate, int *__restrict__ counts,
    int *__restrict__ offsets, int *__restrict__ perm, int *__restrict__ slot_row,
    int *__restrict__ ticket, CounterReset reset) {
  constexpr int EPC = kDecodeEPC, TG = 16, NW = kDecodeWarps;
  constexpr int MAXC = kDecodeMaxD / (NW * 8) / 32;
  static_assert(EPC * TG == 32, "one butterfly value per lane");
  __shared__ float red[NW][32];
  __shared__ int s_last;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int e0 = blockIdx.x * EPC;
  const int slice = d / NW;        // this warp's K range
  const int chunks = slice / 8;    // 16-byte chunks in it
  uint4 w[MAXC][EPC];
#pragma unroll
  for (int ci = 0; ci < MAXC; ++ci) {
    const int c = lane + 32 * ci;
#pragma unroll
    for (int e = 0; e < EPC; ++e) {
      w[ci][e] = make_uint4(0u, 0u, 0u, 0u);
      if (c < chunks && e0 + e < E)
        w[ci][e] = __ldg(reinterpret_cast<const uint4 *>(wr + (size_t)(e0 + e) * d +
                                                         warp * slice + c * 8));
    }
  }
  griddep_wait();
  griddep_launch_dependents();
  for (int tg = 0; tg < T; tg += TG) {
    float a[EPC * TG];  // value j = e * TG + t
#pragma unroll
    for (int j = 0; j < EPC * TG; ++j) a[j] = 0.f;
    // tokens past T read token T-1 (clamped, so the loads are unconditional and issue
    // together); their sums are never stored
#pragma unroll
    for (int ci = 0; ci < MAXC; ++ci) {
      const int c = lane + 32 * ci;
      if (ci * 32 < chunks) {  // warp-uniform
        const int cc = min(c, chunks - 1);
#pragma unroll
        for (int t0 = 0; t0 < TG; t0 += 8) {
          uint4 xv[8];
#pragma unroll
          for (int t = 0; t < 8; ++t)
            xv[t] = __ldg(reinterpret_cast<const uint4 *>(
                x + (size_t)min(tg + t0 + t, T - 1) * d + warp * slice + cc * 8));
          if (c < chunks) {
#pragma unroll
            for (int t = 0; t < 8; ++t)
#pragma unroll
              for (int e = 0; e < EPC; ++e) a[e * TG + t0 + t] += dot8_bf16(xv[t], w[ci][e]);
          }
        }
      }
    }
    // butterfly: after the step with offset o a lane keeps the half of its 2o values whose
    // index bit matches its lane bit, so lane j ends with the warp's sum of value j
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) {
      const bool upper = (lane & o) != 0;
#pragma unroll
      for (int i = 0; i < o; ++i) {
        const float send = upper ? a[i] : a[i + o];
        const float keep = upper ? a[i + o] : a[i];
        a[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
      }
    }
    red[warp][lane] = a[0];
    __syncthreads();
    if (threadIdx.x < 32) {
      float v = 0.f;
#pragma unroll
      for (int ww = 0; ww < NW; ++ww) v += red[ww][threadIdx.x];
      const int e = threadIdx.x / TG, t = threadIdx.x % TG;
      if (tg + t < T && e0 + e < E) logits[(size_t)(tg + t) * E + e0 + e] = v;
    }
    __syncthreads();
  }
  // the last CTA to finish its experts routes all tokens
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) {
    const int v = atomicAdd(ticket, 1);
    s_last = (v == (int)gridDim.x - 1);
    if (s_last) *ticket = 0;  // ready for the next call
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  reset.run();
  route_small_block<9>(logits, bias, T, E, k, nullptr, topk_idx, topk_gate, counts, offsets,
                       perm, slot_row);
}

// ------------------------------------------------------------------ permutation (scatter)
// CTA c: totals and this chunk's prefix over the chunk histograms, exclusive scan over
// experts -> offsets, then each (t, j) of the chunk gets position
//   offsets[e] + (tokens of earlier chunks that chose e) + (earlier tokens of this chunk
//   that chose e)
// where the last term is a popcount over a per-expert token bitmap.  No atomics decide
// any position, so perm and slot_row are deterministic (ascending t within an expert).
__global__ void __launch_bounds__(256) permute_scatter_kernel(
    const int *__restrict__ topk_idx, const int *__restrict__ chunk_hist, int T, int E, int k,
    int n_chunks, int *__restrict__ counts, int *__restrict__ offsets, int *__restrict__ perm,
    int *__restrict__ slot_row, CounterReset reset) {
  griddep_wait();
  griddep_launch_dependents();
  reset.apply();
  __shared__ int s_tot[kMaxExperts];
  __shared__ int s_base[kMaxExperts];
  __shared__ uint32_t bits[kMaxExperts][kChunk / 32];
  __shared__ int warp_sum[32];
  const int c = blockIdx.x;
  const int tid = threadIdx.x;
  for (int e = tid; e < E; e += blockDim.x) {
    int tot = 0, pre = 0;
    // 16 chunk counts loaded before they are summed: independent L2 loads in flight
    for (int cc0 = 0; cc0 < n_chunks; cc0 += 16) {
      int v[16];
#pragma unroll
      for (int u = 0; u < 16; ++u)
        v[u] = (cc0 + u < n_chunks) ? chunk_hist[(size_t)(cc0 + u) * E + e] : 0;
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        tot += v[u];
        pre += (cc0 + u < c) ? v[u] : 0;
      }
    }
    s_tot[e] = tot;
    s_base[e] = pre;
#pragma unroll
    for (int w = 0; w < kChunk / 32; ++w) bits[e][w] = 0u;
  }
  __syncthreads();
  // exclusive scan of s_tot over experts: each thread owns a contiguous run
  {
    const int per = (E + blockDim.x - 1) / blockDim.x;
    const int lo = min(E, tid * per), hi = min(E, lo + per);
    int run = 0;
    for (int e = lo; e < hi; ++e) run += s_tot[e];
    // block exclusive scan of `run`
    const int lane = tid & 31, warp = tid >> 5;
    int incl = run;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    if (lane == 31) warp_sum[warp] = incl;
    __syncthreads();
    if (warp == 0) {
      const int nw = blockDim.x >> 5;
      int v = (lane < nw) ? warp_sum[lane] : 0;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += y;
      }
      if (lane < nw) warp_sum[lane] = v;  // inclusive warp totals
    }
    __syncthreads();
    int excl = incl - run + (warp > 0 ? warp_sum[warp - 1] : 0);
    for (int e = lo; e < hi; ++e) {
      const int cnt = s_tot[e];
      if (c == 0) {
        counts[e] = cnt;
        offsets[e] = excl;
      }
      s_base[e] += excl;
      excl += cnt;
    }
    if (c == 0 && tid == 0) offsets[E] = T * k;
  }
  __syncthreads();
  const int tbeg = c * kChunk, tend = min(T, tbeg + kChunk);
  const int npair = (tend - tbeg) * k;
  for (int q = tid; q < npair; q += blockDim.x) {
    const int tl = q / k;
    const int e = topk_idx[(size_t)tbeg * k + q];
    atomicOr(&bits[e][tl >> 5], 1u << (tl & 31));
  }
  __syncthreads();
  for (int q = tid; q < npair; q += blockDim.x) {
    const int tl = q / k;
    const int e = topk_idx[(size_t)tbeg * k + q];
    int rank = 0;
#pragma unroll
    for (int w = 0; w < kChunk / 32; ++w) {
      const uint32_t word = bits[e][w];
      if (w < (tl >> 5)) rank += __popc(word);
      else if (w == (tl >> 5)) rank += __popc(word & ((1u << (tl & 31)) - 1u));
    }
    const int p = s_base[e] + rank;
    const int pair = tbeg * k + q;
    perm[p] = pair;
    slot_row[pair] = p;
  }
}

// ------------------------------------------------------------------ row gather
// xs[p, :] = x[t, :] for every row p = slot_row[t, j] of the expert-sorted space (the sorted
// copy of x that the up GEMM's larger token tiles load).
// Written token by token: one warp per token reads its x row once
// (chunks of four 16-byte vectors per lane in flight) and stores it to the k rows
// slot_row[t, 0..k) of xs (rows at or past *n_rows_dev, when given, are skipped).  x is read
// from HBM once instead of once per slot.
__global__ void __launch_bounds__(256) gather_rows_by_token_kernel(
    const uint4 *__restrict__ x, const int *__restrict__ slot_row, int T, int k,
    int vec_per_row, uint4 *__restrict__ xs, const int *__restrict__ n_rows_dev) {
  griddep_wait();
  griddep_launch_dependents();
  const int lane = threadIdx.x & 31;
  const int n_warps = gridDim.x * (blockDim.x >> 5);
  const int n_rows = n_rows_dev ? *n_rows_dev : 0x7fffffff;
  for (int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); t < T; t += n_warps) {
    const int my_row = lane < k ? __ldg(slot_row + (size_t)t * k + lane) : -1;
    const uint4 *__restrict__ src = x + (size_t)t * vec_per_row;
    for (int v0 = 0; v0 < vec_per_row; v0 += 128) {
      uint4 r[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int v = v0 + 32 * i + lane;
        if (v < vec_per_row) r[i] = __ldg(src + v);
      }
      for (int j = 0; j < k; ++j) {
        const int p = __shfl_sync(0xffffffffu, my_row, j);
        if (p >= n_rows) continue;
        uint4 *__restrict__ dst = xs + (size_t)p * vec_per_row;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int v = v0 + 32 * i + lane;
          if (v < vec_per_row) dst[v] = r[i];
        }
      }
    }
  }
}

}  // namespace moe
