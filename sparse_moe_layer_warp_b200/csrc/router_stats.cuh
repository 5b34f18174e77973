// router_stats.cuh -- balancing by-products of the router.
//
// "Step 3.5 Flash: Open Frontier-Level Intelligence with 11B Active Parameters",
// section 2.2.2: the EP-group balance loss L_EP = G sum_g f_g p_g with p_e the mean routing
// probability and f_e the selection frequency of expert e, summed over G disjoint expert
// groups; section 5.2.3: routing confidence, the mean probability mass of the activated
// experts.  The routing probability p[t,e] is the softmax over all E unbiased logits of token
// t.  "Step 3.5 Flash 技术论文深度解读", architecture item 1: balancing by a per-expert bias
// (the step below is this library's sign-rule reading; the pages give no rule).
//
// Deterministic: per-chunk partials are summed in fixed warp and chunk order, selection
// counts are integers.
#pragma once
#include <stdint.h>

#include "ptx_sm100.cuh"
#include "routing.cuh"

namespace moe {

constexpr int kStatWarps = 16;

// CTA c: tokens [c*kChunk, (c+1)*kChunk); warp w takes tokens w, w+16, ...  Writes
// part_p[c][e] = sum of p[t,e] over the chunk, part_cnt[c][e] = selections of e in the
// chunk and part_conf[c] = sum over the chunk's tokens of the selected probability mass.
// Dynamic shared memory: kStatWarps * E floats.
template <int MAXV>
__global__ void __launch_bounds__(kStatWarps * 32) router_stats_partial_kernel(
    const float *__restrict__ logits, const int *__restrict__ topk_idx, int T, int E, int k,
    float *__restrict__ part_p, int *__restrict__ part_cnt, float *__restrict__ part_conf) {
  griddep_wait();
  griddep_launch_dependents();
  extern __shared__ float wsum[];  // [kStatWarps][E]
  __shared__ int cnt[kMaxExperts];
  __shared__ float conf_w[kStatWarps];
  const int c = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int e = threadIdx.x; e < E; e += blockDim.x) cnt[e] = 0;
  __syncthreads();
  float acc[MAXV];
#pragma unroll
  for (int v = 0; v < MAXV; ++v) acc[v] = 0.f;
  float conf = 0.f;
  const int tbeg = c * kChunk, tend = min(T, tbeg + kChunk);
  for (int t = tbeg + warp; t < tend; t += kStatWarps) {
    float l[MAXV];
    float m = -INFINITY;
#pragma unroll
    for (int v = 0; v < MAXV; ++v) {
      const int e = lane + 32 * v;
      l[v] = (e < E) ? logits[(size_t)t * E + e] : -INFINITY;
      m = fmaxf(m, l[v]);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    float z = 0.f;
#pragma unroll
    for (int v = 0; v < MAXV; ++v) {
      l[v] = (lane + 32 * v < E) ? expf(l[v] - m) : 0.f;
      z += l[v];
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
    const float inv = 1.f / z;
#pragma unroll
    for (int v = 0; v < MAXV; ++v) {
      l[v] *= inv;  // p[t, lane + 32v]
      acc[v] += l[v];
    }
    float mass = 0.f;
    for (int j = 0; j < k; ++j) {
      const int e = topk_idx[(size_t)t * k + j];
      const int owner = e & 31, vv = e >> 5;
      float mine = 0.f;
#pragma unroll
      for (int v = 0; v < MAXV; ++v)
        if (v == vv) mine = l[v];
      mass += __shfl_sync(0xffffffffu, mine, owner);
      if (lane == 0) atomicAdd(&cnt[e], 1);
    }
    conf += mass;
  }
#pragma unroll
  for (int v = 0; v < MAXV; ++v) {
    const int e = lane + 32 * v;
    if (e < E) wsum[warp * E + e] = acc[v];
  }
  if (lane == 0) conf_w[warp] = conf;
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    float s = 0.f;
    for (int w = 0; w < kStatWarps; ++w) s += wsum[w * E + e];
    part_p[(size_t)c * E + e] = s;
    part_cnt[(size_t)c * E + e] = cnt[e];
  }
  if (threadIdx.x == 0) {
    float s = 0.f;
    for (int w = 0; w < kStatWarps; ++w) s += conf_w[w];
    part_conf[c] = s;
  }
}

// One CTA: sums the chunk partials in chunk order, then
//   p_mean[e] = sum_t p[t,e] / T,  f_sel[e] = selections of e / (T k),
//   scalars[0] = L_EP = G sum_g f_g p_g  (groups of E/G consecutive experts),
//   scalars[1] = routing confidence = sum_t sum_{e in S_t} p[t,e] / T.
__global__ void __launch_bounds__(256) router_stats_final_kernel(
    const float *__restrict__ part_p, const int *__restrict__ part_cnt,
    const float *__restrict__ part_conf, int n_chunks, int T, int E, int k, int G,
    float *__restrict__ p_mean, float *__restrict__ f_sel, float *__restrict__ scalars) {
  griddep_wait();
  griddep_launch_dependents();
  __shared__ float sp[kMaxExperts];
  __shared__ float sf[kMaxExperts];
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    float p = 0.f;
    long long n = 0;
    for (int c = 0; c < n_chunks; ++c) {
      p += part_p[(size_t)c * E + e];
      n += part_cnt[(size_t)c * E + e];
    }
    sp[e] = p / (float)T;
    sf[e] = (float)((double)n / ((double)T * k));
    p_mean[e] = sp[e];
    f_sel[e] = sf[e];
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const int per = E / G;
    double loss = 0.0;
    for (int g = 0; g < G; ++g) {
      double pg = 0.0, fg = 0.0;
      for (int e = g * per; e < (g + 1) * per; ++e) {
        pg += sp[e];
        fg += sf[e];
      }
      loss += pg * fg;
    }
    double conf = 0.0;
    for (int c = 0; c < n_chunks; ++c) conf += part_conf[c];
    scalars[0] = (float)(G * loss);
    scalars[1] = (float)(conf / T);
  }
}

// Loss-free balancing step (sign rule, see the header of this file):
//   bias[e] += gamma * sign(T k / E - counts[e])
__global__ void __launch_bounds__(256) bias_update_kernel(const int *__restrict__ counts, int E,
                                                          int Tk, float gamma,
                                                          float *__restrict__ bias) {
  griddep_wait();
  griddep_launch_dependents();
  const float mean = (float)Tk / (float)E;
  for (int e = blockIdx.x * blockDim.x + threadIdx.x; e < E; e += gridDim.x * blockDim.x) {
    const float gap = mean - (float)counts[e];
    const float s = (gap > 0.f) ? 1.f : ((gap < 0.f) ? -1.f : 0.f);
    bias[e] = bias[e] + gamma * s;
  }
}

}  // namespace moe
