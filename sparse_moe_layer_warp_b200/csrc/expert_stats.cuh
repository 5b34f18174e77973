// expert_stats.cuh -- expert health signals of the layer.
//
// "Step 3.5 Flash: Open Frontier-Level Intelligence with 11B Active Parameters", section
// 4.1.2: expert collapse shows as vanishing expert activations and stalling parameter norms,
// so per-expert activation and parameter norms are to be monitored; "Step 3.5 Flash
// 技术论文深度解读", training stability, "expert collapse": the per-expert activation RMS norm
// and the min-to-median ratio of the parameter Frobenius norms.
//
//   act_rms[g]    = RMS of the SwiGLU activation h of expert g over the rows of its group
//                   (the tokens routed to it; every token for the shared expert), 0 if empty
//   param_norm[g] = Frobenius norm of W_gate[g], W_up[g] and W_down[g] together
//   ratios[0]     = median / max of act_rms over the routed experts some token chose
//   ratios[1]     = min / median of param_norm over the routed experts
// (median of an even count: mean of the two middle values).  Sums of squares are taken in
// fp64 per slice and added over the slices in a fixed order: deterministic.
#pragma once
#include <cuda_bf16.h>
#include <stdint.h>

#include "ptx_sm100.cuh"

namespace moe {

constexpr int kHealthSlices = 16;        // blocks per expert in the sum-of-squares kernels
constexpr int kMaxExpertsHealth = 1024;  // routed experts handled by the final kernel

__device__ __forceinline__ double sq_of(float v) { return (double)v * (double)v; }
__device__ __forceinline__ double sq_of(__nv_bfloat16 v) {
  const double d = (double)__bfloat162float(v);
  return d * d;
}

// Block-wide fp64 sum (fixed order); result valid in thread 0.
__device__ __forceinline__ double block_sum_f64(double v, double *red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  if (lane == 0) red[warp] = v;
  __syncthreads();
  double s = 0.0;
  if (threadIdx.x == 0)
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) s += red[w];
  __syncthreads();
  return s;
}

// Block (g, s): slice s of the h rows of group g.  part[g * kHealthSlices + s].
template <typename Th>
__global__ void __launch_bounds__(256) expert_act_sumsq_kernel(
    const Th *__restrict__ h, const int *__restrict__ offsets, int E, int T, int Tk, int f,
    double *__restrict__ part) {
  griddep_wait();
  griddep_launch_dependents();
  __shared__ double red[8];
  const int g = blockIdx.x, s = blockIdx.y;
  const int row0 = (g < E) ? offsets[g] : Tk + (g - E) * T;
  const int rows = (g < E) ? offsets[g + 1] - row0 : T;
  const long long n = (long long)rows * f;
  const long long per = (n + kHealthSlices - 1) / kHealthSlices;
  const long long lo = min(n, per * s), hi = min(n, lo + per);
  const Th *base = h + (size_t)row0 * f;
  double acc = 0.0;
  for (long long i = lo + threadIdx.x; i < hi; i += blockDim.x) acc += sq_of(base[i]);
  const double tot = block_sum_f64(acc, red);
  if (threadIdx.x == 0) part[g * kHealthSlices + s] = tot;
}

// Block (g, s): slice s of expert g's three weight matrices (each f*d elements).
template <typename Tw>
__global__ void __launch_bounds__(256) expert_param_sumsq_kernel(
    const Tw *__restrict__ wg, const Tw *__restrict__ wu, const Tw *__restrict__ wd,
    long long per_matrix, double *__restrict__ part) {
  griddep_wait();
  griddep_launch_dependents();
  __shared__ double red[8];
  const int g = blockIdx.x, s = blockIdx.y;
  const long long per = (per_matrix + kHealthSlices - 1) / kHealthSlices;
  const long long lo = min(per_matrix, per * s), hi = min(per_matrix, lo + per);
  const size_t off = (size_t)g * per_matrix;
  double acc = 0.0;
  for (long long i = lo + threadIdx.x; i < hi; i += blockDim.x)
    acc += sq_of(wg[off + i]) + sq_of(wu[off + i]) + sq_of(wd[off + i]);
  const double tot = block_sum_f64(acc, red);
  if (threadIdx.x == 0) part[g * kHealthSlices + s] = tot;
}

// One CTA of 1024 threads: slice sums in order, norms, and the two ratios.  A value's place
// in sorted order is its rank (smaller values first, equal values by index), so the median
// needs no sort.
__global__ void __launch_bounds__(1024) expert_health_final_kernel(
    const double *__restrict__ act_part, const double *__restrict__ par_part,
    const int *__restrict__ offsets, int E, int G, int T, int f, float *__restrict__ act_rms,
    float *__restrict__ param_norm, float *__restrict__ ratios) {
  griddep_wait();
  griddep_launch_dependents();
  __shared__ double va[kMaxExpertsHealth];
  __shared__ double vp[kMaxExpertsHealth];
  __shared__ double sa[kMaxExpertsHealth];
  __shared__ double sp[kMaxExpertsHealth];
  __shared__ int chosen[kMaxExpertsHealth];
  __shared__ int n_chosen;
  if (threadIdx.x == 0) n_chosen = 0;
  __syncthreads();
  for (int g = threadIdx.x; g < G; g += blockDim.x) {
    double a = 0.0, p = 0.0;
    for (int s = 0; s < kHealthSlices; ++s) {
      a += act_part[g * kHealthSlices + s];
      p += par_part[g * kHealthSlices + s];
    }
    const int rows = (g < E) ? offsets[g + 1] - offsets[g] : T;
    const double rms = rows > 0 ? sqrt(a / ((double)rows * f)) : 0.0;
    act_rms[g] = (float)rms;
    param_norm[g] = (float)sqrt(p);
    if (g < E) {
      va[g] = rms;
      vp[g] = sqrt(p);
      chosen[g] = rows > 0;
    }
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int ra = 0, rp = 0;
    for (int j = 0; j < E; ++j) {
      if (chosen[j] && (va[j] < va[e] || (va[j] == va[e] && j < e))) ++ra;
      if (vp[j] < vp[e] || (vp[j] == vp[e] && j < e)) ++rp;
    }
    if (chosen[e]) {
      sa[ra] = va[e];
      atomicAdd(&n_chosen, 1);
    }
    sp[rp] = vp[e];
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const int n = n_chosen;
    const double med_a = n == 0 ? 0.0 : ((n & 1) ? sa[n / 2] : 0.5 * (sa[n / 2 - 1] + sa[n / 2]));
    const double max_a = n == 0 ? 0.0 : sa[n - 1];
    const double med_p = (E & 1) ? sp[E / 2] : 0.5 * (sp[E / 2 - 1] + sp[E / 2]);
    ratios[0] = max_a > 0.0 ? (float)(med_a / max_a) : 0.f;
    ratios[1] = med_p > 0.0 ? (float)(sp[0] / med_p) : 0.f;
  }
}

}  // namespace moe
