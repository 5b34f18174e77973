// expert_simt.cuh -- exact-fp32 expert FFNs (CUDA-core FFMA, no TF32) and the
// gate-weighted combine shared by both precisions.
//
// Expert FFN: SwiGLU with gate and up branches ("Step 3.5 Flash 技术论文深度解读",
// training stability, local activation explosion, root cause 3); the routed sum carries an
// explicit scale ("Step 3.5 Flash: Open Frontier-Level Intelligence with 11B Active
// Parameters", section 4.1.2) and the shared expert is always on (section 2.2).
#pragma once
#include <cuda_bf16.h>
#include <stdint.h>

#include "ptx_sm100.cuh"

namespace moe {

// Row p of the expert-sorted space: p < Tk is pair perm[p] = t*k + j of expert
// topk_idx[perm[p]]; p >= Tk is the shared expert on token p - Tk.
__device__ __forceinline__ void sorted_row_owner(int p, int Tk, int k, int E,
                                                 const int *__restrict__ perm,
                                                 const int *__restrict__ topk_idx, int &t,
                                                 int &g) {
  if (p < Tk) {
    const int pair = perm[p];
    t = pair / k;
    g = topk_idx[pair];
  } else {
    t = p - Tk;
    g = E;
  }
}

// h[p, r] = silu(x_t . W_g[g, r]) * (x_t . W_u[g, r]), one thread per (p, r), fp32.
__global__ void __launch_bounds__(256) ffn_up_f32_kernel(
    const float *__restrict__ x, const float *__restrict__ wg, const float *__restrict__ wu,
    const int *__restrict__ perm, const int *__restrict__ topk_idx, int Tk, int k, int E,
    int n_rows, int d, int f, float *__restrict__ h) {
  griddep_wait();
  griddep_launch_dependents();
  const size_t total = (size_t)n_rows * f;
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (size_t)gridDim.x * blockDim.x) {
    const int p = (int)(i / f), r = (int)(i % f);
    int t, g;
    sorted_row_owner(p, Tk, k, E, perm, topk_idx, t, g);
    const float *xr = x + (size_t)t * d;
    const float *gr = wg + ((size_t)g * f + r) * d;
    const float *ur = wu + ((size_t)g * f + r) * d;
    float a = 0.f, b = 0.f;
    for (int c = 0; c < d; ++c) {
      a = fmaf(xr[c], gr[c], a);
      b = fmaf(xr[c], ur[c], b);
    }
    h[i] = a / (1.f + expf(-a)) * b;
  }
}

// y[p, c] = scale_p * sum_r h[p, r] W_d[g, c, r]; scale_p = routed_scale * gate of the pair
// for routed rows, 1 for shared rows.  One thread per (p, c), fp32.
__global__ void __launch_bounds__(256) ffn_down_f32_kernel(
    const float *__restrict__ h, const float *__restrict__ wd, const int *__restrict__ perm,
    const int *__restrict__ topk_idx, const float *__restrict__ topk_gate, float routed_scale,
    int Tk, int k, int E, int n_rows, int d, int f, float *__restrict__ y) {
  griddep_wait();
  griddep_launch_dependents();
  const size_t total = (size_t)n_rows * d;
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (size_t)gridDim.x * blockDim.x) {
    const int p = (int)(i / d), c = (int)(i % d);
    int t, g;
    sorted_row_owner(p, Tk, k, E, perm, topk_idx, t, g);
    const float *hr = h + (size_t)p * f;
    const float *wr = wd + ((size_t)g * d + c) * f;
    float a = 0.f;
    for (int r = 0; r < f; ++r) a = fmaf(hr[r], wr[r], a);
    const float scale = (p < Tk) ? routed_scale * topk_gate[perm[p]] : 1.f;
    y[i] = a * scale;
  }
}

// out[t, :] = sum_{j < k} y[slot_row[t, j], :] (+ y[Tk + t, :] if shared): y rows are
// fp32, summed in this fixed order in fp32 and rounded once to the output type.  Each
// thread owns 4 consecutive columns (16-byte loads of y), grid-stride.
__device__ __forceinline__ void store4(float *p, const float4 &v) {
  *reinterpret_cast<float4 *>(p) = v;
}
__device__ __forceinline__ void store4(__nv_bfloat16 *p, const float4 &v) {
  uint2 u;
  *reinterpret_cast<__nv_bfloat162 *>(&u.x) = __floats2bfloat162_rn(v.x, v.y);
  *reinterpret_cast<__nv_bfloat162 *>(&u.y) = __floats2bfloat162_rn(v.z, v.w);
  *reinterpret_cast<uint2 *>(p) = u;
}

template <typename Tout>
__global__ void __launch_bounds__(256) combine_kernel(const float *__restrict__ y,
                                                      const int *__restrict__ slot_row,
                                                      int n_tokens, int k, int Tk,
                                                      int n_shared, int d,
                                                      Tout *__restrict__ out) {
  griddep_wait();
  griddep_launch_dependents();
  const int vpr = d / 4;
  const size_t total = (size_t)n_tokens * vpr;
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (size_t)gridDim.x * blockDim.x) {
    const int t = (int)(i / vpr);
    const int c = (int)(i % vpr) * 4;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    // eight slots at a time: their row indices, then their rows, are loaded before the
    // first add, so the loads are in flight together; the sum keeps slot order
    for (int j0 = 0; j0 < k; j0 += 8) {
      int p[8];
      float4 v[8];
#pragma unroll
      for (int j = 0; j < 8; ++j)
        p[j] = (j0 + j < k) ? __ldg(slot_row + (size_t)t * k + j0 + j) : 0;
#pragma unroll
      for (int j = 0; j < 8; ++j)
        v[j] = (j0 + j < k) ? __ldg(reinterpret_cast<const float4 *>(y + (size_t)p[j] * d + c))
                            : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (j0 + j < k) {
          acc.x += v[j].x;
          acc.y += v[j].y;
          acc.z += v[j].z;
          acc.w += v[j].w;
        }
      }
    }
    if (n_shared) {
      const float4 v = __ldg(reinterpret_cast<const float4 *>(y + (size_t)(Tk + t) * d + c));
      acc.x += v.x;
      acc.y += v.y;
      acc.z += v.z;
      acc.w += v.w;
    }
    store4(out + (size_t)t * d + c, acc);
  }
}

}  // namespace moe
