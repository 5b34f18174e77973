// backward.cuh -- backward of the sparse-MoE FFN layer (CUDA-core fp32 kernels).
//
// The chain rule through the forward ("Step 3.5 Flash: Open Frontier-Level Intelligence with
// 11B Active Parameters", sections 2.2 / 2.2.2 / 4.1.2 and section 3.2.4 for the expert-sorted
// layout; SwiGLU experts, "Step 3.5 Flash 技术论文深度解读", training stability, root cause 3)
// for the forward's own selection, which carries no gradient (the bias only selects).  Per
// row p of the expert-sorted space (group g, token t, scale s = routed_scale * gate, 1 for
// the shared expert):
//   a = W_g[g] x_t,  b = W_u[g] x_t,  h = silu(a) b,  yhat = W_d[g] h
//   dy = s dout_t,  dh = W_d[g]^T dy,  da = dh b silu'(a),  db = dh silu(a)
//   dX_p = W_g[g]^T da + W_u[g]^T db
//   dW_d[g] += sum_p dy h^T,  dW_g[g] += sum_p da x_t^T,  dW_u[g] += sum_p db x_t^T
//   (weight gradients accumulate into the caller's buffers, as over micro-batches; experts
//   no token chose are not touched)
//   routed rows: dgate = routed_scale * (dout_t . yhat)
// and for the router (gates = softmax of the selected unbiased logits):
//   dl_j = g_j (dgate_j - sum_i g_i dgate_i),  dW_r[e] = sum dl x_t,  dx_t += sum dl W_r[e]
//   dx_t = sum_j dX[slot_row[t,j]] + dX[shared row of t] + router term  (fixed order)
// Every sum runs in a fixed order in fp32 (no atomics): results are deterministic.
//
// Three grouped row kernels do the matrix work (tiles of 16 rows of one group):
//   bw_nt_kernel   out[p][m] = sum_k W[g][m][k] v_p[k]      (W row-major [M, K])
//   bw_nn_kernel   out[p][n] = sum_k W[g][k][n] v_p[k]      (W row-major [K, N])
//   bw_wgrad_kernel dW[g][m][n] += sum_{p in g} u_p[m] v_p[n]
// with the row vectors v_p, u_p produced on the fly by small source functors.
#pragma once
#include <cuda_bf16.h>
#include <stdint.h>

#include "ptx_sm100.cuh"

namespace moe {

constexpr int kBwRows = 16;  // rows of one group per tile
constexpr int kBwK = 32;     // reduction chunk staged in shared memory

__device__ __forceinline__ float bw_f32(float v) { return v; }
__device__ __forceinline__ float bw_f32(__nv_bfloat16 v) { return __bfloat162float(v); }

__device__ __forceinline__ float bw_silu(float a) { return a / (1.f + expf(-a)); }

// ---------------------------------------------------------------------- row sources
template <typename Tin>
struct SrcX {  // x of the row's token
  const Tin *x;
  const int *row_token;
  int d;
  __device__ __forceinline__ float operator()(int p, int k) const {
    return bw_f32(x[(size_t)row_token[p] * d + k]);
  }
};

template <typename Tin>
struct SrcDy {  // s_p * dout of the row's token
  const Tin *dout;
  const int *row_token;
  const float *row_scale;
  int d;
  __device__ __forceinline__ float operator()(int p, int k) const {
    return row_scale[p] * bw_f32(dout[(size_t)row_token[p] * d + k]);
  }
};

struct SrcRow {  // a stored fp32 row
  const float *v;
  int ld;
  __device__ __forceinline__ float operator()(int p, int k) const {
    return v[(size_t)p * ld + k];
  }
};

struct SrcH {  // h = silu(a) * b from the stored pre-activations
  const float *a, *b;
  int f;
  __device__ __forceinline__ float operator()(int p, int k) const {
    const size_t i = (size_t)p * f + k;
    return bw_silu(a[i]) * b[i];
  }
};

// ------------------------------------------------------------- row bookkeeping
// Per sorted row: token, group and scale; per group: the prefix of 16-row tiles.
__global__ void __launch_bounds__(256) bw_rows_kernel(const int *__restrict__ perm,
                                                      const int *__restrict__ topk_idx,
                                                      const float *__restrict__ topk_gate,
                                                      int T, int k, int E, int n_shared,
                                                      float routed_scale, int *row_token,
                                                      int *row_group, float *row_scale) {
  griddep_wait();
  griddep_launch_dependents();
  const int Tk = T * k, P = Tk + n_shared * T;
  for (int p = blockIdx.x * blockDim.x + threadIdx.x; p < P; p += gridDim.x * blockDim.x) {
    if (p < Tk) {
      const int q = perm[p];
      row_token[p] = q / k;
      row_group[p] = topk_idx[q];
      row_scale[p] = routed_scale * topk_gate[q];
    } else {
      row_token[p] = p - Tk;
      row_group[p] = E;
      row_scale[p] = 1.f;
    }
  }
}

__global__ void __launch_bounds__(32) bw_tiles_kernel(const int *__restrict__ offsets, int E,
                                                      int G, int T, int R, int *tile_prefix) {
  griddep_wait();
  griddep_launch_dependents();
  if (threadIdx.x != 0) return;
  int acc = 0;
  for (int g = 0; g < G; ++g) {
    tile_prefix[g] = acc;
    const int cnt = (g < E) ? offsets[g + 1] - offsets[g] : T;
    acc += (cnt + R - 1) / R;
  }
  tile_prefix[G] = acc;
}

// Tile b of the row-tile list (tiles of R rows) -> group, first row, rows.  Returns false
// past the list.
template <int R>
__device__ __forceinline__ bool bw_tile(int b, const int *tile_prefix, const int *offsets,
                                        int E, int G, int T, int Tk, int &g, int &row0,
                                        int &rows) {
  if (b >= tile_prefix[G]) return false;
  int lo = 0, hi = G - 1;
  while (lo < hi) {  // last g with tile_prefix[g] <= b
    const int mid = (lo + hi + 1) >> 1;
    if (tile_prefix[mid] <= b) lo = mid;
    else hi = mid - 1;
  }
  g = lo;
  const int base = (g < E) ? offsets[g] : Tk + (g - E) * T;
  const int cnt = (g < E) ? offsets[g + 1] - offsets[g] : T;
  const int i = b - tile_prefix[g];
  row0 = base + i * R;
  rows = min(R, cnt - i * R);
  return true;
}

// 8 consecutive weights as floats (16 bytes of bf16, or 32 of fp32).
__device__ __forceinline__ void bw_load8(const __nv_bfloat16 *p, float (&v)[8]) {
  const uint4 r = __ldg(reinterpret_cast<const uint4 *>(p));
  const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&r);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __bfloat1622float2(h[i]);
    v[2 * i] = f.x;
    v[2 * i + 1] = f.y;
  }
}
__device__ __forceinline__ void bw_load8(const float *p, float (&v)[8]) {
  const float4 a = __ldg(reinterpret_cast<const float4 *>(p));
  const float4 b = __ldg(reinterpret_cast<const float4 *>(p + 4));
  v[0] = a.x, v[1] = a.y, v[2] = a.z, v[3] = a.w;
  v[4] = b.x, v[5] = b.y, v[6] = b.z, v[7] = b.w;
}

// ---------------------------------------------------------------------------- NT
// Block (tile of R rows, m block of 64): out_j[p][m] = sum_k W_j[g][m][k] v_p[k] for j < NW
// (the matrices share v).  K and M are multiples of 8 (the weight tile is staged with one
// 16-byte load per thread and matrix).  Thread (r = tid / 16, c = tid % 16) owns rows
// r + 16 a (a < R / 16) and m = c + 16 i: R / 16 x 4 outputs.
template <int NW, int R, typename Tw, typename Src>
__global__ void __launch_bounds__(256) bw_nt_kernel(const Tw *__restrict__ W0,
                                                    const Tw *__restrict__ W1, int M, int K,
                                                    Src src, const int *__restrict__ tile_prefix,
                                                    const int *__restrict__ offsets, int E,
                                                    int G, int T, int Tk, float *out0,
                                                    float *out1) {
  griddep_wait();
  griddep_launch_dependents();
  constexpr int RA = R / 16;
  __shared__ float ws[NW][64][kBwK + 1];
  __shared__ float vs[R][kBwK + 1];
  int g, row0, rows;
  if (!bw_tile<R>(blockIdx.x, tile_prefix, offsets, E, G, T, Tk, g, row0, rows)) return;
  const int m0 = blockIdx.y * 64;
  const int r = threadIdx.x >> 4, c = threadIdx.x & 15;
  float acc[NW][RA][4];
#pragma unroll
  for (int j = 0; j < NW; ++j)
#pragma unroll
    for (int a = 0; a < RA; ++a)
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[j][a][i] = 0.f;
  const Tw *Wj[2] = {W0, W1};
  // weight tile staging: thread -> (row mm = tid / 4, 8 columns at kq = 8 (tid % 4))
  const int mm = threadIdx.x >> 2, kq = (threadIdx.x & 3) * 8;
  for (int k0 = 0; k0 < K; k0 += kBwK) {
#pragma unroll
    for (int j = 0; j < NW; ++j) {
      float w8[8];
      if (m0 + mm < M && k0 + kq < K) {
        bw_load8(Wj[j] + ((size_t)g * M + m0 + mm) * K + k0 + kq, w8);
      } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) w8[i] = 0.f;
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) ws[j][mm][kq + i] = w8[i];
    }
    for (int e = threadIdx.x; e < R * kBwK; e += blockDim.x) {
      const int rr = e / kBwK, kk = e % kBwK;
      vs[rr][kk] = (rr < rows && k0 + kk < K) ? src(row0 + rr, k0 + kk) : 0.f;
    }
    __syncthreads();
#pragma unroll 4
    for (int kk = 0; kk < kBwK; ++kk) {
      float v[RA], w[NW][4];
#pragma unroll
      for (int a = 0; a < RA; ++a) v[a] = vs[r + 16 * a][kk];
#pragma unroll
      for (int j = 0; j < NW; ++j)
#pragma unroll
        for (int i = 0; i < 4; ++i) w[j][i] = ws[j][c + 16 * i][kk];
#pragma unroll
      for (int j = 0; j < NW; ++j)
#pragma unroll
        for (int a = 0; a < RA; ++a)
#pragma unroll
          for (int i = 0; i < 4; ++i) acc[j][a][i] = fmaf(w[j][i], v[a], acc[j][a][i]);
    }
    __syncthreads();
  }
  float *outs[2] = {out0, out1};
#pragma unroll
  for (int a = 0; a < RA; ++a) {
    if (r + 16 * a >= rows) continue;
#pragma unroll
    for (int j = 0; j < NW; ++j)
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int m = m0 + c + 16 * i;
        if (m < M) outs[j][(size_t)(row0 + r + 16 * a) * M + m] = acc[j][a][i];
      }
  }
}

// ---------------------------------------------------------------------------- NN
// Block (tile of R rows, n block of 64): out[p][n] = sum_j sum_k W_j[g][k][n] v_j,p[k]; N a
// multiple of 8 (one 16-byte weight load per thread and matrix per stage).  Thread
// (r, c) owns rows r + 16 a and n = c + 16 i.
template <int NW, int R, typename Tw, typename Src0, typename Src1>
__global__ void __launch_bounds__(256) bw_nn_kernel(const Tw *__restrict__ W0,
                                                    const Tw *__restrict__ W1, int K, int N,
                                                    Src0 src0, Src1 src1,
                                                    const int *__restrict__ tile_prefix,
                                                    const int *__restrict__ offsets, int E,
                                                    int G, int T, int Tk, float *out) {
  griddep_wait();
  griddep_launch_dependents();
  constexpr int RA = R / 16;
  __shared__ float ws[NW][kBwK][64 + 1];
  __shared__ float vs[NW][R][kBwK + 1];
  int g, row0, rows;
  if (!bw_tile<R>(blockIdx.x, tile_prefix, offsets, E, G, T, Tk, g, row0, rows)) return;
  const int n0 = blockIdx.y * 64;
  const int r = threadIdx.x >> 4, c = threadIdx.x & 15;
  float acc[RA][4];
#pragma unroll
  for (int a = 0; a < RA; ++a)
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[a][i] = 0.f;
  const Tw *Wj[2] = {W0, W1};
  // weight tile staging: thread -> (row kk = tid / 8, 8 columns at nq = 8 (tid % 8))
  const int kr = threadIdx.x >> 3, nq = (threadIdx.x & 7) * 8;
  for (int k0 = 0; k0 < K; k0 += kBwK) {
#pragma unroll
    for (int j = 0; j < NW; ++j) {
      float w8[8];
      if (k0 + kr < K && n0 + nq < N) {
        bw_load8(Wj[j] + ((size_t)g * K + k0 + kr) * N + n0 + nq, w8);
      } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) w8[i] = 0.f;
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) ws[j][kr][nq + i] = w8[i];
    }
    for (int e = threadIdx.x; e < R * kBwK; e += blockDim.x) {
      const int rr = e / kBwK, kk = e % kBwK;
      const bool in = rr < rows && k0 + kk < K;
      vs[0][rr][kk] = in ? src0(row0 + rr, k0 + kk) : 0.f;
      if (NW > 1) vs[NW - 1][rr][kk] = in ? src1(row0 + rr, k0 + kk) : 0.f;
    }
    __syncthreads();
#pragma unroll 4
    for (int kk = 0; kk < kBwK; ++kk)
#pragma unroll
      for (int j = 0; j < NW; ++j) {
        float v[RA], w[4];
#pragma unroll
        for (int a = 0; a < RA; ++a) v[a] = vs[j][r + 16 * a][kk];
#pragma unroll
        for (int i = 0; i < 4; ++i) w[i] = ws[j][kk][c + 16 * i];
#pragma unroll
        for (int a = 0; a < RA; ++a)
#pragma unroll
          for (int i = 0; i < 4; ++i) acc[a][i] = fmaf(w[i], v[a], acc[a][i]);
      }
    __syncthreads();
  }
#pragma unroll
  for (int a = 0; a < RA; ++a) {
    if (r + 16 * a >= rows) continue;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int n = n0 + c + 16 * i;
      if (n < N) out[(size_t)(row0 + r + 16 * a) * N + n] = acc[a][i];
    }
  }
}

// ------------------------------------------------------------------------- WGRAD
// Block (g, m block of 64, n block of 128): dW[g][m][n] += sum over the group's rows p of
// u_p[m] v_p[n], rows in order, 16 at a time.  Thread (mi = tid / 16, ni = tid % 16) owns
// m = m0 + 4 mi + {0..3} and n = n0 + 8 ni + {0..7} (N a multiple of 8: the gradient is
// read and written as float4).  Groups with no rows are left untouched.
template <typename SrcU, typename SrcV>
__global__ void __launch_bounds__(256) bw_wgrad_kernel(SrcU u, SrcV v, int M, int N,
                                                       const int *__restrict__ offsets, int E,
                                                       int T, int Tk, float *dW) {
  griddep_wait();
  griddep_launch_dependents();
  __shared__ float us[kBwRows][64 + 4];
  __shared__ float vsm[kBwRows][128 + 4];
  const int g = blockIdx.x;
  const int m0 = blockIdx.y * 64, n0 = blockIdx.z * 128;
  const int base = (g < E) ? offsets[g] : Tk + (g - E) * T;
  const int cnt = (g < E) ? offsets[g + 1] - offsets[g] : T;
  if (cnt == 0) return;
  const int mi = threadIdx.x >> 4, ni = threadIdx.x & 15;
  float acc[4][8];
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[a][j] = 0.f;
  for (int r0 = 0; r0 < cnt; r0 += kBwRows) {
    const int rows = min(kBwRows, cnt - r0);
    for (int e = threadIdx.x; e < kBwRows * 64; e += blockDim.x) {
      const int rr = e / 64, mm = e % 64;
      us[rr][mm] = (rr < rows && m0 + mm < M) ? u(base + r0 + rr, m0 + mm) : 0.f;
    }
    for (int e = threadIdx.x; e < kBwRows * 128; e += blockDim.x) {
      const int rr = e / 128, nn = e % 128;
      vsm[rr][nn] = (rr < rows && n0 + nn < N) ? v(base + r0 + rr, n0 + nn) : 0.f;
    }
    __syncthreads();
    for (int rr = 0; rr < rows; ++rr) {
      const float4 ua = *reinterpret_cast<const float4 *>(&us[rr][4 * mi]);
      const float4 v0 = *reinterpret_cast<const float4 *>(&vsm[rr][8 * ni]);
      const float4 v1 = *reinterpret_cast<const float4 *>(&vsm[rr][8 * ni + 4]);
      const float uu[4] = {ua.x, ua.y, ua.z, ua.w};
      const float vv[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[a][j] = fmaf(uu[a], vv[j], acc[a][j]);
    }
    __syncthreads();
  }
  const int n = n0 + 8 * ni;
  if (n >= N) return;
#pragma unroll
  for (int a = 0; a < 4; ++a) {
    const int m = m0 + 4 * mi + a;
    if (m >= M) continue;
    float4 *dst = reinterpret_cast<float4 *>(dW + ((size_t)g * M + m) * N + n);
    float4 x0 = dst[0], x1 = dst[1];
    x0.x += acc[a][0], x0.y += acc[a][1], x0.z += acc[a][2], x0.w += acc[a][3];
    x1.x += acc[a][4], x1.y += acc[a][5], x1.z += acc[a][6], x1.w += acc[a][7];
    dst[0] = x0;
    dst[1] = x1;
  }
}

// ------------------------------------------------------------------ elementwise steps
// da, db from dh and the pre-activations (in place: da over dh).
__global__ void __launch_bounds__(256) bw_swiglu_kernel(const float *__restrict__ a,
                                                        const float *__restrict__ b, float *dh,
                                                        float *db, size_t n) {
  griddep_wait();
  griddep_launch_dependents();
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n;
       i += (size_t)gridDim.x * blockDim.x) {
    const float av = a[i], g = dh[i];
    const float sg = 1.f / (1.f + expf(-av));
    db[i] = g * av * sg;
    dh[i] = g * b[i] * sg * (1.f + av * (1.f - sg));
  }
}

// dgate of routed row p = routed_scale * (dout_t . yhat_p): one warp per row.
template <typename Tin>
__global__ void __launch_bounds__(256) bw_dgate_kernel(const Tin *__restrict__ dout,
                                                       const float *__restrict__ yhat,
                                                       const int *__restrict__ row_token,
                                                       const int *__restrict__ perm, int Tk,
                                                       int d, float routed_scale,
                                                       float *dgate) {
  griddep_wait();
  griddep_launch_dependents();
  const int lane = threadIdx.x & 31;
  const int n_warps = gridDim.x * (blockDim.x >> 5);
  for (int p = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); p < Tk; p += n_warps) {
    const Tin *o = dout + (size_t)row_token[p] * d;
    const float *y = yhat + (size_t)p * d;
    float s = 0.f;
    for (int i = lane; i < d; i += 32) s = fmaf(bw_f32(o[i]), y[i], s);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
    if (lane == 0) dgate[perm[p]] = routed_scale * s;  // indexed by pair t*k + j
  }
}

// Router: dl[t, j] = g_j (dgate_j - sum_i g_i dgate_i), one thread per token.
__global__ void __launch_bounds__(256) bw_router_dl_kernel(const float *__restrict__ gate,
                                                           const float *__restrict__ dgate,
                                                           int T, int k, float *dl) {
  griddep_wait();
  griddep_launch_dependents();
  for (int t = blockIdx.x * blockDim.x + threadIdx.x; t < T; t += gridDim.x * blockDim.x) {
    float s = 0.f;
    for (int j = 0; j < k; ++j) s = fmaf(gate[t * k + j], dgate[t * k + j], s);
    for (int j = 0; j < k; ++j) dl[t * k + j] = gate[t * k + j] * (dgate[t * k + j] - s);
  }
}

// Two consecutive inputs as floats (4 bytes of bf16, 8 of fp32); four (8 / 16 bytes).
__device__ __forceinline__ float2 bw_load2(const __nv_bfloat16 *p) {
  return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(p));
}
__device__ __forceinline__ float2 bw_load2(const float *p) {
  return *reinterpret_cast<const float2 *>(p);
}
__device__ __forceinline__ float4 bw_load4(const __nv_bfloat16 *p) {
  const uint2 r = __ldg(reinterpret_cast<const uint2 *>(p));
  const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&r.x));
  const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&r.y));
  return make_float4(a.x, a.y, b.x, b.y);
}
__device__ __forceinline__ float4 bw_load4(const float *p) {
  return __ldg(reinterpret_cast<const float4 *>(p));
}

// dW_r[e][i] += sum over the rows of routed group e (ascending token) of dl x_t[i]; experts
// no token chose are left untouched (overwrite: dW_r[e][i] = the sum, zero for them).  Block
// (e, 512 columns): each thread two columns, the rows four at a time (their loads issued
// together, the sums still in row order).
template <typename Tin>
__global__ void __launch_bounds__(256) bw_router_dw_kernel(const Tin *__restrict__ x,
                                                           const float *__restrict__ dl,
                                                           const int *__restrict__ perm,
                                                           const int *__restrict__ offsets,
                                                           int k, int d, float *dw_r,
                                                           int overwrite) {
  griddep_wait();
  griddep_launch_dependents();
  const int e = blockIdx.x;
  const int i = 2 * (blockIdx.y * blockDim.x + threadIdx.x);
  const int lo = offsets[e], hi = offsets[e + 1];
  if (i >= d) return;
  if (lo == hi) {
    if (overwrite)
      *reinterpret_cast<float2 *>(dw_r + (size_t)e * d + i) = make_float2(0.f, 0.f);
    return;
  }
  float2 acc = make_float2(0.f, 0.f);
  int p = lo;
  for (; p + 4 <= hi; p += 4) {
    int q[4];
    float w[4];
    float2 v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) q[u] = perm[p + u];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      w[u] = dl[q[u]];
      v[u] = bw_load2(x + (size_t)(q[u] / k) * d + i);
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      acc.x = fmaf(w[u], v[u].x, acc.x);
      acc.y = fmaf(w[u], v[u].y, acc.y);
    }
  }
  for (; p < hi; ++p) {
    const int q = perm[p];
    const float w = dl[q];
    const float2 v = bw_load2(x + (size_t)(q / k) * d + i);
    acc.x = fmaf(w, v.x, acc.x);
    acc.y = fmaf(w, v.y, acc.y);
  }
  float2 *o = reinterpret_cast<float2 *>(dw_r + (size_t)e * d + i);
  if (overwrite) {
    *o = acc;
  } else {
    const float2 old = *o;
    *o = make_float2(old.x + acc.x, old.y + acc.y);
  }
}

// dx[t][i] = sum_j dX[slot_row[t,j]][i] + dX[shared row][i] + sum_j dl[t,j] W_r[e_j][i],
// four consecutive columns per thread (16-byte rows of dX, d a multiple of 4).
template <typename Tw>
__global__ void __launch_bounds__(256) bw_dx_kernel(const float *__restrict__ dX,
                                                    const int *__restrict__ slot_row,
                                                    const int *__restrict__ topk_idx,
                                                    const float *__restrict__ dl,
                                                    const Tw *__restrict__ w_r, int T, int k,
                                                    int Tk, int n_shared, int d, float *dx) {
  griddep_wait();
  griddep_launch_dependents();
  const int d4 = d / 4;
  const size_t total = (size_t)T * d4;
  for (size_t id = blockIdx.x * (size_t)blockDim.x + threadIdx.x; id < total;
       id += (size_t)gridDim.x * blockDim.x) {
    const int t = (int)(id / d4), i = 4 * (int)(id % d4);
    float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int j = 0; j < k; ++j) {
      const float4 v = __ldg(reinterpret_cast<const float4 *>(
          dX + (size_t)slot_row[t * k + j] * d + i));
      s.x += v.x;
      s.y += v.y;
      s.z += v.z;
      s.w += v.w;
    }
    if (n_shared) {
      const float4 v = __ldg(reinterpret_cast<const float4 *>(dX + (size_t)(Tk + t) * d + i));
      s.x += v.x;
      s.y += v.y;
      s.z += v.z;
      s.w += v.w;
    }
    for (int j = 0; j < k; ++j) {
      const float g = dl[t * k + j];
      const float4 w = bw_load4(w_r + (size_t)topk_idx[t * k + j] * d + i);
      s.x = fmaf(g, w.x, s.x);
      s.y = fmaf(g, w.y, s.y);
      s.z = fmaf(g, w.z, s.z);
      s.w = fmaf(g, w.w, s.w);
    }
    *reinterpret_cast<float4 *>(dx + (size_t)t * d + i) = s;
  }
}

}  // namespace moe
