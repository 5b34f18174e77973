// expert_parallel.cuh -- the layer split by experts over ranks (expert parallelism).
//
// "Step 3.5 Flash: Open Frontier-Level Intelligence with 11B Active Parameters" deploys the
// MoE layers expert-parallel (section 3: EP8 within a node over NVLink / NVSwitch) and
// balances the load across EP groups of experts (section 2.2.2: the EP-group balance loss
// over G groups).  Here rank q of R holds the experts of EP group q, the E / R consecutive
// expert ids [q E / R, (q + 1) E / R) (the grouping the router statistics use), plus the
// always-on shared expert.  Every rank routes its own tokens with the full router.
//
// The kernels below are the device side of the two exchanges:
//   * partial forward: a rank computes, for the tokens it holds, only the routed slots whose
//     expert lies in its range (ep_local_hist_kernel maps the selection to local expert
//     groups, with one "drop" bucket for the other slots, and the forward's permutation
//     kernel sorts them), and adds the shared expert on a token range it owns;
//     combine_partial_kernel sums those contributions in fp32 without rounding;
//   * dispatch plan (all-to-all): which tokens go to which rank, in a deterministic order
//     (ep_plan_mask_kernel + the permutation kernel over R + 1 buckets), the packing of the
//     send buffer (ep_pack_kernel) and the final combine of the partial rows that come back
//     (ep_combine_kernel: ranks in order, then the shared expert, one rounding).
#pragma once
#include <cuda_bf16.h>
#include <stdint.h>

#include "expert_simt.cuh"
#include "ptx_sm100.cuh"
#include "routing.cuh"

namespace moe {

// Slot (t, j) of the selection -> local group: idx - e0 for an expert in [e0, e1), else the
// drop bucket (e1 - e0) + j of slot j (also for an id outside [0, E): a caller-supplied
// selection is checked, not trusted).  One drop bucket per slot keeps every (token, bucket)
// pair unique, as the permutation kernel's per-bucket token ranks need (a token selects
// distinct experts).  The gate is copied next to it when gate_out differs from gate_in.
// CTA c counts its kChunk tokens per bucket into chunk_hist[c][0 .. e1 - e0 + k).
__global__ void __launch_bounds__(256) ep_local_hist_kernel(
    const int *idx_in, const float *gate_in, int T, int k, int E, int e0, int e1,
    int *lidx_out, float *gate_out, int *__restrict__ chunk_hist) {
  griddep_wait();
  griddep_launch_dependents();
  __shared__ int hist[kMaxExperts];
  const int nb = e1 - e0 + k;  // local groups + one drop bucket per slot
  for (int b = threadIdx.x; b < nb; b += blockDim.x) hist[b] = 0;
  __syncthreads();
  const int c = blockIdx.x;
  const int q0 = c * kChunk * k, q1 = min(T, (c + 1) * kChunk) * k;
  for (int q = q0 + threadIdx.x; q < q1; q += blockDim.x) {
    const int e = idx_in[q];
    const int l = (e >= e0 && e < e1 && e < E) ? e - e0 : (e1 - e0) + q % k;
    if (gate_out != gate_in) gate_out[q] = gate_in[q];
    lidx_out[q] = l;  // may be idx_in itself: each thread rewrites only what it read
    atomicAdd(&hist[l], 1);
  }
  __syncthreads();
  for (int b = threadIdx.x; b < nb; b += blockDim.x) chunk_hist[(size_t)c * nb + b] = hist[b];
}

// out[t, :] = sum over slots j of t (in order) whose row slot_row[t, j] lies below *n_valid
// (the rows of the routed groups this launch computed) of y[row, :], then + y[Tk + t - s0, :]
// for s0 <= t < s1 (the shared expert's rows): fp32, not rounded.
__global__ void __launch_bounds__(256) combine_partial_kernel(
    const float *__restrict__ y, const int *__restrict__ slot_row,
    const int *__restrict__ n_valid, int n_tokens, int k, int Tk, int s0, int s1, int d,
    float *__restrict__ out) {
  griddep_wait();
  griddep_launch_dependents();
  const int valid = *n_valid;
  const int vpr = d / 4;
  const size_t total = (size_t)n_tokens * vpr;
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (size_t)gridDim.x * blockDim.x) {
    const int t = (int)(i / vpr);
    const int c = (int)(i % vpr) * 4;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int j = 0; j < k; ++j) {
      const int p = __ldg(slot_row + (size_t)t * k + j);
      if (p < valid) {
        const float4 v = __ldg(reinterpret_cast<const float4 *>(y + (size_t)p * d + c));
        acc.x += v.x;
        acc.y += v.y;
        acc.z += v.z;
        acc.w += v.w;
      }
    }
    if (t >= s0 && t < s1) {
      const float4 v =
          __ldg(reinterpret_cast<const float4 *>(y + (size_t)(Tk + t - s0) * d + c));
      acc.x += v.x;
      acc.y += v.y;
      acc.z += v.z;
      acc.w += v.w;
    }
    *reinterpret_cast<float4 *>(out + (size_t)t * d + c) = acc;
  }
}

// Dispatch plan, step 1: pair (t, q) of token t and rank q gets bucket q when some slot of t
// selects an expert of rank q's range [q E / R, (q + 1) E / R), else the drop bucket R + q
// (one per rank, so every (token, bucket) pair is unique).  CTA c counts its kChunk tokens'
// pairs per bucket into chunk_hist[c][0 .. 2R).  The forward's permutation kernel then sorts
// the pairs (ascending t within a bucket): rows [0, offsets[R]) are the send order.
__global__ void __launch_bounds__(256) ep_plan_mask_kernel(const int *__restrict__ topk_idx,
                                                           int T, int k, int E, int R,
                                                           int *__restrict__ pidx,
                                                           int *__restrict__ chunk_hist) {
  griddep_wait();
  griddep_launch_dependents();
  __shared__ int hist[kMaxExperts];
  for (int b = threadIdx.x; b < 2 * R; b += blockDim.x) hist[b] = 0;
  __syncthreads();
  const int c = blockIdx.x;
  const int tbeg = c * kChunk, tend = min(T, tbeg + kChunk);
  const int per = E / R;
  for (int pq = threadIdx.x; pq < (tend - tbeg) * R; pq += blockDim.x) {
    const int t = tbeg + pq / R, q = pq % R;
    bool need = false;
    for (int j = 0; j < k; ++j) {
      const int e = topk_idx[(size_t)t * k + j];
      need |= (e >= q * per && e < (q + 1) * per);
    }
    const int b = need ? q : R + q;
    pidx[(size_t)t * R + q] = b;
    atomicAdd(&hist[b], 1);
  }
  __syncthreads();
  for (int b = threadIdx.x; b < 2 * R; b += blockDim.x)
    chunk_hist[(size_t)c * (2 * R) + b] = hist[b];
}

// Send buffer rows r < send_offsets[R]: token t = send_perm[r] / R, its x row (16-byte
// vectors) and its k selected expert ids and gates.  One warp per row.
template <typename Tin>
__global__ void __launch_bounds__(256) ep_pack_kernel(
    const Tin *__restrict__ x, const int *__restrict__ topk_idx,
    const float *__restrict__ topk_gate, const int *__restrict__ send_perm,
    const int *__restrict__ send_offsets, int R, int n_pairs, int d, int k,
    Tin *__restrict__ x_send, int *__restrict__ idx_send, float *__restrict__ gate_send) {
  griddep_wait();
  griddep_launch_dependents();
  const int n_rows = min(send_offsets[R], n_pairs);
  const int lane = threadIdx.x & 31;
  const int n_warps = gridDim.x * (blockDim.x >> 5);
  const int vpr = d * (int)sizeof(Tin) / 16;
  for (int r = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); r < n_rows; r += n_warps) {
    const int t = __ldg(send_perm + r) / R;
    const uint4 *src = reinterpret_cast<const uint4 *>(x + (size_t)t * d);
    uint4 *dst = reinterpret_cast<uint4 *>(x_send + (size_t)r * d);
    for (int v = lane; v < vpr; v += 32) dst[v] = __ldg(src + v);
    for (int j = lane; j < k; j += 32) {
      idx_send[(size_t)r * k + j] = __ldg(topk_idx + (size_t)t * k + j);
      gate_send[(size_t)r * k + j] = __ldg(topk_gate + (size_t)t * k + j);
    }
  }
}

// out[t, :] = round( sum_{q = 0 .. R-1, pair (t, q) sent} back[send_slot[t R + q], :]
//                    + shared[t, :] )
// with back = the partial rows returned by the ranks, in the send buffer's order (null: none)
// and shared = fp32 [T, d] (null: none): fp32 adds in this fixed order, one rounding to the
// output type.
template <typename Tout>
__global__ void __launch_bounds__(256) ep_combine_kernel(
    const float *__restrict__ back, const int *__restrict__ send_slot,
    const int *__restrict__ send_offsets, const float *__restrict__ shared, int n_tokens,
    int R, int d, Tout *__restrict__ out) {
  griddep_wait();
  griddep_launch_dependents();
  const int n_sent = back ? send_offsets[R] : 0;
  const int vpr = d / 4;
  const size_t total = (size_t)n_tokens * vpr;
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (size_t)gridDim.x * blockDim.x) {
    const int t = (int)(i / vpr);
    const int c = (int)(i % vpr) * 4;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    if (back) {
      for (int q = 0; q < R; ++q) {
        const int r = __ldg(send_slot + (size_t)t * R + q);
        if (r < n_sent) {
          const float4 v = __ldg(reinterpret_cast<const float4 *>(back + (size_t)r * d + c));
          acc.x += v.x;
          acc.y += v.y;
          acc.z += v.z;
          acc.w += v.w;
        }
      }
    }
    if (shared) {
      const float4 v = __ldg(reinterpret_cast<const float4 *>(shared + (size_t)t * d + c));
      acc.x += v.x;
      acc.y += v.y;
      acc.z += v.z;
      acc.w += v.w;
    }
    store4(out + (size_t)t * d + c, acc);
  }
}

}  // namespace moe
