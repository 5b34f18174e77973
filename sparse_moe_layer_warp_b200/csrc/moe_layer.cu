// moe_layer.cu -- C ABI of the sparse-MoE FFN layer (declared in include/moe_layer.h) and
// the host logic around the kernels: argument checks, workspace layout, TMA descriptors,
// launch configuration.  The library never allocates device memory.
//
// One call of moe_forward launches, in stream order:
//   router logits -> top-k + chunk histograms -> permutation scatter     (routing.cuh)
//   bf16: [row gather] -> grouped GEMM up+SwiGLU -> grouped GEMM down   (grouped_gemm.cuh)
//         (small token tiles: the up GEMM gathers the rows of x itself)
//   fp32: SIMT up+SwiGLU -> SIMT down                                    (expert_simt.cuh)
//   -> gate-weighted combine                                             (expert_simt.cuh)
// (decode-sized batches: routing in one launch; large groups: CTA-pair GEMMs,
// grouped_gemm_pair.cuh).  One call of moe_backward (bf16) launches:
//   the forward's routing -> row bookkeeping, padded offsets, padded sorted rows
//   -> [up GEMM recompute of a, b] -> DH -> dgate -> DX + weight gradients (one launch on
//   CTA pairs, or two) -> router dl, dW_r -> dx                        (grouped_gemm_bw.cuh)
// and the fp32 layer's backward runs the CUDA-core row kernels of backward.cuh.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#include <mutex>
#include <utility>

#include "moe_layer.h"
#include "backward.cuh"
#include "expert_parallel.cuh"
#include "expert_simt.cuh"
#include "expert_stats.cuh"
#include "grouped_gemm.cuh"
#include "grouped_gemm_bw.cuh"
#include "grouped_gemm_pair.cuh"
#include "ptx_sm100.cuh"
#include "router_stats.cuh"
#include "routing.cuh"

using namespace moe;

struct moe_layer {
  moe_config cfg;
  moe_weights w;
  int device;
  int num_sms;
  int smem_optin;
  int pair_grid[2];  // CTAs of the CTA-pair GEMM (up, down): 2 x co-resident clusters
  CUtensorMap tm_wg, tm_wu, tm_wd, tm_wr;
  CUtensorMap tm_wr2;  // W_r with a box of half the experts (256 < E <= 288, see below)
  // the same weights as MN-major operands of the backward (box {64, 64}): W_gate and W_up
  // as [G*f, d], W_down as [G*d, f]
  CUtensorMap tm_wg_mn, tm_wu_mn, tm_wd_mn;
  int wg_pair_grid;  // CTAs of the CTA-pair weight-gradient kernel (0: not available)
  int bw_pair_grid;  // CTAs of the CTA-pair dgrad kernels (0: not available)
  int tail_pair_grid;  // CTAs of the CTA-pair dx + weight-gradient kernel (0: not available)
  // Per-group hand-over of h from the up to the down GEMM (see GemmParams::done):
  // handover_fits is the init-time occupancy check (every persistent up grid the forward
  // can launch fits on the device at once), opt_handover the caller's switch
  // (MOE_OPTION_H_HANDOVER).  Without it the down GEMM waits for the whole up GEMM.
  int handover_fits;
  int opt_handover;
  int opt_gather_in_gemm;  // MOE_OPTION_ROW_GATHER_IN_GEMM
  int opt_gemm_clock;      // MOE_OPTION_GEMM_CLOCK
  // experts whose weights the handle holds: [e0, e1) (the whole layer: [0, E)); the weight
  // tensors hold e1 - e0 routed experts then the shared expert (moe_layer_init_ep)
  int e0, e1;
  // Shared expert beside the routing (MOE_OPTION_SHARED_SIDE_SMS): a stream of the handle on
  // which the shared expert's up and down GEMMs run while the caller's stream routes, on
  // side_sms SMs (0: off), forked from and joined back into the caller's stream by events.
  int side_sms;
  cudaStream_t side;
  cudaEvent_t ev_fork, ev_join;
};

namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// Row-major bf16 matrix [rows, cols] -> tiled map with box {64 columns, box_rows rows} and
// 128-byte swizzle (the K-major operand layout of the tcgen05 descriptors).
bool encode_bf16_2d(CUtensorMap *m, const void *base, uint64_t cols, uint64_t rows,
                    uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides,
            box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

// Row-major fp32 matrix [rows, cols] -> tiled map with box {32 columns, 32 rows} and
// 128-byte swizzle (the staging tiles of the weight-gradient reductions).
bool encode_f32_2d(CUtensorMap *m, void *base, uint64_t cols, uint64_t rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 4};
  cuuint32_t box[2] = {32, 32};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, base, dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// The same matrix with token-row boxes of 16, 32 and 64 rows (the CTA-pair GEMMs' loads for
// units of few tokens; see GemmParams::tmBr).
bool encode_row_boxes(CUtensorMap (&m)[3], const void *base, uint64_t cols, uint64_t rows) {
  for (int i = 0; i < 3; ++i)
    if (!encode_bf16_2d(&m[i], base, cols, rows, 16u << i)) return false;
  return true;
}

// Every kernel of the library starts with griddepcontrol.wait, so each launch may use
// programmatic stream serialisation: its CTAs can be scheduled (and run their set-up)
// while the previous kernel drains.
template <typename... KArgs, typename... Args>
moe_status launch_cl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                     cudaStream_t st, int cluster, Args &&...args) {
  cudaLaunchConfig_t cfg;
  memset(&cfg, 0, sizeof cfg);
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  int n = 1;
  if (cluster > 1) {
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = cluster;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    n = 2;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...) == cudaSuccess
             ? MOE_OK
             : MOE_ERR_CUDA;
}

template <typename... KArgs, typename... Args>
moe_status launch(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                  Args &&...args) {
  return launch_cl(kern, grid, block, smem, st, 1, std::forward<Args>(args)...);
}

int n_splits(const moe_config &c) { return (c.d_model + kSplitKSlice - 1) / kSplitKSlice; }

size_t esize(const moe_config &c) { return c.dtype == MOE_BF16 ? 2 : 4; }

// Workspace regions (256-byte aligned).  P = T*k + n_shared*T rows of the sorted space.
struct WsLayout {
  size_t status, logits, part, idx, gate, counts, offsets, perm, slot_row, chunk_hist, stats,
      xs, h, y, done, health, total;
};

int pick_bn(const moe_config &c, int T, int mode);

// The bf16 up GEMM gathers its token rows from x when its token tile is small; larger
// tiles read an expert-sorted copy xs written by gather_rows_by_token_kernel.
bool up_gathers_rows(const moe_config &c, int T) {
  return pick_bn(c, T, MODE_UP) <= kGatherMaxBN;
}

WsLayout ws_layout(const moe_config &c, int T) {
  WsLayout L;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off += (bytes + 255) & ~static_cast<size_t>(255);
    return o;
  };
  const size_t Tk = (size_t)T * c.top_k;
  const size_t P = Tk + (size_t)c.n_shared * T;
  const size_t nch = ((size_t)T + kChunk - 1) / kChunk;
  L.status = take(sizeof(DevStatus));
  L.logits = take((size_t)T * c.n_experts * 4);
  L.part = take((T <= kSplitKTokens ? (size_t)n_splits(c) : 0) * T * c.n_experts * 4);
  L.idx = take(Tk * 4);
  L.gate = take(Tk * 4);
  // counts, offsets and chunk histograms hold kMaxTopK more buckets than experts: the drop
  // buckets (one per slot) of an expert-range (partial) forward
  L.counts = take(((size_t)c.n_experts + kMaxTopK) * 4);
  L.offsets = take(((size_t)c.n_experts + kMaxTopK + 1) * 4);
  L.perm = take(Tk * 4);
  L.slot_row = take(Tk * 4);
  L.chunk_hist = take(nch * ((size_t)c.n_experts + kMaxTopK) * 4);
  L.stats = take(nch * (2 * (size_t)c.n_experts + 1) * 4);  // router statistics partials
  L.xs = (c.dtype == MOE_BF16 && !up_gathers_rows(c, T)) ? take(Tk * c.d_model * 2) : off;
  L.h = take(P * c.d_ff * esize(c));
  L.y = take(P * c.d_model * 4);  // fp32 in both precisions
  L.done = take(((size_t)c.n_experts + c.n_shared) * 4);  // per-group up completion counts
  // expert health: slice sums of squares, activations then parameters
  L.health = take(2 * ((size_t)c.n_experts + c.n_shared) * kHealthSlices * 8);
  L.total = off;
  return L;
}

template <typename P>
P *at(void *ws, size_t off) {
  return reinterpret_cast<P *>(static_cast<char *>(ws) + off);
}

int grid_for(size_t work, int per_block, int num_sms) {
  size_t b = (work + per_block - 1) / per_block;
  const size_t cap = (size_t)num_sms * 16;
  if (b > cap) b = cap;
  return b < 1 ? 1 : (int)b;
}

// Token tile of the grouped GEMM from the mean tokens per routed expert.  Larger tiles
// raise the tensor work per staged byte; the smallest tile that holds a typical group keeps
// the token rows a TMA box loads mostly useful.
// The up kernel stops at 128: at 256 its gate + up accumulators fill all 512 TMEM columns,
// the epilogue can no longer overlap the next tile's MMAs, and it runs slower (measured).
int pick_bn(const moe_config &c, int T, int mode) {
  const double mean = (double)T * c.top_k / c.n_experts;
  if (mean <= 4.0) return 16;
  if (mean <= 12.0) return 32;
  if (mean <= 40.0) return 64;
  if (mean <= 160.0 || mode == MODE_UP) return 128;
  return 256;
}

// ------------------------------------------------------------------ routing launches
moe_status launch_gemm_logits(const moe_layer *L, const void *x, int T, float *logits,
                              DevStatus *status, cudaStream_t st);

// Router logits [T][E] into `logits`; for small T the split-K partials go to `part`.
moe_status launch_logits(const moe_layer *L, const void *x, int T, float *logits, float *part,
                         DevStatus *status, cudaStream_t st) {
  const moe_config &c = L->cfg;
  if (T <= kSplitKTokens) {
    dim3 grid((c.n_experts + 31) / 32, n_splits(c));
    if (c.dtype == MOE_BF16)
      return launch(router_logits_splitk_kernel<__nv_bfloat16>, grid, dim3(256), 0, st,
                    static_cast<const __nv_bfloat16 *>(x),
                    static_cast<const __nv_bfloat16 *>(L->w.w_router), T, c.d_model,
                    c.n_experts, part, logits, status->router_ticket);
    return launch(router_logits_splitk_kernel<float>, grid, dim3(256), 0, st,
                  static_cast<const float *>(x), static_cast<const float *>(L->w.w_router), T,
                  c.d_model, c.n_experts, part, logits, status->router_ticket);
  }
  if (c.dtype == MOE_BF16) return launch_gemm_logits(L, x, T, logits, status, st);
  dim3 grid((T + 63) / 64, (c.n_experts + 63) / 64);
  return launch(router_logits_tiled_kernel<float>, grid, dim3(256), 0, st,
                static_cast<const float *>(x), static_cast<const float *>(L->w.w_router), T,
                c.d_model, c.n_experts, logits);
}

// T <= kChunk: selection and permutation in one launch of one CTA.
moe_status launch_route_small(const moe_layer *L, const float *logits, int T, float *logits_out,
                              int *idx, float *gate, int *counts, int *offsets, int *perm,
                              int *slot_row, CounterReset reset, cudaStream_t st) {
  const moe_config &c = L->cfg;
  const int need = (c.n_experts + 31) / 32;
  const float *bias = L->w.router_bias;
  const dim3 thr(kRouteWarps * 32);
#define MOE_SMALL(V)                                                                         \
  launch(route_small_kernel<V>, dim3(1), thr, 0, st, logits, bias, T, c.n_experts, c.top_k, \
         logits_out, idx, gate, counts, offsets, perm, slot_row, reset)
  if (need <= 1) return MOE_SMALL(1);
  if (need <= 2) return MOE_SMALL(2);
  if (need <= 4) return MOE_SMALL(4);
  if (need <= 9) return MOE_SMALL(9);
  if (need <= 16) return MOE_SMALL(16);
  return MOE_SMALL(32);
#undef MOE_SMALL
}

moe_status launch_select_permute(const moe_layer *L, const float *logits, int T,
                                 float *logits_out, int *idx, float *gate, int *counts,
                                 int *offsets, int *perm, int *slot_row, int *chunk_hist,
                                 CounterReset reset, cudaStream_t st,
                                 void *const *events = nullptr, int mark_index = 0) {
  const moe_config &c = L->cfg;
  const int nch = (T + kChunk - 1) / kChunk;
  const int need = (c.n_experts + 31) / 32;
  const float *bias = L->w.router_bias;
  const dim3 thr(kRouteWarps * 32);
  moe_status s;
  if (T <= kChunk) {
    s = launch_route_small(L, logits, T, logits_out, idx, gate, counts, offsets, perm, slot_row,
                           reset, st);
    if (s == MOE_OK && events &&
        cudaEventRecord(static_cast<cudaEvent_t>(events[mark_index]), st) != cudaSuccess)
      return MOE_ERR_CUDA;
    return s;
  }
#define MOE_TOPK(V)                                                                        \
  launch(topk_hist_kernel<V>, dim3(nch), thr, 0, st, logits, bias, T, c.n_experts, c.top_k, \
         logits_out, idx, gate, chunk_hist)
  if (need <= 1) s = MOE_TOPK(1);
  else if (need <= 2) s = MOE_TOPK(2);
  else if (need <= 4) s = MOE_TOPK(4);
  else if (need <= 9) s = MOE_TOPK(9);
  else if (need <= 16) s = MOE_TOPK(16);
  else s = MOE_TOPK(32);
#undef MOE_TOPK
  if (s != MOE_OK) return s;
  if (events && cudaEventRecord(static_cast<cudaEvent_t>(events[mark_index]), st) != cudaSuccess)
    return MOE_ERR_CUDA;
  return launch(permute_scatter_kernel, dim3(nch), dim3(256), 0, st, idx, chunk_hist, T,
                c.n_experts, c.top_k, nch, counts, offsets, perm, slot_row, reset);
}

// ------------------------------------------------------------------ grouped GEMM launch
template <int MODE, int BN>
moe_status launch_gemm_bn(const moe_layer *L, const GemmParams &p, cudaStream_t st) {
  using C = GemmCfg<MODE, BN>;
  const size_t smem = C::smem_bytes(p.n_groups);
  if (smem > (size_t)L->smem_optin) return MOE_ERR_UNSUPPORTED;
  if (cudaFuncSetAttribute(grouped_gemm_kernel<MODE, BN>,
                           cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
      cudaSuccess)
    return MOE_ERR_CUDA;
  return launch(grouped_gemm_kernel<MODE, BN>, dim3(L->num_sms), dim3(kGemmThreads), smem, st,
                p);
}

template <int MODE>
moe_status launch_gemm(const moe_layer *L, int bn, const GemmParams &p, cudaStream_t st) {
  switch (bn) {
    case 16: return launch_gemm_bn<MODE, 16>(L, p, st);
    case 32: return launch_gemm_bn<MODE, 32>(L, p, st);
    case 64: return launch_gemm_bn<MODE, 64>(L, p, st);
  }
  if (bn == 128) return launch_gemm_bn<MODE, 128>(L, p, st);
  if constexpr (MODE == MODE_DOWN) {
    if (bn == 256) return launch_gemm_bn<MODE, 256>(L, p, st);
  }
  return MOE_ERR_UNSUPPORTED;
}

// ------------------------------------------------------------------ CTA-pair GEMM launch
// Large expert groups (prefill) run on CTA pairs: 256 weight rows x 256 tokens per unit.
constexpr double kPairMinMeanTokens = 96.0;

bool use_pair(const moe_layer *L, int T) {
  const moe_config &c = L->cfg;
  const double mean = (double)T * c.top_k / c.n_experts;
  return mean >= kPairMinMeanTokens && c.d_ff % kPairBM == 0 && c.d_model % kPairBM == 0 &&
         L->pair_grid[0] >= 2 && L->pair_grid[1] >= 2;
}

template <int MODE>
size_t pair_smem(const moe_config &c) {
  return PairCfg<MODE>::smem_bytes(c.n_experts + c.n_shared);
}

// CTAs of a persistent pair-kernel grid: two per cluster that can be resident at once.
template <int MODE>
int pair_grid_size(const moe_layer *L) {
  const size_t smem = pair_smem<MODE>(L->cfg);
  if (smem > (size_t)L->smem_optin) return 0;
  if (cudaFuncSetAttribute(grouped_gemm_pair_kernel<MODE>,
                           cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return 0;
  cudaLaunchConfig_t cfg;
  memset(&cfg, 0, sizeof cfg);
  cfg.gridDim = dim3(L->num_sms & ~1);
  cfg.blockDim = dim3(PairCfg<MODE>::THREADS);
  cfg.dynamicSmemBytes = smem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, grouped_gemm_pair_kernel<MODE>, &cfg) != cudaSuccess)
    return 0;
  return 2 * n;
}

// CTAs of the persistent CTA-pair weight-gradient kernel (two per co-resident cluster).
int wgrad_pair_grid_size(const moe_layer *L) {
  const size_t smem = BwWgradPairCfg::smem_bytes(L->cfg.n_experts + L->cfg.n_shared);
  if (smem > (size_t)L->smem_optin) return 0;
  if (cudaFuncSetAttribute(bw_wgrad_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem) != cudaSuccess)
    return 0;
  cudaLaunchConfig_t cfg;
  memset(&cfg, 0, sizeof cfg);
  cfg.gridDim = dim3(L->num_sms & ~1);
  cfg.blockDim = dim3(kWgPairThreads);
  cfg.dynamicSmemBytes = smem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, bw_wgrad_pair_kernel, &cfg) != cudaSuccess) return 0;
  return 2 * n;
}

// CTAs of a persistent cluster-of-two kernel: two per cluster that can be resident at once.
template <typename KP>
int cluster_grid_size(void (*kern)(KP), size_t smem, int threads, const moe_layer *L) {
  if (smem > (size_t)L->smem_optin) return 0;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
      cudaSuccess)
    return 0;
  cudaLaunchConfig_t cfg;
  memset(&cfg, 0, sizeof cfg);
  cfg.gridDim = dim3(L->num_sms & ~1);
  cfg.blockDim = dim3(threads);
  cfg.dynamicSmemBytes = smem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess) return 0;
  return 2 * n;
}

// CTAs of the persistent CTA-pair dgrad kernels (both modes share the configuration).
int dgrad_pair_grid_size(const moe_layer *L) {
  const size_t smem = BwDgradPairCfg::smem_bytes(L->cfg.n_experts + L->cfg.n_shared);
  if (smem > (size_t)L->smem_optin) return 0;
  int n[2] = {0, 0};
  void (*kern[2])(BwDgradParams) = {bw_dgrad_pair_kernel<BW_DH>, bw_dgrad_pair_kernel<BW_DX>};
  for (int i = 0; i < 2; ++i) {
    if (cudaFuncSetAttribute(kern[i], cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
        cudaSuccess)
      return 0;
    cudaLaunchConfig_t cfg;
    memset(&cfg, 0, sizeof cfg);
    cfg.gridDim = dim3(L->num_sms & ~1);
    cfg.blockDim = dim3(kBwPairThreads);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaOccupancyMaxActiveClusters(&n[i], kern[i], &cfg) != cudaSuccess) return 0;
  }
  return 2 * (n[0] < n[1] ? n[0] : n[1]);
}

template <int MODE>
moe_status launch_gemm_pair(const moe_layer *L, const GemmParams &p, cudaStream_t st,
                            int max_ctas = 0) {
  // sized for this launch's groups (the kernel lays out its group table from p.n_groups)
  const size_t smem = PairCfg<MODE>::smem_bytes(p.n_groups);
  if (smem > (size_t)L->smem_optin) return MOE_ERR_UNSUPPORTED;
  if (cudaFuncSetAttribute(grouped_gemm_pair_kernel<MODE>,
                           cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return MOE_ERR_CUDA;
  int grid = L->pair_grid[MODE == MODE_UP ? 0 : 1];
  if (max_ctas >= 2 && max_ctas < grid) grid = max_ctas & ~1;
  return launch_cl(grouped_gemm_pair_kernel<MODE>, dim3(grid), dim3(PairCfg<MODE>::THREADS), smem,
                   st, 2,
                   p);
}

// The per-group hand-over of h lets the down GEMM start while the up GEMM still runs.  Its
// waits end because every up unit is claimed by an up CTA that is resident: a dependent
// launch starts only after every CTA of the up grid has started (and signalled), and a CTA
// leaves only once no unit is left to claim.  The persistent up grids are sized to be
// co-resident (one CTA per SM, or the co-resident cluster count); this check repeats that
// sizing with the occupancy calculator for every up kernel the forward can launch, and the
// forward plans the down GEMM with a whole-grid wait instead when it fails.
template <int BN>
bool up_grid_fits(const moe_layer *L) {
  using C = GemmCfg<MODE_UP, BN>;
  const size_t smem = C::smem_bytes(L->cfg.n_experts + L->cfg.n_shared);
  if (smem > (size_t)L->smem_optin) return true;  // not launchable: the forward refuses it
  if (cudaFuncSetAttribute(grouped_gemm_kernel<MODE_UP, BN>,
                           cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return false;
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, grouped_gemm_kernel<MODE_UP, BN>,
                                                    kGemmThreads, smem) != cudaSuccess)
    return false;
  return (long long)per_sm * L->num_sms >= L->num_sms;  // grid = num_sms CTAs
}

bool up_grids_fit(const moe_layer *L) {
  // the CTA-pair up grid is itself the occupancy calculator's co-resident cluster count
  // (pair_grid_size), so only the one-CTA grids (num_sms CTAs) need the check
  return up_grid_fits<16>(L) && up_grid_fits<32>(L) && up_grid_fits<64>(L) &&
         up_grid_fits<128>(L);
}

// Token tile of the router GEMM.
int pick_bn_router(int T) { return T <= 256 ? 16 : (T <= 1024 ? 32 : 64); }

// Expert tile of the tokens-on-M router GEMM for 256 < E <= 288: two tiles of 144 experts
// (0: tiles of 128).
constexpr int kRouterHalfTile = 144;
int router_half_tile(const moe_config &c) {
  return (c.dtype == MOE_BF16 && c.n_experts > 256 && c.n_experts <= 2 * kRouterHalfTile)
             ? kRouterHalfTile
             : 0;
}

// From this many tokens the router GEMM puts tokens on M (see MODE_LOGITS, out_trans).
constexpr int kRouterTokensOnM = 1024;

moe_status launch_gemm_logits(const moe_layer *L, const void *x, int T, float *logits,
                              DevStatus *status, cudaStream_t st) {
  const moe_config &c = L->cfg;
  GemmParams p;
  memset(&p, 0, sizeof p);
  if (T >= kRouterTokensOnM) {
    // tokens on M (128 per unit), the E experts as the N side in tiles of 128
    if (!encode_bf16_2d(&p.tmA0, x, c.d_model, T, kBM)) return MOE_ERR_CUDA;
    // experts as the N side: tiles of 128 (rows past E zero-filled by TMA), or for
    // 256 < E <= 288 two tiles of half of them, so the units of 128 tokens x one expert tile
    // are 2 per token tile instead of 3 (8192 tokens: 128 units, one wave on 148 SMs)
    const int half = router_half_tile(c);
    p.tmB = half ? L->tm_wr2 : L->tm_wr;
    p.out = logits;
    p.status = status;
    p.E = 0;  // one group of E "rows": the experts
    p.n_groups = 1;
    p.T = c.n_experts;
    p.Tk = 0;
    p.M = T;
    p.K = c.d_model;
    p.ld_out = c.n_experts;
    p.out_trans = 1;
    if (half) return launch_gemm_bn<MODE_LOGITS, kRouterHalfTile>(L, p, st);
    return launch_gemm<MODE_LOGITS>(L, 128, p, st);
  }
  const int bn = pick_bn_router(T);
  p.tmA0 = L->tm_wr;
  if (!encode_bf16_2d(&p.tmB, x, c.d_model, T, bn)) return MOE_ERR_CUDA;
  p.out = logits;
  p.status = status;
  p.E = 0;  // one group: all T tokens, rows [0, T)
  p.n_groups = 1;
  p.T = T;
  p.Tk = 0;
  p.M = c.n_experts;
  p.K = c.d_model;
  p.ld_out = c.n_experts;
  return launch_gemm<MODE_LOGITS>(L, bn, p, st);
}

// The bf16 backward runs its matrix products on the tensor cores (its weight dimensions are
// multiples of the 128-row tile, as the forward requires); the fp32 one on CUDA cores.
bool backward_on_tensor_cores(const moe_config &c) { return c.dtype == MOE_BF16; }

// Backward workspace: the forward's layout, then the backward's own regions.
struct BwLayout {
  size_t row_token, row_group, row_scale, tile_prefix, a, b, dh, db, wide, dgate, dl;
  // tensor-core path: padded expert-sorted rows (bw_rows() of them) of x, dout, da, db,
  // s*h (bf16), the routed groups' padded starts, the (token, slot) pair of each padded
  // row, and the partial sums of dgate
  size_t xs16, dys16, da16, db16, hs16, poff, perm_pad, dgate_part;
  size_t total;
};

// Padded sorted rows of the tensor-core backward: routed groups rounded up to 16 rows
// (at most T*k + 15*E rows), then the shared group at s0 = T*k + 15*E.
int bw_s0(const moe_config &c, int T) { return T * c.top_k + 15 * c.n_experts; }
int bw_rows(const moe_config &c, int T) {
  return bw_s0(c, T) + (c.n_shared ? (T + 15) / 16 * 16 : 0);
}

BwLayout bw_layout(const moe_config &c, int T) {
  BwLayout B;
  size_t off = ws_layout(c, T).total;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off += (bytes + 255) & ~static_cast<size_t>(255);
    return o;
  };
  const bool tc = backward_on_tensor_cores(c);
  const size_t Tk = (size_t)T * c.top_k, P = Tk + (size_t)c.n_shared * T;
  const size_t G = (size_t)c.n_experts + c.n_shared;
  const size_t R = tc ? (size_t)bw_rows(c, T) : P;  // rows of a and b
  B.row_token = take(P * 4);
  B.row_group = take(P * 4);
  B.row_scale = take(P * 4);
  B.tile_prefix = take((G + 1) * 4);
  B.a = take(R * c.d_ff * 4);
  B.b = take(R * c.d_ff * 4);
  B.dh = take(tc ? 0 : P * c.d_ff * 4);
  B.db = take(tc ? 0 : P * c.d_ff * 4);
  B.wide = take(P * c.d_model * 4);  // unscaled expert outputs, then the rows of dx
  B.dgate = take(Tk * 4);
  B.dl = take(Tk * 4);
  const size_t Rt = tc ? R : 0;
  B.xs16 = take(Rt * c.d_model * 2);
  B.dys16 = take(Rt * c.d_model * 2);
  B.da16 = take(Rt * c.d_ff * 2);
  B.db16 = take(Rt * c.d_ff * 2);
  B.hs16 = take(Rt * c.d_ff * 2);
  B.poff = take(tc ? ((size_t)c.n_experts + 1) * 4 : 0);
  B.perm_pad = take(Rt * 4);
  B.dgate_part = take(tc ? Tk * (c.d_ff / 32) * 4 : 0);
  B.total = off;
  return B;
}

moe_status backward_tc(const moe_layer *L, const __nv_bfloat16 *x, const __nv_bfloat16 *dout,
                       int T, float *dx, float *dw_router, float *dw_gate, float *dw_up,
                       float *dw_down, void *ws, cudaStream_t st, const float *saved,
                       bool overwrite);
moe_status backward_f32(const moe_layer *L, const float *x, const float *dout, int T, float *dx,
                        float *dw_router, float *dw_gate, float *dw_up, float *dw_down, void *ws,
                        cudaStream_t st);

// Self-test of the device timeout path: an mbarrier nobody arrives on and a workspace flag
// nobody sets, each waited on with the library's bounded waits (limit_ns), as a stuck
// pipeline would be.  Both give up, leaving the status word set; nothing faults or traps.
__global__ void __launch_bounds__(32) wait_timeout_selftest_kernel(DevStatus *status,
                                                                   unsigned long long limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x != 0) return;
  mbar_init(&bar, 1);
  fence_mbar_init();
  abort_flag = 0;
  mbar_wait_bounded(&bar, 0, &abort_flag, status, 101, limit_ns);
  abort_flag = 0;
  int *flag = &status->pad[25];
  *flag = 0;
  counter_wait_bounded(flag, 1, &abort_flag, status, 102, limit_ns);
}

bool holds_all_experts(const moe_layer *L) { return L->e0 == 0 && L->e1 == L->cfg.n_experts; }

moe_status check_call(const moe_layer *L, int T, void *ws, size_t ws_bytes) {
  if (!L) return MOE_ERR_INVALID_ARG;
  if (T < 0 || T > L->cfg.max_tokens) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  if (!ws || ws_bytes < ws_layout(L->cfg, T).total) return MOE_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return MOE_ERR_ALIGNMENT;
  return MOE_OK;
}

}  // namespace

// =============================================================================== C ABI
extern "C" {

const char *moe_status_string(moe_status s) {
  switch (s) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument";
    case MOE_ERR_UNSUPPORTED: return "unsupported shape";
    case MOE_ERR_ALIGNMENT: return "device pointer not 16-byte aligned";
    case MOE_ERR_WORKSPACE: return "workspace missing or too small";
    case MOE_ERR_CUDA: return "CUDA call or kernel launch failed";
    case MOE_ERR_DEVICE_TIMEOUT: return "a bounded device-side wait gave up";
  }
  return "unknown status";
}

static moe_status layer_init(const moe_config *cfg, const moe_weights *w, int e0, int e1,
                             moe_handle *out) {
  if (!cfg || !w || !out) return MOE_ERR_INVALID_ARG;
  *out = nullptr;
  const moe_config c = *cfg;
  if (e0 < 0 || e1 <= e0 || e1 > c.n_experts) return MOE_ERR_INVALID_ARG;
  if (c.max_tokens < 1 || c.d_model < 1 || c.n_experts < 1 || c.top_k < 1 || c.d_ff < 1)
    return MOE_ERR_INVALID_ARG;
  if (c.top_k > c.n_experts || (c.n_shared != 0 && c.n_shared != 1)) return MOE_ERR_INVALID_ARG;
  if (c.dtype != MOE_F32 && c.dtype != MOE_BF16) return MOE_ERR_INVALID_ARG;
  if (c.top_k > kMaxTopK || c.n_experts > kMaxExperts) return MOE_ERR_UNSUPPORTED;
  if ((long long)c.max_tokens * (c.top_k + c.n_shared) >= (1ll << 31)) return MOE_ERR_UNSUPPORTED;
  if (c.d_model % 8 != 0) return MOE_ERR_UNSUPPORTED;
  if (c.dtype == MOE_BF16 && (c.d_model % kBM != 0 || c.d_ff % kBM != 0))
    return MOE_ERR_UNSUPPORTED;
  if (!w->w_router || !w->w_gate || !w->w_up || !w->w_down) return MOE_ERR_INVALID_ARG;
  if (!aligned16(w->w_router) || !aligned16(w->w_gate) || !aligned16(w->w_up) ||
      !aligned16(w->w_down) || !aligned16(w->router_bias))
    return MOE_ERR_ALIGNMENT;

  moe_layer *L = static_cast<moe_layer *>(calloc(1, sizeof(moe_layer)));
  if (!L) return MOE_ERR_INVALID_ARG;
  L->cfg = c;
  L->w = *w;
  L->e0 = e0;
  L->e1 = e1;

  int major = 0;
  if (cudaGetDevice(&L->device) != cudaSuccess ||
      cudaDeviceGetAttribute(&L->num_sms, cudaDevAttrMultiProcessorCount, L->device) !=
          cudaSuccess ||
      cudaDeviceGetAttribute(&L->smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin,
                             L->device) != cudaSuccess ||
      cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, L->device) !=
          cudaSuccess) {
    free(L);
    return MOE_ERR_CUDA;
  }
  if (major != 10) {  // the library is built for sm_100a only
    free(L);
    return MOE_ERR_UNSUPPORTED;
  }
  L->opt_handover = 1;
  L->opt_gather_in_gemm = 1;
  L->opt_gemm_clock = 0;
  if (c.dtype == MOE_BF16) {
    L->pair_grid[0] = pair_grid_size<MODE_UP>(L);
    L->pair_grid[1] = pair_grid_size<MODE_DOWN>(L);
    L->wg_pair_grid = wgrad_pair_grid_size(L);
    L->bw_pair_grid = dgrad_pair_grid_size(L);
    L->tail_pair_grid = cluster_grid_size(bw_tail_pair_kernel,
                                          BwTailPairCfg::smem_bytes(c.n_experts + c.n_shared),
                                          kWgPairThreads, L);
    L->handover_fits = up_grids_fit(L);
    cudaGetLastError();  // an unavailable cluster query only disables the pair path
    const uint64_t G = (uint64_t)(e1 - e0) + c.n_shared;  // weight groups held
    if (!encode_bf16_2d(&L->tm_wg, w->w_gate, c.d_model, G * c.d_ff, kBM) ||
        !encode_bf16_2d(&L->tm_wu, w->w_up, c.d_model, G * c.d_ff, kBM) ||
        !encode_bf16_2d(&L->tm_wd, w->w_down, c.d_ff, G * c.d_model, kBM) ||
        !encode_bf16_2d(&L->tm_wr, w->w_router, c.d_model, c.n_experts, kBM) ||
        (router_half_tile(c) &&
         !encode_bf16_2d(&L->tm_wr2, w->w_router, c.d_model, c.n_experts,
                         (uint32_t)router_half_tile(c))) ||
        !encode_bf16_2d(&L->tm_wg_mn, w->w_gate, c.d_model, G * c.d_ff, 64) ||
        !encode_bf16_2d(&L->tm_wu_mn, w->w_up, c.d_model, G * c.d_ff, 64) ||
        !encode_bf16_2d(&L->tm_wd_mn, w->w_down, c.d_ff, G * c.d_model, 64)) {
      free(L);
      return MOE_ERR_CUDA;
    }
  }
  *out = L;
  return MOE_OK;
}

moe_status moe_layer_init(const moe_config *cfg, const moe_weights *w, moe_handle *out) {
  return layer_init(cfg, w, 0, cfg ? cfg->n_experts : 0, out);
}

moe_status moe_layer_init_ep(const moe_config *cfg, const moe_weights *w, int expert_begin,
                             int expert_end, moe_handle *out) {
  if (cfg && cfg->dtype != MOE_BF16) return MOE_ERR_UNSUPPORTED;
  return layer_init(cfg, w, expert_begin, expert_end, out);
}

moe_status moe_layer_destroy(moe_handle h) {
  if (!h) return MOE_ERR_INVALID_ARG;
  if (h->side) cudaStreamDestroy(h->side);
  if (h->ev_fork) cudaEventDestroy(h->ev_fork);
  if (h->ev_join) cudaEventDestroy(h->ev_join);
  free(h);
  return MOE_OK;
}

moe_status moe_set_option(moe_handle h, int option, int value) {
  if (!h) return MOE_ERR_INVALID_ARG;
  switch (option) {
    case MOE_OPTION_H_HANDOVER:
      if (value != 0 && value != 1) return MOE_ERR_INVALID_ARG;
      h->opt_handover = value;
      return MOE_OK;
    case MOE_OPTION_SHARED_SIDE_SMS:
      if (value < 0 || value > h->num_sms) return MOE_ERR_INVALID_ARG;
      if (value > 0 && !h->side) {
        int cur = -1;
        if (cudaGetDevice(&cur) != cudaSuccess || cur != h->device) return MOE_ERR_INVALID_ARG;
        if (cudaStreamCreateWithFlags(&h->side, cudaStreamNonBlocking) != cudaSuccess ||
            cudaEventCreateWithFlags(&h->ev_fork, cudaEventDisableTiming) != cudaSuccess ||
            cudaEventCreateWithFlags(&h->ev_join, cudaEventDisableTiming) != cudaSuccess)
          return MOE_ERR_CUDA;
      }
      h->side_sms = value & ~1;  // whole CTA pairs
      return MOE_OK;
    case MOE_OPTION_ROW_GATHER_IN_GEMM:
      if (value < 0 || value > 2) return MOE_ERR_INVALID_ARG;
      h->opt_gather_in_gemm = value;
      return MOE_OK;
    case MOE_OPTION_GEMM_CLOCK:
      if (value != 0 && value != 1) return MOE_ERR_INVALID_ARG;
      h->opt_gemm_clock = value;
      return MOE_OK;
  }
  return MOE_ERR_INVALID_ARG;
}

size_t moe_workspace_size(moe_handle h, int n_tokens) {
  if (!h || n_tokens < 0 || n_tokens > h->cfg.max_tokens) return 0;
  return ws_layout(h->cfg, n_tokens < 1 ? 1 : n_tokens).total;
}

moe_status moe_workspace_init(moe_handle h, void *ws, size_t ws_bytes, void *stream) {
  // zeroes the status word and the router's split-K tickets
  if (!h || !ws || ws_bytes < sizeof(DevStatus)) return MOE_ERR_INVALID_ARG;
  return cudaMemsetAsync(ws, 0, sizeof(DevStatus), static_cast<cudaStream_t>(stream)) ==
                 cudaSuccess
             ? MOE_OK
             : MOE_ERR_CUDA;
}

moe_status moe_selftest_wait_timeout(moe_handle h, void *ws, size_t ws_bytes, int limit_us,
                                     void *stream) {
  if (!h || !ws || ws_bytes < sizeof(DevStatus) || limit_us < 1 || limit_us > 2000000)
    return MOE_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return MOE_ERR_ALIGNMENT;
  return launch(wait_timeout_selftest_kernel, dim3(1), dim3(32), 0,
                static_cast<cudaStream_t>(stream), static_cast<DevStatus *>(ws),
                (unsigned long long)limit_us * 1000ull);
}

size_t moe_backward_workspace_size(moe_handle h, int n_tokens) {
  if (!h || n_tokens < 0 || n_tokens > h->cfg.max_tokens) return 0;
  return bw_layout(h->cfg, n_tokens).total;
}

static moe_status backward_entry(moe_handle h, const void *x, int n_tokens, const void *dout,
                                 const float *saved, bool overwrite, float *dx,
                                 float *dw_router, float *dw_gate, float *dw_up,
                                 float *dw_down, void *ws, size_t ws_bytes, void *stream);

moe_status moe_backward(moe_handle h, const void *x, int n_tokens, const void *dout, float *dx,
                        float *dw_router, float *dw_gate, float *dw_up, float *dw_down,
                        void *ws, size_t ws_bytes, void *stream) {
  return backward_entry(h, x, n_tokens, dout, nullptr, false, dx, dw_router, dw_gate, dw_up,
                        dw_down, ws, ws_bytes, stream);
}

moe_status moe_backward_ex(moe_handle h, const void *x, int n_tokens, const void *dout,
                           const float *saved, size_t saved_bytes, unsigned flags, float *dx,
                           float *dw_router, float *dw_gate, float *dw_up, float *dw_down,
                           void *ws, size_t ws_bytes, void *stream) {
  if (!h) return MOE_ERR_INVALID_ARG;
  if (flags & ~(unsigned)MOE_BACKWARD_OVERWRITE) return MOE_ERR_INVALID_ARG;
  if (saved) {
    if (h->cfg.dtype != MOE_BF16) return MOE_ERR_UNSUPPORTED;
    if (n_tokens > 0 && saved_bytes < moe_saved_size(h, n_tokens)) return MOE_ERR_INVALID_ARG;
    if (!aligned16(saved)) return MOE_ERR_ALIGNMENT;
  }
  return backward_entry(h, x, n_tokens, dout, saved, (flags & MOE_BACKWARD_OVERWRITE) != 0, dx,
                        dw_router, dw_gate, dw_up, dw_down, ws, ws_bytes, stream);
}

moe_status moe_backward_saved(moe_handle h, const void *x, int n_tokens, const void *dout,
                              const float *saved, size_t saved_bytes, float *dx,
                              float *dw_router, float *dw_gate, float *dw_up, float *dw_down,
                              void *ws, size_t ws_bytes, void *stream) {
  if (!h) return MOE_ERR_INVALID_ARG;
  if (h->cfg.dtype != MOE_BF16) return MOE_ERR_UNSUPPORTED;
  if (n_tokens > 0 && !saved) return MOE_ERR_INVALID_ARG;
  return moe_backward_ex(h, x, n_tokens, dout, saved, saved_bytes, 0u, dx, dw_router, dw_gate,
                         dw_up, dw_down, ws, ws_bytes, stream);
}

static moe_status backward_entry(moe_handle h, const void *x, int n_tokens, const void *dout,
                                 const float *saved, bool overwrite, float *dx,
                                 float *dw_router, float *dw_gate, float *dw_up,
                                 float *dw_down, void *ws, size_t ws_bytes, void *stream) {
  if (!h) return MOE_ERR_INVALID_ARG;
  if (n_tokens < 0 || n_tokens > h->cfg.max_tokens) return MOE_ERR_INVALID_ARG;
  if (!holds_all_experts(h)) return MOE_ERR_UNSUPPORTED;  // an expert-parallel slice
  if (n_tokens == 0) return MOE_OK;
  if (!x || !dout || !dx || !dw_router || !dw_gate || !dw_up || !dw_down)
    return MOE_ERR_INVALID_ARG;
  if (!ws || ws_bytes < bw_layout(h->cfg, n_tokens).total) return MOE_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return MOE_ERR_ALIGNMENT;
  if (!aligned16(x) || !aligned16(dout) || !aligned16(dx) || !aligned16(dw_router) ||
      !aligned16(dw_gate) || !aligned16(dw_up) || !aligned16(dw_down))
    return MOE_ERR_ALIGNMENT;
  if (h->cfg.d_ff % 8 != 0) return MOE_ERR_UNSUPPORTED;  // 8-wide weight and gradient rows
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (h->cfg.dtype == MOE_BF16)
    return backward_tc(h, static_cast<const __nv_bfloat16 *>(x),
                       static_cast<const __nv_bfloat16 *>(dout), n_tokens, dx, dw_router, dw_gate,
                       dw_up, dw_down, ws, st, saved, overwrite);
  if (overwrite) {  // fp32 layer: clear, then accumulate
    const moe_config &c = h->cfg;
    const size_t G = (size_t)c.n_experts + c.n_shared, fd = (size_t)c.d_ff * c.d_model;
    if (cudaMemsetAsync(dw_router, 0, (size_t)c.n_experts * c.d_model * 4, st) != cudaSuccess ||
        cudaMemsetAsync(dw_gate, 0, G * fd * 4, st) != cudaSuccess ||
        cudaMemsetAsync(dw_up, 0, G * fd * 4, st) != cudaSuccess ||
        cudaMemsetAsync(dw_down, 0, G * fd * 4, st) != cudaSuccess)
      return MOE_ERR_CUDA;
  }
  return backward_f32(h, static_cast<const float *>(x), static_cast<const float *>(dout),
                      n_tokens, dx, dw_router, dw_gate, dw_up, dw_down, ws, st);
}

moe_status moe_expert_health(moe_handle h, int n_tokens, float *act_rms, float *param_norm,
                             float *ratios, void *ws, size_t ws_bytes, void *stream) {
  moe_status s = check_call(h, n_tokens, ws, ws_bytes);
  if (s != MOE_OK) return s;
  if (!holds_all_experts(h)) return MOE_ERR_UNSUPPORTED;  // an expert-parallel slice
  if (n_tokens == 0 || !act_rms || !param_norm || !ratios) return MOE_ERR_INVALID_ARG;
  const moe_config &c = h->cfg;
  const int T = n_tokens, Tk = T * c.top_k, G = c.n_experts + c.n_shared;
  const WsLayout W = ws_layout(c, T);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  double *act_part = at<double>(ws, W.health);
  double *par_part = act_part + (size_t)G * kHealthSlices;
  const int *offsets = at<int>(ws, W.offsets);
  const dim3 grid(G, kHealthSlices);
  const long long per = (long long)c.d_ff * c.d_model;
  if (c.dtype == MOE_BF16) {
    if ((s = launch(expert_act_sumsq_kernel<__nv_bfloat16>, grid, dim3(256), 0, st,
                    at<const __nv_bfloat16>(ws, W.h), offsets, c.n_experts, T, Tk, c.d_ff,
                    act_part)) != MOE_OK ||
        (s = launch(expert_param_sumsq_kernel<__nv_bfloat16>, grid, dim3(256), 0, st,
                    static_cast<const __nv_bfloat16 *>(h->w.w_gate),
                    static_cast<const __nv_bfloat16 *>(h->w.w_up),
                    static_cast<const __nv_bfloat16 *>(h->w.w_down), per, par_part)) != MOE_OK)
      return s;
  } else {
    if ((s = launch(expert_act_sumsq_kernel<float>, grid, dim3(256), 0, st,
                    at<const float>(ws, W.h), offsets, c.n_experts, T, Tk, c.d_ff,
                    act_part)) != MOE_OK ||
        (s = launch(expert_param_sumsq_kernel<float>, grid, dim3(256), 0, st,
                    static_cast<const float *>(h->w.w_gate),
                    static_cast<const float *>(h->w.w_up),
                    static_cast<const float *>(h->w.w_down), per, par_part)) != MOE_OK)
      return s;
  }
  return launch(expert_health_final_kernel, dim3(1), dim3(1024), 0, st, (const double *)act_part,
                (const double *)par_part, offsets, c.n_experts, G, T, c.d_ff, act_rms,
                param_norm, ratios);
}

moe_status moe_gemm_clock(moe_handle h, void *ws, size_t ws_bytes, double *mhz, void *stream) {
  if (!h || !ws || !mhz || ws_bytes < sizeof(DevStatus)) return MOE_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  DevStatus *d = static_cast<DevStatus *>(ws);
  unsigned long long v[4];
  if (cudaStreamSynchronize(st) != cudaSuccess ||
      cudaMemcpy(v, d->gemm_clock, sizeof v, cudaMemcpyDeviceToHost) != cudaSuccess ||
      cudaMemset(d->gemm_clock, 0, sizeof v) != cudaSuccess)
    return MOE_ERR_CUDA;
  for (int i = 0; i < 2; ++i)  // cycles per microsecond
    mhz[i] = v[2 * i + 1] ? 1e3 * (double)v[2 * i] / (double)v[2 * i + 1] : 0.0;
  return MOE_OK;
}

moe_status moe_device_status(moe_handle h, void *ws, size_t ws_bytes, void *stream) {
  if (!h || !ws || ws_bytes < sizeof(DevStatus)) return MOE_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  DevStatus s;
  if (cudaStreamSynchronize(st) != cudaSuccess) return MOE_ERR_CUDA;
  if (cudaMemcpy(&s, ws, sizeof s, cudaMemcpyDeviceToHost) != cudaSuccess) return MOE_ERR_CUDA;
  if (s.error == 0) return MOE_OK;
  if (cudaMemset(ws, 0, sizeof(DevStatus)) != cudaSuccess) return MOE_ERR_CUDA;
  return MOE_ERR_DEVICE_TIMEOUT;
}

}  // extern "C"

namespace {
// bf16 decode batches: router logits, selection and permutation in one launch
bool decode_route_ok(const moe_config &c, int T) {
  return T <= kChunk && c.dtype == MOE_BF16 && c.n_experts <= kDecodeMaxExperts &&
         c.d_model % (kDecodeWarps * 8) == 0 && c.d_model <= kDecodeMaxD;
}

moe_status launch_route_decode(const moe_layer *L, const void *x, int T, float *logits,
                               int *idx, float *gate, int *counts, int *offsets, int *perm,
                               int *slot_row, DevStatus *status, CounterReset reset,
                               cudaStream_t st) {
  const moe_config &c = L->cfg;
  return launch(route_decode_kernel, dim3((c.n_experts + kDecodeEPC - 1) / kDecodeEPC),
                dim3(kDecodeWarps * 32), 0, st, static_cast<const __nv_bfloat16 *>(x),
                static_cast<const __nv_bfloat16 *>(L->w.w_router), L->w.router_bias, T,
                c.d_model, c.n_experts, c.top_k, logits, idx, gate, counts, offsets, perm,
                slot_row, &status->router_ticket[31], reset);
}
}  // namespace

extern "C" {

static moe_status route_common(moe_handle h, const void *x, const float *logits_in, int T,
                               float *logits_out, int *idx, float *gate, int *counts,
                               int *offsets, int *perm, int *slot_row, void *ws,
                               size_t ws_bytes, void *stream) {
  moe_status s = check_call(h, T, ws, ws_bytes);
  if (s != MOE_OK || T == 0) return s;
  if (!idx || !gate || !counts || !offsets || !perm || !slot_row) return MOE_ERR_INVALID_ARG;
  if (!x && !logits_in) return MOE_ERR_INVALID_ARG;
  if (x && !aligned16(x)) return MOE_ERR_ALIGNMENT;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const WsLayout W = ws_layout(h->cfg, T);
  DevStatus *status = at<DevStatus>(ws, W.status);
  if (!logits_in && decode_route_ok(h->cfg, T)) {
    // the forward's decode routing: logits straight into logits_out when it is given
    float *dst = logits_out ? logits_out : at<float>(ws, W.logits);
    return launch_route_decode(h, x, T, dst, idx, gate, counts, offsets, perm, slot_row, status,
                               CounterReset{status->sched, nullptr, 0}, st);
  }
  const float *logits = logits_in;
  float *copy_out = nullptr;
  if (!logits) {
    float *dst = at<float>(ws, W.logits);
    if ((s = launch_logits(h, x, T, dst, at<float>(ws, W.part), at<DevStatus>(ws, W.status),
                           st)) != MOE_OK)
      return s;
    logits = dst;
    copy_out = logits_out;
  }
  return launch_select_permute(h, logits, T, copy_out, idx, gate, counts, offsets, perm,
                               slot_row, at<int>(ws, W.chunk_hist),
                               CounterReset{at<DevStatus>(ws, W.status)->sched, nullptr, 0}, st);
}

moe_status moe_route(moe_handle h, const void *x, int n_tokens, float *logits_out,
                     int *topk_idx, float *topk_gate, int *expert_counts, int *expert_offsets,
                     int *perm, int *slot_row, void *ws, size_t ws_bytes, void *stream) {
  if (!x) return MOE_ERR_INVALID_ARG;
  return route_common(h, x, nullptr, n_tokens, logits_out, topk_idx, topk_gate, expert_counts,
                      expert_offsets, perm, slot_row, ws, ws_bytes, stream);
}

moe_status moe_route_from_logits(moe_handle h, const float *logits, int n_tokens,
                                 int *topk_idx, float *topk_gate, int *expert_counts,
                                 int *expert_offsets, int *perm, int *slot_row, void *ws,
                                 size_t ws_bytes, void *stream) {
  if (!logits) return MOE_ERR_INVALID_ARG;
  return route_common(h, nullptr, logits, n_tokens, nullptr, topk_idx, topk_gate,
                      expert_counts, expert_offsets, perm, slot_row, ws, ws_bytes, stream);
}

}  // extern "C"

namespace {
// Which kernels a forward of T tokens runs (shared by forward_impl and the launch count).
struct ForwardPlan {
  bool decode_route;  // router logits + selection + permutation in one launch
  bool small_route;   // selection + permutation in one launch after the router
  bool pair;          // CTA-pair grouped GEMMs
  bool gather_in_gemm;  // the up GEMM gathers x rows itself (no gather launch)
  bool gather_in_pair;  // the CTA-pair up GEMM's gather warps write the sorted copy of x
                        // during the shared expert's units (no gather launch)
  bool handover;        // the down GEMM takes h from the up GEMM group by group
  bool side_shared;     // the shared expert's GEMMs run on the side stream during routing
  int launches;
};

// The CTA-pair up GEMM writes the sorted copy of x itself (MOE_OPTION_ROW_GATHER_IN_GEMM):
// 2 always with a shared expert; 1 when the shared expert's n_shared_tokens rows make at
// least one up unit per CTA pair, so the copy's writes have a wave of shared units to overlap.
bool gather_in_pair_ok(const moe_layer *L, bool pair, bool side_shared, int n_shared_tokens) {
  const moe_config &c = L->cfg;
  if (!pair || !c.n_shared || side_shared || n_shared_tokens <= 0) return false;
  if (L->opt_gather_in_gemm == 2) return true;
  const long long units = (long long)(c.d_ff / kPairBM) *
                          ((n_shared_tokens + kPairBN - 1) / kPairBN) * c.n_shared;
  return L->opt_gather_in_gemm == 1 && units >= L->pair_grid[0] / 2;
}

ForwardPlan plan_forward(const moe_layer *L, int T) {
  const moe_config &c = L->cfg;
  ForwardPlan f;
  f.decode_route = decode_route_ok(c, T);
  f.small_route = !f.decode_route && T <= kChunk;
  f.pair = c.dtype == MOE_BF16 && use_pair(L, T);
  f.gather_in_gemm = c.dtype == MOE_BF16 && !f.pair && up_gathers_rows(c, T);
  f.handover = c.dtype == MOE_BF16 && L->handover_fits && L->opt_handover;
  f.side_shared = f.pair && c.n_shared && L->side_sms >= 2 && L->side != nullptr;
  f.gather_in_pair = gather_in_pair_ok(L, f.pair, f.side_shared, T);
  if (T == 0) {
    f.launches = 0;
    return f;
  }
  const int routing = f.decode_route ? 1 : (f.small_route ? 2 : 3);
  const int gather = (c.dtype == MOE_BF16 && !f.gather_in_gemm && !f.gather_in_pair) ? 1 : 0;
  f.launches = routing + gather + 3 + (f.side_shared ? 2 : 0);  // + up, down, combine
  return f;
}

// bf16: the expert-sorted copy of x rows, unless the up GEMM gathers them itself.
moe_status launch_row_gather(const moe_layer *h, const void *x, int T, void *ws,
                             const WsLayout &W, const ForwardPlan &plan, cudaStream_t st,
                             const int *n_rows_dev = nullptr) {
  if (plan.gather_in_gemm || plan.gather_in_pair) return MOE_OK;
  const moe_config &c = h->cfg;
  return launch(gather_rows_by_token_kernel, dim3(grid_for((size_t)T, 8, h->num_sms)),
                dim3(256), 0, st, static_cast<const uint4 *>(x),
                (const int *)at<int>(ws, W.slot_row), T, c.top_k, c.d_model / 8,
                at<uint4>(ws, W.xs), n_rows_dev);
}

// bf16 expert up GEMM over the routing in `ws`: h (bf16, `out`) -- or, with out2 set, the
// fp32 pre-activations x W_g^T (`out`) and x W_u^T (`out2`).  done: the per-group h
// hand-over counts (null: none).  *used receives the parameters (the down GEMM's start).
// Row layout of an up GEMM that does not use the forward's (the backward's padded rows):
// group starts (routed groups; counts from consecutive starts), the (token, slot) pair of
// each row, the shared group's first row, and the sorted copy of x with its row count.
struct UpRows {
  const int *offsets;
  const int *perm;
  int shared_row;
  const void *xs;
  int xs_rows;
};

// Expert-range launch of the expert GEMMs (moe_forward_partial): `n_routed` routed groups
// (the sorted space's first n_routed groups) whose weights start at weight group
// wg_off_routed, and the shared expert (weight group n_routed + wg_off_shared) over the
// shared_n tokens from shared_t0 on.  The whole layer: {E, 0, 0, 0, T}.
struct Slice {
  int n_routed, wg_off_routed, wg_off_shared, shared_t0, shared_n;
};

// gather_rows: the CTA-pair kernel writes the sorted copy of x itself (rows at or past
// *n_rows_dev skipped, when given) and claims the shared group's units first.
moe_status launch_expert_up(const moe_layer *h, const void *x, int T, void *ws,
                            const WsLayout &W, const ForwardPlan &plan, void *out, float *out2,
                            int *done, cudaStream_t st, GemmParams *used,
                            const UpRows *rows = nullptr, float *save_a = nullptr,
                            float *save_b = nullptr, const Slice *slice = nullptr,
                            bool gather_rows = false, const int *n_rows_dev = nullptr) {
  const moe_config &c = h->cfg;
  const int Tk = T * c.top_k;
  // token rows per TMA box: the pair kernels stage half of a 256-token tile per CTA
  const int bn = plan.pair ? PairCfg<MODE_UP>::HALF_BN : pick_bn(c, T, MODE_UP);
  GemmParams &p1 = *used;
  memset(&p1, 0, sizeof p1);
  p1.tmA0 = h->tm_wg;
  p1.tmA1 = h->tm_wu;
  const void *xs = rows ? rows->xs : at<void>(ws, W.xs);
  const int xs_rows = rows ? rows->xs_rows : Tk;
  if (plan.gather_in_gemm) {
    if (!encode_bf16_2d(&p1.tmB, x, c.d_model, T, 1)) return MOE_ERR_CUDA;  // gather4 map
  } else if (!encode_bf16_2d(&p1.tmB, xs, c.d_model, xs_rows, bn) ||
             !encode_bf16_2d(&p1.tmBs, x, c.d_model, T, bn)) {
    return MOE_ERR_CUDA;
  }
  if (plan.pair) {  // smaller token-row boxes for units of few tokens
    if (!encode_row_boxes(p1.tmBr, xs, c.d_model, xs_rows) ||
        !encode_row_boxes(p1.tmBsr, x, c.d_model, T))
      return MOE_ERR_CUDA;
    p1.b_boxes = 1;
  }
  p1.offsets = at<int>(ws, W.offsets);
  p1.perm = at<int>(ws, W.perm);
  p1.topk_gate = at<float>(ws, W.gate);
  p1.out = out;
  p1.out2 = out2;
  p1.status = at<DevStatus>(ws, W.status);
  p1.routed_scale = c.routed_scale;
  p1.E = c.n_experts;
  p1.n_groups = c.n_experts + c.n_shared;
  p1.T = T;
  p1.Tk = Tk;
  p1.M = c.d_ff;
  p1.K = c.d_model;
  p1.ld_out = c.d_ff;
  p1.sched = &at<DevStatus>(ws, W.status)->sched[0];  // dynamic unit claiming
  p1.topk = c.top_k;
  p1.done = done;
  p1.save_a = save_a;
  p1.save_b = save_b;
  if (rows) {
    p1.offsets = rows->offsets;
    p1.perm = rows->perm;
    p1.Tk = rows->shared_row;
  }
  if (slice) {
    p1.E = slice->n_routed;
    p1.n_groups = slice->n_routed + c.n_shared;
    p1.T = slice->shared_n;
    p1.shared_t0 = slice->shared_t0;
    p1.wg_off_routed = slice->wg_off_routed;
    p1.wg_off_shared = slice->wg_off_shared;
  }
  if (h->opt_gemm_clock && !rows) p1.clock_sum = at<DevStatus>(ws, W.status)->gemm_clock;
  if (gather_rows && plan.pair && !rows) {
    DevStatus *status = at<DevStatus>(ws, W.status);
    p1.shared_first = 1;
    p1.gx_src = static_cast<const uint4 *>(x);
    p1.gx_dst = at<uint4>(ws, W.xs);
    p1.gx_slot_row = at<int>(ws, W.slot_row);
    p1.gx_n_rows = n_rows_dev;
    p1.gx_claim = &status->sched[4];
    p1.gx_done = &status->sched[5];
    p1.gx_T = T;
    p1.gx_vec = c.d_model / 8;
  }
  return plan.pair ? launch_gemm_pair<MODE_UP>(h, p1, st) : launch_gemm<MODE_UP>(h, bn, p1, st);
}

// bf16 expert stage of a forward, after the routing: [row gather] -> up + SwiGLU -> down,
// leaving the per-row expert outputs in y.  events (if given) mark the ends of the gather,
// up and down stages (indices 4, 5, 6); slice / n_rows_dev: an expert-range launch.
moe_status launch_experts_bf16(const moe_layer *h, const void *x, int T, void *ws,
                               const WsLayout &W, const ForwardPlan &plan, cudaStream_t st,
                               void *const *events, float *saved, const Slice *slice,
                               const int *n_rows_dev) {
  const moe_config &c = h->cfg;
  const int Tk = T * c.top_k;
  const int P = Tk + (slice ? slice->shared_n : c.n_shared * T);
  auto mark = [&](int i) -> moe_status {
    if (!events) return MOE_OK;
    return cudaEventRecord(static_cast<cudaEvent_t>(events[i]), st) == cudaSuccess ? MOE_OK
                                                                                 : MOE_ERR_CUDA;
  };
  moe_status s;
  ForwardPlan pl = plan;
  // the up kernel gathers the rows while it runs the shared expert's units: an expert-range
  // launch decides by its own shared rows
  if (slice) pl.gather_in_pair = gather_in_pair_ok(h, pl.pair, pl.side_shared, slice->shared_n);
  const bool pair = pl.pair;
  const int bn = pair ? PairCfg<MODE_UP>::HALF_BN : pick_bn(c, T, MODE_UP);
  if ((s = launch_row_gather(h, x, T, ws, W, pl, st, n_rows_dev)) != MOE_OK ||
      (s = mark(4)) != MOE_OK)
    return s;
  const int bn2 = pair ? PairCfg<MODE_DOWN>::HALF_BN : pick_bn(c, T, MODE_DOWN);
  __nv_bfloat16 *hbuf = at<__nv_bfloat16>(ws, W.h);
  // the down kernel starts on the SMs the up kernel leaves in its last wave and waits per
  // expert group for that group's rows of h (see grouped_gemm_kernel)
  GemmParams p1;
  if ((s = launch_expert_up(h, x, T, ws, W, pl, hbuf, nullptr,
                            pl.handover ? at<int>(ws, W.done) : nullptr, st, &p1, nullptr,
                            saved, saved ? saved + (size_t)P * c.d_ff : nullptr, slice,
                            pl.gather_in_pair, n_rows_dev)) != MOE_OK)
    return s;
  if ((s = mark(5)) != MOE_OK) return s;
  GemmParams p2 = p1;  // shared_first carries over: the shared group's h is complete first
  p2.gx_dst = nullptr;
  if (p1.clock_sum) p2.clock_sum = p1.clock_sum + 2;
  p2.tmA0 = h->tm_wd;
  if (!encode_bf16_2d(&p2.tmB, hbuf, c.d_ff, P, bn2)) return MOE_ERR_CUDA;
  p2.b_boxes = 0;
  if (pair) {
    if (!encode_row_boxes(p2.tmBr, hbuf, c.d_ff, P)) return MOE_ERR_CUDA;
    p2.b_boxes = 1;
  }
  p2.out = at<float>(ws, W.y);
  p2.sched = &at<DevStatus>(ws, W.status)->sched[1];
  p2.M = c.d_model;
  p2.K = c.d_ff;
  p2.ld_out = c.d_model;
  // the up kernel's weight tiles per token tile, its token tile and its epilogue warps
  p2.done_mt = c.d_ff / (pair ? kPairBM : kBM);
  p2.done_bn = pair ? kPairBN : bn;
  p2.done_warps = pair ? 2 * kPairEpiWarps : 4;
  if ((s = pair ? launch_gemm_pair<MODE_DOWN>(h, p2, st)
                : launch_gemm<MODE_DOWN>(h, bn2, p2, st)) != MOE_OK)
    return s;
  return mark(6);
}

// The shared expert of a CTA-pair forward on the handle's side stream: forked from `st`
// before the routing (it reads only x and writes only the shared rows of h and y, which no
// routing kernel touches), up and down GEMMs on side_sms SMs with their own work counters,
// and the join event recorded after them (the caller's stream waits for it before the
// combine).
moe_status launch_shared_side(const moe_layer *h, const void *x, int T, void *ws,
                              const WsLayout &W, cudaStream_t st) {
  const moe_config &c = h->cfg;
  const int Tk = T * c.top_k;
  DevStatus *status = at<DevStatus>(ws, W.status);
  cudaStream_t sd = h->side;
  if (cudaEventRecord(h->ev_fork, st) != cudaSuccess ||
      cudaStreamWaitEvent(sd, h->ev_fork, 0) != cudaSuccess ||
      cudaMemsetAsync(status->side_sched, 0, sizeof(status->side_sched), sd) != cudaSuccess)
    return MOE_ERR_CUDA;
  const Slice shared{0, 0, h->e1 - h->e0, 0, T};  // no routed group; weight group E
  __nv_bfloat16 *hbuf = at<__nv_bfloat16>(ws, W.h);
  GemmParams p1;
  memset(&p1, 0, sizeof p1);
  p1.tmA0 = h->tm_wg;
  p1.tmA1 = h->tm_wu;
  if (!encode_bf16_2d(&p1.tmB, x, c.d_model, T, PairCfg<MODE_UP>::HALF_BN) ||
      !encode_bf16_2d(&p1.tmBs, x, c.d_model, T, PairCfg<MODE_UP>::HALF_BN) ||
      !encode_row_boxes(p1.tmBr, x, c.d_model, T) || !encode_row_boxes(p1.tmBsr, x, c.d_model, T))
    return MOE_ERR_CUDA;
  p1.b_boxes = 1;
  p1.offsets = at<int>(ws, W.offsets);  // not read: no routed group
  p1.perm = at<int>(ws, W.perm);
  p1.topk_gate = at<float>(ws, W.gate);
  p1.out = hbuf;
  p1.status = status;
  p1.routed_scale = c.routed_scale;
  p1.E = shared.n_routed;
  p1.n_groups = shared.n_routed + 1;
  p1.T = T;
  p1.Tk = Tk;
  p1.M = c.d_ff;
  p1.K = c.d_model;
  p1.ld_out = c.d_ff;
  p1.sched = &status->side_sched[0];
  p1.topk = c.top_k;
  p1.wg_off_shared = shared.wg_off_shared;
  moe_status s;
  if ((s = launch_gemm_pair<MODE_UP>(h, p1, sd, h->side_sms)) != MOE_OK) return s;
  GemmParams p2 = p1;
  p2.tmA0 = h->tm_wd;
  if (!encode_bf16_2d(&p2.tmB, hbuf, c.d_ff, Tk + T, PairCfg<MODE_DOWN>::HALF_BN) ||
      !encode_row_boxes(p2.tmBr, hbuf, c.d_ff, Tk + T))
    return MOE_ERR_CUDA;
  p2.out = at<float>(ws, W.y);
  p2.sched = &status->side_sched[1];
  p2.M = c.d_model;
  p2.K = c.d_ff;
  p2.ld_out = c.d_model;
  if ((s = launch_gemm_pair<MODE_DOWN>(h, p2, sd, h->side_sms)) != MOE_OK) return s;
  return cudaEventRecord(h->ev_join, sd) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
}  // namespace

extern "C" {

int moe_forward_launch_count(moe_handle h, int n_tokens) {
  if (!h || n_tokens < 0 || n_tokens > h->cfg.max_tokens) return -1;
  return plan_forward(h, n_tokens).launches;
}

static moe_status forward_impl(moe_handle h, const void *x, int n_tokens, void *out, void *ws,
                               size_t ws_bytes, void *stream, void *const *events,
                               float *saved = nullptr) {
  moe_status s = check_call(h, n_tokens, ws, ws_bytes);
  if (s != MOE_OK) return s;
  if (!holds_all_experts(h)) return MOE_ERR_UNSUPPORTED;  // an expert-parallel slice
  if (n_tokens == 0) return MOE_OK;
  if (!x || !out) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(out)) return MOE_ERR_ALIGNMENT;
  const moe_config &c = h->cfg;
  const int T = n_tokens;
  const int Tk = T * c.top_k;
  const int P = Tk + c.n_shared * T;
  const WsLayout W = ws_layout(c, T);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int *idx = at<int>(ws, W.idx);
  float *gate = at<float>(ws, W.gate);
  int *offsets = at<int>(ws, W.offsets);
  int *perm = at<int>(ws, W.perm);
  int *slot_row = at<int>(ws, W.slot_row);
  float *logits = at<float>(ws, W.logits);
  // events[i] (if given) marks the end of stage i (events[0]: the start)
  auto mark = [&](int i) -> moe_status {
    if (!events) return MOE_OK;
    return cudaEventRecord(static_cast<cudaEvent_t>(events[i]), st) == cudaSuccess ? MOE_OK
                                                                                 : MOE_ERR_CUDA;
  };
  if ((s = mark(0)) != MOE_OK) return s;
  // the expert kernels' counters start from zero in every forward
  const CounterReset reset{at<DevStatus>(ws, W.status)->sched, at<int>(ws, W.done),
                           c.n_experts + c.n_shared};
  ForwardPlan plan = plan_forward(h, T);
  // the shared expert beside the routing: not with per-stage events (their stages would
  // overlap) nor with kept pre-activations (the training forward stores all rows in one up
  // launch)
  if (events || saved) {
    plan.side_shared = false;
    plan.gather_in_pair = gather_in_pair_ok(h, plan.pair, false, T);
  }
  if (plan.side_shared && (s = launch_shared_side(h, x, T, ws, W, st)) != MOE_OK) return s;
  if (plan.decode_route) {
    if ((s = launch_route_decode(h, x, T, logits, idx, gate, at<int>(ws, W.counts), offsets,
                                 perm, slot_row, at<DevStatus>(ws, W.status), reset, st)) !=
        MOE_OK)
      return s;
    if ((s = mark(1)) != MOE_OK || (s = mark(2)) != MOE_OK) return s;
  } else {
    if ((s = launch_logits(h, x, T, logits, at<float>(ws, W.part), at<DevStatus>(ws, W.status),
                           st)) != MOE_OK ||
        (s = mark(1)) != MOE_OK)
      return s;
    if (plan.small_route) {
      if ((s = launch_route_small(h, logits, T, nullptr, idx, gate, at<int>(ws, W.counts),
                                  offsets, perm, slot_row, reset, st)) != MOE_OK ||
          (s = mark(2)) != MOE_OK)
        return s;
    } else if ((s = launch_select_permute(h, logits, T, nullptr, idx, gate,
                                          at<int>(ws, W.counts), offsets, perm, slot_row,
                                          at<int>(ws, W.chunk_hist), reset, st, events, 2)) !=
               MOE_OK) {
      return s;
    }
  }
  if ((s = mark(3)) != MOE_OK) return s;

  if (c.dtype == MOE_BF16) {
    const Slice routed_only{c.n_experts, 0, 0, 0, 0};
    if ((s = launch_experts_bf16(h, x, T, ws, W, plan, st, events, saved,
                                 plan.side_shared ? &routed_only : nullptr, nullptr)) != MOE_OK)
      return s;
    if (plan.side_shared && cudaStreamWaitEvent(st, h->ev_join, 0) != cudaSuccess)
      return MOE_ERR_CUDA;
    const float *ybuf = at<float>(ws, W.y);
    if ((s = launch(combine_kernel<__nv_bfloat16>,
                    dim3(grid_for((size_t)T * (c.d_model / 4), 256, h->num_sms)), dim3(256), 0,
                    st, (const float *)ybuf, (const int *)slot_row, T, c.top_k, Tk, c.n_shared,
                    c.d_model, static_cast<__nv_bfloat16 *>(out))) != MOE_OK)
      return s;
    return mark(7);
  }

  float *hbuf = at<float>(ws, W.h);
  float *ybuf = at<float>(ws, W.y);
  if ((s = mark(4)) != MOE_OK) return s;
  if ((s = launch(ffn_up_f32_kernel, dim3(grid_for((size_t)P * c.d_ff, 256, h->num_sms)),
                  dim3(256), 0, st, static_cast<const float *>(x),
                  static_cast<const float *>(h->w.w_gate), static_cast<const float *>(h->w.w_up),
                  (const int *)perm, (const int *)idx, Tk, c.top_k, c.n_experts, P, c.d_model,
                  c.d_ff, hbuf)) != MOE_OK)
    return s;
  if ((s = mark(5)) != MOE_OK) return s;
  if ((s = launch(ffn_down_f32_kernel, dim3(grid_for((size_t)P * c.d_model, 256, h->num_sms)),
                  dim3(256), 0, st, (const float *)hbuf,
                  static_cast<const float *>(h->w.w_down), (const int *)perm, (const int *)idx,
                  (const float *)gate, c.routed_scale, Tk, c.top_k, c.n_experts, P, c.d_model,
                  c.d_ff, ybuf)) != MOE_OK)
    return s;
  if ((s = mark(6)) != MOE_OK) return s;
  if ((s = launch(combine_kernel<float>,
                  dim3(grid_for((size_t)T * (c.d_model / 4), 256, h->num_sms)), dim3(256), 0, st,
                  (const float *)ybuf, (const int *)slot_row, T, c.top_k, Tk, c.n_shared,
                  c.d_model, static_cast<float *>(out))) != MOE_OK)
    return s;
  return mark(7);
}

size_t moe_saved_size(moe_handle h, int n_tokens) {
  if (!h || n_tokens < 0 || n_tokens > h->cfg.max_tokens) return 0;
  const moe_config &c = h->cfg;
  return 2 * (size_t)n_tokens * (c.top_k + c.n_shared) * c.d_ff * sizeof(float);
}

moe_status moe_forward_save(moe_handle h, const void *x, int n_tokens, void *out, float *saved,
                            size_t saved_bytes, void *ws, size_t ws_bytes, void *stream) {
  if (!h) return MOE_ERR_INVALID_ARG;
  if (h->cfg.dtype != MOE_BF16) return MOE_ERR_UNSUPPORTED;
  if (n_tokens < 0 || n_tokens > h->cfg.max_tokens) return MOE_ERR_INVALID_ARG;
  if (n_tokens > 0 && (!saved || saved_bytes < moe_saved_size(h, n_tokens)))
    return MOE_ERR_INVALID_ARG;
  if (saved && !aligned16(saved)) return MOE_ERR_ALIGNMENT;
  return forward_impl(h, x, n_tokens, out, ws, ws_bytes, stream, nullptr, saved);
}

moe_status moe_forward(moe_handle h, const void *x, int n_tokens, void *out, void *ws,
                       size_t ws_bytes, void *stream) {
  return forward_impl(h, x, n_tokens, out, ws, ws_bytes, stream, nullptr);
}

moe_status moe_forward_profiled(moe_handle h, const void *x, int n_tokens, void *out,
                                void *ws, size_t ws_bytes, void *stream, void *const *events,
                                int n_events) {
  if (!events || n_events < MOE_PROFILE_STAGES + 1) return MOE_ERR_INVALID_ARG;
  for (int i = 0; i <= MOE_PROFILE_STAGES; ++i)
    if (!events[i]) return MOE_ERR_INVALID_ARG;
  return forward_impl(h, x, n_tokens, out, ws, ws_bytes, stream, events);
}

moe_status moe_router_stats(moe_handle h, const float *logits, const int *topk_idx,
                            int n_tokens, int n_groups, float *p_mean, float *f_sel,
                            float *scalars, void *ws, size_t ws_bytes, void *stream) {
  moe_status s = check_call(h, n_tokens, ws, ws_bytes);
  if (s != MOE_OK) return s;
  if (n_tokens == 0 || !logits || !topk_idx || !p_mean || !f_sel || !scalars)
    return MOE_ERR_INVALID_ARG;
  const moe_config &c = h->cfg;
  if (n_groups < 1 || c.n_experts % n_groups != 0) return MOE_ERR_INVALID_ARG;
  const WsLayout W = ws_layout(c, n_tokens);
  const int nch = (n_tokens + kChunk - 1) / kChunk;
  float *part_p = at<float>(ws, W.stats);
  int *part_cnt = reinterpret_cast<int *>(part_p + (size_t)nch * c.n_experts);
  float *part_conf = reinterpret_cast<float *>(part_cnt + (size_t)nch * c.n_experts);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t smem = (size_t)kStatWarps * c.n_experts * 4;
  const int need = (c.n_experts + 31) / 32;
#define MOE_STATS(V)                                                                        \
  (cudaFuncSetAttribute(router_stats_partial_kernel<V>,                                     \
                        cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess \
       ? MOE_ERR_CUDA                                                                       \
       : launch(router_stats_partial_kernel<V>, dim3(nch), dim3(kStatWarps * 32), smem, st,  \
                logits, topk_idx, n_tokens, c.n_experts, c.top_k, part_p, part_cnt, part_conf))
  if (need <= 1) s = MOE_STATS(1);
  else if (need <= 2) s = MOE_STATS(2);
  else if (need <= 4) s = MOE_STATS(4);
  else if (need <= 9) s = MOE_STATS(9);
  else if (need <= 16) s = MOE_STATS(16);
  else s = MOE_STATS(32);
#undef MOE_STATS
  if (s != MOE_OK) return s;
  return launch(router_stats_final_kernel, dim3(1), dim3(256), 0, st, (const float *)part_p,
                (const int *)part_cnt, (const float *)part_conf, nch, n_tokens, c.n_experts,
                c.top_k, n_groups, p_mean, f_sel, scalars);
}

moe_status moe_update_router_bias(moe_handle h, const int *expert_counts, int n_tokens,
                                  float gamma, float *bias, void *stream) {
  if (!h || !expert_counts || !bias || n_tokens < 0) return MOE_ERR_INVALID_ARG;
  const moe_config &c = h->cfg;
  return launch(bias_update_kernel, dim3((c.n_experts + 255) / 256), dim3(256), 0,
                static_cast<cudaStream_t>(stream), expert_counts, c.n_experts,
                n_tokens * c.top_k, gamma, bias);
}

}  // extern "C"

// ================================================================ expert parallelism
// The layer split by experts over ranks (expert_parallel.cuh): a forward of an expert range
// returning unrounded fp32 partial outputs, the dispatch plan of an all-to-all exchange, the
// packing of its send buffer and the combine of the partial rows that come back.
extern "C" {

moe_status moe_forward_partial(moe_handle h, const void *x, int n_tokens, const int *topk_idx,
                               const float *topk_gate, int expert_begin, int expert_end,
                               int shared_begin, int shared_end, float *out, void *ws,
                               size_t ws_bytes, void *stream) {
  moe_status s = check_call(h, n_tokens, ws, ws_bytes);
  if (s != MOE_OK) return s;
  const moe_config &c = h->cfg;
  if (c.dtype != MOE_BF16) return MOE_ERR_UNSUPPORTED;
  if (expert_begin < h->e0 || expert_end < expert_begin || expert_end > h->e1)
    return MOE_ERR_INVALID_ARG;
  if (expert_end - expert_begin + c.top_k > kMaxExperts) return MOE_ERR_UNSUPPORTED;
  if (shared_end < shared_begin || shared_begin < 0 || shared_end > n_tokens)
    return MOE_ERR_INVALID_ARG;
  if (shared_end > shared_begin && !c.n_shared) return MOE_ERR_INVALID_ARG;
  if ((topk_idx == nullptr) != (topk_gate == nullptr)) return MOE_ERR_INVALID_ARG;
  if (n_tokens == 0) return MOE_OK;
  if (!x || !out) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(out)) return MOE_ERR_ALIGNMENT;
  const int T = n_tokens, k = c.top_k, Tk = T * k;
  const int El = expert_end - expert_begin;  // routed groups of this launch
  const WsLayout W = ws_layout(c, T);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  DevStatus *status = at<DevStatus>(ws, W.status);
  int *idx = at<int>(ws, W.idx);
  float *gate = at<float>(ws, W.gate);
  int *offsets = at<int>(ws, W.offsets);
  int *perm = at<int>(ws, W.perm);
  int *slot_row = at<int>(ws, W.slot_row);
  int *lidx = at<int>(ws, W.y);  // local groups of the slots (y is written only later)
  const CounterReset reset{status->sched, at<int>(ws, W.done), El + c.n_shared};
  // 1. the selection: given, or the layer's own routing of x (full router, all E experts)
  if (!topk_idx) {
    if ((s = route_common(h, x, nullptr, T, nullptr, idx, gate, at<int>(ws, W.counts), offsets,
                          perm, slot_row, ws, ws_bytes, stream)) != MOE_OK)
      return s;
    topk_idx = idx;
    topk_gate = gate;
  }
  // 2. slots -> local groups (drop bucket El for other experts), sorted by group
  const int nch = (T + kChunk - 1) / kChunk;
  if ((s = launch(ep_local_hist_kernel, dim3(nch), dim3(256), 0, st, topk_idx, topk_gate, T, k,
                  c.n_experts, expert_begin, expert_end, lidx, gate,
                  at<int>(ws, W.chunk_hist))) != MOE_OK ||
      (s = launch(permute_scatter_kernel, dim3(nch), dim3(256), 0, st, (const int *)lidx,
                  (const int *)at<int>(ws, W.chunk_hist), T, El + k, k, nch,
                  at<int>(ws, W.counts), offsets, perm, slot_row, reset)) != MOE_OK)
    return s;
  const int *n_valid = offsets + El;  // rows of the routed groups of this launch
  // 3. the expert GEMMs over the local groups and the shared expert's token range
  const ForwardPlan plan = plan_forward(h, T);
  const Slice slice{El, expert_begin - h->e0, (h->e1 - h->e0) - El, shared_begin,
                    shared_end - shared_begin};
  if ((s = launch_experts_bf16(h, x, T, ws, W, plan, st, nullptr, nullptr, &slice, n_valid)) !=
      MOE_OK)
    return s;
  // 4. per token: its slots in range, then the shared expert, fp32, not rounded
  return launch(combine_partial_kernel,
                dim3(grid_for((size_t)T * (c.d_model / 4), 256, h->num_sms)), dim3(256), 0, st,
                (const float *)at<float>(ws, W.y), (const int *)slot_row, n_valid, T, k, Tk,
                shared_begin, shared_end, c.d_model, out);
}

moe_status moe_ep_plan(moe_handle h, const int *topk_idx, int n_tokens, int n_ranks,
                       int *send_counts, int *send_offsets, int *send_perm, int *send_slot,
                       void *ws, size_t ws_bytes, void *stream) {
  moe_status s = check_call(h, n_tokens, ws, ws_bytes);
  if (s != MOE_OK) return s;
  const moe_config &c = h->cfg;
  if (n_ranks < 1 || 2 * n_ranks > kMaxExperts || c.n_experts % n_ranks != 0)
    return MOE_ERR_INVALID_ARG;
  if (n_tokens == 0) return MOE_OK;
  if (!topk_idx || !send_counts || !send_offsets || !send_perm || !send_slot)
    return MOE_ERR_INVALID_ARG;
  if ((long long)n_tokens * n_ranks >= (1ll << 31)) return MOE_ERR_UNSUPPORTED;
  const WsLayout W = ws_layout(c, n_tokens);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int nch = (n_tokens + kChunk - 1) / kChunk;
  int *pidx = at<int>(ws, W.y);  // (token, rank) buckets: scratch in the expert-output region
  if ((s = launch(ep_plan_mask_kernel, dim3(nch), dim3(256), 0, st, topk_idx, n_tokens,
                  c.top_k, c.n_experts, n_ranks, pidx, at<int>(ws, W.chunk_hist))) != MOE_OK)
    return s;
  return launch(permute_scatter_kernel, dim3(nch), dim3(256), 0, st, (const int *)pidx,
                (const int *)at<int>(ws, W.chunk_hist), n_tokens, 2 * n_ranks, n_ranks, nch,
                send_counts, send_offsets, send_perm, send_slot, CounterReset{nullptr, nullptr, 0});
}

moe_status moe_ep_pack(moe_handle h, const void *x, const int *topk_idx, const float *topk_gate,
                       int n_tokens, int n_ranks, const int *send_perm,
                       const int *send_offsets, void *x_send, int *idx_send, float *gate_send,
                       void *stream) {
  if (!h) return MOE_ERR_INVALID_ARG;
  const moe_config &c = h->cfg;
  if (n_tokens < 0 || n_tokens > c.max_tokens || n_ranks < 1 || c.n_experts % n_ranks != 0)
    return MOE_ERR_INVALID_ARG;
  if (n_tokens == 0) return MOE_OK;
  if (!x || !topk_idx || !topk_gate || !send_perm || !send_offsets || !x_send || !idx_send ||
      !gate_send)
    return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(x_send)) return MOE_ERR_ALIGNMENT;
  const int n_pairs = n_tokens * n_ranks;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const dim3 grid(grid_for((size_t)n_pairs, 8, h->num_sms));
  if (c.dtype == MOE_BF16)
    return launch(ep_pack_kernel<__nv_bfloat16>, grid, dim3(256), 0, st,
                  static_cast<const __nv_bfloat16 *>(x), topk_idx, topk_gate, send_perm,
                  send_offsets, n_ranks, n_pairs, c.d_model, c.top_k,
                  static_cast<__nv_bfloat16 *>(x_send), idx_send, gate_send);
  return launch(ep_pack_kernel<float>, grid, dim3(256), 0, st, static_cast<const float *>(x),
                topk_idx, topk_gate, send_perm, send_offsets, n_ranks, n_pairs, c.d_model,
                c.top_k, static_cast<float *>(x_send), idx_send, gate_send);
}

moe_status moe_ep_combine(moe_handle h, const float *back, const int *send_slot,
                          const int *send_offsets, const float *shared, int n_tokens,
                          int n_ranks, void *out, void *stream) {
  if (!h) return MOE_ERR_INVALID_ARG;
  const moe_config &c = h->cfg;
  if (n_tokens < 0 || n_tokens > c.max_tokens || n_ranks < 1 || c.n_experts % n_ranks != 0)
    return MOE_ERR_INVALID_ARG;
  if (n_tokens == 0) return MOE_OK;
  if (!out || (back && (!send_slot || !send_offsets))) return MOE_ERR_INVALID_ARG;
  if (!aligned16(out) || (back && !aligned16(back)) || (shared && !aligned16(shared)))
    return MOE_ERR_ALIGNMENT;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const dim3 grid(grid_for((size_t)n_tokens * (c.d_model / 4), 256, h->num_sms));
  if (c.dtype == MOE_BF16)
    return launch(ep_combine_kernel<__nv_bfloat16>, grid, dim3(256), 0, st, back, send_slot,
                  send_offsets, shared, n_tokens, n_ranks, c.d_model,
                  static_cast<__nv_bfloat16 *>(out));
  return launch(ep_combine_kernel<float>, grid, dim3(256), 0, st, back, send_slot, send_offsets,
                shared, n_tokens, n_ranks, c.d_model, static_cast<float *>(out));
}

}  // extern "C"

// ================================================== router logits with library-held scratch
// For callers that cannot allocate device memory (see moe_router_logits_static in the
// header): the split-K router's scratch -- partial sums [splits][T][E] and the per-expert-
// block arrival counters -- lives in this file-scope device array instead of a caller
// workspace.  In host code the array's name is only a host-side stand-in, so the device
// address is looked up once per device with cudaGetSymbolAddress and passed to the kernel.
namespace {
constexpr size_t kStaticScratchBytes = size_t(2) << 20;  // partial sums
constexpr int kStaticTickets = 32;                        // one per block of 32 experts
constexpr int kMaxDevices = 64;
static __device__ __align__(256) unsigned char g_router_scratch[kStaticScratchBytes +
                                                                 kStaticTickets * 4];
std::mutex g_static_mu;
void *g_static_ptr[kMaxDevices];  // device address of g_router_scratch per device
}  // namespace

extern "C" moe_status moe_router_logits_static(moe_handle h, const void *x, int n_tokens,
                                               float *logits_out, void *stream) {
  if (!h || !x || !logits_out) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(logits_out)) return MOE_ERR_ALIGNMENT;
  const moe_config &c = h->cfg;
  if (n_tokens < 1 || n_tokens > c.max_tokens) return MOE_ERR_INVALID_ARG;
  const int S = n_splits(c);
  if (n_tokens > kSplitKTokens || (c.n_experts + 31) / 32 > kStaticTickets ||
      (size_t)S * n_tokens * c.n_experts * 4 > kStaticScratchBytes)
    return MOE_ERR_UNSUPPORTED;  // beyond the fixed scratch size
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MOE_ERR_CUDA;
  // the scratch and the launch belong to the current device; the handle's weight pointers
  // to the device it was created on
  if (dev != h->device) return MOE_ERR_INVALID_ARG;
  void *base = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_static_mu);
    if (!g_static_ptr[dev]) {
      void *ptr = nullptr;
      if (cudaGetSymbolAddress(&ptr, g_router_scratch) != cudaSuccess || !ptr)
        return MOE_ERR_CUDA;
      g_static_ptr[dev] = ptr;
    }
    base = g_static_ptr[dev];
  }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  float *part = static_cast<float *>(base);
  int *tickets = reinterpret_cast<int *>(static_cast<char *>(base) + kStaticScratchBytes);
  // the counters must start at zero; the buffer keeps whatever the previous call left
  if (cudaMemsetAsync(tickets, 0, kStaticTickets * 4, st) != cudaSuccess) return MOE_ERR_CUDA;
  dim3 grid((c.n_experts + 31) / 32, S);
  if (c.dtype == MOE_BF16)
    return launch(router_logits_splitk_kernel<__nv_bfloat16>, grid, dim3(256), 0, st,
                  static_cast<const __nv_bfloat16 *>(x),
                  static_cast<const __nv_bfloat16 *>(h->w.w_router), n_tokens, c.d_model,
                  c.n_experts, part, logits_out, tickets);
  return launch(router_logits_splitk_kernel<float>, grid, dim3(256), 0, st,
                static_cast<const float *>(x), static_cast<const float *>(h->w.w_router),
                n_tokens, c.d_model, c.n_experts, part, logits_out, tickets);
}


namespace {

// The forward's routing kernels over x (same experts, gates and sorted order), with the
// grouped GEMMs' work counters reset.
moe_status backward_select(const moe_layer *L, const void *x, int T, void *ws, cudaStream_t st) {
  const WsLayout W = ws_layout(L->cfg, T);
  DevStatus *status = at<DevStatus>(ws, W.status);
  int *idx = at<int>(ws, W.idx), *offsets = at<int>(ws, W.offsets), *perm = at<int>(ws, W.perm);
  int *slot_row = at<int>(ws, W.slot_row), *counts = at<int>(ws, W.counts);
  float *gate = at<float>(ws, W.gate), *logits = at<float>(ws, W.logits);
  const ForwardPlan plan = plan_forward(L, T);
  const CounterReset reset{status->sched, nullptr, 0};
  if (plan.decode_route)
    return launch_route_decode(L, x, T, logits, idx, gate, counts, offsets, perm, slot_row,
                               status, reset, st);
  moe_status s = launch_logits(L, x, T, logits, at<float>(ws, W.part), status, st);
  if (s != MOE_OK) return s;
  return plan.small_route
             ? launch_route_small(L, logits, T, nullptr, idx, gate, counts, offsets, perm,
                                  slot_row, reset, st)
             : launch_select_permute(L, logits, T, nullptr, idx, gate, counts, offsets, perm,
                                     slot_row, at<int>(ws, W.chunk_hist), reset, st);
}

// R: rows of one expert group per tile of the row kernels (16 for decode-sized groups, 64
// when groups average 32 rows or more)
template <typename T_, int R>
moe_status backward_rows(const moe_layer *L, const T_ *x, const T_ *dout, int T, float *dx,
                         float *dw_router, float *dw_gate, float *dw_up, float *dw_down,
                         void *ws, cudaStream_t st) {
  const moe_config &c = L->cfg;
  const int E = c.n_experts, G = E + c.n_shared, k = c.top_k, d = c.d_model, f = c.d_ff;
  const int Tk = T * k, P = Tk + c.n_shared * T;
  const WsLayout W = ws_layout(c, T);
  const BwLayout B = bw_layout(c, T);
  int *idx = at<int>(ws, W.idx), *offsets = at<int>(ws, W.offsets), *perm = at<int>(ws, W.perm);
  int *slot_row = at<int>(ws, W.slot_row);
  float *gate = at<float>(ws, W.gate);
  const T_ *wg = static_cast<const T_ *>(L->w.w_gate);
  const T_ *wu = static_cast<const T_ *>(L->w.w_up);
  const T_ *wd = static_cast<const T_ *>(L->w.w_down);
  const T_ *wr = static_cast<const T_ *>(L->w.w_router);
  moe_status s;
  // 1. the forward's selection (same kernels, so the same experts and gates)
  if ((s = backward_select(L, x, T, ws, st)) != MOE_OK) return s;
  // 2. row bookkeeping
  int *row_token = at<int>(ws, B.row_token), *row_group = at<int>(ws, B.row_group);
  float *row_scale = at<float>(ws, B.row_scale);
  int *tile_prefix = at<int>(ws, B.tile_prefix);
  float *a = at<float>(ws, B.a), *b = at<float>(ws, B.b), *dh = at<float>(ws, B.dh);
  float *db = at<float>(ws, B.db), *wide = at<float>(ws, B.wide);
  float *dgate = at<float>(ws, B.dgate), *dl = at<float>(ws, B.dl);
  if ((s = launch(bw_rows_kernel, dim3(grid_for(P, 256, L->num_sms)), dim3(256), 0, st,
                  (const int *)perm, (const int *)idx, (const float *)gate, T, k, E, c.n_shared,
                  c.routed_scale, row_token, row_group, row_scale)) != MOE_OK ||
      (s = launch(bw_tiles_kernel, dim3(1), dim3(32), 0, st, (const int *)offsets, E, G, T, R,
                  tile_prefix)) != MOE_OK)
    return s;
  const int n_tiles = P / R + G;  // upper bound of the row-tile list
  auto cdiv = [](int n, int m) { return (n + m - 1) / m; };
  const SrcX<T_> src_x{x, row_token, d};
  const SrcDy<T_> src_dy{dout, row_token, row_scale, d};
  const SrcH src_h{a, b, f};
  const SrcRow src_da{dh, f}, src_db{db, f};
  // 3. pre-activations a, b; unscaled expert outputs; dgate
  if ((s = launch(bw_nt_kernel<2, R, T_, SrcX<T_>>, dim3(n_tiles, cdiv(f, 64)), dim3(256), 0, st,
                  wg, wu, f, d, src_x, (const int *)tile_prefix, (const int *)offsets, E, G, T,
                  Tk, a, b)) != MOE_OK)
    return s;
  if ((s = launch(bw_nt_kernel<1, R, T_, SrcH>, dim3(n_tiles, cdiv(d, 64)), dim3(256), 0, st, wd,
                  wd, d, f, src_h, (const int *)tile_prefix, (const int *)offsets, E, G, T, Tk,
                  wide, wide)) != MOE_OK ||
      (s = launch(bw_dgate_kernel<T_>, dim3(grid_for(Tk, 8, L->num_sms)), dim3(256), 0, st,
                  dout, (const float *)wide, (const int *)row_token, (const int *)perm, Tk, d,
                  c.routed_scale, dgate)) != MOE_OK)
    return s;
  // 4. dh, dW_d, then da (over dh) and db
  if ((s = launch(bw_nn_kernel<1, R, T_, SrcDy<T_>, SrcDy<T_>>, dim3(n_tiles, cdiv(f, 64)),
                  dim3(256), 0, st, wd, wd, d, f, src_dy, src_dy, (const int *)tile_prefix,
                  (const int *)offsets, E, G, T, Tk, dh)) != MOE_OK ||
      (s = launch(bw_wgrad_kernel<SrcDy<T_>, SrcH>, dim3(G, cdiv(d, 64), cdiv(f, 128)),
                  dim3(256), 0, st, src_dy, src_h, d, f, (const int *)offsets, E, T, Tk,
                  dw_down)) != MOE_OK ||
      (s = launch(bw_swiglu_kernel, dim3(grid_for((size_t)P * f, 256, L->num_sms)), dim3(256),
                  0, st, (const float *)a, (const float *)b, dh, db, (size_t)P * f)) != MOE_OK)
    return s;
  // 5. rows of dx (over the unscaled outputs, no longer needed), dW_g, dW_u
  if ((s = launch(bw_nn_kernel<2, R, T_, SrcRow, SrcRow>, dim3(n_tiles, cdiv(d, 64)), dim3(256),
                  0, st, wg, wu, f, d, src_da, src_db, (const int *)tile_prefix,
                  (const int *)offsets, E, G, T, Tk, wide)) != MOE_OK ||
      (s = launch(bw_wgrad_kernel<SrcRow, SrcX<T_>>, dim3(G, cdiv(f, 64), cdiv(d, 128)),
                  dim3(256), 0, st, src_da, src_x, f, d, (const int *)offsets, E, T, Tk,
                  dw_gate)) != MOE_OK ||
      (s = launch(bw_wgrad_kernel<SrcRow, SrcX<T_>>, dim3(G, cdiv(f, 64), cdiv(d, 128)),
                  dim3(256), 0, st, src_db, src_x, f, d, (const int *)offsets, E, T, Tk,
                  dw_up)) != MOE_OK)
    return s;
  // 6. router and dx
  if ((s = launch(bw_router_dl_kernel, dim3(grid_for(T, 256, L->num_sms)), dim3(256), 0, st,
                  (const float *)gate, (const float *)dgate, T, k, dl)) != MOE_OK ||
      (s = launch(bw_router_dw_kernel<T_>, dim3(E, cdiv(d, 512)), dim3(256), 0, st, x,
                  (const float *)dl, (const int *)perm, (const int *)offsets, k, d, dw_router,
                  0)) != MOE_OK)
    return s;
  return launch(bw_dx_kernel<T_>, dim3(grid_for((size_t)T * d / 4, 256, L->num_sms)), dim3(256),
                0, st, (const float *)wide, (const int *)slot_row, (const int *)idx,
                (const float *)dl, wr, T, k, Tk, c.n_shared, d, dx);
}

// ------------------------------------------------------- tensor-core backward launches
template <int MODE, int BN>
moe_status launch_bw_dgrad_bn(const moe_layer *L, const BwDgradParams &p, cudaStream_t st) {
  using C = BwDgradCfg<BN>;
  const size_t smem = C::smem_bytes(p.n_groups);
  if (smem > (size_t)L->smem_optin) return MOE_ERR_UNSUPPORTED;
  if (cudaFuncSetAttribute(bw_dgrad_kernel<MODE, BN>,
                           cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
      cudaSuccess)
    return MOE_ERR_CUDA;
  return launch(bw_dgrad_kernel<MODE, BN>, dim3(L->num_sms), dim3(kGemmThreads), smem, st, p);
}

template <int MODE>
moe_status launch_bw_dgrad(const moe_layer *L, int bn, const BwDgradParams &p, cudaStream_t st) {
  switch (bn) {
    case 16: return launch_bw_dgrad_bn<MODE, 16>(L, p, st);
    case 32: return launch_bw_dgrad_bn<MODE, 32>(L, p, st);
    case 64: return launch_bw_dgrad_bn<MODE, 64>(L, p, st);
    case 128: return launch_bw_dgrad_bn<MODE, 128>(L, p, st);
    case 256: return launch_bw_dgrad_bn<MODE, 256>(L, p, st);
  }
  return MOE_ERR_UNSUPPORTED;
}

template <int BNW>
moe_status launch_bw_wgrad(const moe_layer *L, const BwWgradParams &p, cudaStream_t st) {
  using C = BwWgradCfg<BNW>;
  const size_t smem = C::smem_bytes(p.n_groups);
  if (smem > (size_t)L->smem_optin) return MOE_ERR_UNSUPPORTED;
  if (cudaFuncSetAttribute(bw_wgrad_kernel<BNW>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem) != cudaSuccess)
    return MOE_ERR_CUDA;
  return launch(bw_wgrad_kernel<BNW>, dim3(L->num_sms), dim3(kGemmThreads), smem, st, p);
}

template <int MODE>
moe_status launch_bw_dgrad_pair(const moe_layer *L, const BwDgradParams &p, cudaStream_t st) {
  const size_t smem = BwDgradPairCfg::smem_bytes(p.n_groups);
  if (smem > (size_t)L->smem_optin) return MOE_ERR_UNSUPPORTED;
  if (cudaFuncSetAttribute(bw_dgrad_pair_kernel<MODE>,
                           cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return MOE_ERR_CUDA;
  return launch_cl(bw_dgrad_pair_kernel<MODE>, dim3(L->bw_pair_grid), dim3(kBwPairThreads), smem,
                   st, 2, p);
}

moe_status launch_bw_tail_pair(const moe_layer *L, const BwTailParams &p, cudaStream_t st) {
  const size_t smem = BwTailPairCfg::smem_bytes(p.wg.n_groups);
  if (smem > (size_t)L->smem_optin) return MOE_ERR_UNSUPPORTED;
  if (cudaFuncSetAttribute(bw_tail_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem) != cudaSuccess)
    return MOE_ERR_CUDA;
  return launch_cl(bw_tail_pair_kernel, dim3(L->tail_pair_grid), dim3(kWgPairThreads), smem, st,
                   2, p);
}

// Mean routed rows per expert from which the weight gradients run on CTA pairs.
constexpr double kWgradPairMinRows = 16.0;

moe_status launch_bw_wgrad_pair(const moe_layer *L, const BwWgradParams &p, cudaStream_t st) {
  const size_t smem = BwWgradPairCfg::smem_bytes(p.n_groups);
  if (smem > (size_t)L->smem_optin) return MOE_ERR_UNSUPPORTED;
  if (cudaFuncSetAttribute(bw_wgrad_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem) != cudaSuccess)
    return MOE_ERR_CUDA;
  return launch_cl(bw_wgrad_pair_kernel, dim3(L->wg_pair_grid), dim3(kWgPairThreads), smem, st,
                   2, p);
}

// bf16 backward with every matrix product on the tensor cores (grouped_gemm_bw.cuh):
//   selection -> row bookkeeping -> padded sorted bf16 rows of x and dout -> a, b (the
//   forward's up GEMM on the padded rows) -> DH (dh, SwiGLU backward, dgate partials) ->
//   dgate -> DX (rows of dx) -> the three weight gradients in one launch -> router terms
//   and dx.
moe_status backward_tc(const moe_layer *L, const __nv_bfloat16 *x, const __nv_bfloat16 *dout,
                       int T, float *dx, float *dw_router, float *dw_gate, float *dw_up,
                       float *dw_down, void *ws, cudaStream_t st, const float *saved,
                       bool overwrite) {
  const moe_config &c = L->cfg;
  const int E = c.n_experts, G = E + c.n_shared, k = c.top_k, d = c.d_model, f = c.d_ff;
  const int Tk = T * k, P = Tk + c.n_shared * T;
  const int R = bw_rows(c, T);
  const WsLayout W = ws_layout(c, T);
  const BwLayout B = bw_layout(c, T);
  DevStatus *status = at<DevStatus>(ws, W.status);
  int *idx = at<int>(ws, W.idx), *offsets = at<int>(ws, W.offsets), *perm = at<int>(ws, W.perm);
  int *slot_row = at<int>(ws, W.slot_row);
  float *gate = at<float>(ws, W.gate);
  int *row_token = at<int>(ws, B.row_token), *row_group = at<int>(ws, B.row_group);
  float *row_scale = at<float>(ws, B.row_scale);
  float *a = at<float>(ws, B.a), *b = at<float>(ws, B.b), *wide = at<float>(ws, B.wide);
  float *dgate = at<float>(ws, B.dgate), *dl = at<float>(ws, B.dl);
  __nv_bfloat16 *xs = at<__nv_bfloat16>(ws, B.xs16), *dys = at<__nv_bfloat16>(ws, B.dys16);
  __nv_bfloat16 *da = at<__nv_bfloat16>(ws, B.da16), *db = at<__nv_bfloat16>(ws, B.db16);
  __nv_bfloat16 *hs = at<__nv_bfloat16>(ws, B.hs16);
  int *poff = at<int>(ws, B.poff), *perm_pad = at<int>(ws, B.perm_pad);
  float *dgate_part = at<float>(ws, B.dgate_part);
  const __nv_bfloat16 *wr = static_cast<const __nv_bfloat16 *>(L->w.w_router);
  const BwRows rows{offsets, poff, E, T, Tk, bw_s0(c, T)};
  moe_status s;
  if ((s = backward_select(L, x, T, ws, st)) != MOE_OK) return s;
  if ((s = launch(bw_rows_kernel, dim3(grid_for(P, 256, L->num_sms)), dim3(256), 0, st,
                  (const int *)perm, (const int *)idx, (const float *)gate, T, k, E, c.n_shared,
                  c.routed_scale, row_token, row_group, row_scale)) != MOE_OK ||
      (s = launch(bw_pad_offsets_kernel, dim3(1), dim3(32), 0, st, (const int *)offsets, E,
                  poff)) != MOE_OK ||
      (s = launch(bw_sorted_rows_kernel, dim3(grid_for((size_t)R, 8, L->num_sms)), dim3(256), 0,
                  st, x, dout, (const int *)perm, k, rows, c.n_shared, R, d, f, xs, dys, da, db,
                  hs, perm_pad)) != MOE_OK)
    return s;
  // pre-activations a, b: kept by a training forward (unpadded rows), or recomputed by the
  // forward's up GEMM over the padded rows
  const ForwardPlan plan = plan_forward(L, T);
  if (!saved) {
    const UpRows up_rows{poff, perm_pad, rows.s0, xs, R};
    GemmParams pu;
    if ((s = launch_expert_up(L, x, T, ws, W, plan, a, b, nullptr, st, &pu, &up_rows)) != MOE_OK)
      return s;
  }
  // DH (CTA pairs for groups as large as the forward's pair threshold)
  const bool pair_dg = plan.pair && d % 256 == 0 && f % 256 == 0 && L->bw_pair_grid >= 2;
  const int bn = pair_dg ? BwDgradPairCfg::HALF_BN : pick_bn(c, T, MODE_DOWN);
  BwDgradParams pd;
  memset(&pd, 0, sizeof pd);
  pd.tmA0 = L->tm_wd_mn;
  if (!encode_bf16_2d(&pd.tmB0, dys, d, (uint64_t)R, bn)) return MOE_ERR_CUDA;
  pd.rows = rows;
  pd.row_scale = row_scale;
  pd.pre_a = saved ? saved : a;
  pd.pre_b = saved ? saved + (size_t)P * f : b;
  pd.pre_unpadded = saved ? 1 : 0;
  pd.da = da;
  pd.db = db;
  pd.hs = hs;
  pd.dgate_part = dgate_part;
  pd.status = status;
  pd.n_groups = G;
  pd.M = f;
  pd.K = d;
  pd.n_pairs = 1;
  pd.n_part = f / 32;
  pd.sched = &status->sched[1];
  if ((s = pair_dg ? launch_bw_dgrad_pair<BW_DH>(L, pd, st)
                   : launch_bw_dgrad<BW_DH>(L, bn, pd, st)) != MOE_OK ||
      (s = launch(bw_dgate_reduce_kernel, dim3(grid_for(Tk, 256, L->num_sms)), dim3(256), 0, st,
                  (const float *)dgate_part, f / 32, (const int *)perm, Tk, c.routed_scale,
                  dgate)) != MOE_OK)
    return s;
  // DX: rows of dx = W_gate^T da + W_up^T db
  BwDgradParams px = pd;
  px.tmA0 = L->tm_wg_mn;
  px.tmA1 = L->tm_wu_mn;
  if (!encode_bf16_2d(&px.tmB0, da, f, (uint64_t)R, bn) ||
      !encode_bf16_2d(&px.tmB1, db, f, (uint64_t)R, bn))
    return MOE_ERR_CUDA;
  px.out = wide;
  px.M = d;
  px.K = f;
  px.n_pairs = 2;
  px.sched = &status->sched[2];
  // weight gradients: dW_down += dout^T (s h), dW_gate += da^T x, dW_up += db^T x
  BwWgradParams pw;
  memset(&pw, 0, sizeof pw);
  __nv_bfloat16 *ops[kWgOps] = {dys, hs, da, db, xs};
  const int widths[kWgOps] = {d, f, f, f, d};
  for (int i = 0; i < kWgOps; ++i)
    if (!encode_bf16_2d(&pw.box[i], ops[i], widths[i], (uint64_t)R, 64)) return MOE_ERR_CUDA;
  if (!encode_f32_2d(&pw.out[0], dw_down, f, (uint64_t)G * d) ||
      !encode_f32_2d(&pw.out[1], dw_gate, d, (uint64_t)G * f) ||
      !encode_f32_2d(&pw.out[2], dw_up, d, (uint64_t)G * f))
    return MOE_ERR_CUDA;
  const int a_op[kWgProbs] = {0, 2, 3}, b_op[kWgProbs] = {1, 4, 4};
  const int Ms[kWgProbs] = {d, f, f}, Ns[kWgProbs] = {f, d, d};
  for (int i = 0; i < kWgProbs; ++i) {
    pw.a_op[i] = a_op[i];
    pw.b_op[i] = b_op[i];
    pw.M[i] = Ms[i];
    pw.N[i] = Ns[i];
  }
  pw.n_prob = kWgProbs;
  pw.rows = rows;
  pw.status = status;
  pw.n_groups = G;
  pw.sched = &status->sched[3];
  pw.overwrite = overwrite ? 1 : 0;
  // CTA pairs (256 x 256 tiles) when the groups' K loops are long enough for their operand
  // traffic to matter; decode-sized groups (a row or two each) are bound by the gradient
  // read-modify-write, where the one-CTA kernel's shorter per-unit path is faster
  const bool pair_wg = (double)T * k / E >= kWgradPairMinRows;
  if (pair_dg && pair_wg && L->tail_pair_grid >= 2) {
    // dx rows and weight gradients in one launch, their units interleaved
    BwTailParams pt;
    pt.dx = px;
    pt.wg = pw;
    s = launch_bw_tail_pair(L, pt, st);
  } else {
    s = pair_dg ? launch_bw_dgrad_pair<BW_DX>(L, px, st) : launch_bw_dgrad<BW_DX>(L, bn, px, st);
    if (s != MOE_OK) return s;
    if (pair_wg && d % 256 == 0 && f % 256 == 0 && L->wg_pair_grid >= 2)
      s = launch_bw_wgrad_pair(L, pw, st);
    else
      s = (d % 256 == 0 && f % 256 == 0) ? launch_bw_wgrad<256>(L, pw, st)
                                         : launch_bw_wgrad<128>(L, pw, st);
  }
  if (s != MOE_OK) return s;
  // router and dx
  if ((s = launch(bw_router_dl_kernel, dim3(grid_for(T, 256, L->num_sms)), dim3(256), 0, st,
                  (const float *)gate, (const float *)dgate, T, k, dl)) != MOE_OK ||
      (s = launch(bw_router_dw_kernel<__nv_bfloat16>, dim3(E, (d + 511) / 512), dim3(256), 0,
                  st, x, (const float *)dl, (const int *)perm, (const int *)offsets, k, d,
                  dw_router, overwrite ? 1 : 0)) != MOE_OK)
    return s;
  return launch(bw_dx_kernel<__nv_bfloat16>, dim3(grid_for((size_t)T * d / 4, 256, L->num_sms)),
                dim3(256), 0, st, (const float *)wide, (const int *)slot_row, (const int *)idx,
                (const float *)dl, wr, T, k, Tk, c.n_shared, d, dx);
}

// fp32 layer: CUDA-core row kernels (64-row tiles when groups average 32 rows or more)
moe_status backward_f32(const moe_layer *L, const float *x, const float *dout, int T, float *dx,
                        float *dw_router, float *dw_gate, float *dw_up, float *dw_down, void *ws,
                        cudaStream_t st) {
  const moe_config &c = L->cfg;
  const long long P = (long long)T * (c.top_k + c.n_shared);
  const long long G = c.n_experts + c.n_shared;
  if (P >= 32 * G)
    return backward_rows<float, 64>(L, x, dout, T, dx, dw_router, dw_gate, dw_up, dw_down, ws,
                                    st);
  return backward_rows<float, 16>(L, x, dout, T, dx, dw_router, dw_gate, dw_up, dw_down, ws, st);
}

}  // namespace
