// grouped_gemm.cuh -- persistent, warp-specialised grouped expert GEMM on tcgen05.
//
// "Fused MoE gather/scatter with grouped GEMM" ("Step 3.5 Flash: Open Frontier-Level
// Intelligence with 11B Active Parameters", section 3.2.4) over SwiGLU experts with gate
// and up branches ("Step 3.5 Flash 技术论文深度解读", training stability, root cause 3),
// one always-on shared expert (first page, section 2.2) and an explicit routed scale
// (first page, section 4.1.2).
//
// Orientation ("weights on M"): every unit computes D[128 weight rows, n tokens] =
//   W[g][m0:m0+128, :] . B[rows of group g]^T
// so the weight tile is the 128-row MMA A operand and the group's tokens are the N side
// (N = 16 .. 256 in steps of 16, chosen per unit from the group's real token count).  In
// decode a group holds one or two tokens, so this keeps the tensor-core work tiny while
// every SM streams weight tiles from HBM through TMA.
//
//   MODE_UP   : A0 = W_gate, A1 = W_up (two accumulators), B = the group's x rows;
//               epilogue h = silu(G) * U -> bf16 (with out2 set: G and U in fp32, for the
//               backward's recompute).  With token tiles of up to 32 rows the
//               rows are gathered from x by token id with tile::gather4 (four rows per copy:
//               the "gather" of section 3.2.4 fused into the operand load, no expert-sorted
//               copy of x); larger tiles load expert-sorted rows xs written by the gather
//               kernel, and the shared group reads x directly.  (Gathering 128-row tiles,
//               32 gather4 copies per stage, measured 1.6x slower than the row box.)
//   MODE_LOGITS: router logits, fp32 out[t, e].  out_trans = 0: one group of all T tokens,
//               A0 = W_r (rows past E zero-filled by TMA), B = x.  out_trans = 1 (many
//               tokens): A0 = x (128 tokens per unit), one "group" of all E experts as B = W_r,
//               so x is streamed about once and no MMA rows are spent on padding experts.
//   MODE_DOWN : A0 = W_down, B = h rows; epilogue y = acc * scale -> fp32, scale =
//               routed_scale * gate for routed rows and 1 for shared rows.  y stays fp32:
//               rounding it to bf16 as well as h and the output would put the layer's
//               error above 2e-2 x RMS(out) even with exact accumulation.
//
// Roles (192 threads): warp 0 = TMA producer (lane 0 claims units and loads weight tiles;
// in MODE_UP each lane gathers four token rows per stage), warp 1 lane 0 = MMA issuer (warp 1
// also owns the TMEM allocation), warps 2..5 = epilogue (TMEM lane quadrant = warp % 4).
// Pipelines: STAGES shared-memory slots (full / empty mbarriers) and two TMEM accumulator
// buffers (tmem_full / tmem_empty) so the epilogue of unit i overlaps the MMAs of i + 1.
// Every wait is bounded (ptx_sm100.cuh); on a time-out the CTA drains its in-flight
// copies and MMAs, frees TMEM and returns with the workspace status word set.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "ptx_sm100.cuh"

namespace moe {

enum GemmMode { MODE_UP = 0, MODE_DOWN = 1, MODE_LOGITS = 2 };

struct GemmParams {
  CUtensorMap tmA0;  // UP: W_gate [G*f, d]; DOWN: W_down [G*d, f]     box {64, 128}
  CUtensorMap tmA1;  // UP: W_up [G*f, d]                               box {64, 128}
  CUtensorMap tmB;   // UP, BN <= 32: x [T, d] box {64, 1} (tile::gather4 by token id);
                     // UP, BN > 32: xs [Tk, d]; DOWN: h [Tk + n_shared*T, f]; LOGITS: x
                     // (box {64, BN} for all but the gather map)
  CUtensorMap tmBs;  // UP, BN > 32: x [T, d] (shared group)            box {64, BN}
  // CTA-pair kernels with b_boxes set: the same matrices as tmB / tmBs with boxes of 16, 32
  // and 64 rows, so a unit of few tokens stages only the rows it multiplies
  CUtensorMap tmBr[3], tmBsr[3];
  int b_boxes;
  const int *offsets;       // [E + 1] expert offsets in the sorted space
  const int *perm;          // [Tk] sorted row -> t*k + j (UP: token of a row; DOWN: gate)
  const float *topk_gate;   // [Tk] (DOWN)
  void *out;                // UP: h [P, f] bf16; DOWN: y [P, d] fp32; LOGITS: [T, E] fp32
  float *out2;              // UP with out2 set: out = fp32 pre-activation x W_g^T, out2 =
                            // x W_u^T, [P, f] each, instead of h (for the backward)
  float *save_a, *save_b;   // UP, training forward: h to out as usual and, in addition, the
                            // fp32 pre-activations x W_g^T, x W_u^T [P, f] (null: not kept)
  DevStatus *status;
  float routed_scale;
  int E, n_groups, T, Tk;
  int M;      // weight rows per group: f (UP), d (DOWN), E (LOGITS)
  int K;      // reduction length: d (UP, LOGITS) or f (DOWN)
  int ld_out; // f (UP), d (DOWN), E (LOGITS)
  int *sched;  // work counter (zero at launch) for dynamic unit claiming; null: round-robin
  int topk;    // k (UP: token of routed sorted row q = perm[q] / k)
  int out_trans;  // LOGITS: 0 = A is W_r (experts on M), 1 = A is x (tokens on M, B = W_r)
  // Per-group hand-over of h from the up kernel to the down kernel (null: none).  UP: each
  // epilogue warp adds 1 to done[g] once its rows of h for group g are stored.  DOWN: the
  // kernel does not wait for the up kernel to finish; before loading h rows of group g it
  // waits until done[g] = done_warps * done_mt * (token tiles of g at done_bn tokens).
  int *done;
  int done_mt, done_bn;
  int done_warps;  // arrivals per up unit: its epilogue warps (all CTAs of the unit)
  // Expert-range launches (a slice of the layer's experts, e.g. one expert-parallel rank's):
  // routed group g reads the weights of weight group g + wg_off_routed, the shared group
  // (g = E) those of E + wg_off_shared, and the shared group covers the T tokens from x row
  // shared_t0 on.  All zero for the whole layer.
  int wg_off_routed, wg_off_shared;
  int shared_t0;
  // Claim the shared groups' units before all others (build_unit_table).
  int shared_first;
  // CTA-pair up kernel with gx_dst set: its gather warps write the expert-sorted copy of x
  // (gx_dst [rows, d] = gx_src rows; token t to rows gx_slot_row[t*k .. t*k + k), rows at or
  // past *gx_n_rows skipped when gx_n_rows is set) while the shared groups' units, which read
  // x itself, run; a routed unit's loads wait until *gx_done = gx_T.  gx_claim and gx_done
  // are zero at launch; gx_vec = 16-byte vectors per row.
  // Effective SM clock (null: not measured): each CTA adds its SM cycles and %globaltimer ns
  // from entry to exit to clock_sum[0] and clock_sum[1].
  unsigned long long *clock_sum;
  const uint4 *gx_src;
  uint4 *gx_dst;
  const int *gx_slot_row;
  const int *gx_n_rows;
  int *gx_claim, *gx_done;
  int gx_T, gx_vec;
};

// Weight group of work group g (see GemmParams::wg_off_routed).
__device__ __forceinline__ int weight_group(const GemmParams &p, int g) {
  return g + (g < p.E ? p.wg_off_routed : p.wg_off_shared);
}

constexpr int kUnitQ = 4;  // depth of the producer -> MMA/epilogue unit queue
constexpr int kGatherMaxBN = 32;  // MODE_UP token tiles up to this size gather rows from x

// Launches with at most this many groups order their units by cost (build_unit_table);
// larger ones keep the plain group order (the ordered list would not fit in shared memory
// beside the deepest pipelines).
constexpr int kOrderMaxGroups = 512;
__host__ __device__ constexpr int order_words(int n_groups) {
  return n_groups <= kOrderMaxGroups ? n_groups : 0;
}

constexpr int kBM = 128;         // weight rows per unit (MMA M)
constexpr int kBK = 64;          // K per stage: one 128-byte swizzle atom of bf16
constexpr int kGemmThreads = 192;

template <int MODE, int BN>
struct GemmCfg {
  static constexpr int NA = (MODE == MODE_UP) ? 2 : 1;
  static constexpr int A_BYTES = kBM * kBK * 2;
  static constexpr int B_BYTES = BN * kBK * 2;
  static constexpr int STAGE_BYTES = NA * A_BYTES + B_BYTES;
  static constexpr int ACC_COLS = NA * BN;
  // two accumulator buffers (epilogue of unit i overlaps MMAs of unit i+1) when they fit in
  // the 512 TMEM columns; the up kernel at BN = 256 (gate + up = 512 columns) has one
  static constexpr int ACC_BUFS = (2 * ACC_COLS <= 512) ? 2 : 1;
  static constexpr int TMEM_COLS_RAW = ACC_BUFS * ACC_COLS;
  static constexpr int TMEM_COLS = TMEM_COLS_RAW <= 32    ? 32
                                   : TMEM_COLS_RAW <= 64  ? 64
                                   : TMEM_COLS_RAW <= 128 ? 128
                                   : TMEM_COLS_RAW <= 256 ? 256
                                                          : 512;
  static constexpr int SMEM_BUDGET = 208 * 1024;
  static constexpr int STAGES_RAW = SMEM_BUDGET / STAGE_BYTES;
  static constexpr int STAGES = STAGES_RAW > 12 ? 12 : STAGES_RAW;
  static_assert(STAGES >= 2, "pipeline too shallow");
  static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "N of the MMA");
  static_assert(TMEM_COLS_RAW <= 512, "TMEM has 512 columns");
  // barriers: full[S], empty[S], tfull[2], tempty[2], drain[1], uq_full[Q], uq_empty[Q]
  static constexpr int BAR_BYTES = (2 * STAGES + 5 + 2 * kUnitQ) * 8;
  static constexpr size_t smem_bytes(int n_groups) {
    return 1024 /*alignment slack*/ + (size_t)STAGES * STAGE_BYTES + BAR_BYTES + 64 +
           (size_t)(3 * n_groups + 1 + order_words(n_groups)) * 4 +
           ACC_BUFS * BN * 4 /*row scales*/ +
           4 * 16 * 32 * 4 /*epilogue transpose buffers*/ + 16 /*alignment*/;
  }
};

// silu(g) * u with the fast exponential and division (relative error ~1e-6, far below the
// bf16 rounding of the result); silu(z) = z / (1 + exp(-z)) -> 0 for z -> -inf.
__device__ __forceinline__ float swiglu(float g, float u) {
  return __fdividef(g, 1.f + __expf(-g)) * u;
}

// Epilogue store of one 32-row x 16-token block held by a warp (lane = row, vals[n] = token
// column c0 + n) into a row-major [token][column] output: the block is transposed through a
// per-warp shared-memory buffer (16 x 32 fp32) so every lane writes 16-byte vectors along an
// output row.  Rows (tokens) at or past `valid` are not written.
__device__ __forceinline__ void store_block16_bf16(__nv_bfloat16 *out, int ld, int row0, int c0,
                                                   int valid, int col_base, const float (&vals)[16],
                                                   float *wbuf, int lane) {
#pragma unroll
  for (int n = 0; n < 16; ++n) wbuf[n * 32 + lane] = vals[n];
  __syncwarp();
#pragma unroll
  for (int i = 0; i < 2; ++i) {  // 16 tokens x 4 chunks of 8 columns = 64 chunks
    const int c = lane + 32 * i;
    const int j = c >> 2, k = c & 3;
    if (c0 + j < valid) {
      const float4 a = *reinterpret_cast<const float4 *>(wbuf + j * 32 + 8 * k);
      const float4 b = *reinterpret_cast<const float4 *>(wbuf + j * 32 + 8 * k + 4);
      uint4 v;
      *reinterpret_cast<__nv_bfloat162 *>(&v.x) = __floats2bfloat162_rn(a.x, a.y);
      *reinterpret_cast<__nv_bfloat162 *>(&v.y) = __floats2bfloat162_rn(a.z, a.w);
      *reinterpret_cast<__nv_bfloat162 *>(&v.z) = __floats2bfloat162_rn(b.x, b.y);
      *reinterpret_cast<__nv_bfloat162 *>(&v.w) = __floats2bfloat162_rn(b.z, b.w);
      *reinterpret_cast<uint4 *>(out + (size_t)(row0 + c0 + j) * ld + col_base + 8 * k) = v;
    }
  }
  __syncwarp();
}

__device__ __forceinline__ void store_block16_f32(float *out, int ld, int row0, int c0,
                                                  int valid, int col_base, const float (&vals)[16],
                                                  float *wbuf, int lane) {
#pragma unroll
  for (int n = 0; n < 16; ++n) wbuf[n * 32 + lane] = vals[n];
  __syncwarp();
#pragma unroll
  for (int i = 0; i < 4; ++i) {  // 16 tokens x 8 chunks of 4 columns = 128 chunks
    const int c = lane + 32 * i;
    const int j = c >> 3, k = c & 7;
    if (c0 + j < valid)
      *reinterpret_cast<float4 *>(out + (size_t)(row0 + c0 + j) * ld + col_base + 4 * k) =
          *reinterpret_cast<const float4 *>(wbuf + j * 32 + 4 * k);
  }
  __syncwarp();
}

// Work list of a grouped GEMM launch, built by every CTA from the routing's offsets:
// grp_count / grp_row [G] by group id; order [G] = the shared groups when p.shared_first is
// set ("first"), then the groups with at least one full token tile of BN rows ("heavy":
// tensor-bound, their weight tiles shared by several token tiles), then the others ("light":
// a few tokens each, bound by streaming their weights from HBM), each class in id order;
// unit_prefix [G + 1] = exclusive prefix of the units (m tiles x token tiles) over that
// order.  *n_first = units of the first class, *n_heavy = units of the heavy class.  With more
// than kOrderMaxGroups groups the order is the identity (no array) and both are 0.  Called by
// all threads of the CTA (it synchronises them).
template <int BN>
__device__ __forceinline__ void build_unit_table(const GemmParams &p, int mtiles,
                                                 int *unit_prefix, int *grp_count,
                                                 int *grp_row, int *order, int *n_first,
                                                 int *n_heavy) {
  const int G = p.n_groups;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int g = threadIdx.x; g < G; g += blockDim.x) {
    int cnt, row;
    if (g < p.E) {
      row = p.offsets[g];
      cnt = p.offsets[g + 1] - row;
    } else {
      row = p.Tk + (g - p.E) * p.T;
      cnt = p.T;
    }
    grp_count[g] = cnt;
    grp_row[g] = row;
  }
  __syncthreads();
  if (warp == 0) {
    // each lane a contiguous run of groups, partitioned stably into the three classes
    const int per = (G + 31) / 32;
    const int lo = min(G, lane * per), hi = min(G, lo + per);
    auto cls = [&](int g) {
      return (p.shared_first && g >= p.E) ? 0 : (grp_count[g] >= BN ? 1 : 2);
    };
    int nf = 0, nh = 0;
    if (order)
      for (int g = lo; g < hi; ++g) {
        const int c = cls(g);
        nf += c == 0;
        nh += c == 1;
      }
    int inf = nf, inh = nh;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int yf = __shfl_up_sync(0xffffffffu, inf, o);
      const int yh = __shfl_up_sync(0xffffffffu, inh, o);
      if (lane >= o) {
        inf += yf;
        inh += yh;
      }
    }
    const int first_groups = __shfl_sync(0xffffffffu, inf, 31);
    const int heavy_groups = __shfl_sync(0xffffffffu, inh, 31);
    int fpos = inf - nf, hpos = first_groups + inh - nh;
    int lpos = first_groups + heavy_groups + (lo - (inf - nf) - (inh - nh));
    if (order)
      for (int g = lo; g < hi; ++g) {
        const int c = cls(g);
        if (c == 0) order[fpos++] = g;
        else if (c == 1) order[hpos++] = g;
        else order[lpos++] = g;
      }
    __syncwarp();
    // exclusive scan of the units over the ordered positions
    auto grp_at = [&](int i) { return order ? order[i] : i; };
    int run = 0;
    for (int i = lo; i < hi; ++i) run += mtiles * ((grp_count[grp_at(i)] + BN - 1) / BN);
    int incl = run;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    int excl = incl - run;
    for (int i = lo; i < hi; ++i) {
      const int u = mtiles * ((grp_count[grp_at(i)] + BN - 1) / BN);
      unit_prefix[i] = excl;
      excl += u;
    }
    if (lane == 31) unit_prefix[G] = incl;
    __syncwarp();
    if (lane == 0) {
      *n_first = unit_prefix[first_groups];
      *n_heavy = unit_prefix[first_groups + heavy_groups] - unit_prefix[first_groups];
    }
  }
  __syncthreads();
}

// Claim order: ticket c of [0, total) -> unit.  The first n_first tickets take the first
// class's units in order; over the rest the heavy units (the next n_heavy of the ordered
// list) are spread evenly (ticket c' = c - n_first of rest = total - n_first is heavy iff
// floor((c'+1) n_heavy / rest) > floor(c' n_heavy / rest)) and the light ones fill the gaps in
// order, so the CTAs run tensor-bound and HBM-bound units side by side instead of one kind
// after the other.  A bijection of [0, total).
__device__ __forceinline__ int unit_of_ticket(int c, int n_first, int n_heavy, int total) {
  if (c < n_first) return c;
  c -= n_first;
  const int rest = total - n_first;
  const long long h0 = (long long)c * n_heavy / rest;
  const long long h1 = (long long)(c + 1) * n_heavy / rest;
  return n_first + (h1 > h0 ? (int)h0 : n_heavy + (c - (int)h0));
}

// unit -> (group, m tile, token tile) over the ordered list: token tile innermost, so the
// units that share a weight tile are claimed close together and run at about the same time
// on different SMs (the tile is read from HBM about once).
__device__ __forceinline__ void decode_unit(int u, int G, const int *unit_prefix,
                                            const int *order, const int *grp_count, int bn,
                                            int &g, int &mt, int &nt) {
  int lo = 0, hi = G - 1;
  while (lo < hi) {  // last position with unit_prefix <= u
    const int mid = (lo + hi + 1) >> 1;
    if (unit_prefix[mid] <= u) lo = mid;
    else hi = mid - 1;
  }
  g = order ? order[lo] : lo;
  const int nts = (grp_count[g] + bn - 1) / bn;
  const int loc = u - unit_prefix[lo];
  mt = loc / nts;
  nt = loc % nts;
}

template <int MODE, int BN>
__global__ void __launch_bounds__(kGemmThreads, 1)
    grouped_gemm_kernel(const __grid_constant__ GemmParams p) {
  using C = GemmCfg<MODE, BN>;
  constexpr int S = C::STAGES;
  constexpr bool kGather = (MODE == MODE_UP) && (BN <= kGatherMaxBN);
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t *sA0 = smem;
  uint8_t *sA1 = sA0 + S * C::A_BYTES;  // only used by MODE_UP
  uint8_t *sB = sA0 + C::NA * S * C::A_BYTES;
  uint64_t *bars = reinterpret_cast<uint64_t *>(sB + S * C::B_BYTES);
  uint64_t *full = bars;
  uint64_t *empty = bars + S;
  uint64_t *tfull = bars + 2 * S;
  uint64_t *tempty = bars + 2 * S + 2;
  uint64_t *drain = bars + 2 * S + 4;
  uint64_t *uq_full = bars + 2 * S + 5;
  uint64_t *uq_empty = uq_full + kUnitQ;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(uq_empty + kUnitQ);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
  volatile int *uq = reinterpret_cast<volatile int *>(tmem_slot + 4);  // [kUnitQ] unit ids
  int *n_heavy_s = reinterpret_cast<int *>(tmem_slot + 8);
  int *n_first_s = reinterpret_cast<int *>(tmem_slot + 9);
  uint64_t *epi_bar = reinterpret_cast<uint64_t *>(tmem_slot + 2);  // epilogue warps' barrier
  ClockSpan *span = reinterpret_cast<ClockSpan *>(tmem_slot + 12);  // effective-clock probe
  if (p.clock_sum && threadIdx.x == 0) *span = clock_span_start();
  int *unit_prefix = reinterpret_cast<int *>(tmem_slot + 16);  // [G + 1]
  int *grp_count = unit_prefix + p.n_groups + 1;                // [G]
  int *grp_row = grp_count + p.n_groups;                        // [G]
  // [G] when G <= kOrderMaxGroups, else none (identity order)
  int *order = order_words(p.n_groups) ? grp_row + p.n_groups : nullptr;
  // [ACC_BUFS][BN], 16-byte aligned: read as float4
  float *row_scale = reinterpret_cast<float *>(
      (reinterpret_cast<uintptr_t>(grp_row + p.n_groups + order_words(p.n_groups)) + 15) &
      ~static_cast<uintptr_t>(15));
  float *xbuf = row_scale + C::ACC_BUFS * BN;  // [4 warps][16][32] epilogue transposes

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = p.n_groups;
  const int mtiles = (p.M + kBM - 1) / kBM;
  const int kblocks = p.K / kBK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 128);
    }
    mbar_init(drain, 1);
    mbar_init(epi_bar, 4);
    for (int q = 0; q < kUnitQ; ++q) {
      mbar_init(&uq_full[q], 1);
      mbar_init(&uq_empty[q], 5);  // the MMA thread and the four epilogue warps
    }
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&p.tmA0);
    if (MODE == MODE_UP) {
      tma_prefetch_desc(&p.tmA1);
      if (BN > kGatherMaxBN) tma_prefetch_desc(&p.tmBs);
    }
    tma_prefetch_desc(&p.tmB);
  }
  if (warp == 1) tmem_alloc(tmem_slot, C::TMEM_COLS);
  // Programmatic dependent launch: the set-up above overlaps the previous kernel's tail;
  // the expert offsets, the token rows and the outputs may all belong to it, so everything
  // below waits for it to complete.  A down kernel with the per-group hand-over (p.done)
  // only reads what the routing kernel wrote, complete before the up kernel (its
  // predecessor) could let it launch, and h, which it takes group by group through done[].
  if (!(MODE == MODE_DOWN && p.done)) griddep_wait();
  griddep_launch_dependents();
  // group table (token count, first row in the sorted space) and the cost-ordered work list
  build_unit_table<BN>(p, mtiles, unit_prefix, grp_count, grp_row, order, n_first_s,
                       n_heavy_s);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int total_units = unit_prefix[G];
  const int n_heavy = *n_heavy_s;
  const int n_first = *n_first_s;

  auto decode = [&](int u, int &g, int &mt, int &nt) {
    decode_unit(u, G, unit_prefix, order, grp_count, BN, g, mt, nt);
  };

  // Work distribution: the producer claims units (from the shared counter when p.sched is
  // set, so units that share weight or token tiles run at about the same time on different
  // SMs and a slow unit delays nothing else; round-robin otherwise) and publishes each id
  // through a small shared-memory queue; the MMA thread and the epilogue warps take the ids
  // in the same order.  Id -1 ends the sequence.
  auto claim = [&](int prev) -> int {
    if (p.sched) return atomicAdd(p.sched, 1);
    return prev < 0 ? (int)blockIdx.x : prev + (int)gridDim.x;
  };

  if (warp == 0) {
    // -------------------------------------------------------------- TMA producer (warp 0)
    // Lane 0 claims units, publishes them, waits for free slots and loads the weight tiles.
    // Gathering (MODE_UP, BN <= kGatherMaxBN): every lane then gathers four of the unit's
    // token rows of x per stage (lane l: tile rows 4l..4l+3), n_mma rows in all; rows past
    // the group's last token repeat its first token (their accumulator columns are never
    // read).  Otherwise lane 0 loads the contiguous token-row box.
    const uint64_t pol_w = policy_evict_first();  // weights read once
    const uint64_t pol_b = policy_evict_last();   // activations: re-read per m tile
    int stage = 0;
    uint32_t phase = 0;
    int issued = 0;
    bool ok = true;
    int qi = 0;
    uint32_t qph = 0;
    int u = -1;             // lane 0's claim cursor
    int ready_group = -1;   // lane 0, down kernel: group whose h is known to be complete
    for (;;) {
      int uid = -1;
      if (lane == 0) {
        u = claim(u);
        uid = (u < total_units) ? unit_of_ticket(u, n_first, n_heavy, total_units) : -1;
        if (mbar_wait_bounded(&uq_empty[qi], qph ^ 1, abort_flag, p.status, 5)) {
          uq[qi] = uid;
          mbar_arrive(&uq_full[qi]);
        } else {
          ok = false;
        }
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      uid = __shfl_sync(0xffffffffu, uid, 0);
      if (++qi == kUnitQ) {
        qi = 0;
        qph ^= 1;
      }
      if (uid < 0) break;
      int g, mt, nt;
      decode(uid, g, mt, nt);
      const int a_row = weight_group(p, g) * p.M + mt * kBM;
      const int valid = min(BN, grp_count[g] - nt * BN);
      // the shared group of a non-gathering up kernel reads x, not the sorted rows
      const bool shared_x = (MODE == MODE_UP) && !kGather && (g >= p.E);
      const CUtensorMap *bmap = shared_x ? &p.tmBs : &p.tmB;
      const int b_row = shared_x ? p.shared_t0 + nt * BN : grp_row[g] + nt * BN;
      // gathering: this lane's four token ids and the rows the MMA reads
      int tok[4] = {0, 0, 0, 0};
      int n_rows = BN;
      if (kGather) {
        n_rows = (valid + 15) & ~15;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int pos = 4 * lane + i;
          const int q = b_row + ((pos < valid) ? pos : 0);
          if (4 * lane < n_rows)
            tok[i] = (g < p.E) ? p.perm[q] / p.topk : p.shared_t0 + q - grp_row[g];
        }
      }
      if (MODE == MODE_DOWN && p.done) {
        if (lane == 0 && g != ready_group) {
          const int target =
              p.done_warps * p.done_mt * ((grp_count[g] + p.done_bn - 1) / p.done_bn);
          ok = counter_wait_bounded(p.done + g, target, abort_flag, p.status, 8);
          fence_proxy_async_global();  // the h rows are read through TMA below
          ready_group = g;
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
      }
      const uint32_t stage_bytes = C::NA * C::A_BYTES + (uint32_t)n_rows * kBK * 2;
      // a weight tile read by one unit only is streamed with evict-first priority; one
      // shared by several token tiles keeps normal priority so its neighbours hit L2
      const bool single_use = grp_count[g] <= BN;
      for (int kb = 0; kb < kblocks; ++kb) {
        const int kc = kb * kBK;
        if (lane == 0) {
          ok = mbar_wait_bounded(&empty[stage], phase ^ 1, abort_flag, p.status, 1);
          if (ok) {
            mbar_arrive_expect_tx(&full[stage], stage_bytes);
            if (single_use) {
              tma_load_2d_hint(sA0 + stage * C::A_BYTES, &p.tmA0, &full[stage], kc, a_row,
                               pol_w);
              if (MODE == MODE_UP)
                tma_load_2d_hint(sA1 + stage * C::A_BYTES, &p.tmA1, &full[stage], kc, a_row,
                                 pol_w);
            } else {
              tma_load_2d(sA0 + stage * C::A_BYTES, &p.tmA0, &full[stage], kc, a_row);
              if (MODE == MODE_UP)
                tma_load_2d(sA1 + stage * C::A_BYTES, &p.tmA1, &full[stage], kc, a_row);
            }
            if (!kGather)
              tma_load_2d_hint(sB + stage * C::B_BYTES, bmap, &full[stage], kc, b_row, pol_b);
          }
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
        if (kGather && 4 * lane < n_rows)
          tma_gather4(sB + stage * C::B_BYTES + lane * 4 * kBK * 2, &p.tmB, &full[stage], kc,
                      tok[0], tok[1], tok[2], tok[3], pol_b);
        ++issued;
        if (++stage == S) {
          stage = 0;
          phase ^= 1;
        }
      }
      if (!ok) break;
    }
    if (!ok && lane == 0) {
      // drain: wait (time-bounded, ignoring the abort flag) for the copies still in flight
      int n = issued < S ? issued : S;
      int st = stage, ph = phase;
      for (int i = 0; i < n; ++i) {
        if (--st < 0) {
          st = S - 1;
          ph ^= 1;
        }
        volatile int no_abort = 0;
        mbar_wait_bounded(&full[st], ph, &no_abort, nullptr, 0);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------------ MMA issuer
      int stage = 0;
      uint32_t phase = 0;
      int it = 0;
      bool ok = true;
      int qi = 0;
      uint32_t qph = 0;
      while (ok) {
        if (!mbar_wait_bounded(&uq_full[qi], qph, abort_flag, p.status, 6)) break;
        const int u = uq[qi];
        mbar_arrive(&uq_empty[qi]);
        if (++qi == kUnitQ) {
          qi = 0;
          qph ^= 1;
        }
        if (u < 0) break;
        const int acc = it % C::ACC_BUFS;
        const uint32_t acc_phase = (it / C::ACC_BUFS) & 1;
        ++it;
        if (!mbar_wait_bounded(&tempty[acc], acc_phase ^ 1, abort_flag, p.status, 2)) break;
        tc_fence_after();
        int g, mt, nt;
        decode(u, g, mt, nt);
        const int valid = min(BN, grp_count[g] - nt * BN);
        const int n_mma = (valid + 15) & ~15;
        const uint32_t idesc = idesc_bf16_f32(kBM, n_mma);
        const uint32_t d0 = tmem_base + acc * C::ACC_COLS;
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!mbar_wait_bounded(&full[stage], phase, abort_flag, p.status, 3)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(sA0 + stage * C::A_BYTES);
          const uint32_t a1 = smem_u32(sA1 + stage * C::A_BYTES);
          const uint32_t b = smem_u32(sB + stage * C::B_BYTES);
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk) {
            const uint32_t accum = (kb | kk) ? 1u : 0u;
            const uint64_t bd = sdesc_k_sw128(b + kk * 32);
            tc_mma_bf16(d0, sdesc_k_sw128(a0 + kk * 32), bd, idesc, accum);
            if (MODE == MODE_UP) tc_mma_bf16(d0 + BN, sdesc_k_sw128(a1 + kk * 32), bd, idesc, accum);
          }
          tc_commit(&empty[stage]);  // slot free once these MMAs have read it
          if (++stage == S) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (ok) tc_commit(&tfull[acc]);
      }
      // every MMA issued by this thread has completed once `drain` flips
      tc_commit(drain);
      volatile int no_abort = 0;
      mbar_wait_bounded(drain, 0, &no_abort, nullptr, 0);
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------------- epilogue
    // Lane 0 of each warp polls the barriers and the warp follows it, so every lane takes
    // the same path into the warp-wide tcgen05.ld instructions.
    const int q = warp & 3;              // TMEM lane quadrant of this warp
    const int r = q * 32 + lane;         // weight row within the unit
    auto warp_wait = [&](uint64_t *bar, uint32_t parity, int where) -> bool {
      int ok = 1;
      if (lane == 0) ok = mbar_wait_bounded(bar, parity, abort_flag, p.status, where) ? 1 : 0;
      ok = __shfl_sync(0xffffffffu, ok, 0);
      __syncwarp();
      return ok != 0;
    };
    int it = 0;
    int qi = 0;
    uint32_t qph = 0;
    while (true) {
      if (!warp_wait(&uq_full[qi], qph, 7)) break;
      const int u = uq[qi];
      __syncwarp();
      if (lane == 0) mbar_arrive(&uq_empty[qi]);
      if (++qi == kUnitQ) {
        qi = 0;
        qph ^= 1;
      }
      if (u < 0) break;
      const int acc = it % C::ACC_BUFS;
      const uint32_t acc_phase = (it / C::ACC_BUFS) & 1;
      ++it;
      if (!warp_wait(&tfull[acc], acc_phase, 4)) break;
      tc_fence_after();
      int g, mt, nt;
      decode(u, g, mt, nt);
      const int valid = min(BN, grp_count[g] - nt * BN);
      const int row0 = grp_row[g] + nt * BN;
      const int col = mt * kBM + r;
      const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + acc * C::ACC_COLS;
      if (MODE == MODE_DOWN) {
        // gate * routed_scale of each token column, staged once per unit (one copy per
        // accumulator buffer, so a fast warp never overwrites scales a slow warp still reads)
        for (int n = threadIdx.x - 64; n < BN; n += 128) {
          float sc = 0.f;
          if (n < valid) sc = (g < p.E) ? p.routed_scale * p.topk_gate[p.perm[row0 + n]] : 1.f;
          row_scale[acc * BN + n] = sc;
        }
        // all epilogue warps' scales are staged before any reads them: a bounded mbarrier (one
        // arrival per warp) instead of bar.sync, so a warp that aborts leaves none waiting
        __syncwarp();
        if (lane == 0) mbar_arrive(epi_bar);
        if (!warp_wait(epi_bar, (uint32_t)(it - 1) & 1, 71)) break;
      }
      float *wbuf = xbuf + q * 16 * 32;
      const int col_base = mt * kBM + q * 32;  // first output column of this warp
      // TMEM loads run one 16-column chunk ahead of their use
      uint32_t n0[16], n1[16];
      tmem_ld16(taddr, n0);
      if (MODE == MODE_UP) tmem_ld16(taddr + BN, n1);
      for (int c0 = 0; c0 < valid; c0 += 16) {
        uint32_t v0[16], v1[16];
        if (MODE == MODE_UP) tmem_ld_wait_regs(n0, n1);
        else tmem_ld_wait_regs(n0);
#pragma unroll
        for (int n = 0; n < 16; ++n) {
          v0[n] = n0[n];
          v1[n] = n1[n];
        }
        if (c0 + 16 < valid) {
          tmem_ld16(taddr + c0 + 16, n0);
          if (MODE == MODE_UP) tmem_ld16(taddr + BN + c0 + 16, n1);
        }
        float vals[16];
        if (MODE == MODE_UP && p.out2) {  // the pre-activations themselves (backward)
#pragma unroll
          for (int n = 0; n < 16; ++n) vals[n] = __uint_as_float(v0[n]);
          store_block16_f32(static_cast<float *>(p.out), p.ld_out, row0, c0, valid, col_base,
                            vals, wbuf, lane);
#pragma unroll
          for (int n = 0; n < 16; ++n) vals[n] = __uint_as_float(v1[n]);
          store_block16_f32(p.out2, p.ld_out, row0, c0, valid, col_base, vals, wbuf, lane);
        } else if (MODE == MODE_UP) {
#pragma unroll
          for (int n = 0; n < 16; ++n)
            vals[n] = swiglu(__uint_as_float(v0[n]), __uint_as_float(v1[n]));
          store_block16_bf16(static_cast<__nv_bfloat16 *>(p.out), p.ld_out, row0, c0, valid,
                             col_base, vals, wbuf, lane);
          if (p.save_a) {  // training forward: keep the pre-activations for the backward
#pragma unroll
            for (int n = 0; n < 16; ++n) vals[n] = __uint_as_float(v0[n]);
            store_block16_f32(p.save_a, p.ld_out, row0, c0, valid, col_base, vals, wbuf, lane);
#pragma unroll
            for (int n = 0; n < 16; ++n) vals[n] = __uint_as_float(v1[n]);
            store_block16_f32(p.save_b, p.ld_out, row0, c0, valid, col_base, vals, wbuf, lane);
          }
        } else if (MODE == MODE_DOWN) {
          const float4 *sc = reinterpret_cast<const float4 *>(row_scale + acc * BN + c0);
#pragma unroll
          for (int n4 = 0; n4 < 4; ++n4) {
            const float4 s4 = sc[n4];
            vals[4 * n4 + 0] = __uint_as_float(v0[4 * n4 + 0]) * s4.x;
            vals[4 * n4 + 1] = __uint_as_float(v0[4 * n4 + 1]) * s4.y;
            vals[4 * n4 + 2] = __uint_as_float(v0[4 * n4 + 2]) * s4.z;
            vals[4 * n4 + 3] = __uint_as_float(v0[4 * n4 + 3]) * s4.w;
          }
          store_block16_f32(static_cast<float *>(p.out), p.ld_out, row0, c0, valid, col_base,
                            vals, wbuf, lane);
        } else if (!p.out_trans) {  // MODE_LOGITS, experts on M: scalar masked stores
          if (col < p.M) {
#pragma unroll
            for (int n = 0; n < 16; ++n) {
              if (c0 + n < valid)
                static_cast<float *>(p.out)[(size_t)(row0 + c0 + n) * p.ld_out + col] =
                    __uint_as_float(v0[n]);
            }
          }
        } else if (col < p.M) {  // MODE_LOGITS, tokens on M: lane = token, 16 experts
          float *dst = static_cast<float *>(p.out) + (size_t)col * p.ld_out + row0 + c0;
          if ((p.ld_out & 3) == 0 && c0 + 16 <= valid) {
#pragma unroll
            for (int n4 = 0; n4 < 4; ++n4)
              reinterpret_cast<float4 *>(dst)[n4] =
                  make_float4(__uint_as_float(v0[4 * n4]), __uint_as_float(v0[4 * n4 + 1]),
                              __uint_as_float(v0[4 * n4 + 2]), __uint_as_float(v0[4 * n4 + 3]));
          } else {
#pragma unroll
            for (int n = 0; n < 16; ++n)
              if (c0 + n < valid) dst[n] = __uint_as_float(v0[n]);
          }
        }
      }
      // every TMEM load of this unit has completed (tcgen05.wait::ld before each use), so
      // the accumulator is handed back to the MMA thread before this warp's global stores
      // drain: the h hand-over's fences below wait for them, off the MMA's critical path
      tc_fence_before();
      mbar_arrive(&tempty[acc]);
      if (MODE == MODE_UP && p.done) {
        // publish this warp's rows of h for group g: stores, then a release of the count
        __threadfence();
        __syncwarp();
        if (lane == 0) {
          __threadfence();
          atomicAdd(p.done + g, 1);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
  if (p.clock_sum && threadIdx.x == 0) clock_span_add(*span, p.clock_sum);
}

}  // namespace moe
