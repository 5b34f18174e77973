// grouped_gemm_bw.cuh -- tcgen05 grouped GEMMs of the bf16 layer's backward.
//
// The chain rule through the SwiGLU experts ("Step 3.5 Flash: Open Frontier-Level
// Intelligence with 11B Active Parameters", sections 2.2 and 4.1.2; "Step 3.5 Flash
// 技术论文深度解读", training stability, root cause 3) as grouped GEMMs over the
// expert-sorted rows ("fused MoE gather/scatter with grouped GEMM", first page, section
// 3.2.4).  Per sorted row p of group g (token t, scale s_p = routed_scale * gate, 1 for the
// shared expert), with a = W_g[g] x_t and b = W_u[g] x_t recomputed by the forward's up GEMM
// (or kept by a training forward):
//
//   DH    dhu_p = W_d[g]^T dout_t                (weights on M: f rows; K = d)
//         epilogue: h = silu(a) b, dgate partial sum dhu . h, dh = s_p dhu,
//                   da = dh b silu'(a), db = dh silu(a), hs = s_p h  -> bf16 rows
//   DX    dX_p = W_g[g]^T da_p + W_u[g]^T db_p   (weights on M: d rows; K = 2 f)
//   WGRAD dW_d[g] += sum_p dout_p hs_p^T,  dW_g[g] += sum_p da_p x_p^T,
//         dW_u[g] += sum_p db_p x_p^T            (K = the group's rows)
//
// Operand layouts.  The weights enter the dgrad GEMMs transposed: W_d[g] is [d, f] with f
// contiguous, and DH wants f on M, so the weight tile is an M-major ("MN-major") operand:
// TMA boxes of 64 M elements x 64 K rows, one 128-byte swizzled row per K index.  The
// weight gradients reduce over rows, so both of their operands are MN-major tiles of the
// expert-sorted activations.  Both are described to tcgen05.mma by shared-memory
// descriptors whose leading byte offset steps between 64-element M (or N) blocks and whose
// stride byte offset steps between 8-row K groups (the canonical MN-major layout of the
// tcgen05 shared-memory descriptor), with the instruction descriptor's A/B major bits set.
//
// Row layout.  The backward keeps its expert-sorted rows (x, dout, da, db, s*h and the
// recomputed a, b) with every group padded to a multiple of 16 rows: routed group g starts at
// poff[g] (an exclusive scan of the padded counts, computed on the device), the shared group
// at a fixed row s0 = T*k + 15*E past any possible routed end, and the padding rows of the
// bf16 operands are zero.  The dgrad GEMMs tile a group's rows on N as the forward does
// (columns past the group's rows are never stored).  The weight gradients take a group's
// rows as K in blocks of 64 box-loaded rows and issue only the 16-row MMA steps that reach
// the group's padded end, so rows of a neighbouring group are loaded but never multiplied and
// the padding adds zeros.  Each dW tile is owned by one unit, which adds its finished
// accumulator into the caller's fp32 gradient with TMA reductions (cp.reduce.async.bulk
// .tensor add): one addition per element and call, so the result is deterministic.
//
// Kernels: bw_dgrad_kernel (one CTA per unit, DH or DX), bw_dgrad_pair_kernel (the same on a
// CTA pair, 256 weight rows per unit), bw_wgrad_kernel / bw_wgrad_pair_kernel (weight
// gradients, 128 x 256 or 256 x 256 tiles), bw_tail_pair_kernel (DX and the weight gradients
// in one persistent launch with interleaved units), and the small row-layout kernels.
// Roles, pipelines and bounded waits are those of grouped_gemm.cuh and grouped_gemm_pair.cuh:
// warp 0 produces (lane 0 claims units; on a pair the leader claims and publishes), warp 1
// lane 0 issues the MMAs, warps 2..5 (2..9 on a pair) run the epilogue, STAGES shared-memory
// slots and two TMEM accumulators; every wait gives up after the time limit, drains its
// in-flight copies and MMAs, frees TMEM and reports through the status word.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "grouped_gemm.cuh"
#include "ptx_sm100.cuh"

namespace moe {

// ------------------------------------------------------------------------ PTX helpers
// MN-major operand tile written by TMA boxes {64 elements, rows} with the 128-byte swizzle:
// one 128-byte row per K index, 8-row K groups 1024 B apart (stride byte offset, bits 32-45),
// consecutive 64-element M (or N) blocks `lbo` bytes apart (leading byte offset, bits 16-29);
// version 1 (bit 46), layout type 2 = 128-byte swizzle (bits 61-63).
__device__ __forceinline__ uint64_t sdesc_mn_sw128(uint32_t smem_addr, uint32_t lbo) {
  uint64_t d = 0;
  d |= (uint64_t)((smem_addr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)(1024u >> 4) << 32;
  d |= (uint64_t)1u << 46;
  d |= (uint64_t)2u << 61;
  return d;
}

// .kind::f16 instruction descriptor with the A (bit 15) and B (bit 16) major bits:
// 0 = K-major, 1 = MN-major.
__host__ __device__ constexpr uint32_t idesc_bf16_f32_major(int M, int N, bool a_mn,
                                                            bool b_mn) {
  return idesc_bf16_f32(M, N) | ((a_mn ? 1u : 0u) << 15) | ((b_mn ? 1u : 0u) << 16);
}

// global[tile at (c0, c1)] += shared tile, through the TMA unit (bulk-group completion).
__device__ __forceinline__ void tma_reduce_add_2d(const CUtensorMap *map, const void *src, int c0,
                                                  int c1) {
  asm volatile(
      "cp.reduce.async.bulk.tensor.2d.global.shared::cta.add.bulk_group [%0, {%2, %3}], [%1];" ::
          "l"(reinterpret_cast<uint64_t>(map)),
      "r"(smem_u32(src)), "r"(c0), "r"(c1)
      : "memory");
}
// global[tile at (c0, c1)] = shared tile (bulk-group completion).
__device__ __forceinline__ void tma_store_2d(const CUtensorMap *map, const void *src, int c0,
                                             int c1) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::
                   "l"(reinterpret_cast<uint64_t>(map)),
               "r"(smem_u32(src)), "r"(c0), "r"(c1)
               : "memory");
}
__device__ __forceinline__ void bulk_commit_group() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// at most N of this thread's bulk groups still reading shared memory
template <int N>
__device__ __forceinline__ void bulk_wait_group_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ void bulk_wait_group_all() {
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}
// order this thread's generic-proxy shared-memory writes before later async-proxy reads
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// -------------------------------------------------------------------- row layout
struct BwRows {
  const int *offsets;  // [E + 1] group starts in the unpadded sorted rows
  const int *poff;     // [E + 1] starts of the routed groups in the padded rows
  int E, T, Tk;
  int s0;              // padded start of the shared group (n_shared is 0 or 1)
  // group g: first padded row, first unpadded row, rows
  __device__ __forceinline__ void group(int g, int &rowp, int &rowu, int &cnt) const {
    if (g < E) {
      rowu = offsets[g];
      cnt = offsets[g + 1] - rowu;
      rowp = poff[g];
    } else {
      rowu = Tk;
      cnt = T;
      rowp = s0;
    }
  }
};

// --------------------------------------------------------------------- dgrad GEMMs
enum BwDgradMode { BW_DH = 0, BW_DX = 1 };

struct BwDgradParams {
  CUtensorMap tmA0;  // DH: W_down as [G*d, f]; DX: W_gate as [G*f, d]      box {64, 64}
  CUtensorMap tmA1;  // DX: W_up as [G*f, d]                                box {64, 64}
  CUtensorMap tmB0;  // DH: dout rows [R, d]; DX: da [R, f] (padded rows)  box {64, BN}
  CUtensorMap tmB1;  // DX: db [R, f]                                      box {64, BN}
  BwRows rows;
  const float *row_scale;      // [P] s_p by unpadded row (DH)
  const float *pre_a, *pre_b;  // fp32 pre-activations (DH): [R, f] at the padded rows, or
                               // [P, f] at the unpadded rows when pre_unpadded is set (kept
                               // by a training forward)
  int pre_unpadded;
  __nv_bfloat16 *da, *db, *hs; // [R, f] padded rows (DH)
  float *dgate_part;           // [Tk, n_part] by unpadded row (DH): partial sums of dhu . h
  float *out;                  // DX: dX rows [P, d] fp32, unpadded rows
  DevStatus *status;
  int n_groups;
  int M;       // weight rows per group on M: f (DH), d (DX)
  int K;       // reduction length per operand pair: d (DH), f (DX)
  int n_pairs; // 1 (DH) or 2 (DX: W_gate with da, then W_up with db)
  int n_part;  // DH: M / 32 (one partial per epilogue warp and m tile)
  int *sched;  // work counter (zero at launch)
};

template <int BN>
struct BwDgradCfg {
  static constexpr int A_BYTES = kBM * kBK * 2;  // two boxes of 64 M x 64 K
  static constexpr int B_BYTES = BN * kBK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int ACC_COLS = BN;
  static constexpr int ACC_BUFS = 2;
  static constexpr int TMEM_COLS_RAW = ACC_BUFS * ACC_COLS;
  static constexpr int TMEM_COLS = TMEM_COLS_RAW <= 32    ? 32
                                   : TMEM_COLS_RAW <= 64  ? 64
                                   : TMEM_COLS_RAW <= 128 ? 128
                                   : TMEM_COLS_RAW <= 256 ? 256
                                                          : 512;
  static constexpr int SMEM_BUDGET = 200 * 1024;
  static constexpr int STAGES_RAW = SMEM_BUDGET / STAGE_BYTES;
  static constexpr int STAGES = STAGES_RAW > 12 ? 12 : STAGES_RAW;
  static_assert(STAGES >= 2, "pipeline too shallow");
  static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "N of the MMA");
  static constexpr int BAR_BYTES = (2 * STAGES + 5 + 2 * kUnitQ) * 8;
  static constexpr size_t smem_bytes(int n_groups) {
    return 1024 + (size_t)STAGES * STAGE_BYTES + BAR_BYTES + 64 + (size_t)(4 * n_groups + 1) * 4 +
           ACC_BUFS * BN * 4 /*row scales*/ + 4 * 16 * 32 * 4 /*store transposes*/ +
           4 * 16 * 33 * 4 /*dgate reductions*/ + 16;
  }
};

template <int MODE, int BN>
__global__ void __launch_bounds__(kGemmThreads, 1)
    bw_dgrad_kernel(const __grid_constant__ BwDgradParams p) {
  using C = BwDgradCfg<BN>;
  constexpr int S = C::STAGES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t *sA = smem;
  uint8_t *sB = sA + S * C::A_BYTES;
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
  uint64_t *epi_bar = reinterpret_cast<uint64_t *>(tmem_slot + 2);  // epilogue warps' barrier
  volatile int *uq = reinterpret_cast<volatile int *>(tmem_slot + 4);  // [kUnitQ]
  int *unit_prefix = reinterpret_cast<int *>(tmem_slot + 16);        // [G + 1]
  int *grp_count = unit_prefix + p.n_groups + 1;                     // [G]
  int *grp_row = grp_count + p.n_groups;                             // [G] padded
  int *grp_rowu = grp_row + p.n_groups;                              // [G] unpadded
  float *row_scale = reinterpret_cast<float *>(
      (reinterpret_cast<uintptr_t>(grp_rowu + p.n_groups) + 15) & ~static_cast<uintptr_t>(15));
  float *xbuf = row_scale + C::ACC_BUFS * BN;  // [4 warps][16][32] store transposes
  float *rbuf = xbuf + 4 * 16 * 32;            // [4 warps][16][33] dgate reductions

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = p.n_groups;
  const int mtiles = p.M / kBM;
  const int kpp = p.K / kBK;  // k blocks per operand pair
  const int kblocks = p.n_pairs * kpp;

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
      mbar_init(&uq_empty[q], 5);
    }
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&p.tmA0);
    tma_prefetch_desc(&p.tmB0);
    if (MODE == BW_DX) {
      tma_prefetch_desc(&p.tmA1);
      tma_prefetch_desc(&p.tmB1);
    }
  }
  if (warp == 1) tmem_alloc(tmem_slot, C::TMEM_COLS);
  griddep_wait();
  griddep_launch_dependents();
  for (int g = threadIdx.x; g < G; g += blockDim.x) {
    int rowp, rowu, cnt;
    p.rows.group(g, rowp, rowu, cnt);
    grp_count[g] = cnt;
    grp_row[g] = rowp;
    grp_rowu[g] = rowu;
    unit_prefix[g] = mtiles * ((cnt + BN - 1) / BN);
  }
  __syncthreads();
  if (warp == 0) {  // exclusive scan of units per group
    const int per = (G + 31) / 32;
    const int lo = min(G, lane * per), hi = min(G, lo + per);
    int run = 0;
    for (int g = lo; g < hi; ++g) run += unit_prefix[g];
    int incl = run;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    int excl = incl - run;
    for (int g = lo; g < hi; ++g) {
      const int u = unit_prefix[g];
      unit_prefix[g] = excl;
      excl += u;
    }
    if (lane == 31) unit_prefix[G] = incl;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int total_units = unit_prefix[G];

  auto decode = [&](int u, int &g, int &mt, int &nt) {
    int lo = 0, hi = G - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (unit_prefix[mid] <= u) lo = mid;
      else hi = mid - 1;
    }
    g = lo;
    const int nts = (grp_count[g] + BN - 1) / BN;
    const int loc = u - unit_prefix[g];
    mt = loc / nts;
    nt = loc % nts;
  };

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    if (lane == 0) {
      const uint64_t pol_w = policy_evict_first();
      const uint64_t pol_b = policy_evict_last();
      int stage = 0;
      uint32_t phase = 0;
      int issued = 0;
      bool ok = true;
      int qi = 0;
      uint32_t qph = 0;
      for (;;) {
        const int u = atomicAdd(p.sched, 1);
        const int uid = (u < total_units) ? u : -1;
        if (!mbar_wait_bounded(&uq_empty[qi], qph ^ 1, abort_flag, p.status, 21)) {
          ok = false;
          break;
        }
        uq[qi] = uid;
        mbar_arrive(&uq_full[qi]);
        if (++qi == kUnitQ) {
          qi = 0;
          qph ^= 1;
        }
        if (uid < 0) break;
        int g, mt, nt;
        decode(uid, g, mt, nt);
        const int b_row = grp_row[g] + nt * BN;
        const bool single_use = grp_count[g] <= BN;
        for (int kb = 0; kb < kblocks; ++kb) {
          const int pair = kb / kpp;
          const int kc = (kb - pair * kpp) * kBK;
          if (!mbar_wait_bounded(&empty[stage], phase ^ 1, abort_flag, p.status, 22)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[stage], C::STAGE_BYTES);
          const CUtensorMap *amap = pair ? &p.tmA1 : &p.tmA0;
          const CUtensorMap *bmap = pair ? &p.tmB1 : &p.tmB0;
          uint8_t *a_dst = sA + stage * C::A_BYTES;
          const int a_row = g * p.K + kc;
          if (single_use) {
            tma_load_2d_hint(a_dst, amap, &full[stage], mt * kBM, a_row, pol_w);
            tma_load_2d_hint(a_dst + C::A_BYTES / 2, amap, &full[stage], mt * kBM + 64, a_row,
                             pol_w);
          } else {
            tma_load_2d(a_dst, amap, &full[stage], mt * kBM, a_row);
            tma_load_2d(a_dst + C::A_BYTES / 2, amap, &full[stage], mt * kBM + 64, a_row);
          }
          tma_load_2d_hint(sB + stage * C::B_BYTES, bmap, &full[stage], kc, b_row, pol_b);
          ++issued;
          if (++stage == S) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
      }
      if (!ok) {
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
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------------------------------------------------------- MMA issuer
      int stage = 0;
      uint32_t phase = 0;
      int it = 0;
      bool ok = true;
      int qi = 0;
      uint32_t qph = 0;
      while (ok) {
        if (!mbar_wait_bounded(&uq_full[qi], qph, abort_flag, p.status, 23)) break;
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
        if (!mbar_wait_bounded(&tempty[acc], acc_phase ^ 1, abort_flag, p.status, 24)) break;
        tc_fence_after();
        int g, mt, nt;
        decode(u, g, mt, nt);
        const int valid = min(BN, grp_count[g] - nt * BN);
        const int n_mma = (valid + 15) & ~15;
        const uint32_t idesc = idesc_bf16_f32_major(kBM, n_mma, true, false);
        const uint32_t d0 = tmem_base + acc * C::ACC_COLS;
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!mbar_wait_bounded(&full[stage], phase, abort_flag, p.status, 25)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a = smem_u32(sA + stage * C::A_BYTES);
          const uint32_t b = smem_u32(sB + stage * C::B_BYTES);
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk)
            tc_mma_bf16(d0, sdesc_mn_sw128(a + kk * 16 * 128, C::A_BYTES / 2),
                        sdesc_k_sw128(b + kk * 32), idesc, (kb | kk) ? 1u : 0u);
          tc_commit(&empty[stage]);
          if (++stage == S) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (ok) tc_commit(&tfull[acc]);
      }
      tc_commit(drain);
      volatile int no_abort = 0;
      mbar_wait_bounded(drain, 0, &no_abort, nullptr, 0);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------------- epilogue
    const int q = warp & 3;
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
    float *wbuf = xbuf + q * 16 * 32;
    float *red = rbuf + q * 16 * 33;
    while (true) {
      if (!warp_wait(&uq_full[qi], qph, 26)) break;
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
      if (!warp_wait(&tfull[acc], acc_phase, 27)) break;
      tc_fence_after();
      int g, mt, nt;
      decode(u, g, mt, nt);
      const int valid = min(BN, grp_count[g] - nt * BN);
      const int row0 = grp_row[g] + nt * BN;    // padded
      const int rowu0 = grp_rowu[g] + nt * BN;  // unpadded
      const int col_base = mt * kBM + q * 32;  // first output column (M index) of this warp
      const int col = col_base + lane;
      const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + acc * C::ACC_COLS;
      if (MODE == BW_DH) {
        for (int n = threadIdx.x - 64; n < BN; n += 128)
          row_scale[acc * BN + n] = (n < valid) ? p.row_scale[rowu0 + n] : 0.f;
        // all epilogue warps' scales are staged before any reads them: a bounded mbarrier (one
        // arrival per warp) instead of bar.sync, so a warp that aborts leaves none waiting
        __syncwarp();
        if (lane == 0) mbar_arrive(epi_bar);
        if (!warp_wait(epi_bar, (uint32_t)(it - 1) & 1, 73)) break;
      }
      uint32_t nx[16];
      tmem_ld16(taddr, nx);
      for (int c0 = 0; c0 < valid; c0 += 16) {
        uint32_t v[16];
        tmem_ld_wait_regs(nx);
#pragma unroll
        for (int n = 0; n < 16; ++n) v[n] = nx[n];
        if (c0 + 16 < valid) tmem_ld16(taddr + c0 + 16, nx);
        float vals[16];
        if (MODE == BW_DX) {
#pragma unroll
          for (int n = 0; n < 16; ++n) vals[n] = __uint_as_float(v[n]);
          store_block16_f32(p.out, p.M, rowu0, c0, valid, col_base, vals, wbuf, lane);
        } else {
          // pre-activations of the chunk's rows (coalesced: lanes read consecutive columns)
          float av[16], bv[16];
#pragma unroll
          for (int n = 0; n < 16; ++n) {
            const bool in = c0 + n < valid;
            const size_t i = (size_t)((p.pre_unpadded ? rowu0 : row0) + c0 + n) * p.M + col;
            av[n] = in ? p.pre_a[i] : 0.f;
            bv[n] = in ? p.pre_b[i] : 0.f;
          }
          float dav[16], dbv[16], hsv[16];
          const float4 *sc = reinterpret_cast<const float4 *>(row_scale + acc * BN + c0);
#pragma unroll
          for (int n4 = 0; n4 < 4; ++n4) {
            const float4 s4 = sc[n4];
            const float ss[4] = {s4.x, s4.y, s4.z, s4.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int n = 4 * n4 + e;
              const float a = av[n], b = bv[n], s = ss[e];
              const float dhu = __uint_as_float(v[n]);
              const float sig = __fdividef(1.f, 1.f + __expf(-a));
              const float silu = a * sig;
              const float h = silu * b;
              const float dh = s * dhu;
              vals[n] = dhu * h;  // dgate partial
              dav[n] = dh * b * sig * (1.f + a * (1.f - sig));
              dbv[n] = dh * silu;
              hsv[n] = s * h;
            }
          }
          store_block16_bf16(p.da, p.M, row0, c0, valid, col_base, dav, wbuf, lane);
          store_block16_bf16(p.db, p.M, row0, c0, valid, col_base, dbv, wbuf, lane);
          store_block16_bf16(p.hs, p.M, row0, c0, valid, col_base, hsv, wbuf, lane);
          // sum of dhu . h over this warp's 32 columns for each of the 16 rows, lanes in
          // order (fixed order: deterministic)
#pragma unroll
          for (int n = 0; n < 16; ++n) red[n * 33 + lane] = vals[n];
          __syncwarp();
          if (lane < 16 && c0 + lane < valid && g < p.rows.E) {
            float sum = 0.f;
#pragma unroll 8
            for (int i = 0; i < 32; ++i) sum += red[lane * 33 + i];
            p.dgate_part[(size_t)(rowu0 + c0 + lane) * p.n_part + mt * 4 + q] = sum;
          }
          __syncwarp();
        }
      }
      tc_fence_before();
      mbar_arrive(&tempty[acc]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

// CTA-pair dgrad kernel for large groups: 256 weight rows x up to 256 tokens per unit on a
// cluster of two CTAs (tcgen05 cta_group::2), the layout of grouped_gemm_pair.cuh with the
// weight tile MN-major.  CTA r stages weight rows [128 r, 128 r + 128) of the unit (two
// 64-wide MN-major boxes) and token rows [n0 + r*half, n0 + (r+1)*half) (half the token
// tile, K-major), so each CTA loads half the token tile of the one-CTA kernel per MMA.
constexpr int kBwPairEpiWarps = 8;
constexpr int kBwPairThreads = 32 * (2 + kBwPairEpiWarps);

struct BwDgradPairCfg {
  static constexpr int BN = 256;
  static constexpr int HALF_BN = BN / 2;
  static constexpr int A_BYTES = 128 * kBK * 2;       // this CTA's 128 weight rows
  static constexpr int B_BYTES = HALF_BN * kBK * 2;   // this CTA's token rows
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int ACC_COLS = BN;
  static constexpr int TMEM_COLS = 2 * ACC_COLS;
  static constexpr int STAGES_RAW = (160 * 1024) / STAGE_BYTES;
  static constexpr int STAGES = STAGES_RAW > 8 ? 8 : STAGES_RAW;
  static constexpr int BAR_BYTES = (2 * STAGES + 5 + 2 * kUnitQ) * 8;
  static constexpr size_t smem_bytes(int n_groups) {
    return 1024 + (size_t)STAGES * STAGE_BYTES + BAR_BYTES + 64 +
           (size_t)(4 * n_groups + 1) * 4 + 2 * BN * 4 /*row scales*/ +
           kBwPairEpiWarps * 16 * 32 * 4 /*store transposes*/ +
           kBwPairEpiWarps * 16 * 33 * 4 /*dgate reductions*/ + 16;
  }
};

template <int MODE>
__global__ void __launch_bounds__(kBwPairThreads, 1)
    bw_dgrad_pair_kernel(const __grid_constant__ BwDgradParams p) {
  using C = BwDgradPairCfg;
  constexpr int S = C::STAGES;
  constexpr int BN = C::BN;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t *sA = smem;
  uint8_t *sB = sA + S * C::A_BYTES;
  uint64_t *bars = reinterpret_cast<uint64_t *>(sB + S * C::B_BYTES);
  uint64_t *full = bars;
  uint64_t *empty = bars + S;
  uint64_t *tfull = bars + 2 * S;
  uint64_t *tempty = bars + 2 * S + 2;
  uint64_t *drain = bars + 2 * S + 4;
  uint64_t *uq_full = bars + 2 * S + 5;
  uint64_t *uq_empty = uq_full + kUnitQ;  // used in the leader only
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(uq_empty + kUnitQ);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
  uint64_t *epi_bar = reinterpret_cast<uint64_t *>(tmem_slot + 2);  // epilogue warps' barrier
  volatile int *uq = reinterpret_cast<volatile int *>(tmem_slot + 4);  // [kUnitQ]
  int *unit_prefix = reinterpret_cast<int *>(tmem_slot + 16);        // [G + 1]
  int *grp_count = unit_prefix + p.n_groups + 1;                     // [G]
  int *grp_row = grp_count + p.n_groups;                             // [G] padded
  int *grp_rowu = grp_row + p.n_groups;                              // [G] unpadded
  float *row_scale = reinterpret_cast<float *>(
      (reinterpret_cast<uintptr_t>(grp_rowu + p.n_groups) + 15) & ~static_cast<uintptr_t>(15));
  float *xbuf = row_scale + 2 * BN;             // [8 warps][16][32] store transposes
  float *rbuf = xbuf + kBwPairEpiWarps * 16 * 32;  // [8 warps][16][33] dgate reductions

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int G = p.n_groups;
  const int mtiles = p.M / 256;
  const int kpp = p.K / kBK;
  const int kblocks = p.n_pairs * kpp;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 2 * kBwPairEpiWarps);
    }
    mbar_init(drain, 1);
    mbar_init(epi_bar, kBwPairEpiWarps);
    for (int q = 0; q < kUnitQ; ++q) {
      mbar_init(&uq_full[q], 1);
      mbar_init(&uq_empty[q], 2 + 2 * kBwPairEpiWarps);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc_pair(tmem_slot, C::TMEM_COLS);
  griddep_wait();
  griddep_launch_dependents();
  for (int g = threadIdx.x; g < G; g += blockDim.x) {
    int rowp, rowu, cnt;
    p.rows.group(g, rowp, rowu, cnt);
    grp_count[g] = cnt;
    grp_row[g] = rowp;
    grp_rowu[g] = rowu;
    unit_prefix[g] = mtiles * ((cnt + BN - 1) / BN);
  }
  __syncthreads();
  if (warp == 0) {
    const int per = (G + 31) / 32;
    const int lo = min(G, lane * per), hi = min(G, lo + per);
    int run = 0;
    for (int g = lo; g < hi; ++g) run += unit_prefix[g];
    int incl = run;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    int excl = incl - run;
    for (int g = lo; g < hi; ++g) {
      const int u = unit_prefix[g];
      unit_prefix[g] = excl;
      excl += u;
    }
    if (lane == 31) unit_prefix[G] = incl;
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int total_units = unit_prefix[G];

  auto decode = [&](int u, int &g, int &mt, int &nt) {
    int lo = 0, hi = G - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (unit_prefix[mid] <= u) lo = mid;
      else hi = mid - 1;
    }
    g = lo;
    const int nts = (grp_count[g] + BN - 1) / BN;
    const int loc = u - unit_prefix[g];
    mt = loc / nts;
    nt = loc % nts;
  };
  // token split: CTA r holds tokens [n0 + r*half, n0 + (r+1)*half), N = 2*half
  auto split = [&](int g, int nt) {
    const int valid = min(BN, grp_count[g] - nt * BN);
    return (((valid + 1) >> 1) + 7) & ~7;
  };

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ TMA producer
      const uint64_t pol_w = policy_evict_first();
      const uint64_t pol_b = policy_evict_last();
      int stage = 0;
      uint32_t phase = 0;
      int issued = 0;
      bool ok = true;
      int qi = 0;
      uint32_t qph = 0;
      int u = -1;
      while (ok) {
        if (leader) {
          const int c = atomicAdd(p.sched, 1);
          const int uid = (c < total_units) ? c : -1;
          if (!mbar_wait_bounded<true>(&uq_empty[qi], qph ^ 1, abort_flag, p.status, 51)) {
            ok = false;
            break;
          }
          uq[qi] = uid;
          st_shared_remote(mapa_shared(smem_u32((const void *)&uq[qi]), 1), uid);
          mbar_arrive(&uq_full[qi]);
          mbar_arrive_remote(mapa_shared(smem_u32(&uq_full[qi]), 1));
          u = uid;
        } else {
          if (!mbar_wait_bounded<true>(&uq_full[qi], qph, abort_flag, p.status, 52)) {
            ok = false;
            break;
          }
          u = uq[qi];
          mbar_arrive_remote(mapa_shared(smem_u32(&uq_empty[qi]), 0));
        }
        if (++qi == kUnitQ) {
          qi = 0;
          qph ^= 1;
        }
        if (u < 0) break;
        int g, mt, nt;
        decode(u, g, mt, nt);
        const int half = split(g, nt);
        const int a_x = mt * 256 + (int)rank * 128;
        const int b_row = grp_row[g] + nt * BN + (int)rank * half;
        for (int kb = 0; kb < kblocks; ++kb) {
          const int pair = kb / kpp;
          const int kc = (kb - pair * kpp) * kBK;
          if (!mbar_wait_bounded(&empty[stage], phase ^ 1, abort_flag, p.status, 53)) {
            ok = false;
            break;
          }
          const uint32_t fbar = mapa_shared(smem_u32(&full[stage]), 0);
          if (leader) mbar_arrive_expect_tx(&full[stage], 2 * C::STAGE_BYTES);
          const CUtensorMap *amap = pair ? &p.tmA1 : &p.tmA0;
          const CUtensorMap *bmap = pair ? &p.tmB1 : &p.tmB0;
          uint8_t *a_dst = sA + stage * C::A_BYTES;
          const int a_row = g * p.K + kc;
          tma_load_2d_pair(a_dst, amap, fbar, a_x, a_row, pol_w);
          tma_load_2d_pair(a_dst + C::A_BYTES / 2, amap, fbar, a_x + 64, a_row, pol_w);
          tma_load_2d_pair(sB + stage * C::B_BYTES, bmap, fbar, kc, b_row, pol_b);
          ++issued;
          if (++stage == S) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      if (!ok && leader) {
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
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      // ------------------------------------------------------------ MMA issuer (leader)
      int stage = 0;
      uint32_t phase = 0;
      int it = 0;
      bool ok = true;
      int qi = 0;
      uint32_t qph = 0;
      while (ok) {
        if (!mbar_wait_bounded<true>(&uq_full[qi], qph, abort_flag, p.status, 54)) break;
        const int u = uq[qi];
        mbar_arrive(&uq_empty[qi]);
        if (++qi == kUnitQ) {
          qi = 0;
          qph ^= 1;
        }
        if (u < 0) break;
        const int acc = it & 1;
        const uint32_t acc_phase = (it >> 1) & 1;
        ++it;
        if (!mbar_wait_bounded(&tempty[acc], acc_phase ^ 1, abort_flag, p.status, 55)) break;
        tc_fence_after();
        int g, mt, nt;
        decode(u, g, mt, nt);
        const uint32_t idesc = idesc_bf16_f32_major(256, 2 * split(g, nt), true, false);
        const uint32_t d0 = tmem_base + acc * C::ACC_COLS;
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!mbar_wait_bounded(&full[stage], phase, abort_flag, p.status, 56)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a = smem_u32(sA + stage * C::A_BYTES);
          const uint32_t b = smem_u32(sB + stage * C::B_BYTES);
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk)
            tc_mma_bf16_pair(d0, sdesc_mn_sw128(a + kk * 16 * 128, C::A_BYTES / 2),
                             sdesc_k_sw128(b + kk * 32), idesc, (kb | kk) ? 1u : 0u);
          tc_commit_pair_both(&empty[stage]);
          if (++stage == S) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (ok) tc_commit_pair_both(&tfull[acc]);
      }
      tc_commit_pair_local(drain);
      volatile int no_abort = 0;
      mbar_wait_bounded(drain, 0, &no_abort, nullptr, 0);
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------------- epilogue (both CTAs)
    const int q = warp & 3;
    const int eh = (warp - 2) >> 2;  // chunks 2i + eh of the quadrant's token columns
    const uint32_t tempty_leader = mapa_shared(smem_u32(&tempty[0]), 0);
    const uint32_t uq_empty_leader = mapa_shared(smem_u32(&uq_empty[0]), 0);
    auto warp_wait = [&](uint64_t *bar, uint32_t parity, int where, bool cluster) -> bool {
      int ok = 1;
      if (lane == 0)
        ok = (cluster ? mbar_wait_bounded<true>(bar, parity, abort_flag, p.status, where)
                      : mbar_wait_bounded(bar, parity, abort_flag, p.status, where))
                 ? 1
                 : 0;
      ok = __shfl_sync(0xffffffffu, ok, 0);
      __syncwarp();
      return ok != 0;
    };
    float *wbuf = xbuf + (warp - 2) * 16 * 32;
    float *red = rbuf + (warp - 2) * 16 * 33;
    int it = 0;
    int qi = 0;
    uint32_t qph = 0;
    while (true) {
      if (!warp_wait(&uq_full[qi], qph, 57, true)) break;
      const int u = uq[qi];
      __syncwarp();
      if (lane == 0) {
        if (leader) mbar_arrive(&uq_empty[qi]);
        else mbar_arrive_remote(uq_empty_leader + qi * 8);
      }
      if (++qi == kUnitQ) {
        qi = 0;
        qph ^= 1;
      }
      if (u < 0) break;
      const int acc = it & 1;
      const uint32_t acc_phase = (it >> 1) & 1;
      ++it;
      if (!warp_wait(&tfull[acc], acc_phase, 58, false)) break;
      tc_fence_after();
      int g, mt, nt;
      decode(u, g, mt, nt);
      const int valid = min(BN, grp_count[g] - nt * BN);
      const int row0 = grp_row[g] + nt * BN;    // padded
      const int rowu0 = grp_rowu[g] + nt * BN;  // unpadded
      const int col_base = mt * 256 + (int)rank * 128 + q * 32;
      const int col = col_base + lane;
      const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + acc * C::ACC_COLS;
      if (MODE == BW_DH) {
        for (int n = threadIdx.x - 64; n < BN; n += 32 * kBwPairEpiWarps)
          row_scale[acc * BN + n] = (n < valid) ? p.row_scale[rowu0 + n] : 0.f;
        // all epilogue warps' scales are staged before any reads them: a bounded mbarrier (one
        // arrival per warp) instead of bar.sync, so a warp that aborts leaves none waiting
        __syncwarp();
        if (lane == 0) mbar_arrive(epi_bar);
        if (!warp_wait(epi_bar, (uint32_t)(it - 1) & 1, 74, false)) break;
      }
      uint32_t nx[16];
      const int c_first = 16 * eh;
      if (c_first < valid) tmem_ld16(taddr + c_first, nx);
      for (int c0 = c_first; c0 < valid; c0 += 32) {
        uint32_t v[16];
        tmem_ld_wait_regs(nx);
#pragma unroll
        for (int n = 0; n < 16; ++n) v[n] = nx[n];
        if (c0 + 32 < valid) tmem_ld16(taddr + c0 + 32, nx);
        float vals[16];
        if (MODE == BW_DX) {
#pragma unroll
          for (int n = 0; n < 16; ++n) vals[n] = __uint_as_float(v[n]);
          store_block16_f32(p.out, p.M, rowu0, c0, valid, col_base, vals, wbuf, lane);
        } else {
          float av[16], bv[16];
#pragma unroll
          for (int n = 0; n < 16; ++n) {
            const bool in = c0 + n < valid;
            const size_t i = (size_t)((p.pre_unpadded ? rowu0 : row0) + c0 + n) * p.M + col;
            av[n] = in ? p.pre_a[i] : 0.f;
            bv[n] = in ? p.pre_b[i] : 0.f;
          }
          float dav[16], dbv[16], hsv[16];
          const float4 *sc = reinterpret_cast<const float4 *>(row_scale + acc * BN + c0);
#pragma unroll
          for (int n4 = 0; n4 < 4; ++n4) {
            const float4 s4 = sc[n4];
            const float ss[4] = {s4.x, s4.y, s4.z, s4.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int n = 4 * n4 + e;
              const float a = av[n], b = bv[n], s = ss[e];
              const float dhu = __uint_as_float(v[n]);
              const float sig = __fdividef(1.f, 1.f + __expf(-a));
              const float silu = a * sig;
              const float h = silu * b;
              const float dh = s * dhu;
              vals[n] = dhu * h;
              dav[n] = dh * b * sig * (1.f + a * (1.f - sig));
              dbv[n] = dh * silu;
              hsv[n] = s * h;
            }
          }
          store_block16_bf16(p.da, p.M, row0, c0, valid, col_base, dav, wbuf, lane);
          store_block16_bf16(p.db, p.M, row0, c0, valid, col_base, dbv, wbuf, lane);
          store_block16_bf16(p.hs, p.M, row0, c0, valid, col_base, hsv, wbuf, lane);
#pragma unroll
          for (int n = 0; n < 16; ++n) red[n * 33 + lane] = vals[n];
          __syncwarp();
          if (lane < 16 && c0 + lane < valid && g < p.rows.E) {
            float sum = 0.f;
#pragma unroll 8
            for (int i = 0; i < 32; ++i) sum += red[lane * 33 + i];
            p.dgate_part[(size_t)(rowu0 + c0 + lane) * p.n_part + col_base / 32] = sum;
          }
          __syncwarp();
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (leader) mbar_arrive(&tempty[acc]);
        else mbar_arrive_remote(tempty_leader + acc * 8);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, C::TMEM_COLS);
  }
}

// ---------------------------------------------------------------------- wgrad GEMMs
constexpr int kWgOps = 5;    // sorted operands: dout, s*h, da, db, x
constexpr int kWgProbs = 3;  // dW_down, dW_gate, dW_up

struct BwWgradParams {
  CUtensorMap box[kWgOps];   // padded sorted rows [R, width] bf16, box {64, 64}
  CUtensorMap out[kWgProbs]; // dW as [G * M, N] fp32, box {32, 32}, 128-byte swizzle
  int a_op[kWgProbs], b_op[kWgProbs];  // operand of the M side and of the N side
  int M[kWgProbs], N[kWgProbs];        // dW[g] is [M, N]; M, N multiples of the unit tile
  int n_prob;
  BwRows rows;
  DevStatus *status;
  int n_groups;
  int *sched;     // work counter (zero at launch)
  int overwrite;  // 1: dW = this call's gradient (tiles stored, not added; experts no row
                  // chose get zero tiles); 0: dW += it (experts no row chose untouched)
};

constexpr int kWgStgBytes = 32 * 32 * 4;  // one 32 x 32 fp32 reduction tile

// Warp-wide epilogue of one weight-gradient unit: the warp's 32 accumulator rows (TMEM lane
// quadrant at `taddr`), 32-column chunks c = c_first, c_first + c_step, ... < n_cols, each
// registers -> swizzled staging tile -> TMA reduction into dW at (col0 + 32 c, row).  The
// warp cycles through NBUF staging tiles; lane 0 issues and tracks the reductions.  TMEM
// loads run one chunk ahead.
// `store`: tiles are stored instead of added; `zero`: the tiles are zeros (an expert no row
// chose, in the overwrite mode; TMEM is not read).
template <int NBUF>
__device__ __forceinline__ void wgrad_epilogue(uint32_t taddr, int c_first, int c_step, int n_cols,
                                               const CUtensorMap *omap, int col0, int row,
                                               uint8_t *stg, int &n_red, int lane, bool store,
                                               bool zero) {
  uint32_t n0[16], n1[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) n0[i] = n1[i] = 0u;
  if (!zero && 32 * c_first < n_cols) {
    tmem_ld16(taddr + 32 * c_first, n0);
    tmem_ld16(taddr + 32 * c_first + 16, n1);
  }
  for (int c = c_first; 32 * c < n_cols; c += c_step) {
    uint32_t v0[16], v1[16];
    if (!zero) tmem_ld_wait_regs(n0, n1);
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      v0[i] = n0[i];
      v1[i] = n1[i];
    }
    if (!zero && 32 * (c + c_step) < n_cols) {
      tmem_ld16(taddr + 32 * (c + c_step), n0);
      tmem_ld16(taddr + 32 * (c + c_step) + 16, n1);
    }
    uint8_t *buf = stg + (n_red % NBUF) * kWgStgBytes;
    if (n_red >= NBUF) {  // the reduction that last read this tile is done reading it
      if (lane == 0) bulk_wait_group_read<NBUF - 1>();
      __syncwarp();
    }
    // row `lane`, 16-byte chunk j of the row at position j ^ (lane & 7) (128-byte swizzle)
    uint8_t *r = buf + lane * 128;
#pragma unroll
    for (int j = 0; j < 4; ++j)
      *reinterpret_cast<float4 *>(r + ((j ^ (lane & 7)) << 4)) =
          make_float4(__uint_as_float(v0[4 * j]), __uint_as_float(v0[4 * j + 1]),
                      __uint_as_float(v0[4 * j + 2]), __uint_as_float(v0[4 * j + 3]));
#pragma unroll
    for (int j = 0; j < 4; ++j)
      *reinterpret_cast<float4 *>(r + (((j + 4) ^ (lane & 7)) << 4)) =
          make_float4(__uint_as_float(v1[4 * j]), __uint_as_float(v1[4 * j + 1]),
                      __uint_as_float(v1[4 * j + 2]), __uint_as_float(v1[4 * j + 3]));
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
      if (store) tma_store_2d(omap, buf, col0 + 32 * c, row);
      else tma_reduce_add_2d(omap, buf, col0 + 32 * c, row);
      bulk_commit_group();
    }
    ++n_red;
  }
}

// Group table and unit scan shared by both weight-gradient kernels: units of (problem,
// group) with rows, mtiles(pr) x ntiles(pr) each; exclusive prefix in unit_prefix.
template <int BMW, int BNW>
__device__ __forceinline__ void wgrad_unit_table(const BwWgradParams &p, int *unit_prefix,
                                                 int *grp_count, int *grp_row) {
  const int G = p.n_groups, NP = p.n_prob;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int g = threadIdx.x; g < G; g += blockDim.x) {
    int rowp, rowu, cnt;
    p.rows.group(g, rowp, rowu, cnt);
    grp_count[g] = cnt;
    grp_row[g] = rowp;
    for (int pr = 0; pr < NP; ++pr)
      unit_prefix[pr * G + g] =
          (cnt > 0 || p.overwrite) ? (p.M[pr] / BMW) * (p.N[pr] / BNW) : 0;
  }
  __syncthreads();
  if (warp == 0) {
    const int n = NP * G;
    const int per = (n + 31) / 32;
    const int lo = min(n, lane * per), hi = min(n, lo + per);
    int run = 0;
    for (int i = lo; i < hi; ++i) run += unit_prefix[i];
    int incl = run;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    int excl = incl - run;
    for (int i = lo; i < hi; ++i) {
      const int u = unit_prefix[i];
      unit_prefix[i] = excl;
      excl += u;
    }
    if (lane == 31) unit_prefix[n] = incl;
  }
}

// unit -> (problem, group, m tile, n tile), n tile innermost
template <int BNW>
__device__ __forceinline__ void wgrad_decode(const BwWgradParams &p, const int *unit_prefix, int u,
                                             int &pr, int &g, int &mt, int &nt) {
  const int G = p.n_groups;
  int lo = 0, hi = p.n_prob * G - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (unit_prefix[mid] <= u) lo = mid;
    else hi = mid - 1;
  }
  pr = lo / G;
  g = lo - pr * G;
  const int nts = p.N[pr] / BNW;
  const int loc = u - unit_prefix[lo];
  mt = loc / nts;
  nt = loc % nts;
}

template <int BNW>
struct BwWgradCfg {
  static constexpr int NB = BNW / 64;             // 64-element boxes on the N side
  static constexpr int BOX_BYTES = 64 * kBK * 2;  // 8 KB
  static constexpr int A_BYTES = 2 * BOX_BYTES;   // 128 M x 64 rows
  static constexpr int B_BYTES = NB * BOX_BYTES;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int ACC_COLS = BNW;
  static constexpr int TMEM_COLS = 2 * BNW;
  static constexpr int STG_BUFS = 2;
  static constexpr int STG_TOTAL = 4 * STG_BUFS * kWgStgBytes;
  static constexpr int STAGES_RAW = (220 * 1024 - STG_TOTAL) / STAGE_BYTES;
  static constexpr int STAGES = STAGES_RAW > 8 ? 8 : STAGES_RAW;
  static_assert(STAGES >= 2, "pipeline too shallow");
  static_assert(BNW == 128 || BNW == 256, "N tile");
  static constexpr int BAR_BYTES = (2 * STAGES + 5 + 2 * kUnitQ) * 8;
  static constexpr size_t smem_bytes(int n_groups) {
    return 1024 + (size_t)STAGES * STAGE_BYTES + STG_TOTAL + BAR_BYTES + 64 +
           (size_t)(kWgProbs * n_groups + 1) * 4 + (size_t)n_groups * 2 * 4 + 16;
  }
};

// One CTA per unit: 128 x BNW tile of dW[g].
template <int BNW>
__global__ void __launch_bounds__(kGemmThreads, 1)
    bw_wgrad_kernel(const __grid_constant__ BwWgradParams p) {
  using C = BwWgradCfg<BNW>;
  constexpr int S = C::STAGES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t *sA = smem;
  uint8_t *sB = sA + S * C::A_BYTES;
  uint8_t *stg = sB + S * C::B_BYTES;  // 1024-byte aligned
  uint64_t *bars = reinterpret_cast<uint64_t *>(stg + C::STG_TOTAL);
  uint64_t *full = bars;
  uint64_t *empty = bars + S;
  uint64_t *tfull = bars + 2 * S;
  uint64_t *tempty = bars + 2 * S + 2;
  uint64_t *drain = bars + 2 * S + 4;
  uint64_t *uq_full = bars + 2 * S + 5;
  uint64_t *uq_empty = uq_full + kUnitQ;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(uq_empty + kUnitQ);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
  volatile int *uq = reinterpret_cast<volatile int *>(tmem_slot + 4);  // [kUnitQ]
  const int G = p.n_groups;
  int *unit_prefix = reinterpret_cast<int *>(tmem_slot + 16);  // [NP * G + 1]
  int *grp_count = unit_prefix + p.n_prob * G + 1;              // [G]
  int *grp_row = grp_count + G;                                 // [G] padded

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

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
    for (int q = 0; q < kUnitQ; ++q) {
      mbar_init(&uq_full[q], 1);
      mbar_init(&uq_empty[q], 5);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(tmem_slot, C::TMEM_COLS);
  griddep_wait();
  griddep_launch_dependents();
  wgrad_unit_table<kBM, BNW>(p, unit_prefix, grp_count, grp_row);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int total_units = unit_prefix[p.n_prob * G];

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int issued = 0;
      bool ok = true;
      int qi = 0;
      uint32_t qph = 0;
      for (;;) {
        const int u = atomicAdd(p.sched, 1);
        const int uid = (u < total_units) ? u : -1;
        if (!mbar_wait_bounded(&uq_empty[qi], qph ^ 1, abort_flag, p.status, 31)) {
          ok = false;
          break;
        }
        uq[qi] = uid;
        mbar_arrive(&uq_full[qi]);
        if (++qi == kUnitQ) {
          qi = 0;
          qph ^= 1;
        }
        if (uid < 0) break;
        int pr, g, mt, nt;
        wgrad_decode<BNW>(p, unit_prefix, uid, pr, g, mt, nt);
        const CUtensorMap *abox = &p.box[p.a_op[pr]], *bbox = &p.box[p.b_op[pr]];
        const int m0 = mt * kBM, n0 = nt * BNW;
        const int kbs = (grp_count[g] + kBK - 1) / kBK;
        for (int kb = 0; kb < kbs; ++kb) {
          const int r0 = grp_row[g] + kb * kBK;
          if (!mbar_wait_bounded(&empty[stage], phase ^ 1, abort_flag, p.status, 32)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[stage], C::STAGE_BYTES);
          uint8_t *a_dst = sA + stage * C::A_BYTES;
          uint8_t *b_dst = sB + stage * C::B_BYTES;
          tma_load_2d(a_dst, abox, &full[stage], m0, r0);
          tma_load_2d(a_dst + C::BOX_BYTES, abox, &full[stage], m0 + 64, r0);
#pragma unroll
          for (int h = 0; h < C::NB; ++h)
            tma_load_2d(b_dst + h * C::BOX_BYTES, bbox, &full[stage], n0 + 64 * h, r0);
          ++issued;
          if (++stage == S) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
      }
      if (!ok) {
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
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------------------ MMA issuer
      int stage = 0;
      uint32_t phase = 0;
      int it = 0;
      bool ok = true;
      int qi = 0;
      uint32_t qph = 0;
      constexpr uint32_t idesc = idesc_bf16_f32_major(kBM, BNW, true, true);
      while (ok) {
        if (!mbar_wait_bounded(&uq_full[qi], qph, abort_flag, p.status, 33)) break;
        const int u = uq[qi];
        mbar_arrive(&uq_empty[qi]);
        if (++qi == kUnitQ) {
          qi = 0;
          qph ^= 1;
        }
        if (u < 0) break;
        int pr, g, mt, nt;
        wgrad_decode<BNW>(p, unit_prefix, u, pr, g, mt, nt);
        const int cnt = grp_count[g];
        if (cnt == 0) continue;  // zero tile of the overwrite mode: no MMA, no accumulator
        const int acc = it & 1;
        const uint32_t acc_phase = (it >> 1) & 1;
        ++it;
        if (!mbar_wait_bounded(&tempty[acc], acc_phase ^ 1, abort_flag, p.status, 34)) break;
        tc_fence_after();
        const int kbs = (cnt + kBK - 1) / kBK;
        const uint32_t d0 = tmem_base + acc * C::ACC_COLS;
        for (int kb = 0; kb < kbs; ++kb) {
          if (!mbar_wait_bounded(&full[stage], phase, abort_flag, p.status, 35)) {
            ok = false;
            break;
          }
          tc_fence_after();
          // 16-row steps up to the group's padded end (padding rows are zero)
          const int k16 = (min(kBK, cnt - kb * kBK) + 15) >> 4;
          const uint32_t a = smem_u32(sA + stage * C::A_BYTES);
          const uint32_t b = smem_u32(sB + stage * C::B_BYTES);
          for (int kk = 0; kk < k16; ++kk)
            tc_mma_bf16(d0, sdesc_mn_sw128(a + kk * 16 * 128, C::BOX_BYTES),
                        sdesc_mn_sw128(b + kk * 16 * 128, C::BOX_BYTES), idesc,
                        (kb | kk) ? 1u : 0u);
          tc_commit(&empty[stage]);
          if (++stage == S) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (ok) tc_commit(&tfull[acc]);
      }
      tc_commit(drain);
      volatile int no_abort = 0;
      mbar_wait_bounded(drain, 0, &no_abort, nullptr, 0);
    }
    __syncwarp();
  } else {
    // --------------------------------------------------------------------- epilogue
    const int q = warp & 3;
    auto warp_wait = [&](uint64_t *bar, uint32_t parity, int where) -> bool {
      int ok = 1;
      if (lane == 0) ok = mbar_wait_bounded(bar, parity, abort_flag, p.status, where) ? 1 : 0;
      ok = __shfl_sync(0xffffffffu, ok, 0);
      __syncwarp();
      return ok != 0;
    };
    uint8_t *my_stg = stg + q * C::STG_BUFS * kWgStgBytes;
    int it = 0, n_red = 0;
    int qi = 0;
    uint32_t qph = 0;
    while (true) {
      if (!warp_wait(&uq_full[qi], qph, 36)) break;
      const int u = uq[qi];
      __syncwarp();
      if (lane == 0) mbar_arrive(&uq_empty[qi]);
      if (++qi == kUnitQ) {
        qi = 0;
        qph ^= 1;
      }
      if (u < 0) break;
      int pr, g, mt, nt;
      wgrad_decode<BNW>(p, unit_prefix, u, pr, g, mt, nt);
      const int out_row = g * p.M[pr] + mt * kBM + q * 32;
      if (grp_count[g] == 0) {  // overwrite mode, expert no row chose: a zero tile
        wgrad_epilogue<C::STG_BUFS>(0, 0, 1, BNW, &p.out[pr], nt * BNW, out_row, my_stg, n_red,
                                    lane, true, true);
        continue;
      }
      const int acc = it & 1;
      const uint32_t acc_phase = (it >> 1) & 1;
      ++it;
      if (!warp_wait(&tfull[acc], acc_phase, 37)) break;
      tc_fence_after();
      const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + acc * C::ACC_COLS;
      wgrad_epilogue<C::STG_BUFS>(taddr, 0, 1, BNW, &p.out[pr], nt * BNW, out_row, my_stg, n_red,
                                  lane, p.overwrite != 0, false);
      tc_fence_before();
      mbar_arrive(&tempty[acc]);
    }
    if (lane == 0) bulk_wait_group_all();
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

// CTA-pair weight-gradient kernel: 256 x 256 tiles of dW[g] on a cluster of two CTAs
// (tcgen05 cta_group::2).  CTA r stages rows [128 r, 128 r + 128) of the unit's M range and
// columns [128 r, 128 r + 128) of its N range for every 64-row K block (32 KB), the leader
// issues M = 256, N = 256 MMAs, and each CTA's TMEM receives its 128 rows for all 256
// columns.  Per staged byte this is 1.5x the MMA work of the one-CTA 128 x 256 tile, which
// matters because the K loops are short (a group's rows) and the tiles are re-read from L2
// for every output tile.  Barriers and unit publication as in grouped_gemm_pair.cuh: full[s]
// lives in the leader and counts both CTAs' bytes, the MMA commits arrive in both CTAs, and
// tempty / uq_empty (leader) collect the arrivals of both CTAs' warps.
constexpr int kWgPairEpiWarps = 8;  // two per TMEM lane quadrant, alternating 32-column chunks
constexpr int kWgPairThreads = 32 * (2 + kWgPairEpiWarps);

struct BwWgradPairCfg {
  static constexpr int BOX_BYTES = 64 * kBK * 2;  // 8 KB
  static constexpr int A_BYTES = 2 * BOX_BYTES;   // this CTA's 128 M x 64 rows
  static constexpr int B_BYTES = 2 * BOX_BYTES;   // this CTA's 128 N x 64 rows
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int ACC_COLS = 256;
  static constexpr int TMEM_COLS = 512;
  static constexpr int STG_BUFS = 2;
  static constexpr int STG_TOTAL = kWgPairEpiWarps * STG_BUFS * kWgStgBytes;
  static constexpr int STAGES_RAW = (220 * 1024 - STG_TOTAL) / STAGE_BYTES;
  static constexpr int STAGES = STAGES_RAW > 8 ? 8 : STAGES_RAW;
  static_assert(STAGES >= 2, "pipeline too shallow");
  static constexpr int BAR_BYTES = (2 * STAGES + 5 + 2 * kUnitQ) * 8;
  static constexpr size_t smem_bytes(int n_groups) {
    return 1024 + (size_t)STAGES * STAGE_BYTES + STG_TOTAL + BAR_BYTES + 64 +
           (size_t)(kWgProbs * n_groups + 1) * 4 + (size_t)n_groups * 2 * 4 + 16;
  }
};

__global__ void __launch_bounds__(kWgPairThreads, 1)
    bw_wgrad_pair_kernel(const __grid_constant__ BwWgradParams p) {
  using C = BwWgradPairCfg;
  constexpr int S = C::STAGES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t *sA = smem;
  uint8_t *sB = sA + S * C::A_BYTES;
  uint8_t *stg = sB + S * C::B_BYTES;  // 1024-byte aligned
  uint64_t *bars = reinterpret_cast<uint64_t *>(stg + C::STG_TOTAL);
  uint64_t *full = bars;
  uint64_t *empty = bars + S;
  uint64_t *tfull = bars + 2 * S;
  uint64_t *tempty = bars + 2 * S + 2;
  uint64_t *drain = bars + 2 * S + 4;
  uint64_t *uq_full = bars + 2 * S + 5;
  uint64_t *uq_empty = uq_full + kUnitQ;  // used in the leader only
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(uq_empty + kUnitQ);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
  volatile int *uq = reinterpret_cast<volatile int *>(tmem_slot + 4);  // [kUnitQ]
  const int G = p.n_groups;
  int *unit_prefix = reinterpret_cast<int *>(tmem_slot + 16);  // [NP * G + 1]
  int *grp_count = unit_prefix + p.n_prob * G + 1;              // [G]
  int *grp_row = grp_count + G;                                 // [G] padded

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 2 * kWgPairEpiWarps);  // one per epilogue warp of both CTAs
    }
    mbar_init(drain, 1);
    for (int q = 0; q < kUnitQ; ++q) {
      mbar_init(&uq_full[q], 1);
      // readers of a published unit id: the leader's MMA thread and epilogue warps, the
      // peer's producer and epilogue warps
      mbar_init(&uq_empty[q], 2 + 2 * kWgPairEpiWarps);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc_pair(tmem_slot, C::TMEM_COLS);
  griddep_wait();
  griddep_launch_dependents();
  wgrad_unit_table<2 * kBM, 256>(p, unit_prefix, grp_count, grp_row);
  // both CTAs' barriers are initialised and TMEM allocated before any cross-CTA traffic
  tc_fence_before();
  __syncthreads();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int total_units = unit_prefix[p.n_prob * G];

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ TMA producer
      const uint64_t pol = policy_evict_last();
      int stage = 0;
      uint32_t phase = 0;
      int issued = 0;
      bool ok = true;
      int qi = 0;
      uint32_t qph = 0;
      int u = -1;
      while (ok) {
        if (leader) {
          const int c = atomicAdd(p.sched, 1);
          const int uid = (c < total_units) ? c : -1;
          if (!mbar_wait_bounded<true>(&uq_empty[qi], qph ^ 1, abort_flag, p.status, 41)) {
            ok = false;
            break;
          }
          uq[qi] = uid;
          st_shared_remote(mapa_shared(smem_u32((const void *)&uq[qi]), 1), uid);
          mbar_arrive(&uq_full[qi]);
          mbar_arrive_remote(mapa_shared(smem_u32(&uq_full[qi]), 1));
          u = uid;
        } else {
          if (!mbar_wait_bounded<true>(&uq_full[qi], qph, abort_flag, p.status, 42)) {
            ok = false;
            break;
          }
          u = uq[qi];
          mbar_arrive_remote(mapa_shared(smem_u32(&uq_empty[qi]), 0));
        }
        if (++qi == kUnitQ) {
          qi = 0;
          qph ^= 1;
        }
        if (u < 0) break;
        int pr, g, mt, nt;
        wgrad_decode<256>(p, unit_prefix, u, pr, g, mt, nt);
        const CUtensorMap *abox = &p.box[p.a_op[pr]], *bbox = &p.box[p.b_op[pr]];
        const int ma = mt * 256 + (int)rank * 128, nb = nt * 256 + (int)rank * 128;
        const int kbs = (grp_count[g] + kBK - 1) / kBK;
        for (int kb = 0; kb < kbs; ++kb) {
          const int r0 = grp_row[g] + kb * kBK;
          if (!mbar_wait_bounded(&empty[stage], phase ^ 1, abort_flag, p.status, 43)) {
            ok = false;
            break;
          }
          const uint32_t fbar = mapa_shared(smem_u32(&full[stage]), 0);
          if (leader) mbar_arrive_expect_tx(&full[stage], 2 * C::STAGE_BYTES);
          uint8_t *a_dst = sA + stage * C::A_BYTES;
          uint8_t *b_dst = sB + stage * C::B_BYTES;
          tma_load_2d_pair(a_dst, abox, fbar, ma, r0, pol);
          tma_load_2d_pair(a_dst + C::BOX_BYTES, abox, fbar, ma + 64, r0, pol);
          tma_load_2d_pair(b_dst, bbox, fbar, nb, r0, pol);
          tma_load_2d_pair(b_dst + C::BOX_BYTES, bbox, fbar, nb + 64, r0, pol);
          ++issued;
          if (++stage == S) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      if (!ok && leader) {
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
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      // ------------------------------------------------------------ MMA issuer (leader)
      int stage = 0;
      uint32_t phase = 0;
      int it = 0;
      bool ok = true;
      int qi = 0;
      uint32_t qph = 0;
      constexpr uint32_t idesc = idesc_bf16_f32_major(2 * kBM, 256, true, true);
      while (ok) {
        if (!mbar_wait_bounded<true>(&uq_full[qi], qph, abort_flag, p.status, 44)) break;
        const int u = uq[qi];
        mbar_arrive(&uq_empty[qi]);
        if (++qi == kUnitQ) {
          qi = 0;
          qph ^= 1;
        }
        if (u < 0) break;
        int pr, g, mt, nt;
        wgrad_decode<256>(p, unit_prefix, u, pr, g, mt, nt);
        const int cnt = grp_count[g];
        if (cnt == 0) continue;  // zero tile of the overwrite mode
        const int acc = it & 1;
        const uint32_t acc_phase = (it >> 1) & 1;
        ++it;
        if (!mbar_wait_bounded(&tempty[acc], acc_phase ^ 1, abort_flag, p.status, 45)) break;
        tc_fence_after();
        const int kbs = (cnt + kBK - 1) / kBK;
        const uint32_t d0 = tmem_base + acc * C::ACC_COLS;
        for (int kb = 0; kb < kbs; ++kb) {
          if (!mbar_wait_bounded(&full[stage], phase, abort_flag, p.status, 46)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const int k16 = (min(kBK, cnt - kb * kBK) + 15) >> 4;
          const uint32_t a = smem_u32(sA + stage * C::A_BYTES);
          const uint32_t b = smem_u32(sB + stage * C::B_BYTES);
          for (int kk = 0; kk < k16; ++kk)
            tc_mma_bf16_pair(d0, sdesc_mn_sw128(a + kk * 16 * 128, C::BOX_BYTES),
                             sdesc_mn_sw128(b + kk * 16 * 128, C::BOX_BYTES), idesc,
                             (kb | kk) ? 1u : 0u);
          tc_commit_pair_both(&empty[stage]);  // slot free in both CTAs once read
          if (++stage == S) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (ok) tc_commit_pair_both(&tfull[acc]);
      }
      tc_commit_pair_local(drain);
      volatile int no_abort = 0;
      mbar_wait_bounded(drain, 0, &no_abort, nullptr, 0);
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------------- epilogue (both CTAs)
    const int q = warp & 3;          // TMEM lane quadrant
    const int eh = (warp - 2) >> 2;  // which of the quadrant's two warps: chunks eh, eh + 2, ..
    const uint32_t tempty_leader = mapa_shared(smem_u32(&tempty[0]), 0);
    const uint32_t uq_empty_leader = mapa_shared(smem_u32(&uq_empty[0]), 0);
    auto warp_wait = [&](uint64_t *bar, uint32_t parity, int where, bool cluster) -> bool {
      int ok = 1;
      if (lane == 0)
        ok = (cluster ? mbar_wait_bounded<true>(bar, parity, abort_flag, p.status, where)
                      : mbar_wait_bounded(bar, parity, abort_flag, p.status, where))
                 ? 1
                 : 0;
      ok = __shfl_sync(0xffffffffu, ok, 0);
      __syncwarp();
      return ok != 0;
    };
    uint8_t *my_stg = stg + (warp - 2) * C::STG_BUFS * kWgStgBytes;
    int it = 0, n_red = 0;
    int qi = 0;
    uint32_t qph = 0;
    while (true) {
      if (!warp_wait(&uq_full[qi], qph, 47, true)) break;
      const int u = uq[qi];
      __syncwarp();
      if (lane == 0) {
        if (leader) mbar_arrive(&uq_empty[qi]);
        else mbar_arrive_remote(uq_empty_leader + qi * 8);
      }
      if (++qi == kUnitQ) {
        qi = 0;
        qph ^= 1;
      }
      if (u < 0) break;
      int pr, g, mt, nt;
      wgrad_decode<256>(p, unit_prefix, u, pr, g, mt, nt);
      const int out_row = g * p.M[pr] + mt * 256 + (int)rank * 128 + q * 32;
      if (grp_count[g] == 0) {  // overwrite mode, expert no row chose: a zero tile
        wgrad_epilogue<C::STG_BUFS>(0, eh, 2, 256, &p.out[pr], nt * 256, out_row, my_stg, n_red,
                                    lane, true, true);
        continue;
      }
      const int acc = it & 1;
      const uint32_t acc_phase = (it >> 1) & 1;
      ++it;
      if (!warp_wait(&tfull[acc], acc_phase, 48, false)) break;
      tc_fence_after();
      const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + acc * C::ACC_COLS;
      wgrad_epilogue<C::STG_BUFS>(taddr, eh, 2, 256, &p.out[pr], nt * 256, out_row, my_stg,
                                  n_red, lane, p.overwrite != 0, false);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (leader) mbar_arrive(&tempty[acc]);
        else mbar_arrive_remote(tempty_leader + acc * 8);
      }
    }
    if (lane == 0) bulk_wait_group_all();
    __syncwarp();
  }

  // the pair leaves together: the leader's MMAs read the peer's shared memory, and the
  // peer's TMA loads signal the leader's barriers
  tc_fence_before();
  __syncthreads();
  cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, C::TMEM_COLS);
  }
}

// ------------------------------------------------------------ dx rows + weight gradients
// One persistent CTA-pair kernel for the two steps that follow DH: the dgrad units of DX
// (256 d rows x up to 256 tokens, K = 2 f, bound by moving weight and activation tiles into
// the SMs) and the weight-gradient units (256 x 256 tiles of dW, K = the group's rows, bound
// by the fp32 gradient read-modify-write in HBM).  Units are listed group by group, each
// group's DX units first, so the pairs claiming consecutive units run both kinds at once and
// the two bottlenecks overlap.  Stage layout (32 KB per CTA: a 128-row MN-major A tile and a
// 128-row B tile), barriers and unit publication are those of the two pair kernels above.
struct BwTailParams {
  BwDgradParams dx;  // DX: tmA0/tmA1 = W_gate/W_up (MN-major), tmB0/tmB1 = da/db (box {64, 128})
  BwWgradParams wg;  // weight gradients (256 x 256 tiles)
};

struct BwTailPairCfg {
  static constexpr int BOX_BYTES = 64 * kBK * 2;  // 8 KB
  static constexpr int A_BYTES = 2 * BOX_BYTES;   // this CTA's 128 M rows x 64 K
  static constexpr int B_BYTES = 2 * BOX_BYTES;   // 128 N columns (wgrad) / tokens (dx) x 64 K
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int ACC_COLS = 256;
  static constexpr int TMEM_COLS = 512;
  static constexpr int STG_BUFS = 2;
  static constexpr int STG_TOTAL = kWgPairEpiWarps * STG_BUFS * kWgStgBytes;
  static constexpr int XBUF_BYTES = kWgPairEpiWarps * 16 * 32 * 4;
  static constexpr int STAGES_RAW = (212 * 1024 - STG_TOTAL - XBUF_BYTES) / STAGE_BYTES;
  static constexpr int STAGES = STAGES_RAW > 8 ? 8 : STAGES_RAW;
  static_assert(STAGES >= 2, "pipeline too shallow");
  static constexpr int BAR_BYTES = (2 * STAGES + 5 + 2 * kUnitQ) * 8;
  static constexpr size_t smem_bytes(int n_groups) {
    return 1024 + (size_t)STAGES * STAGE_BYTES + STG_TOTAL + XBUF_BYTES + BAR_BYTES + 64 +
           (size_t)(4 * n_groups + 1) * 4 + 16;
  }
};

__global__ void __launch_bounds__(kWgPairThreads, 1)
    bw_tail_pair_kernel(const __grid_constant__ BwTailParams P) {
  using C = BwTailPairCfg;
  constexpr int S = C::STAGES;
  const BwDgradParams &px = P.dx;
  const BwWgradParams &pw = P.wg;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t *sA = smem;
  uint8_t *sB = sA + S * C::A_BYTES;
  uint8_t *stg = sB + S * C::B_BYTES;  // 1024-byte aligned
  float *xbuf = reinterpret_cast<float *>(stg + C::STG_TOTAL);
  uint64_t *bars = reinterpret_cast<uint64_t *>(stg + C::STG_TOTAL + C::XBUF_BYTES);
  uint64_t *full = bars;
  uint64_t *empty = bars + S;
  uint64_t *tfull = bars + 2 * S;
  uint64_t *tempty = bars + 2 * S + 2;
  uint64_t *drain = bars + 2 * S + 4;
  uint64_t *uq_full = bars + 2 * S + 5;
  uint64_t *uq_empty = uq_full + kUnitQ;  // used in the leader only
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(uq_empty + kUnitQ);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
  volatile int *uq = reinterpret_cast<volatile int *>(tmem_slot + 4);  // [kUnitQ]
  const int G = pw.n_groups;
  int *unit_prefix = reinterpret_cast<int *>(tmem_slot + 16);  // [G + 1]
  int *grp_count = unit_prefix + G + 1;                         // [G]
  int *grp_row = grp_count + G;                                 // [G] padded
  int *grp_rowu = grp_row + G;                                  // [G] unpadded

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int dx_mtiles = px.M / 256;
  const int dx_kpp = px.K / kBK;
  const int dx_kblocks = 2 * dx_kpp;
  int wg_units_per_group = 0;  // the same for every group with rows
  for (int pr = 0; pr < pw.n_prob; ++pr) wg_units_per_group += (pw.M[pr] / 256) * (pw.N[pr] / 256);

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 2 * kWgPairEpiWarps);
    }
    mbar_init(drain, 1);
    for (int q = 0; q < kUnitQ; ++q) {
      mbar_init(&uq_full[q], 1);
      mbar_init(&uq_empty[q], 2 + 2 * kWgPairEpiWarps);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc_pair(tmem_slot, C::TMEM_COLS);
  griddep_wait();
  griddep_launch_dependents();
  for (int g = threadIdx.x; g < G; g += blockDim.x) {
    int rowp, rowu, cnt;
    pw.rows.group(g, rowp, rowu, cnt);
    grp_count[g] = cnt;
    grp_row[g] = rowp;
    grp_rowu[g] = rowu;
    unit_prefix[g] = (cnt > 0 ? dx_mtiles * ((cnt + 255) / 256) : 0) +
                     ((cnt > 0 || pw.overwrite) ? wg_units_per_group : 0);
  }
  __syncthreads();
  if (warp == 0) {
    const int per = (G + 31) / 32;
    const int lo = min(G, lane * per), hi = min(G, lo + per);
    int run = 0;
    for (int g = lo; g < hi; ++g) run += unit_prefix[g];
    int incl = run;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    int excl = incl - run;
    for (int g = lo; g < hi; ++g) {
      const int u = unit_prefix[g];
      unit_prefix[g] = excl;
      excl += u;
    }
    if (lane == 31) unit_prefix[G] = incl;
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int total_units = unit_prefix[G];

  // unit -> group and kind: dx (pr = -1; mt, nt over d rows / tokens) or weight gradient
  // (problem pr; mt, nt over the 256 x 256 tiles of dW, n innermost)
  auto decode = [&](int u, int &g, int &pr, int &mt, int &nt) {
    int lo = 0, hi = G - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (unit_prefix[mid] <= u) lo = mid;
      else hi = mid - 1;
    }
    g = lo;
    int loc = u - unit_prefix[g];
    const int nts = (grp_count[g] + 255) / 256;
    if (loc < dx_mtiles * nts) {
      pr = -1;
      mt = loc / nts;
      nt = loc % nts;
      return;
    }
    loc -= dx_mtiles * nts;
    for (pr = 0; pr < pw.n_prob; ++pr) {
      const int n_here = (pw.M[pr] / 256) * (pw.N[pr] / 256);
      if (loc < n_here) break;
      loc -= n_here;
    }
    const int ntw = pw.N[pr] / 256;
    mt = loc / ntw;
    nt = loc % ntw;
  };
  // dx token split: CTA r holds tokens [n0 + r*half, n0 + (r+1)*half), N = 2*half
  auto split = [&](int g, int nt) {
    const int valid = min(256, grp_count[g] - nt * 256);
    return (((valid + 1) >> 1) + 7) & ~7;
  };

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ TMA producer
      const uint64_t pol_w = policy_evict_first();
      const uint64_t pol_b = policy_evict_last();
      int stage = 0;
      uint32_t phase = 0;
      int issued = 0;
      bool ok = true;
      int qi = 0;
      uint32_t qph = 0;
      int u = -1;
      while (ok) {
        if (leader) {
          const int c = atomicAdd(pw.sched, 1);
          const int uid = (c < total_units) ? c : -1;
          if (!mbar_wait_bounded<true>(&uq_empty[qi], qph ^ 1, abort_flag, pw.status, 61)) {
            ok = false;
            break;
          }
          uq[qi] = uid;
          st_shared_remote(mapa_shared(smem_u32((const void *)&uq[qi]), 1), uid);
          mbar_arrive(&uq_full[qi]);
          mbar_arrive_remote(mapa_shared(smem_u32(&uq_full[qi]), 1));
          u = uid;
        } else {
          if (!mbar_wait_bounded<true>(&uq_full[qi], qph, abort_flag, pw.status, 62)) {
            ok = false;
            break;
          }
          u = uq[qi];
          mbar_arrive_remote(mapa_shared(smem_u32(&uq_empty[qi]), 0));
        }
        if (++qi == kUnitQ) {
          qi = 0;
          qph ^= 1;
        }
        if (u < 0) break;
        int g, pr, mt, nt;
        decode(u, g, pr, mt, nt);
        const int kbs = (pr < 0) ? dx_kblocks : (grp_count[g] + kBK - 1) / kBK;
        for (int kb = 0; kb < kbs; ++kb) {
          if (!mbar_wait_bounded(&empty[stage], phase ^ 1, abort_flag, pw.status, 63)) {
            ok = false;
            break;
          }
          const uint32_t fbar = mapa_shared(smem_u32(&full[stage]), 0);
          if (leader) mbar_arrive_expect_tx(&full[stage], 2 * C::STAGE_BYTES);
          uint8_t *a_dst = sA + stage * C::A_BYTES;
          uint8_t *b_dst = sB + stage * C::B_BYTES;
          if (pr < 0) {
            const int pair = kb / dx_kpp;
            const int kc = (kb - pair * dx_kpp) * kBK;
            const CUtensorMap *amap = pair ? &px.tmA1 : &px.tmA0;
            const CUtensorMap *bmap = pair ? &px.tmB1 : &px.tmB0;
            const int a_x = mt * 256 + (int)rank * 128;
            const int a_row = g * px.K + kc;
            tma_load_2d_pair(a_dst, amap, fbar, a_x, a_row, pol_w);
            tma_load_2d_pair(a_dst + C::BOX_BYTES, amap, fbar, a_x + 64, a_row, pol_w);
            tma_load_2d_pair(b_dst, bmap, fbar, kc,
                             grp_row[g] + nt * 256 + (int)rank * split(g, nt), pol_b);
          } else {
            const CUtensorMap *abox = &pw.box[pw.a_op[pr]], *bbox = &pw.box[pw.b_op[pr]];
            const int ma = mt * 256 + (int)rank * 128, nb = nt * 256 + (int)rank * 128;
            const int r0 = grp_row[g] + kb * kBK;
            tma_load_2d_pair(a_dst, abox, fbar, ma, r0, pol_b);
            tma_load_2d_pair(a_dst + C::BOX_BYTES, abox, fbar, ma + 64, r0, pol_b);
            tma_load_2d_pair(b_dst, bbox, fbar, nb, r0, pol_b);
            tma_load_2d_pair(b_dst + C::BOX_BYTES, bbox, fbar, nb + 64, r0, pol_b);
          }
          ++issued;
          if (++stage == S) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      if (!ok && leader) {
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
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      // ------------------------------------------------------------ MMA issuer (leader)
      int stage = 0;
      uint32_t phase = 0;
      int it = 0;
      bool ok = true;
      int qi = 0;
      uint32_t qph = 0;
      while (ok) {
        if (!mbar_wait_bounded<true>(&uq_full[qi], qph, abort_flag, pw.status, 64)) break;
        const int u = uq[qi];
        mbar_arrive(&uq_empty[qi]);
        if (++qi == kUnitQ) {
          qi = 0;
          qph ^= 1;
        }
        if (u < 0) break;
        int g, pr, mt, nt;
        decode(u, g, pr, mt, nt);
        const int cnt = grp_count[g];
        if (cnt == 0) continue;  // zero tile of the overwrite mode
        const int acc = it & 1;
        const uint32_t acc_phase = (it >> 1) & 1;
        ++it;
        if (!mbar_wait_bounded(&tempty[acc], acc_phase ^ 1, abort_flag, pw.status, 65)) break;
        tc_fence_after();
        const int kbs = (pr < 0) ? dx_kblocks : (cnt + kBK - 1) / kBK;
        const uint32_t idesc = (pr < 0)
                                   ? idesc_bf16_f32_major(256, 2 * split(g, nt), true, false)
                                   : idesc_bf16_f32_major(256, 256, true, true);
        const uint32_t d0 = tmem_base + acc * C::ACC_COLS;
        for (int kb = 0; kb < kbs; ++kb) {
          if (!mbar_wait_bounded(&full[stage], phase, abort_flag, pw.status, 66)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a = smem_u32(sA + stage * C::A_BYTES);
          const uint32_t b = smem_u32(sB + stage * C::B_BYTES);
          if (pr < 0) {
#pragma unroll
            for (int kk = 0; kk < kBK / 16; ++kk)
              tc_mma_bf16_pair(d0, sdesc_mn_sw128(a + kk * 16 * 128, C::BOX_BYTES),
                               sdesc_k_sw128(b + kk * 32), idesc, (kb | kk) ? 1u : 0u);
          } else {
            const int k16 = (min(kBK, cnt - kb * kBK) + 15) >> 4;
            for (int kk = 0; kk < k16; ++kk)
              tc_mma_bf16_pair(d0, sdesc_mn_sw128(a + kk * 16 * 128, C::BOX_BYTES),
                               sdesc_mn_sw128(b + kk * 16 * 128, C::BOX_BYTES), idesc,
                               (kb | kk) ? 1u : 0u);
          }
          tc_commit_pair_both(&empty[stage]);
          if (++stage == S) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (ok) tc_commit_pair_both(&tfull[acc]);
      }
      tc_commit_pair_local(drain);
      volatile int no_abort = 0;
      mbar_wait_bounded(drain, 0, &no_abort, nullptr, 0);
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------------- epilogue (both CTAs)
    const int q = warp & 3;
    const int eh = (warp - 2) >> 2;
    const uint32_t tempty_leader = mapa_shared(smem_u32(&tempty[0]), 0);
    const uint32_t uq_empty_leader = mapa_shared(smem_u32(&uq_empty[0]), 0);
    auto warp_wait = [&](uint64_t *bar, uint32_t parity, int where, bool cluster) -> bool {
      int ok = 1;
      if (lane == 0)
        ok = (cluster ? mbar_wait_bounded<true>(bar, parity, abort_flag, pw.status, where)
                      : mbar_wait_bounded(bar, parity, abort_flag, pw.status, where))
                 ? 1
                 : 0;
      ok = __shfl_sync(0xffffffffu, ok, 0);
      __syncwarp();
      return ok != 0;
    };
    uint8_t *my_stg = stg + (warp - 2) * C::STG_BUFS * kWgStgBytes;
    float *wbuf = xbuf + (warp - 2) * 16 * 32;
    int it = 0, n_red = 0;
    int qi = 0;
    uint32_t qph = 0;
    while (true) {
      if (!warp_wait(&uq_full[qi], qph, 67, true)) break;
      const int u = uq[qi];
      __syncwarp();
      if (lane == 0) {
        if (leader) mbar_arrive(&uq_empty[qi]);
        else mbar_arrive_remote(uq_empty_leader + qi * 8);
      }
      if (++qi == kUnitQ) {
        qi = 0;
        qph ^= 1;
      }
      if (u < 0) break;
      int g, pr, mt, nt;
      decode(u, g, pr, mt, nt);
      if (grp_count[g] == 0) {  // overwrite mode, expert no row chose: a zero tile
        wgrad_epilogue<C::STG_BUFS>(0, eh, 2, 256, &pw.out[pr], nt * 256,
                                    g * pw.M[pr] + mt * 256 + (int)rank * 128 + q * 32, my_stg,
                                    n_red, lane, true, true);
        continue;
      }
      const int acc = it & 1;
      const uint32_t acc_phase = (it >> 1) & 1;
      ++it;
      if (!warp_wait(&tfull[acc], acc_phase, 68, false)) break;
      tc_fence_after();
      const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + acc * C::ACC_COLS;
      if (pr < 0) {
        // rows of dx: fp32, tokens of this unit at unpadded rows
        const int valid = min(256, grp_count[g] - nt * 256);
        const int rowu0 = grp_rowu[g] + nt * 256;
        const int col_base = mt * 256 + (int)rank * 128 + q * 32;
        uint32_t nx[16];
        const int c_first = 16 * eh;
        if (c_first < valid) tmem_ld16(taddr + c_first, nx);
        for (int c0 = c_first; c0 < valid; c0 += 32) {
          uint32_t v[16];
          tmem_ld_wait_regs(nx);
#pragma unroll
          for (int n = 0; n < 16; ++n) v[n] = nx[n];
          if (c0 + 32 < valid) tmem_ld16(taddr + c0 + 32, nx);
          float vals[16];
#pragma unroll
          for (int n = 0; n < 16; ++n) vals[n] = __uint_as_float(v[n]);
          store_block16_f32(px.out, px.M, rowu0, c0, valid, col_base, vals, wbuf, lane);
        }
      } else {
        wgrad_epilogue<C::STG_BUFS>(taddr, eh, 2, 256, &pw.out[pr], nt * 256,
                                    g * pw.M[pr] + mt * 256 + (int)rank * 128 + q * 32, my_stg,
                                    n_red, lane, pw.overwrite != 0, false);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (leader) mbar_arrive(&tempty[acc]);
        else mbar_arrive_remote(tempty_leader + acc * 8);
      }
    }
    if (lane == 0) bulk_wait_group_all();
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, C::TMEM_COLS);
  }
}

// --------------------------------------------------------------- small backward kernels
// poff[g] = sum over routed groups g' < g of their row counts rounded up to 16 (g <= E).
// One warp: each lane scans a contiguous run of groups.
__global__ void __launch_bounds__(32) bw_pad_offsets_kernel(const int *__restrict__ offsets,
                                                            int E, int *poff) {
  griddep_wait();
  griddep_launch_dependents();
  const int lane = threadIdx.x;
  const int per = (E + 31) / 32;
  const int lo = min(E, lane * per), hi = min(E, lo + per);
  int run = 0;
  for (int g = lo; g < hi; ++g) run += (offsets[g + 1] - offsets[g] + 15) & ~15;
  int incl = run;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  int excl = incl - run;
  for (int g = lo; g < hi; ++g) {
    poff[g] = excl;
    excl += (offsets[g + 1] - offsets[g] + 15) & ~15;
  }
  if (lane == 31) poff[E] = incl;
}

// Padded expert-sorted rows [0, R): x and dout of the row's token into xs, dys; zero rows of
// xs, dys, da, db, hs at the padding; perm_pad[r] = the (token, slot) pair of routed row r
// (padding rows repeat their group's first pair).  Rows between the routed end and the
// shared group belong to no group and are not written.  One warp per row, 16-byte copies.
__global__ void __launch_bounds__(256) bw_sorted_rows_kernel(
    const __nv_bfloat16 *__restrict__ x, const __nv_bfloat16 *__restrict__ dout,
    const int *__restrict__ perm, int k, BwRows rows, int n_shared, int R, int d, int f,
    __nv_bfloat16 *xs, __nv_bfloat16 *dys, __nv_bfloat16 *da, __nv_bfloat16 *db,
    __nv_bfloat16 *hs, int *perm_pad) {
  griddep_wait();
  griddep_launch_dependents();
  const int lane = threadIdx.x & 31;
  const int nw = (gridDim.x * blockDim.x) >> 5;
  const int vec_d = d / 8, vec_f = f / 8;
  const uint4 z = make_uint4(0, 0, 0, 0);
  const int routed_end = rows.poff[rows.E];
  for (int r = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; r < R; r += nw) {
    int t = -1;  // token of the row; -1: padding
    if (r >= rows.s0) {
      if (n_shared == 0) continue;
      const int i = r - rows.s0;
      if (i < rows.T) t = i;
    } else {
      if (r >= routed_end) continue;  // between the groups: unused
      int lo = 0, hi = rows.E - 1;    // last g with poff[g] <= r
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (rows.poff[mid] <= r) lo = mid;
        else hi = mid - 1;
      }
      const int g = lo;
      const int base = rows.offsets[g], cnt = rows.offsets[g + 1] - base;
      const int i = r - rows.poff[g];
      const int q = perm[base + (i < cnt ? i : 0)];
      if (lane == 0) perm_pad[r] = q;
      if (i < cnt) t = q / k;
    }
    uint4 *xo = reinterpret_cast<uint4 *>(xs + (size_t)r * d);
    uint4 *yo = reinterpret_cast<uint4 *>(dys + (size_t)r * d);
    if (t >= 0) {
      const uint4 *xi = reinterpret_cast<const uint4 *>(x + (size_t)t * d);
      const uint4 *yi = reinterpret_cast<const uint4 *>(dout + (size_t)t * d);
      for (int i = lane; i < vec_d; i += 32) {
        xo[i] = __ldg(xi + i);
        yo[i] = __ldg(yi + i);
      }
    } else {
      for (int i = lane; i < vec_d; i += 32) {
        xo[i] = z;
        yo[i] = z;
      }
      for (int i = lane; i < vec_f; i += 32) {
        reinterpret_cast<uint4 *>(da + (size_t)r * f)[i] = z;
        reinterpret_cast<uint4 *>(db + (size_t)r * f)[i] = z;
        reinterpret_cast<uint4 *>(hs + (size_t)r * f)[i] = z;
      }
    }
  }
}

// dgate of routed slot perm[p] = routed_scale * (sum of the row's partials, in order).
__global__ void __launch_bounds__(256) bw_dgate_reduce_kernel(const float *__restrict__ part,
                                                              int n_part,
                                                              const int *__restrict__ perm,
                                                              int Tk, float routed_scale,
                                                              float *dgate) {
  griddep_wait();
  griddep_launch_dependents();
  for (int p = blockIdx.x * blockDim.x + threadIdx.x; p < Tk; p += gridDim.x * blockDim.x) {
    const float *r = part + (size_t)p * n_part;
    float s = 0.f;
    for (int i = 0; i < n_part; ++i) s += r[i];
    dgate[perm[p]] = routed_scale * s;
  }
}

}  // namespace moe
