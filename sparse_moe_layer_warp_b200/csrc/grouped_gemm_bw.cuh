// grouped_gemm_bw.cuh -- tcgen05 grouped GEMMs of the bf16 layer's backward.
//
// The chain rule through the SwiGLU experts ("Step 3.5 Flash: Open Frontier-Level
// Intelligence with 11B Active Parameters", sections 2.2 and 4.1.2; "Step 3.5 Flash
// 技术论文深度解读", training stability, root cause 3) as grouped GEMMs over the
// expert-sorted rows ("fused MoE gather/scatter with grouped GEMM", first page, section
// 3.2.4).  Per sorted row p of group g (token t, scale s_p = routed_scale * gate, 1 for the
// shared expert), with a = W_g[g] x_t and b = W_u[g] x_t recomputed by the forward's up GEMM:
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
// Ragged groups.  The dgrad GEMMs tile a group's rows on N as the forward does (columns
// past the group's rows are computed from neighbouring rows and never stored).  The weight
// gradients take a group's rows as K in blocks of 64: full blocks are box loads; the last,
// partial block is gathered four rows at a time (tile::gather4) with the rows past the
// group pointing at an all-zero row kept after the sorted rows, so no row of a neighbouring
// group enters the sum.  Each dW tile is owned by one unit, which adds its finished
// accumulator into the caller's fp32 gradient with TMA reductions (cp.reduce.async.bulk
// .tensor add): one addition per element and call, so the result is deterministic.
//
// Roles, pipelines and bounded waits are those of grouped_gemm.cuh: warp 0 produces (lane 0
// claims units), warp 1 lane 0 issues the MMAs, warps 2..5 run the epilogue, STAGES
// shared-memory slots and two TMEM accumulators; every wait gives up after the time limit,
// drains its in-flight copies and MMAs, frees TMEM and reports through the status word.
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

// --------------------------------------------------------------------- dgrad GEMMs
enum BwDgradMode { BW_DH = 0, BW_DX = 1 };

struct BwDgradParams {
  CUtensorMap tmA0;  // DH: W_down as [G*d, f]; DX: W_gate as [G*f, d]      box {64, 64}
  CUtensorMap tmA1;  // DX: W_up as [G*f, d]                                box {64, 64}
  CUtensorMap tmB0;  // DH: dout rows [P+1, d]; DX: da [P+1, f] (sorted)    box {64, BN}
  CUtensorMap tmB1;  // DX: db [P+1, f]                                     box {64, BN}
  const int *offsets;          // [E + 1]
  const float *row_scale;      // [P] s_p (DH)
  const float *pre_a, *pre_b;  // [P, f] fp32 pre-activations (DH)
  __nv_bfloat16 *da, *db, *hs; // [P + 1, f] (DH)
  float *dgate_part;           // [P, n_part] (DH): partial sums of dhu . h
  float *out;                  // DX: dX rows [P, d] fp32
  DevStatus *status;
  int E, n_groups, T, Tk;
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
    return 1024 + (size_t)STAGES * STAGE_BYTES + BAR_BYTES + 64 + (size_t)(3 * n_groups + 1) * 4 +
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
  volatile int *uq = reinterpret_cast<volatile int *>(tmem_slot + 4);  // [kUnitQ]
  int *unit_prefix = reinterpret_cast<int *>(tmem_slot + 16);        // [G + 1]
  int *grp_count = unit_prefix + p.n_groups + 1;                     // [G]
  int *grp_row = grp_count + p.n_groups;                             // [G]
  float *row_scale = reinterpret_cast<float *>(
      (reinterpret_cast<uintptr_t>(grp_row + p.n_groups) + 15) & ~static_cast<uintptr_t>(15));
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
      const int row0 = grp_row[g] + nt * BN;
      const int col_base = mt * kBM + q * 32;  // first output column (M index) of this warp
      const int col = col_base + lane;
      const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + acc * C::ACC_COLS;
      if (MODE == BW_DH) {
        for (int n = threadIdx.x - 64; n < BN; n += 128)
          row_scale[acc * BN + n] = (n < valid) ? p.row_scale[row0 + n] : 0.f;
        named_bar_sync(1, 128);
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
          store_block16_f32(p.out, p.M, row0, c0, valid, col_base, vals, wbuf, lane);
        } else {
          // pre-activations of the chunk's rows (coalesced: lanes read consecutive columns)
          float av[16], bv[16];
#pragma unroll
          for (int n = 0; n < 16; ++n) {
            const bool in = c0 + n < valid;
            const size_t i = (size_t)(row0 + c0 + n) * p.M + col;
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
          if (lane < 16 && c0 + lane < valid && g < p.E) {
            float sum = 0.f;
#pragma unroll 8
            for (int i = 0; i < 32; ++i) sum += red[lane * 33 + i];
            p.dgate_part[(size_t)(row0 + c0 + lane) * p.n_part + mt * 4 + q] = sum;
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

// ---------------------------------------------------------------------- wgrad GEMM
constexpr int kWgOps = 5;    // sorted operands: dout, hs, da, db, x
constexpr int kWgProbs = 3;  // dW_down, dW_gate, dW_up

struct BwWgradParams {
  CUtensorMap box[kWgOps];   // sorted rows [P + 1, width] bf16, box {64, 64}
  CUtensorMap gat[kWgOps];   // the same rows, box {64, 1} (tile::gather4)
  CUtensorMap out[kWgProbs]; // dW as [G * M, N] fp32, box {32, 32}, 128-byte swizzle
  int a_op[kWgProbs], b_op[kWgProbs];  // operand of the M side and of the N side
  int M[kWgProbs], N[kWgProbs];        // dW[g] is [M, N]; M % 128 == 0, N % BNW == 0
  int n_prob;
  const int *offsets;
  DevStatus *status;
  int E, n_groups, T, Tk;
  int zero_row;  // P: the all-zero row after the sorted rows
  int *sched;
};

template <int BNW>
struct BwWgradCfg {
  static constexpr int NB = BNW / 64;             // 64-element boxes on the N side
  static constexpr int A_BYTES = kBM * kBK * 2;   // 2 boxes of 64 M x 64 rows
  static constexpr int B_BYTES = BNW * kBK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int BOX_BYTES = 64 * kBK * 2;  // 8 KB
  static constexpr int ACC_COLS = BNW;
  static constexpr int TMEM_COLS = 2 * BNW;
  static constexpr int STG_BYTES = 32 * 32 * 4;   // one 32 x 32 fp32 reduction tile
#ifndef MOE_WG_STG_BUFS
#define MOE_WG_STG_BUFS 2
#endif
#ifndef MOE_WG_MAX_STAGES
#define MOE_WG_MAX_STAGES 8
#endif
  static constexpr int STG_BUFS = MOE_WG_STG_BUFS;  // staging tiles per epilogue warp
  static constexpr int STG_TOTAL = 4 * STG_BUFS * STG_BYTES;
  static constexpr int SMEM_BUDGET = 220 * 1024 - STG_TOTAL;
  static constexpr int STAGES_RAW = SMEM_BUDGET / STAGE_BYTES;
  static constexpr int STAGES = STAGES_RAW > MOE_WG_MAX_STAGES ? MOE_WG_MAX_STAGES : STAGES_RAW;
  static_assert(STAGES >= 2, "pipeline too shallow");
  static_assert(BNW == 128 || BNW == 256, "N tile");
  static constexpr int BAR_BYTES = (2 * STAGES + 5 + 2 * kUnitQ) * 8;
  static constexpr size_t smem_bytes(int n_groups) {
    return 1024 + (size_t)STAGES * STAGE_BYTES + STG_TOTAL + BAR_BYTES + 64 +
           (size_t)(kWgProbs * n_groups + 1) * 4 + (size_t)n_groups * 2 * 4 + 16;
  }
};

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
  const int NP = p.n_prob;
  int *unit_prefix = reinterpret_cast<int *>(tmem_slot + 16);  // [NP * G + 1]
  int *grp_count = unit_prefix + NP * G + 1;                    // [G]
  int *grp_row = grp_count + G;                                 // [G]

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
    for (int pr = 0; pr < NP; ++pr)
      unit_prefix[pr * G + g] = cnt > 0 ? (p.M[pr] / kBM) * (p.N[pr] / BNW) : 0;
  }
  __syncthreads();
  if (warp == 0) {  // exclusive scan over (problem, group)
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
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int total_units = unit_prefix[NP * G];

  // unit -> (problem, group, m tile, n tile), n tile innermost
  auto decode = [&](int u, int &pr, int &g, int &mt, int &nt) {
    int lo = 0, hi = NP * G - 1;
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
  };

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    // Lane 0 claims units and loads full 64-row blocks as boxes; the last partial block of
    // a group is gathered by the whole warp, rows past the group read from the zero row.
    int stage = 0;
    uint32_t phase = 0;
    int issued = 0;
    bool ok = true;
    int qi = 0;
    uint32_t qph = 0;
    for (;;) {
      int uid = -1;
      if (lane == 0) {
        const int u = atomicAdd(p.sched, 1);
        uid = (u < total_units) ? u : -1;
        if (mbar_wait_bounded(&uq_empty[qi], qph ^ 1, abort_flag, p.status, 31)) {
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
      int pr, g, mt, nt;
      decode(uid, pr, g, mt, nt);
      const CUtensorMap *abox = &p.box[p.a_op[pr]], *bbox = &p.box[p.b_op[pr]];
      const CUtensorMap *agat = &p.gat[p.a_op[pr]], *bgat = &p.gat[p.b_op[pr]];
      const int m0 = mt * kBM, n0 = nt * BNW;
      const int cnt = grp_count[g], start = grp_row[g];
      const int kbs = (cnt + kBK - 1) / kBK;
      for (int kb = 0; kb < kbs; ++kb) {
        const int r0 = start + kb * kBK;
        const int rows_in = min(kBK, cnt - kb * kBK);
        const int n_rows = (rows_in + 15) & ~15;
        if (lane == 0) {
          ok = mbar_wait_bounded(&empty[stage], phase ^ 1, abort_flag, p.status, 32);
          if (ok) {
            mbar_arrive_expect_tx(&full[stage], (uint32_t)(2 + C::NB) * n_rows * 128);
            if (rows_in == kBK) {
              uint8_t *a_dst = sA + stage * C::A_BYTES;
              uint8_t *b_dst = sB + stage * C::B_BYTES;
              tma_load_2d(a_dst, abox, &full[stage], m0, r0);
              tma_load_2d(a_dst + C::BOX_BYTES, abox, &full[stage], m0 + 64, r0);
#pragma unroll
              for (int h = 0; h < C::NB; ++h)
                tma_load_2d(b_dst + h * C::BOX_BYTES, bbox, &full[stage], n0 + 64 * h, r0);
            }
          }
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
        if (rows_in < kBK) {
          // (2 + NB) boxes x n_rows / 4 gathers, spread over the lanes
          const int quads = n_rows / 4;
          const int total = (2 + C::NB) * quads;
          const uint64_t pol = policy_evict_last();
          for (int i = lane; i < total; i += 32) {
            const int bx = i / quads, qd = i - bx * quads;
            int rr[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int r = 4 * qd + e;
              rr[e] = (r < rows_in) ? r0 + r : p.zero_row;
            }
            uint8_t *dst;
            const CUtensorMap *map;
            int x;
            if (bx < 2) {
              dst = sA + stage * C::A_BYTES + bx * C::BOX_BYTES;
              map = agat;
              x = m0 + 64 * bx;
            } else {
              dst = sB + stage * C::B_BYTES + (bx - 2) * C::BOX_BYTES;
              map = bgat;
              x = n0 + 64 * (bx - 2);
            }
            tma_gather4(dst + qd * 4 * 128, map, &full[stage], x, rr[0], rr[1], rr[2], rr[3],
                        pol);
          }
        }
        ++issued;
        if (++stage == S) {
          stage = 0;
          phase ^= 1;
        }
      }
      if (!ok) break;
    }
    if (!ok && lane == 0) {
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
        const int acc = it & 1;
        const uint32_t acc_phase = (it >> 1) & 1;
        ++it;
        if (!mbar_wait_bounded(&tempty[acc], acc_phase ^ 1, abort_flag, p.status, 34)) break;
        tc_fence_after();
        int pr, g, mt, nt;
        decode(u, pr, g, mt, nt);
        const int cnt = grp_count[g];
        const int kbs = (cnt + kBK - 1) / kBK;
        const uint32_t d0 = tmem_base + acc * C::ACC_COLS;
        for (int kb = 0; kb < kbs; ++kb) {
          if (!mbar_wait_bounded(&full[stage], phase, abort_flag, p.status, 35)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const int rows_in = min(kBK, cnt - kb * kBK);
          const int k16 = (rows_in + 15) >> 4;
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
    // Warp q owns accumulator rows 32q..32q+31 (its TMEM lane quadrant).  Each 32-column
    // chunk goes registers -> swizzled staging tile -> TMA reduction into dW; two staging
    // tiles per warp, so the next chunk is written while the previous reduction reads.
    const int q = warp & 3;
    auto warp_wait = [&](uint64_t *bar, uint32_t parity, int where) -> bool {
      int ok = 1;
      if (lane == 0) ok = mbar_wait_bounded(bar, parity, abort_flag, p.status, where) ? 1 : 0;
      ok = __shfl_sync(0xffffffffu, ok, 0);
      __syncwarp();
      return ok != 0;
    };
    uint8_t *my_stg = stg + q * C::STG_BUFS * C::STG_BYTES;
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
      const int acc = it & 1;
      const uint32_t acc_phase = (it >> 1) & 1;
      ++it;
      if (!warp_wait(&tfull[acc], acc_phase, 37)) break;
      tc_fence_after();
      int pr, g, mt, nt;
      decode(u, pr, g, mt, nt);
      const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + acc * C::ACC_COLS;
      const int out_row = g * p.M[pr] + mt * kBM + q * 32;
      const CUtensorMap *omap = &p.out[pr];
      for (int c = 0; c < BNW / 32; ++c) {
        uint32_t v0[16], v1[16];
        tmem_ld16(taddr + 32 * c, v0);
        tmem_ld16(taddr + 32 * c + 16, v1);
        tmem_ld_wait_regs(v0, v1);
        uint8_t *buf = my_stg + (n_red % C::STG_BUFS) * C::STG_BYTES;
        if (n_red >= C::STG_BUFS) {  // the reduction that last read this tile is done reading
          if (lane == 0) bulk_wait_group_read<C::STG_BUFS - 1>();
          __syncwarp();
        }
        // row `lane`, 16-byte chunk j of the row at position j ^ (lane & 7) (128-byte swizzle)
        uint8_t *row = buf + lane * 128;
#pragma unroll
        for (int j = 0; j < 4; ++j)
          *reinterpret_cast<float4 *>(row + ((j ^ (lane & 7)) << 4)) =
              make_float4(__uint_as_float(v0[4 * j]), __uint_as_float(v0[4 * j + 1]),
                          __uint_as_float(v0[4 * j + 2]), __uint_as_float(v0[4 * j + 3]));
#pragma unroll
        for (int j = 0; j < 4; ++j)
          *reinterpret_cast<float4 *>(row + (((j + 4) ^ (lane & 7)) << 4)) =
              make_float4(__uint_as_float(v1[4 * j]), __uint_as_float(v1[4 * j + 1]),
                          __uint_as_float(v1[4 * j + 2]), __uint_as_float(v1[4 * j + 3]));
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_reduce_add_2d(omap, buf, nt * BNW + 32 * c, out_row);
          bulk_commit_group();
        }
        ++n_red;
      }
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

// --------------------------------------------------------------- small backward kernels
// Sorted rows of x and dout (row p of group g: token row_token[p]) with the all-zero row P
// after them; the zero row of da, db and hs as well.  One warp per row, 16-byte copies.
__global__ void __launch_bounds__(256) bw_sorted_rows_kernel(
    const __nv_bfloat16 *__restrict__ x, const __nv_bfloat16 *__restrict__ dout,
    const int *__restrict__ row_token, int P, int d, int f, __nv_bfloat16 *xs,
    __nv_bfloat16 *dys, __nv_bfloat16 *da, __nv_bfloat16 *db, __nv_bfloat16 *hs) {
  griddep_wait();
  griddep_launch_dependents();
  const int lane = threadIdx.x & 31;
  const int nw = (gridDim.x * blockDim.x) >> 5;
  const int vec_d = d / 8, vec_f = f / 8;
  for (int p = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; p <= P; p += nw) {
    uint4 *xo = reinterpret_cast<uint4 *>(xs + (size_t)p * d);
    uint4 *yo = reinterpret_cast<uint4 *>(dys + (size_t)p * d);
    if (p < P) {
      const int t = row_token[p];
      const uint4 *xi = reinterpret_cast<const uint4 *>(x + (size_t)t * d);
      const uint4 *yi = reinterpret_cast<const uint4 *>(dout + (size_t)t * d);
      for (int i = lane; i < vec_d; i += 32) {
        xo[i] = __ldg(xi + i);
        yo[i] = __ldg(yi + i);
      }
    } else {
      const uint4 z = make_uint4(0, 0, 0, 0);
      for (int i = lane; i < vec_d; i += 32) {
        xo[i] = z;
        yo[i] = z;
      }
      for (int i = lane; i < vec_f; i += 32) {
        reinterpret_cast<uint4 *>(da + (size_t)P * f)[i] = z;
        reinterpret_cast<uint4 *>(db + (size_t)P * f)[i] = z;
        reinterpret_cast<uint4 *>(hs + (size_t)P * f)[i] = z;
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
