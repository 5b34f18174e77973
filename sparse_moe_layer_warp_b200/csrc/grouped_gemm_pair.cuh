// grouped_gemm_pair.cuh -- the grouped expert GEMM of grouped_gemm.cuh on CTA pairs
// (tcgen05 cta_group::2) for large expert groups (prefill).
//
// Same work ("fused MoE gather/scatter with grouped GEMM", "Step 3.5 Flash: Open
// Frontier-Level Intelligence with 11B Active Parameters", section 3.2.4; SwiGLU experts,
// "Step 3.5 Flash 技术论文深度解读", training stability, root cause 3) and the same
// parameters and epilogues as grouped_gemm_kernel, with a bigger tile per unit:
// 256 weight rows x up to 256 tokens.  A cluster of two CTAs on one TPC runs it: CTA r stages
// weight rows [128r, 128r + 128) of the unit and token rows [n0 + r*half, n0 + r*half + 128)
// (half = the token tile split point), the leader (rank 0) issues
// tcgen05.mma.cta_group::2 with M = 256, N = 2*half, and each CTA's TMEM receives its 128 rows
// of D for all N token columns (column j = token n0 + j).  Per CTA and 64-wide K step the up
// kernel stages 48 KB for 2 x 128 x 256 x 64 MACs -- twice the tensor work per staged byte of
// the 1-CTA 128 x 128 tile, which is what limits that kernel at prefill sizes (it stays near
// 70 GB/s of TMA delivery per SM).
//
// Barriers: full[s] lives in the leader and counts both CTAs' TMA bytes (the peer's loads
// signal it through the .cta_group::2 load form); the leader's MMA commits arrive on empty[s]
// and tmem_full[a] of both CTAs; tmem_empty[a] (leader) collects one arrival per epilogue
// warp of both CTAs.  All waits are bounded as in grouped_gemm.cuh.
//
// Row gather inside the up kernel (GemmParams::gx_dst): two more warps per CTA write the
// expert-sorted copy of x, token by token (each x row read once, stored to its k rows), in
// chunks claimed from a counter, while the CTAs run the shared expert's units -- claimed
// first (shared_first), they read x itself and are tensor-bound with L2-resident operands, so
// the copy's HBM writes overlap them instead of taking a launch of their own before the GEMM.
// A routed unit's token loads wait (bounded) for the count of gathered tokens.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "grouped_gemm.cuh"
#include "ptx_sm100.cuh"

namespace moe {

constexpr int kPairBM = 256;  // weight rows per unit (both CTAs)
constexpr int kPairBN = 256;  // tokens per unit (both CTAs)
// warps: 0 producer, 1 MMA (leader) / TMEM owner, 2..9 epilogue -- two per TMEM lane
// quadrant (warp % 4), splitting a unit's 16-column chunks between them
constexpr int kPairEpiWarps = 8;
// up kernel: warps 10, 11 gather rows of x (idle when the copy is already written)
constexpr int kPairGatherWarps = 2;
constexpr int kGatherChunk = 4;  // tokens per claim of a gather warp

template <int MODE>
struct PairCfg {
  static constexpr int NA = (MODE == MODE_UP) ? 2 : 1;
  static constexpr int THREADS =
      32 * (2 + kPairEpiWarps + (MODE == MODE_UP ? kPairGatherWarps : 0));
  static constexpr int HALF_BN = kPairBN / 2;
  static constexpr int A_BYTES = 128 * kBK * 2;      // this CTA's 128 weight rows
  static constexpr int B_BYTES = HALF_BN * kBK * 2;  // this CTA's token rows
  static constexpr int STAGE_BYTES = NA * A_BYTES + B_BYTES;
  static constexpr int ACC_COLS = NA * kPairBN;
  static constexpr int ACC_BUFS = (2 * ACC_COLS <= 512) ? 2 : 1;
  static constexpr int TMEM_COLS = ACC_BUFS * ACC_COLS;
  static constexpr int STAGES_RAW = (192 * 1024) / STAGE_BYTES;
  static constexpr int STAGES = STAGES_RAW > 12 ? 12 : STAGES_RAW;
  static_assert(TMEM_COLS <= 512 && (TMEM_COLS & (TMEM_COLS - 1)) == 0, "TMEM allocation");
  // full[S], empty[S], tfull[A], tempty[A], drain, uq_full[Q], uq_empty[Q]
  static constexpr int BAR_BYTES = (2 * STAGES + 2 * ACC_BUFS + 1 + 2 * kUnitQ) * 8;
  static constexpr size_t smem_bytes(int n_groups) {
    return 1024 + (size_t)STAGES * STAGE_BYTES + BAR_BYTES + 64 +
           (size_t)(3 * n_groups + 1 + order_words(n_groups)) * 4 + ACC_BUFS * kPairBN * 4 +
           kPairEpiWarps * 16 * 32 * 4 /*epilogue transpose buffers*/ + 16 /*alignment*/;
  }
};

// One gather warp of the up kernel: claims kGatherChunk tokens at a time until every token is
// claimed; per token the warp reads the x row once (16-byte vectors, up to 16 per lane in
// flight) and stores it to the token's k rows of the sorted copy (L2 evict-first: the copy is
// far larger than L2 and is read back tile by tile later, while x and the running units'
// operands should stay), then publishes the chunk (stores, fence, count).
__device__ __forceinline__ void gather_token_rows(const GemmParams &p, int lane) {
  const int k = p.topk, vec = p.gx_vec, T = p.gx_T;
  const int n_rows = p.gx_n_rows ? *p.gx_n_rows : 0x7fffffff;
  const uint64_t pol = policy_evict_first();
  for (;;) {
    int c = 0;
    if (lane == 0) c = atomicAdd(p.gx_claim, 1);
    c = __shfl_sync(0xffffffffu, c, 0);
    const int t0 = c * kGatherChunk;
    if (t0 >= T) break;
    const int t1 = min(T, t0 + kGatherChunk);
    for (int t = t0; t < t1; ++t) {
      const int my_row = lane < k ? __ldg(p.gx_slot_row + (size_t)t * k + lane) : -1;
      const uint4 *__restrict__ src = p.gx_src + (size_t)t * vec;
      for (int v0 = 0; v0 < vec; v0 += 512) {
        uint4 r[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int v = v0 + 32 * i + lane;
          if (v < vec) r[i] = __ldg(src + v);
        }
        for (int j = 0; j < k; ++j) {
          const int row = __shfl_sync(0xffffffffu, my_row, j);
          if (row >= n_rows) continue;
          uint4 *__restrict__ dst = p.gx_dst + (size_t)row * vec;
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const int v = v0 + 32 * i + lane;
            if (v < vec) st_global_v4_hint(dst + v, r[i], pol);
          }
        }
      }
    }
    // publish: every lane's stores, then the count (as the h hand-over does)
    __threadfence();
    __syncwarp();
    if (lane == 0) {
      __threadfence();
      atomicAdd(p.gx_done, t1 - t0);
    }
  }
}

template <int MODE>
__global__ void __launch_bounds__(PairCfg<MODE>::THREADS, 1)
    grouped_gemm_pair_kernel(const __grid_constant__ GemmParams p) {
  using C = PairCfg<MODE>;
  constexpr int S = C::STAGES;
  constexpr int BN = kPairBN;
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
  uint64_t *tempty = bars + 2 * S + C::ACC_BUFS;
  uint64_t *drain = bars + 2 * S + 2 * C::ACC_BUFS;
  uint64_t *uq_full = drain + 1;
  uint64_t *uq_empty = uq_full + kUnitQ;  // used in the leader only
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
  float *xbuf = row_scale + C::ACC_BUFS * BN;  // [8 warps][16][32] epilogue transposes

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int cluster_id = blockIdx.x >> 1, n_clusters = gridDim.x >> 1;
  const int G = p.n_groups;
  const int mtiles = p.M / kPairBM;
  const int kblocks = p.K / kBK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < C::ACC_BUFS; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 2 * kPairEpiWarps);  // one per epilogue warp of both CTAs
    }
    mbar_init(drain, 1);
    mbar_init(epi_bar, kPairEpiWarps);
    for (int q = 0; q < kUnitQ; ++q) {
      mbar_init(&uq_full[q], 1);
      // readers of a published unit id: the leader's MMA thread and epilogue warps, the
      // peer's producer and epilogue warps
      mbar_init(&uq_empty[q], 2 + 2 * kPairEpiWarps);
    }
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&p.tmA0);
    if (MODE == MODE_UP) {
      tma_prefetch_desc(&p.tmA1);
      tma_prefetch_desc(&p.tmBs);
    }
    tma_prefetch_desc(&p.tmB);
  }
  if (warp == 1) tmem_alloc_pair(tmem_slot, C::TMEM_COLS);
  // programmatic dependent launch: everything below may read the previous kernel's output,
  // except in a down kernel with the per-group hand-over of h (see grouped_gemm_kernel)
  if (!(MODE == MODE_DOWN && p.done)) griddep_wait();
  griddep_launch_dependents();
  // group table and the cost-ordered work list (see build_unit_table)
  build_unit_table<BN>(p, mtiles, unit_prefix, grp_count, grp_row, order, n_first_s,
                       n_heavy_s);
  // both CTAs' barriers are initialised and TMEM allocated before any cross-CTA traffic
  tc_fence_before();
  __syncthreads();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int total_units = unit_prefix[G];
  const int n_heavy = *n_heavy_s;
  const int n_first = *n_first_s;

  auto decode = [&](int u, int &g, int &mt, int &nt) {
    decode_unit(u, G, unit_prefix, order, grp_count, BN, g, mt, nt);
  };
  // token split of a unit: CTA r holds tokens [n0 + r*half, n0 + (r+1)*half), N = 2*half
  auto split = [&](int g, int nt) {
    const int valid = min(BN, grp_count[g] - nt * BN);
    return (((valid + 1) >> 1) + 7) & ~7;
  };

  // unit claiming as in grouped_gemm_kernel, per CTA pair: the leader's producer claims
  auto claim = [&](int prev) -> int {
    if (p.sched) return atomicAdd(p.sched, 1);
    return prev < 0 ? cluster_id : prev + n_clusters;
  };

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ TMA producer
      const uint64_t pol_w = policy_evict_first();
      const uint64_t pol_b = policy_evict_last();
      uint64_t pol_w_shared;
      asm volatile("createpolicy.fractional.L2::evict_normal.b64 %0, 1.0;" : "=l"(pol_w_shared));
      int stage = 0;
      uint32_t phase = 0;
      int issued = 0;
      bool ok = true;
      int qi = 0;
      uint32_t qph = 0;
      int u = -1;
      int ticket = -1;       // leader: its claim cursor
      int ready_group = -1;  // down kernel: group whose h is known to be complete
      bool gathered = !(MODE == MODE_UP && p.gx_dst);  // up: the sorted copy is complete
      while (ok) {
        // the leader claims the next unit and publishes its id to both CTAs; the peer reads it
        if (leader) {
          ticket = claim(ticket);
          const int uid = (ticket < total_units)
                              ? unit_of_ticket(ticket, n_first, n_heavy, total_units)
                              : -1;
          if (!mbar_wait_bounded<true>(&uq_empty[qi], qph ^ 1, abort_flag, p.status, 15)) {
            ok = false;
            break;
          }
          uq[qi] = uid;
          st_shared_remote(mapa_shared(smem_u32((const void *)&uq[qi]), 1), uid);
          mbar_arrive(&uq_full[qi]);
          mbar_arrive_remote(mapa_shared(smem_u32(&uq_full[qi]), 1));
          u = uid;
        } else {
          if (!mbar_wait_bounded<true>(&uq_full[qi], qph, abort_flag, p.status, 16)) {
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
        const int a_row = weight_group(p, g) * p.M + mt * kPairBM + (int)rank * 128;
        const bool shared_x = (MODE == MODE_UP) && (g >= p.E);
        // token rows of this CTA: a box of 16, 32, 64 or 128 rows, the smallest that holds
        // the half tile (rows past it are never read by the MMA)
        const int box = (!p.b_boxes || half > 64) ? 3 : (half > 32 ? 2 : (half > 16 ? 1 : 0));
        const CUtensorMap *bmap = box == 3 ? (shared_x ? &p.tmBs : &p.tmB)
                                           : (shared_x ? &p.tmBsr[box] : &p.tmBr[box]);
        const uint32_t stage_tx = 2u * (C::NA * C::A_BYTES + (16u << box) * kBK * 2);
        const int b_row =
            (shared_x ? p.shared_t0 + nt * BN : grp_row[g] + nt * BN) + (int)rank * half;
        const uint64_t pw = (grp_count[g] <= BN) ? pol_w : pol_w_shared;
        if (MODE == MODE_DOWN && p.done && g != ready_group) {
          // both CTAs load h rows: each waits for every up unit of the group
          const int target =
              p.done_warps * p.done_mt * ((grp_count[g] + p.done_bn - 1) / p.done_bn);
          if (!counter_wait_bounded(p.done + g, target, abort_flag, p.status, 19)) {
            ok = false;
            break;
          }
          fence_proxy_async_global();  // the h rows are read through TMA below
          ready_group = g;
        }
        if (MODE == MODE_UP && !gathered && !shared_x) {
          // both CTAs load rows of the sorted copy: each waits for every token's rows
          if (!counter_wait_bounded(p.gx_done, p.gx_T, abort_flag, p.status, 20)) {
            ok = false;
            break;
          }
          fence_proxy_async_global();  // written by the gather warps' stores, read by TMA
          gathered = true;
        }
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!mbar_wait_bounded(&empty[stage], phase ^ 1, abort_flag, p.status, 11)) {
            ok = false;
            break;
          }
          const uint32_t fbar = mapa_shared(smem_u32(&full[stage]), 0);
          if (leader) mbar_arrive_expect_tx(&full[stage], stage_tx);
          tma_load_2d_pair(sA0 + stage * C::A_BYTES, &p.tmA0, fbar, kb * kBK, a_row, pw);
          if (MODE == MODE_UP)
            tma_load_2d_pair(sA1 + stage * C::A_BYTES, &p.tmA1, fbar, kb * kBK, a_row, pw);
          tma_load_2d_pair(sB + stage * C::B_BYTES, bmap, fbar, kb * kBK, b_row, pol_b);
          ++issued;
          if (++stage == S) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (u < 0) break;
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
      while (ok) {
        if (!mbar_wait_bounded<true>(&uq_full[qi], qph, abort_flag, p.status, 17)) break;
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
        if (!mbar_wait_bounded(&tempty[acc], acc_phase ^ 1, abort_flag, p.status, 12)) break;
        tc_fence_after();
        int g, mt, nt;
        decode(u, g, mt, nt);
        const uint32_t idesc = idesc_bf16_f32(kPairBM, 2 * split(g, nt));
        const uint32_t d0 = tmem_base + acc * C::ACC_COLS;
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!mbar_wait_bounded(&full[stage], phase, abort_flag, p.status, 13)) {
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
            tc_mma_bf16_pair(d0, sdesc_k_sw128(a0 + kk * 32), bd, idesc, accum);
            if (MODE == MODE_UP)
              tc_mma_bf16_pair(d0 + BN, sdesc_k_sw128(a1 + kk * 32), bd, idesc, accum);
          }
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
  } else if (warp >= 2 + kPairEpiWarps) {
    // ---------------------------------------------------------------- row gather (up)
    if (MODE == MODE_UP && p.gx_dst) gather_token_rows(p, lane);
  } else {
    // ---------------------------------------------------------------- epilogue (both CTAs)
    const int q = warp & 3;         // TMEM lane quadrant
    const int eh = (warp - 2) >> 2;  // which of the quadrant's two warps: chunks 2i + eh
    const uint32_t tempty_leader = mapa_shared(smem_u32(&tempty[0]), 0);
    const uint32_t uq_empty_leader = mapa_shared(smem_u32(&uq_empty[0]), 0);
    // lane 0 polls, the warp follows (uniform path into the warp-wide tcgen05.ld)
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
    int it = 0;
    int qi = 0;
    uint32_t qph = 0;
    while (true) {
      if (!warp_wait(&uq_full[qi], qph, 18, true)) break;
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
      const int acc = it % C::ACC_BUFS;
      const uint32_t acc_phase = (it / C::ACC_BUFS) & 1;
      ++it;
      if (!warp_wait(&tfull[acc], acc_phase, 14, false)) break;
      tc_fence_after();
      int g, mt, nt;
      decode(u, g, mt, nt);
      const int valid = min(BN, grp_count[g] - nt * BN);
      const int row0 = grp_row[g] + nt * BN;
      const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + acc * C::ACC_COLS;
      if (MODE == MODE_DOWN) {
        for (int n = threadIdx.x - 64; n < BN; n += 32 * kPairEpiWarps) {
          float sc = 0.f;
          if (n < valid) sc = (g < p.E) ? p.routed_scale * p.topk_gate[p.perm[row0 + n]] : 1.f;
          row_scale[acc * BN + n] = sc;
        }
        // all epilogue warps' scales are staged before any reads them: a bounded mbarrier (one
        // arrival per warp) instead of bar.sync, so a warp that aborts leaves none waiting
        __syncwarp();
        if (lane == 0) mbar_arrive(epi_bar);
        if (!warp_wait(epi_bar, (uint32_t)(it - 1) & 1, 72, false)) break;
      }
      float *wbuf = xbuf + (warp - 2) * 16 * 32;
      const int col_base = mt * kPairBM + (int)rank * 128 + q * 32;
      // TMEM loads run one 16-column chunk ahead of their use
      uint32_t n0[16], n1[16];
      const int c_first = 16 * eh;
      if (c_first < valid) {
        tmem_ld16(taddr + c_first, n0);
        if (MODE == MODE_UP) tmem_ld16(taddr + BN + c_first, n1);
      }
      for (int c0 = c_first; c0 < valid; c0 += 32) {
        uint32_t v0[16], v1[16];
        if (MODE == MODE_UP) tmem_ld_wait_regs(n0, n1);
        else tmem_ld_wait_regs(n0);
#pragma unroll
        for (int n = 0; n < 16; ++n) {
          v0[n] = n0[n];
          v1[n] = n1[n];
        }
        if (c0 + 32 < valid) {
          tmem_ld16(taddr + c0 + 32, n0);
          if (MODE == MODE_UP) tmem_ld16(taddr + BN + c0 + 32, n1);
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
        } else {
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
        }
      }
      // every TMEM load of this unit has completed (tcgen05.wait::ld before each use): the
      // accumulator goes back to the leader's MMA thread before this warp's global stores
      // drain, so the h hand-over's fences below stay off the MMA's critical path (the up
      // kernel has a single accumulator: its next unit's MMAs wait for this arrival)
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (leader) mbar_arrive(&tempty[acc]);
        else mbar_arrive_remote(tempty_leader + acc * 8);
      }
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

  // the pair leaves together: the leader's MMAs read the peer's shared memory, and the
  // peer's TMA loads signal the leader's barriers
  tc_fence_before();
  __syncthreads();
  cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, C::TMEM_COLS);
  }
  if (p.clock_sum && threadIdx.x == 0) clock_span_add(*span, p.clock_sum);
}

}  // namespace moe
