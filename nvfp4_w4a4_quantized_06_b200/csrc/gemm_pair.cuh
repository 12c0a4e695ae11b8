// gemm_pair.cuh -- block-scaled NVFP4 GEMM on CTA pairs (tcgen05 cta_group::2).
//
// Same product as gemm.cuh (D[i, j] = sum_k dec(A)[i, k] * dec(B)[j, k], FP32
// accumulation; web pages on arXiv 2609.04098, ta-paperlens page, "前提1"),
// computed by a cluster of two CTAs on two SMs per 256 x 256 output tile:
//   * each CTA stages its own 128 rows of A and its own 128 rows of the tile's
//     256 B rows, plus the scale atoms of its A rows and of all 256 B rows;
//   * the leader CTA (rank 0) issues one tcgen05.mma.cta_group::2 per 64-deep
//     K block: M = 256 (128 rows from each CTA's shared memory), N = 256 (128
//     B rows from each), the accumulator lands in each CTA's own TMEM;
//   * A/B loads of both CTAs complete on the leader's stage barrier (TMA with
//     .cta_group::2, no multicast); the leader's commits arrive on the stage
//     and accumulator barriers of both CTAs.
// Scale factors reach TMEM through tcgen05.st, not tcgen05.cp: the NVFP4
// scales of a 128 x 256 x 256 slice are 24 KB of replicated TMEM columns per
// SM per stage, which the smem->TMEM copy path moves at ~40 B/clk (slower
// than the MMAs that consume them; the whole GEMM measured 3.86 ms against
// 2.43 ms when the MMA thread issued tcgen05.cp.cta_group::2 per K block),
// while eight "scale warps" (per TMEM lane quarter one for the A scales and
// one for the B scales) store them from registers at several hundred B/clk
// and leave the single MMA-issuing thread nothing but MMAs.  Issuing the
// copies one stage ahead of the MMAs does not help either (4.03 ms): the
// copies and the MMAs share the tensor pipe.  What the scale path still
// costs (about 0.37 ms of the 2.45 ms prefill product) is mostly the shared
// memory reads of the replicated B scales: every lane quarter must hold all
// 256 B-row scales, so four warps each read the same 4 KB per stage; letting
// three of them skip the reads (wrong results, timing only) gives 2.24 ms.
// Each quarter's MMA reads only its own word of the A atom (rows 32q + l),
// but the atom's layout puts those words 16 bytes apart, so reading only
// them takes the same number of shared-memory wavefronts.
//
// BF16 output leaves through TMA stores: each epilogue warp drains its
// accumulator columns, hands TMEM back, converts to BF16 in a 32 x 32 staging
// box in shared memory and one lane stores the box (2.47 ms against 2.97 ms
// with per-lane 16-byte register stores, whose 32 rows per instruction
// crowd the SM's path to L2 that the operand loads share).
//
// Warp roles per CTA: 0 producer (one lane), 1 TMEM allocation + MMA issue
// (one lane of the leader), 2-5 A-scale warps and 6-9 B-scale warps (lane
// quarters 2, 3, 0, 1), 10-25 epilogue (four warps per lane quarter, 64
// columns each).  26 warps fit one SM at <= 72 registers per thread.
#pragma once
#include <cuda_bf16.h>
#include <cstdint>

#include "gemm.cuh"
#include "ptx.cuh"

#ifndef NVFP4_Y_EVICT_FIRST
#define NVFP4_Y_EVICT_FIRST false
#endif

namespace nvfp4 {

struct PairCfg {
  static constexpr int BM = 128;                 // rows of A per CTA (256 per pair)
  static constexpr int BN = 256;                 // columns of the pair's tile
  static constexpr int BN_CTA = 128;             // B rows staged per CTA
  static constexpr int A_BYTES = BM * 128;
  static constexpr int B_BYTES = BN_CTA * 128;
  static constexpr int SFA_BYTES = 4 * 512;
  static constexpr int SFB_BYTES = 2 * 4 * 512;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES;
  static constexpr int STAGES = 5;
  static constexpr int SF_WARPS = 8;
  static constexpr int EPI_WARPS = 16;
  static constexpr int EPI_COLS = 64;            // four warps per lane quarter, 64 columns each
  static constexpr int FIRST_EPI_WARP = 2 + SF_WARPS;
  static constexpr int THREADS = 64 + 32 * (SF_WARPS + EPI_WARPS);
  static constexpr int SF_COLS = 16 + 32;        // per-stage scale region: A (4 x 4), B (4 x 8)
  static constexpr int SFA_COL = BN;
  static constexpr int SFB_COL = BN + 16;
  static constexpr int TMEM_COLS = 512;
  // BF16 output staging: one 32-row x 32-column box (64-byte rows, 64-byte
  // swizzle) per epilogue warp, stored to Y by TMA
  static constexpr int STG_WARP_BYTES = 32 * 64;
  static constexpr int STG_BYTES = EPI_WARPS * STG_WARP_BYTES;
  static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + STG_BYTES + 256;
  static constexpr uint32_t IDESC = (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) |
                                    ((uint32_t)(256 >> 4) << 24);
  static_assert(BN + STAGES * SF_COLS <= TMEM_COLS, "TMEM budget");
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

template <int MODE>
__global__ void __launch_bounds__(PairCfg::THREADS, 1)
    nvfp4_gemm_pair_kernel(const __grid_constant__ CUtensorMap tma, const __grid_constant__ CUtensorMap tmb,
                           const __grid_constant__ CUtensorMap tmsfa, const __grid_constant__ CUtensorMap tmsfb,
                           const __grid_constant__ CUtensorMap tmy, const GemmParams p) {
  using C = PairCfg;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sA = smem;
  uint8_t *sB = sA + C::STAGES * C::A_BYTES;
  uint8_t *sSFA = sB + C::STAGES * C::B_BYTES;
  uint8_t *sSFB = sSFA + C::STAGES * C::SFA_BYTES;
  uint8_t *sStg = sSFB + C::STAGES * C::SFB_BYTES;
  uint64_t *bars = reinterpret_cast<uint64_t *>(sStg + C::STG_BYTES);
  uint64_t *full = bars;                        // leader: A/B of both CTAs + own scales
  uint64_t *sffull = bars + C::STAGES;          // peer: own scales
  uint64_t *sfready = bars + 2 * C::STAGES;     // leader: scales in both TMEMs (8 warps)
  uint64_t *empty = bars + 3 * C::STAGES;       // both: the stage's MMAs have completed
  uint64_t *tfull = bars + 4 * C::STAGES;       // both: accumulator ready
  uint64_t *tempty = tfull + 1;                 // leader: both epilogues drained TMEM
  uint64_t *tdone = tfull + 2;                  // both: all tensor work of the pair done
  uint64_t *pairdone = tfull + 3;               // both: the other CTA has finished
  uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(tfull + 4);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int cluster = blockIdx.x >> 1, nclusters = gridDim.x >> 1;
  const int total_units = p.tiles_a * p.tiles_b;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&sffull[s], 1);
      mbar_init(&sfready[s], 2 * C::SF_WARPS);
      mbar_init(&empty[s], 1);
    }
    mbar_init(tfull, 1);
    mbar_init(tempty, 2 * C::EPI_WARPS);
    mbar_init(tdone, 1);
    mbar_init(pairdone, 1);
    *abort_flag = 0;
    fence_barrier_init();
    prefetch_tmap(&tma);
    prefetch_tmap(&tmb);
    prefetch_tmap(&tmsfa);
    prefetch_tmap(&tmsfb);
    if (p.tma_store) prefetch_tmap(&tmy);
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_holder, C::TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();                 // both CTAs' barriers and TMEM exist before any pair traffic
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ producer
      int st = 0;
      uint32_t ph = 0;
      uint32_t issued = 0;
      bool ok = true;
      for (int u = cluster; u < total_units && ok; u += nclusters) {
        int ta, tb, split;
        unit_coords(p, u, ta, tb, split);
        const int row_a = ta * 256 + (int)rank * C::BM;        // this CTA's A rows
        const int row_b = tb * C::BN + (int)rank * C::BN_CTA;  // this CTA's B rows
        for (int ks = 0; ks < p.kstages; ++ks) {
          if (!mbar_wait(&empty[st], ph ^ 1, p.err, ERR_PRODUCER, abort_flag)) { ok = false; break; }
          const uint32_t fbar = mapa_shared(smem_u32(&full[st]), 0);
          // scales land on a barrier of this CTA (its scale warps wait there)
          const uint32_t sbar = leader ? fbar : mapa_shared(smem_u32(&sffull[st]), rank);
          if (leader) {
            mbar_arrive_expect_tx(&full[st], 2u * (C::A_BYTES + C::B_BYTES) + C::SFA_BYTES + C::SFB_BYTES);
          } else {
            mbar_arrive_expect_tx(&sffull[st], C::SFA_BYTES + C::SFB_BYTES);
          }
          tma_load_2d_pair(sA + st * C::A_BYTES, &tma, fbar, ks * 128, row_a);
          tma_load_2d_pair(sB + st * C::B_BYTES, &tmb, fbar, ks * 128, row_b);
          tma_load_2d_pair(sSFA + st * C::SFA_BYTES, &tmsfa, sbar, ks * 256, row_a >> 7);
          tma_load_2d_pair(sSFB + st * C::SFB_BYTES, &tmsfb, sbar, ks * 256, (tb * C::BN) >> 7);
          ++issued;
          if (++st == C::STAGES) { st = 0; ph ^= 1; }
        }
      }
      // teardown: each issued stage is released by the leader's MMAs (which
      // read this CTA's data) before the CTA may exit
      for (int s = 0; s < C::STAGES; ++s) {
        const uint32_t armed = issued / C::STAGES + ((uint32_t)s < issued % C::STAGES ? 1u : 0u);
        if (armed) {
          volatile int never = 0;
          mbar_wait(&empty[s], (armed - 1) & 1, p.err, ERR_PRODUCER, &never);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      // ------------------------------------------------------------- MMA issue
      // Only MMAs, one commit and one barrier per stage.  The next stage's
      // barrier is probed without suspending before this stage is issued.
      const uint64_t a_desc0 = smem_desc(smem_u32(sA), 16, 1024, 2);
      const uint64_t b_desc0 = smem_desc(smem_u32(sB), 16, 1024, 2);
      int st = 0;
      uint32_t ph = 0;
      uint64_t ad = a_desc0, bd = b_desc0;
      uint32_t reg = tmem;
      int it = 0;
      bool ready = false;
      for (int u = cluster; u < total_units; u += nclusters, ++it) {
        if (!mbar_wait(tempty, (it & 1) ^ 1, p.err, ERR_MMA, abort_flag)) break;
        tc_fence_after();
        bool ok = true;
        for (int ks = 0; ks < p.kstages; ++ks) {
          if (!ready && !mbar_wait(&sfready[st], ph, p.err, ERR_MMA, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const int st1 = st + 1 == C::STAGES ? 0 : st + 1;
          const uint32_t ph1 = st + 1 == C::STAGES ? ph ^ 1u : ph;
          const bool ready1 = mbar_test_wait(smem_u32(&sfready[st1]), ph1);
          const uint32_t acc0 = ks > 0 ? 1u : 0u;
          const int nkb = min(4, p.kblocks - ks * 4);
#pragma unroll
          for (int kb = 0; kb < 4; ++kb)
            if (kb < nkb)
              tc_mma_pair_nvfp4(tmem, ad + (uint64_t)(kb * 2), bd + (uint64_t)(kb * 2), C::IDESC,
                                kb > 0 ? 1u : acc0, reg + C::SFA_COL + 4 * kb, reg + C::SFB_COL + 8 * kb);
          tc_commit_pair(&empty[st], 0x3);
          ready = ready1;
          if (st1 == 0) {
            ad = a_desc0; bd = b_desc0; reg = tmem;
          } else {
            ad += (uint64_t)(C::A_BYTES >> 4); bd += (uint64_t)(C::B_BYTES >> 4); reg += C::SF_COLS;
          }
          st = st1;
          ph = ph1;
        }
        if (!ok) break;
        tc_commit_pair(tfull, 0x3);
      }
      tc_commit_pair(tdone, 0x3);
    }
  } else if (warp < C::FIRST_EPI_WARP) {
    // ----------------------------------------------------------- scale warps
    // Warps 2-5 write the A scales, warps 6-9 the B scales, each for the TMEM
    // lane quarter warp % 4: lane l writes line l of the atoms into lane 32q + l.
    const int q = warp & 3;
    const bool a_role = warp < 6;
    const uint32_t lane_addr = (uint32_t)(q * 32) << 16;
    const uint32_t ready_leader = mapa_shared(smem_u32(&sfready[0]), 0);
    int st = 0;
    uint32_t ph = 0;
    for (int u = cluster; u < total_units; u += nclusters) {
      for (int ks = 0; ks < p.kstages; ++ks) {
        uint64_t *bar = leader ? &full[st] : &sffull[st];
        if (!mbar_wait_warp(bar, ph, p.err, ERR_MMA, abort_flag)) { u = total_units; break; }
        const uint32_t reg = tmem + lane_addr + (uint32_t)(st * C::SF_COLS);
        if (a_role) {
          const uint4 *sa = reinterpret_cast<const uint4 *>(sSFA + st * C::SFA_BYTES) + lane;
          uint32_t ra[16];
#pragma unroll
          for (int kb = 0; kb < 4; ++kb) {
            const uint4 a = sa[kb * 32];
            ra[4 * kb] = a.x; ra[4 * kb + 1] = a.y; ra[4 * kb + 2] = a.z; ra[4 * kb + 3] = a.w;
          }
          tmem_st16(reg + C::SFA_COL, ra);
        } else {
          const uint4 *sb = reinterpret_cast<const uint4 *>(sSFB + st * C::SFB_BYTES) + lane;
          uint32_t rb0[16], rb1[16];
#pragma unroll
          for (int kb = 0; kb < 4; ++kb) {
            const uint4 b0 = sb[kb * 32];
            const uint4 b1 = sb[128 + kb * 32];
            uint32_t *bw = kb < 2 ? rb0 : rb1;
            const int o = (kb & 1) * 8;
            bw[o] = b0.x; bw[o + 1] = b0.y; bw[o + 2] = b0.z; bw[o + 3] = b0.w;
            bw[o + 4] = b1.x; bw[o + 5] = b1.y; bw[o + 6] = b1.z; bw[o + 7] = b1.w;
          }
          tmem_st16(reg + C::SFB_COL, rb0);
          tmem_st16(reg + C::SFB_COL + 16, rb1);
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(ready_leader + (uint32_t)(st * 8));
        if (++st == C::STAGES) { st = 0; ph ^= 1; }
      }
    }
  } else {
    // ------------------------------------------------------------- epilogue
    const int ew = warp - C::FIRST_EPI_WARP;
    const int q = warp & 3;
    const int cbase = (ew >> 2) * C::EPI_COLS;
    const uint32_t lane_addr = (uint32_t)(q * 32) << 16;
    const uint32_t tempty_leader = mapa_shared(smem_u32(tempty), 0);
    const float alpha = __fmul_rn(__ldg(p.ga), __ldg(p.gb));
    int it = 0;
    for (int u = cluster; u < total_units; u += nclusters, ++it) {
      int ta, tb, split;
      unit_coords(p, u, ta, tb, split);
      if (!mbar_wait_warp(tfull, it & 1, p.err, ERR_EPILOGUE, abort_flag)) break;
      tc_fence_after();
      const int i = ta * 256 + (int)rank * C::BM + q * 32 + lane;
      const int j0 = tb * C::BN + cbase;
      if constexpr (MODE == OUT_BF16) {
        // drain all 128 columns as packed bf16 (64 registers), hand TMEM back,
        // then store while the next tile's MMAs run
        uint32_t packed[C::EPI_COLS / 2];
#pragma unroll
        for (int c = 0; c < C::EPI_COLS; c += 32) {
          uint32_t acc[32];
          tmem_ld32(tmem + lane_addr + cbase + c, acc);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            __nv_bfloat162 h = __floats2bfloat162_rn(__fmul_rn(__uint_as_float(acc[2 * e]), alpha),
                                                     __fmul_rn(__uint_as_float(acc[2 * e + 1]), alpha));
            packed[c / 2 + e] = *reinterpret_cast<uint32_t *>(&h);
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(tempty_leader);
        if (p.tma_store) {
          // lane l writes row l of a 32 x 32 box, 16-byte chunk j at j ^ ((l / 2) % 4)
          // (the 64-byte swizzle: conflict-free for eight lanes at a time), then
          // one lane stores the box; rows and columns past Y are not written
          const int row0 = ta * 256 + (int)rank * C::BM + q * 32;
          uint8_t *stg = sStg + ew * C::STG_WARP_BYTES;
          uint4 *dst = reinterpret_cast<uint4 *>(stg + lane * 64);
#pragma unroll
          for (int c = 0; c < C::EPI_COLS; c += 32) {
            if (lane == 0) bulk_wait_read_all();        // the previous box has left the buffer
            __syncwarp();
#pragma unroll
            for (int j = 0; j < 4; ++j)
              dst[j ^ ((lane >> 1) & 3)] = make_uint4(packed[c / 2 + 4 * j], packed[c / 2 + 4 * j + 1],
                                                      packed[c / 2 + 4 * j + 2], packed[c / 2 + 4 * j + 3]);
            fence_proxy_async_shared();
            __syncwarp();
            if (lane == 0 && row0 < p.rows_a && j0 + c < p.rows_b) {
              tma_store_2d<NVFP4_Y_EVICT_FIRST>(&tmy, stg, j0 + c, row0);
              bulk_commit_group();
            }
          }
        } else if (i < p.rows_a) {
          __nv_bfloat16 *o = static_cast<__nv_bfloat16 *>(p.out);
#pragma unroll
          for (int c = 0; c < C::EPI_COLS; c += 8) {
            const int64_t o0 = (int64_t)i * p.out_si + j0 + c;
            if (j0 + c + 8 <= p.rows_b && (o0 & 7) == 0) {
              *reinterpret_cast<uint4 *>(o + o0) =
                  make_uint4(packed[c / 2], packed[c / 2 + 1], packed[c / 2 + 2], packed[c / 2 + 3]);
            } else {
#pragma unroll
              for (int e = 0; e < 8; ++e)
                if (j0 + c + e < p.rows_b) {
                  const uint32_t w = packed[(c + e) / 2];
                  const uint16_t h = (uint16_t)(((c + e) & 1) ? (w >> 16) : (w & 0xFFFFu));
                  reinterpret_cast<uint16_t *>(o)[o0 + e] = h;
                }
            }
          }
        }
      } else {
        // FP32 output: drain and store 32 columns at a time
#pragma unroll 1
        for (int c = 0; c < C::EPI_COLS; c += 32) {
          uint32_t acc[32];
          tmem_ld32(tmem + lane_addr + cbase + c, acc);
          tmem_ld_wait();
          if (i < p.rows_a) {
#pragma unroll
            for (int e = 0; e < 32; e += 8) store_chunk<C::BN, MODE>(p, i, j0 + c + e, &acc[e], alpha, 0);
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(tempty_leader);
      }
    }
    if (lane == 0) bulk_wait_all();                 // Y boxes written before the CTA ends
  }

  // teardown: the leader's MMAs write this CTA's TMEM and read its shared
  // memory, and this CTA's warps arrive on the leader's barriers, so each CTA
  // waits for all tensor work of the pair and for the other CTA to be done
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0) {
    volatile int never = 0;
    mbar_wait(tdone, 0, p.err, ERR_MMA, &never);
    mbar_arrive_cluster(mapa_shared(smem_u32(pairdone), rank ^ 1u));
    mbar_wait(pairdone, 0, p.err, ERR_MMA, &never);
  }
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc_pair(tmem, C::TMEM_COLS);
}

}  // namespace nvfp4
