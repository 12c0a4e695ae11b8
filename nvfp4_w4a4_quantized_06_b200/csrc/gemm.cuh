// gemm.cuh -- block-scaled NVFP4 x NVFP4 GEMM on sm_100a tensor cores.
//
// D[i, j] = sum_k dec(A)[i, k] * dec(B)[j, k]: both operands K-major packed
// E2M1 with swizzled E4M3 scales per 16 elements (web pages on arXiv
// 2609.04098, ta-paperlens page, "前提1": the W4A4 product runs directly on the
// 4-bit tensor cores with FP32 accumulation).  The epilogue multiplies by
// fl32(g_a * g_b) and writes BF16 or FP32, or writes raw FP32 partial sums for
// a later split-K reduction.
//
// Used for the products the CTA-pair kernel (large M and N) and the cluster
// split-K kernel (one operand of at most 128 rows) do not take: both
// operands wider than 128 rows but too few 256 x 256 tiles to fill the
// device with pairs.  This file also holds the parameter block, the tile
// raster and the output helpers the other GEMM kernels share.
//
// Design (one CTA per SM, persistent over output tiles):
//   warp 0      TMA producer: per K-stage of 256 elements, a 2D tiled load of
//               the 128 x 128-byte A tile and the BN x 128-byte B tile (128-byte
//               swizzle), plus 1D bulk copies of the matching 512-byte scale
//               atoms (4 per 128 rows), all completing on one mbarrier.
//   warp 1      MMA issuer (one thread): tcgen05.cp of the scale atoms into
//               TMEM, four tcgen05.mma kind::mxf4nvf4 (K = 64 each) per stage,
//               tcgen05.commit to release the stage; a final commit hands the
//               accumulator to the epilogue.  Also allocates TMEM.
//   warps 2..   epilogue: tcgen05.ld the FP32 accumulator (lane = row i), hand
//               TMEM back as soon as it is in registers, then scale, convert
//               and store while the next tile's MMAs run.
// TMEM columns: [0, BN) accumulator, then one scale region per pipeline stage
// (16 columns of A scales, 4 MMAs x 4 columns, and 16*BN/128 of B scales).  A
// region is rewritten only after the producer has refilled its stage, i.e.
// after the MMAs that read it have completed.
#pragma once
#include <cuda_bf16.h>
#include <cstdint>

#include "ptx.cuh"

namespace nvfp4 {

// OUT_GATES: FP32 GDN gate activations of the fused a/b gate projection
// (output columns [0, n_split) -> exp(-softplus(y)), the rest -> sigmoid(y)).
enum OutMode : int { OUT_BF16 = 0, OUT_F32 = 1, OUT_PARTIAL = 2, OUT_GATES = 3 };

struct GemmParams {
  const uint8_t *sfa;
  const uint8_t *sfb;
  const float *ga;
  const float *gb;
  void *out;
  int64_t out_si, out_sj;   // element strides of D's (A-row i, B-row j) in `out`
  int64_t part_stride;      // elements between split-K partial slices (OUT_PARTIAL)
  int rows_a, rows_b, K;
  int kblocks;              // K / 64
  int kstages;              // ceil(K / 256)
  int tiles_a, tiles_b, splits, group;
  int n_split;              // OUT_GATES: first output column of the b gates
  const void *x;            // fused activation quantize: bf16/fp32 activation [rows_b, K]
  int64_t ld_x;             //   its row stride (elements)
  const float *x_gscale;    //   its global scale (device)
  unsigned *err;
  int tma_store;            // CTA-pair GEMM, BF16 out: store Y through its tensor map
};

template <int BN>
struct GemmCfg {
  static constexpr int BM = 128;
  static constexpr int STAGE_K_BYTES = 128;          // 256 FP4 elements
  static constexpr int A_BYTES = BM * STAGE_K_BYTES;
  static constexpr int B_BYTES = BN * STAGE_K_BYTES;
  static constexpr int SFB_ATOMS = BN >= 128 ? BN / 128 : 1;
  static constexpr int SFA_BYTES = 4 * 512;
  static constexpr int SFB_BYTES = SFB_ATOMS * 4 * 512;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES;
  static constexpr int STAGES = BN >= 256 ? 4 : (BN >= 128 ? 6 : 4);
  static constexpr int EPI_WARPS = BN >= 64 ? 8 : 4;
  static constexpr int EPI_COLS = BN / (EPI_WARPS / 4);   // columns per epilogue warp
  static constexpr int THREADS = 64 + 32 * EPI_WARPS;
  // per-stage scale-factor regions after the accumulator: A scales (4 MMAs x 4
  // columns) then B scales (4 MMAs x 4 columns per 128 rows)
  static constexpr int SF_COLS = 16 + 16 * SFB_ATOMS;
  static constexpr int SFA_COL = BN;
  static constexpr int SFB_COL = BN + 16;
  static constexpr int TMEM_NEEDED = BN + STAGES * SF_COLS;
  static constexpr int TMEM_COLS = TMEM_NEEDED <= 32 ? 32 : TMEM_NEEDED <= 64 ? 64
                                  : TMEM_NEEDED <= 128 ? 128 : TMEM_NEEDED <= 256 ? 256 : 512;
  static constexpr int BAR_BYTES = 256;
  static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + BAR_BYTES;
  // instruction descriptor: A,B = E2M1 (1), K-major, scale type UE4M3, M=128, N=BN
  static constexpr uint32_t IDESC = (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) |
                                    ((uint32_t)(BM >> 4) << 24);
  static_assert(BN % 16 == 0 && BN >= 32 && BN <= 256, "MMA N");
  static_assert(STAGE_BYTES % 1024 == 0, "stage alignment");
  static_assert(EPI_COLS % 32 == 0 && EPI_COLS <= 128, "epilogue chunking");
};

__device__ __forceinline__ void unit_coords(const GemmParams &p, int u, int &ta, int &tb, int &split) {
  split = u % p.splits;
  const int t = u / p.splits;
  const int per_group = p.group * p.tiles_b;
  const int g = t / per_group, r = t - g * per_group;
  const int first = g * p.group;
  const int gs = min(p.group, p.tiles_a - first);
  ta = first + r % gs;
  tb = r / gs;
}

__device__ __forceinline__ void split_range(const GemmParams &p, int split, int &ks0, int &ks1) {
  ks0 = (int)(((int64_t)p.kstages * split) / p.splits);
  ks1 = (int)(((int64_t)p.kstages * (split + 1)) / p.splits);
}

template <int BN, int MODE>
__device__ __forceinline__ void store_chunk(const GemmParams &p, int i, int j0, const uint32_t *acc,
                                            float alpha, int split) {
  // eight consecutive j (B rows) for one i (A row)
  if constexpr (MODE == OUT_PARTIAL) {
    float *o = static_cast<float *>(p.out) + (int64_t)split * p.part_stride;
#pragma unroll
    for (int c = 0; c < 8; ++c)
      if (j0 + c < p.rows_b) o[(int64_t)i * p.out_si + (int64_t)(j0 + c) * p.out_sj] = __uint_as_float(acc[c]);
  } else {
  float v[8];
#pragma unroll
  for (int c = 0; c < 8; ++c) v[c] = __fmul_rn(__uint_as_float(acc[c]), alpha);
  if constexpr (MODE == OUT_BF16) {
    __nv_bfloat16 *o = static_cast<__nv_bfloat16 *>(p.out);
    const int64_t o0 = (int64_t)i * p.out_si + j0;
    if (p.out_sj == 1 && j0 + 8 <= p.rows_b && (o0 & 7) == 0) {
      uint4 w;
      uint32_t *ww = reinterpret_cast<uint32_t *>(&w);
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * c], v[2 * c + 1]);
        ww[c] = *reinterpret_cast<uint32_t *>(&h);
      }
      *reinterpret_cast<uint4 *>(o + o0) = w;
    } else {
#pragma unroll
      for (int c = 0; c < 8; ++c)
        if (j0 + c < p.rows_b) o[(int64_t)i * p.out_si + (int64_t)(j0 + c) * p.out_sj] = __float2bfloat16_rn(v[c]);
    }
  } else {
    float *o = static_cast<float *>(p.out);
    const int64_t o0 = (int64_t)i * p.out_si + j0;
    if (p.out_sj == 1 && j0 + 8 <= p.rows_b && (o0 & 3) == 0) {
      float4 *q = reinterpret_cast<float4 *>(o + o0);
      q[0] = make_float4(v[0], v[1], v[2], v[3]);
      q[1] = make_float4(v[4], v[5], v[6], v[7]);
    } else {
#pragma unroll
      for (int c = 0; c < 8; ++c)
        if (j0 + c < p.rows_b) o[(int64_t)i * p.out_si + (int64_t)(j0 + c) * p.out_sj] = v[c];
    }
  }
  }
}

template <int BN, int MODE>
__global__ void __launch_bounds__(GemmCfg<BN>::THREADS, 1)
    nvfp4_gemm_kernel(const __grid_constant__ CUtensorMap tma, const __grid_constant__ CUtensorMap tmb,
                      const GemmParams p) {
  using C = GemmCfg<BN>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sA = smem;
  uint8_t *sB = sA + C::STAGES * C::A_BYTES;
  uint8_t *sSFA = sB + C::STAGES * C::B_BYTES;
  uint8_t *sSFB = sSFA + C::STAGES * C::SFA_BYTES;
  uint64_t *bars = reinterpret_cast<uint64_t *>(sSFB + C::STAGES * C::SFB_BYTES);
  uint64_t *full = bars;
  uint64_t *empty = bars + C::STAGES;
  uint64_t *tfull = bars + 2 * C::STAGES;
  uint64_t *tempty = tfull + 1;
  uint64_t *tdone = tfull + 2;
  uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(tfull + 3);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int total_units = p.tiles_a * p.tiles_b * p.splits;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(tfull, 1);
    mbar_init(tempty, C::EPI_WARPS);
    mbar_init(tdone, 1);
    *abort_flag = 0;
    fence_barrier_init();
    prefetch_tmap(&tma);
    prefetch_tmap(&tmb);
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ producer
      int st = 0;
      uint32_t ph = 0;
      uint32_t issued = 0;
      bool ok = true;
      const int pad_b = (p.rows_b + 127) & ~127;
      for (int u = blockIdx.x; u < total_units && ok; u += gridDim.x) {
        int ta, tb, split, ks0, ks1;
        unit_coords(p, u, ta, tb, split);
        split_range(p, split, ks0, ks1);
        const int row_a = ta * C::BM, row_b = tb * BN;
        for (int ks = ks0; ks < ks1; ++ks) {
          if (!mbar_wait(&empty[st], ph ^ 1, p.err, ERR_PRODUCER, abort_flag)) { ok = false; break; }
          const int nkb = min(4, p.kblocks - ks * 4);
          int nsfb = 0;
#pragma unroll
          for (int j = 0; j < C::SFB_ATOMS; ++j)
            if (row_b + 128 * j < pad_b) ++nsfb;
          const uint32_t bytes = C::A_BYTES + C::B_BYTES + (uint32_t)nkb * 512u * (1u + nsfb);
          mbar_arrive_expect_tx(&full[st], bytes);
          tma_load_2d(sA + st * C::A_BYTES, &tma, &full[st], ks * C::STAGE_K_BYTES, row_a);
          tma_load_2d(sB + st * C::B_BYTES, &tmb, &full[st], ks * C::STAGE_K_BYTES, row_b);
          bulk_load(sSFA + st * C::SFA_BYTES,
                    p.sfa + ((int64_t)(row_a >> 7) * p.kblocks + ks * 4) * 512, nkb * 512u, &full[st]);
#pragma unroll
          for (int j = 0; j < C::SFB_ATOMS; ++j)
            if (j < nsfb)
              bulk_load(sSFB + st * C::SFB_BYTES + j * 2048,
                        p.sfb + ((int64_t)((row_b >> 7) + j) * p.kblocks + ks * 4) * 512, nkb * 512u,
                        &full[st]);
          ++issued;
          if (++st == C::STAGES) { st = 0; ph ^= 1; }
        }
      }
      // teardown: every armed stage's loads must have landed before the CTA exits
      for (int s = 0; s < C::STAGES; ++s) {
        const uint32_t armed = issued / C::STAGES + ((uint32_t)s < issued % C::STAGES ? 1u : 0u);
        if (armed) {
          volatile int never = 0;
          mbar_wait(&full[s], (armed - 1) & 1, p.err, ERR_PRODUCER, &never);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------------- MMA issue
      // One thread feeds the tensor pipe, so this loop is kept lean: every
      // descriptor is built once and advanced by immediate adds (the start
      // address sits in the low 14 bits, addresses stay below 256 KB), and the
      // four K-blocks of a stage are unrolled.  Per K-block the scale atoms are
      // copied into this stage's TMEM region right before the MMA that reads
      // them; stages rotate through their own regions.
      const uint64_t a_desc0 = smem_desc(smem_u32(sA), 16, 1024, 2);
      const uint64_t b_desc0 = smem_desc(smem_u32(sB), 16, 1024, 2);
      const uint64_t sfa_desc0 = smem_desc(smem_u32(sSFA), 0, 128, 0);
      const uint64_t sfb_desc0 = smem_desc(smem_u32(sSFB), 0, 128, 0);
      int st = 0;
      uint32_t ph = 0;
      int it = 0;
      for (int u = blockIdx.x; u < total_units; u += gridDim.x, ++it) {
        int ta, tb, split, ks0, ks1;
        unit_coords(p, u, ta, tb, split);
        split_range(p, split, ks0, ks1);
        if (!mbar_wait(tempty, (it & 1) ^ 1, p.err, ERR_MMA, abort_flag)) break;
        tc_fence_after();
        bool ok = true;
        for (int ks = ks0; ks < ks1; ++ks) {
          if (!mbar_wait(&full[st], ph, p.err, ERR_MMA, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint64_t ad = a_desc0 + (uint64_t)((st * C::A_BYTES) >> 4);
          const uint64_t bd = b_desc0 + (uint64_t)((st * C::B_BYTES) >> 4);
          const uint64_t sad = sfa_desc0 + (uint64_t)((st * C::SFA_BYTES) >> 4);
          const uint64_t sbd = sfb_desc0 + (uint64_t)((st * C::SFB_BYTES) >> 4);
          const uint32_t reg = tmem + (uint32_t)(st * C::SF_COLS);
          const uint32_t acc0 = ks > ks0 ? 1u : 0u;
          if (ks * 4 + 4 <= p.kblocks) {
#pragma unroll
            for (int kb = 0; kb < 4; ++kb) {
              tc_cp_32x128b_warpx4(reg + C::SFA_COL + 4 * kb, sad + (uint64_t)(kb * 32));
#pragma unroll
              for (int j = 0; j < C::SFB_ATOMS; ++j)
                tc_cp_32x128b_warpx4(reg + C::SFB_COL + kb * 4 * C::SFB_ATOMS + 4 * j,
                                     sbd + (uint64_t)(j * 128 + kb * 32));
              tc_mma_nvfp4(tmem, ad + (uint64_t)(kb * 2), bd + (uint64_t)(kb * 2), C::IDESC,
                           kb > 0 ? 1u : acc0, reg + C::SFA_COL + 4 * kb,
                           reg + C::SFB_COL + kb * 4 * C::SFB_ATOMS);
            }
          } else {
            const int nkb = p.kblocks - ks * 4;      // K tail: 1 to 3 blocks
            for (int kb = 0; kb < nkb; ++kb) {
              tc_cp_32x128b_warpx4(reg + C::SFA_COL + 4 * kb, sad + (uint64_t)(kb * 32));
#pragma unroll
              for (int j = 0; j < C::SFB_ATOMS; ++j)
                tc_cp_32x128b_warpx4(reg + C::SFB_COL + kb * 4 * C::SFB_ATOMS + 4 * j,
                                     sbd + (uint64_t)(j * 128 + kb * 32));
              tc_mma_nvfp4(tmem, ad + (uint64_t)(kb * 2), bd + (uint64_t)(kb * 2), C::IDESC,
                           kb > 0 ? 1u : acc0, reg + C::SFA_COL + 4 * kb,
                           reg + C::SFB_COL + kb * 4 * C::SFB_ATOMS);
            }
          }
          tc_commit(&empty[st]);
          if (++st == C::STAGES) { st = 0; ph ^= 1; }
        }
        if (!ok) break;
        tc_commit(tfull);
      }
      // teardown: all issued tensor-core work must finish before TMEM is freed
      tc_commit(tdone);
      volatile int never = 0;
      mbar_wait(tdone, 0, p.err, ERR_MMA, &never);
    }
  } else {
    // ------------------------------------------------------------- epilogue
    const int ew = warp - 2;
    const int q = warp & 3;                       // TMEM lane quarter this warp may access
    const int cbase = (ew >> 2) * C::EPI_COLS;    // first accumulator column of this warp
    const uint32_t lane_addr = (uint32_t)(q * 32) << 16;
    float alpha = 0.0f;
    if (MODE != OUT_PARTIAL) alpha = __fmul_rn(__ldg(p.ga), __ldg(p.gb));
    int it = 0;
    for (int u = blockIdx.x; u < total_units; u += gridDim.x, ++it) {
      int ta, tb, split;
      unit_coords(p, u, ta, tb, split);
      if (!mbar_wait_warp(tfull, it & 1, p.err, ERR_EPILOGUE, abort_flag)) break;
      tc_fence_after();
      uint32_t acc[C::EPI_COLS];
#pragma unroll
      for (int c = 0; c < C::EPI_COLS; c += 32)
        tmem_ld32(tmem + lane_addr + cbase + c, *reinterpret_cast<uint32_t(*)[32]>(&acc[c]));
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(tempty);
      const int i = ta * C::BM + q * 32 + lane;
      if (i < p.rows_a) {
        const int j0 = tb * BN + cbase;
#pragma unroll
        for (int c = 0; c < C::EPI_COLS; c += 8) store_chunk<BN, MODE>(p, i, j0 + c, &acc[c], alpha, split);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, C::TMEM_COLS);
}

// y[m, n] = cvt(alpha * sum_s part[s][m*N + n]) for split-K
template <int MODE>
__global__ void __launch_bounds__(256) splitk_reduce_kernel(const float *part, int splits, int64_t MN,
                                                            int N, const float *ga, const float *gb,
                                                            void *out, int64_t ld) {
  const float alpha = __fmul_rn(__ldg(ga), __ldg(gb));
  for (int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; e < MN;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    float s = 0.0f;
    for (int k = 0; k < splits; ++k) s += part[(int64_t)k * MN + e];
    const float v = __fmul_rn(s, alpha);
    const int64_t m = e / N, n = e - m * N;
    if (MODE == OUT_BF16) static_cast<__nv_bfloat16 *>(out)[m * ld + n] = __float2bfloat16_rn(v);
    else static_cast<float *>(out)[m * ld + n] = v;
  }
}

}  // namespace nvfp4
