// gemm_cluster.cuh -- block-scaled NVFP4 GEMM with split-K across the CTAs of
// a thread-block cluster, reduced through distributed shared memory.
//
// Same product as gemm.cuh (D[i, j] = sum_k dec(A)[i, k] * dec(B)[j, k], FP32
// accumulation; web pages on arXiv 2609.04098, ta-paperlens page, "前提1"),
// for the shapes where one operand is narrow: decode (a few activation rows,
// the weight on the 128-row MMA side) and small-N projections such as the
// GDN a/b gates (N = 96).  Such products have too few 128-row tiles to fill
// the GPU, so each tile is computed by a cluster of S CTAs, rank r taking
// K stages [r*KS/S, (r+1)*KS/S):
//   warp 0     TMA producer.  The loads of the operand that does not depend
//              on the preceding kernel (the weight) are issued first, then
//              the thread waits for that kernel (programmatic dependent
//              launch) before loading the activation side.
//   warp 1     TMEM allocation and MMA issue: four tcgen05.mma
//              kind::mxf4nvf4 (K = 64) per stage and nothing else.
//   warps 2-5  during the K loop, scale warps (one per TMEM lane quarter):
//              they move each stage's scale atoms from shared memory into
//              the stage's TMEM columns with tcgen05.st (the replicated image
//              a 32x128b.warpx4 copy would make), which keeps the MMA thread
//              from issuing two copies per MMA.  Then the epilogue: each CTA owns a share of the output tile (whole
//              output columns for decode, whole rows otherwise); the FP32
//              partial tile leaves TMEM and every element is stored straight
//              into the owner CTA's shared memory, in the slot of the
//              sending rank (fire-and-forget distributed-shared-memory
//              stores).  After one cluster barrier each CTA sums its share
//              over the S slots in rank order (so the result does not depend
//              on timing), scales by fl32(g_a*g_b) and writes BF16 or FP32.
// No partial sums touch global memory and no second kernel is launched.
#pragma once
#include <cuda_bf16.h>
#include <cstdint>

#include <type_traits>

#include "gemm.cuh"
#include "ptx.cuh"
#include "quantize.cuh"

namespace nvfp4 {

// GDN gate activations of the a and b gate projections (ta-paperlens page,
// "前提2"): a goes through softplus and the exponential, alpha = exp(-softplus(a))
// (the share of the state that is kept), b through the logistic sigmoid,
// beta = 1 / (1 + exp(-b)).  The model's per-head decay scale and bias are
// not part of this layer (unit scale, zero bias).  Since
// exp(-softplus(a)) = exp(-log(1 + e^a)) = 1 / (1 + e^a), both take one CUDA
// expf, one add and one correctly rounded reciprocal (a few ulp in all; an
// overflowing exponential gives the limit 0).
__device__ __forceinline__ float gate_keep(float a) { return __frcp_rn(__fadd_rn(1.0f, expf(a))); }
__device__ __forceinline__ float gate_write(float b) { return __frcp_rn(__fadd_rn(1.0f, expf(-b))); }

// FUSED: the activation (the B operand of decode-shaped products) is read
// as bf16/fp32 and quantized inside the kernel by QWARPS extra warps, which
// write the codes straight into the MMA's swizzled B tiles and the scale
// bytes into the B scale atoms (the quantize fused into the GEMM's producer).
template <int BN, bool FUSED = false>
struct ClusterCfg {
  static constexpr int BM = 128;
  static constexpr int A_BYTES = BM * 128;                 // 256 FP4 per row per stage
  static constexpr int B_BYTES = BN * 128;
  static constexpr int SFB_ATOMS = BN >= 128 ? BN / 128 : 1;
  static constexpr int SFA_BYTES = 4 * 512;
  static constexpr int SFB_BYTES = SFB_ATOMS * 4 * 512;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES;
  static constexpr int STAGES = BN <= 32 ? 8 : (BN <= 64 ? 6 : 4);
  static constexpr int EPI_WARPS = 4;
  // activation encoder warps: a 128-row activation tile (the gate
  // projections' many tokens) needs three times the encoding of a decode tile
  static constexpr int QWARPS = FUSED ? (BN >= 128 ? 24 : 8) : 0;
  static constexpr int THREADS = 64 + 32 * (EPI_WARPS + QWARPS);
  static constexpr int SF_COLS = 16 + 16 * SFB_ATOMS;
  static constexpr int SFA_COL = BN;
  static constexpr int SFB_COL = BN + 16;
  static constexpr int TMEM_NEEDED = BN + STAGES * SF_COLS;
  static constexpr int TMEM_COLS = TMEM_NEEDED <= 64 ? 64 : TMEM_NEEDED <= 128 ? 128
                                  : TMEM_NEEDED <= 256 ? 256 : 512;
  // cluster sizes this configuration serves (the reduction slots of more
  // ranks would not fit next to the 128-wide operand ring)
  static constexpr int MAX_SPLITS = BN >= 128 ? 5 : 8;
  // reduction slots: one per rank in every owner, holding the owner's share
  // of the tile, a multiple of 4 tile rows (share_rows).  A slot is
  // column-major, [BN columns j][slot_pitch], so that for each column the 32
  // lanes of a warp (32 consecutive tile rows) store 32 consecutive floats,
  // and the reduction reads four tile rows with one 16-byte load.  The pitch
  // is the share, plus 4 floats where the share is a multiple of 8, so that
  // lanes walking over columns hit distinct 16-byte bank groups.
  static constexpr int share_rows(int S) { return ((BM + S - 1) / S + 3) / 4 * 4; }
  static constexpr int slot_pitch(int S) { return share_rows(S) % 8 == 0 ? share_rows(S) + 4 : share_rows(S); }
  static constexpr int slot_floats(int S) { return BN * slot_pitch(S); }
  static constexpr int red_need() {
    int m = 0;
    for (int S = 1; S <= MAX_SPLITS; ++S) m = S * slot_floats(S) > m ? S * slot_floats(S) : m;
    return m;
  }
  static constexpr int RED_FLOATS = (red_need() + 31) / 32 * 32;   // 128-byte multiple
  static constexpr int BAR_BYTES = 512;            // barriers, TMEM address, abort flag
  static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + RED_FLOATS * 4 + BAR_BYTES + (FUSED ? 512 : 0);
  static_assert((4 * STAGES + 2) * 8 + 8 <= BAR_BYTES, "barrier area");
  static constexpr uint32_t IDESC = (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) |
                                    ((uint32_t)(BM >> 4) << 24);
  static_assert(BN % 16 == 0 && BN >= 32 && BN <= 128, "MMA N");
  static_assert((STAGES * STAGE_BYTES + RED_FLOATS * 4) % 128 == 0, "mbarrier alignment");
  static_assert(STAGE_BYTES % 1024 == 0, "stage alignment");
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
  static_assert(TMEM_NEEDED <= 512, "TMEM budget");
};

// p.splits = S (the cluster size), p.tiles_a x p.tiles_b tiles (one per
// cluster), p.group != 0 when A is the operand independent of the preceding
// kernel (the weight), 0 when B is.
// XT = void: both operands pre-quantized (TMA); XT = bf16 / float: the B
// operand is the activation p.x [rows_b, K] (row stride p.ld_x), quantized
// here with global scale p.x_gscale (then tmb is unused).
template <int BN, int MODE, typename XT = void>
__global__ void __launch_bounds__(ClusterCfg<BN, !std::is_void<XT>::value>::THREADS, 1)
    nvfp4_gemm_cluster_kernel(const __grid_constant__ CUtensorMap tma, const __grid_constant__ CUtensorMap tmb,
                              const GemmParams p) {
  constexpr bool FUSED = !std::is_void<XT>::value;
  using C = ClusterCfg<BN, FUSED>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sA = smem;
  uint8_t *sB = sA + C::STAGES * C::A_BYTES;
  uint8_t *sSFA = sB + C::STAGES * C::B_BYTES;
  uint8_t *sSFB = sSFA + C::STAGES * C::SFA_BYTES;
  float *red = reinterpret_cast<float *>(sSFB + C::STAGES * C::SFB_BYTES);   // reduction slots
  uint64_t *bars = reinterpret_cast<uint64_t *>(red + C::RED_FLOATS);
  uint64_t *full = bars;
  uint64_t *empty = bars + C::STAGES;
  uint64_t *sfready = bars + 2 * C::STAGES;     // the stage's scales are in TMEM (4 warps)
  uint64_t *bready = bars + 3 * C::STAGES;      // FUSED: the stage's activation tile is encoded
  uint64_t *tfull = bars + 4 * C::STAGES;
  uint64_t *tdone = tfull + 1;
  uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(tfull + 2);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_holder + 1);
  float *rcp_tab = reinterpret_cast<float *>(reinterpret_cast<uint8_t *>(bars) + C::BAR_BYTES);   // FUSED

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int S = p.splits;
  const int rank = (int)cluster_ctarank();
  const int tile = blockIdx.x / S;
  const int ta = tile % p.tiles_a, tb = tile / p.tiles_a;
  int ks0, ks1;
  split_range(p, rank, ks0, ks1);
  // output ownership: decode writes Y[m, n] with n = tile row i contiguous,
  // so a CTA owns whole columns j; otherwise whole rows i
  const bool i_fast = p.out_si == 1;

  // producer helpers (thread 0): the bytes a stage brings and its loads
  const int row_a = ta * C::BM, row_b = tb * BN;
  const int pad_b = (p.rows_b + 127) & ~127;
  const bool a_first = p.group != 0;
  auto stage_bytes = [&](int ks) {
    const int nkb = min(4, p.kblocks - ks * 4);
    int nsfb = 0;
#pragma unroll
    for (int j = 0; j < C::SFB_ATOMS; ++j)
      if (row_b + 128 * j < pad_b) ++nsfb;
    if (FUSED) return (uint32_t)C::A_BYTES + (uint32_t)nkb * 512u;
    return (uint32_t)(C::A_BYTES + C::B_BYTES) + (uint32_t)nkb * 512u * (1u + nsfb);
  };
  auto load_a = [&](int st, int ks) {
    const int nkb = min(4, p.kblocks - ks * 4);
    tma_load_2d(sA + st * C::A_BYTES, &tma, &full[st], ks * 128, row_a);
    bulk_load(sSFA + st * C::SFA_BYTES, p.sfa + ((int64_t)(row_a >> 7) * p.kblocks + ks * 4) * 512,
              nkb * 512u, &full[st]);
  };
  auto load_b = [&](int st, int ks) {
    if (FUSED) return;
    const int nkb = min(4, p.kblocks - ks * 4);
    tma_load_2d(sB + st * C::B_BYTES, &tmb, &full[st], ks * 128, row_b);
#pragma unroll
    for (int j = 0; j < C::SFB_ATOMS; ++j)
      if (row_b + 128 * j < pad_b)
        bulk_load(sSFB + st * C::SFB_BYTES + j * 2048,
                  p.sfb + ((int64_t)((row_b >> 7) + j) * p.kblocks + ks * 4) * 512, nkb * 512u, &full[st]);
  };
  const int pre = min(ks1 - ks0, C::STAGES);

  if (threadIdx.x == 0) {
    // the tensor maps' descriptors are fetched while the barriers are set up
    prefetch_tmap(&tma);
    if (!FUSED) prefetch_tmap(&tmb);
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
      mbar_init(&sfready[s], C::EPI_WARPS);
      if (FUSED) mbar_init(&bready[s], C::QWARPS);
    }
    mbar_init(tfull, 1);
    mbar_init(tdone, 1);
    *abort_flag = 0;
    fence_barrier_init();
    // the first ring's worth of the operand that does not depend on the
    // preceding kernel streams in from here on, while the rest of the CTA
    // sets up (TMEM, tables) and before the preceding kernel has finished.
    // That holds where the preceding kernel is this library's activation
    // quantize, which lets this grid start only after everything before it
    // has completed.  The fused form follows whatever the caller ran last,
    // which may still be writing the weight: it waits first.
    if constexpr (FUSED) griddep_wait();
    for (int i = 0; i < pre; ++i) {
      mbar_arrive_expect_tx(&full[i], stage_bytes(ks0 + i));
      if (a_first) load_a(i, ks0 + i); else load_b(i, ks0 + i);
    }
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, C::TMEM_COLS);
    tmem_relinquish();
  }
  if constexpr (FUSED) {
    fill_rcp_table(rcp_tab);
    // scale atoms of B rows past BN stay zero for the whole kernel
    for (int i = threadIdx.x; i < C::STAGES * C::SFB_BYTES / 16; i += C::THREADS)
      reinterpret_cast<uint4 *>(sSFB)[i] = make_uint4(0u, 0u, 0u, 0u);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  // the next kernel in the stream may be scheduled now; it waits for this
  // grid's completion before it touches anything this grid reads or writes
  if (threadIdx.x == 0) griddep_launch_dependents();

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ producer
      // the independent operand's first stages are in flight (issued at the
      // top); wait for the preceding kernel, then the dependent operand
      griddep_wait();
      for (int i = 0; i < pre; ++i) {
        if (a_first) load_b(i, ks0 + i); else load_a(i, ks0 + i);
      }
      int st = pre == C::STAGES ? 0 : pre;
      uint32_t ph = pre == C::STAGES ? 1u : 0u;
      uint32_t issued = (uint32_t)pre;
      for (int ks = ks0 + pre; ks < ks1; ++ks) {
        if (!mbar_wait(&empty[st], ph ^ 1, p.err, ERR_PRODUCER, abort_flag)) break;
        mbar_arrive_expect_tx(&full[st], stage_bytes(ks));
        load_a(st, ks);
        load_b(st, ks);
        ++issued;
        if (++st == C::STAGES) { st = 0; ph ^= 1; }
      }
      // every armed stage's loads must have landed before the CTA exits
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
      const uint64_t a_desc0 = smem_desc(smem_u32(sA), 16, 1024, 2);
      const uint64_t b_desc0 = smem_desc(smem_u32(sB), 16, 1024, 2);
      int st = 0;
      uint32_t ph = 0;
      bool ok = true;
      for (int ks = ks0; ks < ks1; ++ks) {
        if (!mbar_wait(&sfready[st], ph, p.err, ERR_MMA, abort_flag)) { ok = false; break; }
        if (FUSED && !mbar_wait(&bready[st], ph, p.err, ERR_MMA, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const uint64_t ad = a_desc0 + (uint64_t)((st * C::A_BYTES) >> 4);
        const uint64_t bd = b_desc0 + (uint64_t)((st * C::B_BYTES) >> 4);
        const uint32_t reg = tmem + (uint32_t)(st * C::SF_COLS);
        const int nkb = min(4, p.kblocks - ks * 4);
#pragma unroll
        for (int kb = 0; kb < 4; ++kb)
          if (kb < nkb)
            tc_mma_nvfp4(tmem, ad + (uint64_t)(kb * 2), bd + (uint64_t)(kb * 2), C::IDESC,
                         (ks > ks0 || kb > 0) ? 1u : 0u, reg + C::SFA_COL + 4 * kb,
                         reg + C::SFB_COL + kb * 4 * C::SFB_ATOMS);
        tc_commit(&empty[st]);
        if (++st == C::STAGES) { st = 0; ph ^= 1; }
      }
      if (ok) tc_commit(tfull);
      // all issued tensor-core work must finish before TMEM is freed
      tc_commit(tdone);
      volatile int never = 0;
      mbar_wait(tdone, 0, p.err, ERR_MMA, &never);
    }
  } else if (FUSED && warp >= 2 + C::EPI_WARPS) {
    if constexpr (FUSED) {
      // -------------------------------------------- activation encoder warps
      // Per K stage, the BN x 256 activation slice is encoded (same encoder
      // as the quantize kernels, bit-identical codes) into this stage's B tile
      // in the MMA's 128-byte-swizzled K-major layout (row r, 16-byte chunk c
      // at r*128 + (c ^ (r % 8))*16) and its scale bytes into the stage's B
      // scale atoms.  Rows past rows_b and columns past K encode as zeros.
      const int qt = (int)threadIdx.x - 32 * (2 + C::EPI_WARPS);
      constexpr int QT = 32 * C::QWARPS;
      // blocks of a stage per encoder thread; bf16 blocks are all loaded
      // before any is encoded (their loads overlap), fp32 ones one at a time
      constexpr int NB = sizeof(XT) == 2 ? (BN * 16 + QT - 1) / QT : 1;
      griddep_wait();                                     // x and its scale may come from the preceding kernel
      const EncodeConsts kc = encode_consts(p.x_gscale);
      const XT *x = static_cast<const XT *>(p.x);
      const int row_base = tb * BN;                       // this tile's first activation row
      int st = 0;
      uint32_t ph = 0;
      for (int ks = ks0; ks < ks1; ++ks) {
        // the stage's previous tiles have been consumed by the MMAs
        if (!mbar_wait_warp(&empty[st], ph ^ 1, p.err, ERR_PRODUCER, abort_flag)) break;
        uint8_t *sb = sB + st * C::B_BYTES;
        uint8_t *ssf = sSFB + st * C::SFB_BYTES;
#pragma unroll 1
        for (int bi0 = qt; bi0 < BN * 16; bi0 += NB * QT) {
          Block16<XT> blk[NB];
          bool valid[NB];
#pragma unroll
          for (int n = 0; n < NB; ++n) {
            const int bi = bi0 + n * QT;
            const int r = bi >> 4, b = bi & 15;
            const int64_t col = (int64_t)ks * 256 + b * 16;
            valid[n] = bi < BN * 16 && row_base + r < p.rows_b && col < p.K;
            blk[n].zero();
            if (valid[n]) blk[n].load(x + (int64_t)(row_base + r) * p.ld_x + col);
          }
          if (ks + 1 < ks1) {
            // warm the same blocks of the next stage in L2 while these encode
#pragma unroll
            for (int n = 0; n < NB; ++n) {
              const int bi = bi0 + n * QT;
              const int r = bi >> 4, b = bi & 15;
              const int64_t col = (int64_t)(ks + 1) * 256 + b * 16;
              if (bi < BN * 16 && row_base + r < p.rows_b && col < p.K)
                prefetch_l2(x + (int64_t)(row_base + r) * p.ld_x + col);
            }
          }
#pragma unroll
          for (int n = 0; n < NB; ++n) {
            const int bi = bi0 + n * QT;
            if (bi >= BN * 16) break;
            const int r = bi >> 4, b = bi & 15;
            uint2 w = make_uint2(0u, 0u);
            uint32_t sc = 0u;
            if (valid[n])
              w = encode16(blk[n], kc, rcp_tab, x + (int64_t)(row_base + r) * p.ld_x + (int64_t)ks * 256 + b * 16, &sc);
            *reinterpret_cast<uint2 *>(sb + r * 128 + (((b >> 1) ^ (r & 7)) << 4) + (b & 1) * 8) = w;
            ssf[(b >> 2) * 512 + (r & 31) * 16 + (r >> 5) * 4 + (b & 3)] = (uint8_t)sc;
          }
        }
        fence_proxy_async_shared();                      // the tensor core reads the tile through the async proxy
        __syncwarp();
        if (lane == 0) mbar_arrive(&bready[st]);
        if (++st == C::STAGES) { st = 0; ph ^= 1; }
      }
    }
  } else {
    const int q = warp & 3;                       // TMEM lane quarter of this warp
    const int i = q * 32 + lane;                  // tile row (A row)
    const uint32_t lane_addr = (uint32_t)(q * 32) << 16;
    {
      // ----------------------------------------------------- scale warps
      // Lane l writes, for each 64-deep K block kb of the stage, the 16-byte
      // line l of the A atom and of the B atom(s) into its TMEM lane 32q + l:
      // columns SFA_COL + 4kb .. +3 and SFB_COL + 4kb*SFB_ATOMS .. (the
      // layout the MMA reads).  A stage's columns are rewritten only after
      // its next load has landed, i.e. after the MMAs that read them.
      int st = 0;
      uint32_t ph = 0;
      for (int ks = ks0; ks < ks1; ++ks) {
        if (!mbar_wait_warp(&full[st], ph, p.err, ERR_EPILOGUE, abort_flag)) break;
        if (FUSED && !mbar_wait_warp(&bready[st], ph, p.err, ERR_EPILOGUE, abort_flag)) break;
        const uint4 *sa = reinterpret_cast<const uint4 *>(sSFA + st * C::SFA_BYTES) + lane;
        const uint4 *sb = reinterpret_cast<const uint4 *>(sSFB + st * C::SFB_BYTES) + lane;
        const uint32_t reg = tmem + lane_addr + (uint32_t)(st * C::SF_COLS);
        uint32_t ra[16];
#pragma unroll
        for (int kb = 0; kb < 4; ++kb) {
          const uint4 a = sa[kb * 32];
          ra[4 * kb] = a.x; ra[4 * kb + 1] = a.y; ra[4 * kb + 2] = a.z; ra[4 * kb + 3] = a.w;
        }
        tmem_st16(reg + C::SFA_COL, ra);
#pragma unroll
        for (int h = 0; h < C::SFB_ATOMS; ++h) {
          // B region, 4*SFB_ATOMS words per K block: atom j of the K block at 4j
          uint32_t rb[16];
#pragma unroll
          for (int w = 0; w < 16; ++w) {
            const int kb = (h * 16 + w) / (4 * C::SFB_ATOMS), j = ((h * 16 + w) / 4) % C::SFB_ATOMS;
            const uint4 b = sb[j * 128 + kb * 32];
            rb[w] = (w & 3) == 0 ? b.x : ((w & 3) == 1 ? b.y : ((w & 3) == 2 ? b.z : b.w));
          }
          tmem_st16(reg + C::SFB_COL + 16 * h, rb);
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sfready[st]);
        if (++st == C::STAGES) { st = 0; ph ^= 1; }
      }
    }
    // ------------------------------- epilogue: partial tile -> owners' slots
    // Tile row i belongs to rank i / share; every element goes straight into
    // the owner's slot named after this rank (distributed-shared-memory
    // stores; for each column the warp's 32 lanes write 32 consecutive
    // floats, one transaction).  Columns past the narrow operand's rows hold
    // zeros and are neither sent nor summed.
    const bool ok = mbar_wait_warp(tfull, 0, p.err, ERR_EPILOGUE, abort_flag);
    if (ok) tc_fence_after();
    const int share = C::share_rows(S), pitch = C::slot_pitch(S);
    const int own_r = i / share, a = i - own_r * share;
    const int ncols = min(BN, p.rows_b - tb * BN);
    const uint32_t red_rank = mapa_shared(smem_u32(red) + (uint32_t)(rank * C::slot_floats(S) + a) * 4u,
                                          (uint32_t)own_r);
#pragma unroll 1
    for (int c = 0; c < ncols; c += 32) {
      uint32_t acc[32];
      if (ok) {
        tmem_ld32(tmem + lane_addr + c, acc);
        tmem_ld_wait();
      } else {
#pragma unroll
        for (int e = 0; e < 32; ++e) acc[e] = 0u;
      }
#pragma unroll
      for (int e = 0; e < 32; ++e)
        st_shared_cluster_f32(red_rank + (uint32_t)((c + e) * pitch * 4), __uint_as_float(acc[e]));
    }
  }

  // ------------------------------------------------- cluster-wide reduction
  // After the barrier every slot of this CTA's share holds the partial of
  // the rank it is named after; sum them in rank order (the result does not
  // depend on timing).  Each thread takes four consecutive tile rows of one
  // column (one 16-byte load per slot).  For decode the tile rows run along
  // the output's unit stride: lanes walk over row quads and each writes its
  // four outputs at once.  Otherwise lanes walk over columns, the output's
  // unit stride, and write one row at a time.
  __syncwarp();                   // reconverge the role warps (the cluster barrier is warp-aligned)
  tc_fence_before();
  cluster_sync();
  {
    const float alpha = __fmul_rn(__ldg(p.ga), __ldg(p.gb));
    const int share = C::share_rows(S), pitch = C::slot_pitch(S);
    const int first = rank * share;
    const int n_quads = min(share, C::BM - first) / 4;
    const int ncols = min(BN, p.rows_b - tb * BN);
    const int slot = C::slot_floats(S);
    const uint32_t red_s = smem_u32(red);
    for (int t = threadIdx.x; t < n_quads * ncols; t += C::THREADS) {
      int j, aq;
      if (i_fast) {
        j = t / n_quads;
        aq = t - j * n_quads;
      } else {
        aq = t / ncols;
        j = t - aq * ncols;
      }
      const int a0 = aq * 4;
      const uint32_t off = (uint32_t)(j * pitch + a0) * 4u;
      float4 v = ld_shared_f32x4(red_s + off);
#pragma unroll
      for (int s2 = 1; s2 < C::MAX_SPLITS; ++s2)
        if (s2 < S) {
          const float4 w = ld_shared_f32x4(red_s + off + (uint32_t)(s2 * slot) * 4u);
          v.x = v.x + w.x; v.y = v.y + w.y; v.z = v.z + w.z; v.w = v.w + w.w;
        }
      float o4[4] = {__fmul_rn(v.x, alpha), __fmul_rn(v.y, alpha), __fmul_rn(v.z, alpha), __fmul_rn(v.w, alpha)};
      const int gi0 = ta * C::BM + first + a0, gj = tb * BN + j;
      const int lim = p.rows_a - gi0;              // valid tile rows of the quad
      if (lim <= 0) continue;
      if constexpr (MODE == OUT_GATES) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int n = i_fast ? gi0 + q : gj;             // output column = weight row
          o4[q] = n < p.n_split ? gate_keep(o4[q]) : gate_write(o4[q]);
        }
      }
      const int64_t o = (int64_t)gi0 * p.out_si + (int64_t)gj * p.out_sj;
      if constexpr (MODE == OUT_BF16) {
        __nv_bfloat16 *y = static_cast<__nv_bfloat16 *>(p.out) + o;
        __nv_bfloat162 h0 = __floats2bfloat162_rn(o4[0], o4[1]), h1 = __floats2bfloat162_rn(o4[2], o4[3]);
        if (i_fast && lim >= 4 && (o & 3) == 0) {
          *reinterpret_cast<uint2 *>(y) =
              make_uint2(*reinterpret_cast<uint32_t *>(&h0), *reinterpret_cast<uint32_t *>(&h1));
        } else {
          const __nv_bfloat16 hv[4] = {h0.x, h0.y, h1.x, h1.y};
#pragma unroll
          for (int q = 0; q < 4; ++q)
            if (q < lim) y[(int64_t)q * p.out_si] = hv[q];
        }
      } else {
        float *y = static_cast<float *>(p.out) + o;
        if (i_fast && lim >= 4 && (o & 3) == 0) {
          *reinterpret_cast<float4 *>(y) = make_float4(o4[0], o4[1], o4[2], o4[3]);
        } else {
#pragma unroll
          for (int q = 0; q < 4; ++q)
            if (q < lim) y[(int64_t)q * p.out_si] = o4[q];
        }
      }
    }
  }
  __syncwarp();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, C::TMEM_COLS);
}

}  // namespace nvfp4
