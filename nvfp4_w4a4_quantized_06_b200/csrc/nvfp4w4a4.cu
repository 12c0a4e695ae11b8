// nvfp4w4a4.cu -- the C ABI of the NVFP4 W4A4 linear layer (declared in
// include/nvfp4w4a4.h): argument validation, TMA tensor-map encoding, shape
// dispatch and kernel launches.  No entry point allocates device memory; the
// only library state is a per-device error word and a few cached attributes.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <atomic>
#include <utility>
#include <cstring>
#include <mutex>

#include "nvfp4w4a4.h"
#include "ptx.cuh"
#include "quantize.cuh"
#include "gemm.cuh"
#include "gemm_pair.cuh"
#include "gemm_cluster.cuh"

using namespace nvfp4;

__device__ unsigned g_nvfp4_device_error;
__device__ unsigned g_nvfp4_error_snapshot;   // the word as nvfp4_last_device_status took it

// Fixed scratch of w4a4_gemm_noalloc (see the header): quantized activation
// and split-K partial sums for callers that cannot allocate.
constexpr size_t kNoAllocScratchBytes = size_t(8) << 20;
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

namespace {

constexpr int kMaxDevices = 64;
constexpr int kMaxSplitCluster = 8;
// CTA-pair GEMM raster: consecutive tiles sweep this many 256-row A tiles
// before moving to the next B tile column, so that the group's A rows stay
// in L2 while the B operand streams past them.
#ifndef NVFP4_PAIR_RASTER_GROUP
#define NVFP4_PAIR_RASTER_GROUP 8
#endif
constexpr int kPairRasterGroup = NVFP4_PAIR_RASTER_GROUP;

std::atomic<uint64_t> g_launches{0};
std::mutex g_mu;
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

struct DeviceState {
  bool ready = false;
  int sms = 0;
  unsigned *err = nullptr;
  int pair_clusters = 0;                // co-resident CTA pairs of the pair GEMM
  // co-resident clusters of the split-K cluster GEMM, [BN 32/64/128][size 1..8]
  int split_clusters[3][kMaxSplitCluster + 1] = {};
  // the same for its 128-wide variant with the activation encoded in the kernel
  int fused128_clusters[kMaxSplitCluster + 1] = {};
};
DeviceState g_dev[kMaxDevices];

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline int64_t pad128(int64_t r) { return (r + 127) / 128 * 128; }
inline size_t align256(size_t b) { return (b + 255) / 256 * 256; }

template <typename K>
cudaError_t set_smem(K kernel, int bytes) {
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
}

cudaError_t set_pair_attrs() {
  const int b = PairCfg::SMEM_BYTES;
  cudaError_t e = set_smem(nvfp4_gemm_pair_kernel<OUT_BF16>, b);
  if (e == cudaSuccess) e = set_smem(nvfp4_gemm_pair_kernel<OUT_F32>, b);
  return e;
}

template <int BN>
cudaError_t set_cluster_attrs() {
  const int b = ClusterCfg<BN>::SMEM_BYTES;
  cudaError_t e = set_smem(nvfp4_gemm_cluster_kernel<BN, OUT_BF16>, b);
  if (e == cudaSuccess) e = set_smem(nvfp4_gemm_cluster_kernel<BN, OUT_F32>, b);
  if (e == cudaSuccess) e = set_smem(nvfp4_gemm_cluster_kernel<BN, OUT_GATES>, b);
  const int bf = ClusterCfg<BN, true>::SMEM_BYTES;
  if (e == cudaSuccess) e = set_smem(nvfp4_gemm_cluster_kernel<BN, OUT_BF16, __nv_bfloat16>, bf);
  if (e == cudaSuccess) e = set_smem(nvfp4_gemm_cluster_kernel<BN, OUT_F32, __nv_bfloat16>, bf);
  if (e == cudaSuccess) e = set_smem(nvfp4_gemm_cluster_kernel<BN, OUT_BF16, float>, bf);
  if (e == cudaSuccess) e = set_smem(nvfp4_gemm_cluster_kernel<BN, OUT_F32, float>, bf);
  if (e == cudaSuccess) e = set_smem(nvfp4_gemm_cluster_kernel<BN, OUT_GATES, __nv_bfloat16>, bf);
  if (e == cudaSuccess) e = set_smem(nvfp4_gemm_cluster_kernel<BN, OUT_GATES, float>, bf);
  return e;
}

constexpr int kSmemOptin = 232448;   // 227 KB, the per-CTA opt-in limit of sm_100

template <typename T>
cudaError_t set_quant_attrs() {
  cudaError_t e = set_smem(quantize_tma_kernel<T>, QTmaCfg<T>::SMEM_BYTES);
  if (e == cudaSuccess) e = set_smem(rmsnorm_quantize_warp_kernel<T>, kSmemOptin);
  return e;
}

// How many clusters of `size` CTAs of the split-K GEMM fit on the device at once.
template <int BN, bool FUSED = false>
int max_split_clusters(int size, int sms) {
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = size;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.gridDim = dim3(size * sms);
  cfg.blockDim = dim3(ClusterCfg<BN, FUSED>::THREADS);
  cfg.dynamicSmemBytes = ClusterCfg<BN, FUSED>::SMEM_BYTES;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  cudaError_t e = FUSED ? cudaOccupancyMaxActiveClusters(&n, nvfp4_gemm_cluster_kernel<BN, OUT_BF16, __nv_bfloat16>, &cfg)
                        : cudaOccupancyMaxActiveClusters(&n, nvfp4_gemm_cluster_kernel<BN, OUT_BF16>, &cfg);
  if (e != cudaSuccess) n = 0;
  cudaGetLastError();
  return n;
}

template <int BN>
cudaError_t set_gemm_attrs() {
  const int b = GemmCfg<BN>::SMEM_BYTES;
  cudaError_t e = set_smem(nvfp4_gemm_kernel<BN, OUT_BF16>, b);
  if (e == cudaSuccess) e = set_smem(nvfp4_gemm_kernel<BN, OUT_F32>, b);
  if (e == cudaSuccess) e = set_smem(nvfp4_gemm_kernel<BN, OUT_PARTIAL>, b);
  return e;
}

// Per-device one-time setup with the device current: SM count, the address of
// the error word, the kernels' shared-memory limits, the tensor-map encoder.
nvfp4_status device_state(DeviceState **out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return NVFP4_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  DeviceState &d = g_dev[dev];
  if (!d.ready) {
    if (!g_encode) {
      void *fn = nullptr;
      cudaDriverEntryPointQueryResult q;
      if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
          q != cudaDriverEntryPointSuccess || !fn)
        return NVFP4_ERR_CUDA;
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    }
    int sms = 0, major = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return NVFP4_ERR_CUDA;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return NVFP4_ERR_CUDA;
    if (major != 10) return NVFP4_ERR_UNSUPPORTED;
    void *errp = nullptr;
    if (cudaGetSymbolAddress(&errp, g_nvfp4_device_error) != cudaSuccess) return NVFP4_ERR_CUDA;
    if (set_gemm_attrs<256>() != cudaSuccess || set_gemm_attrs<128>() != cudaSuccess ||
        set_gemm_attrs<64>() != cudaSuccess || set_gemm_attrs<32>() != cudaSuccess ||
        set_pair_attrs() != cudaSuccess || set_cluster_attrs<32>() != cudaSuccess ||
        set_cluster_attrs<64>() != cudaSuccess || set_cluster_attrs<128>() != cudaSuccess ||
        set_quant_attrs<__nv_bfloat16>() != cudaSuccess || set_quant_attrs<float>() != cudaSuccess)
      return NVFP4_ERR_CUDA;
    static_assert(ClusterCfg<32>::MAX_SPLITS == kMaxSplitCluster && ClusterCfg<64>::MAX_SPLITS == kMaxSplitCluster &&
                      ClusterCfg<128>::MAX_SPLITS == 5,
                  "planner limits follow the reduction slots");
    for (int c = 1; c <= kMaxSplitCluster; ++c) {
      d.split_clusters[0][c] = max_split_clusters<32>(c, sms);
      d.split_clusters[1][c] = max_split_clusters<64>(c, sms);
      d.split_clusters[2][c] = max_split_clusters<128>(c, sms);
      d.fused128_clusters[c] = max_split_clusters<128, true>(c, sms);
    }
    {
      cudaLaunchConfig_t cfg = {};
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = 2;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.gridDim = dim3(2 * sms);
      cfg.blockDim = dim3(PairCfg::THREADS);
      cfg.dynamicSmemBytes = PairCfg::SMEM_BYTES;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      if (cudaOccupancyMaxActiveClusters(&d.pair_clusters, nvfp4_gemm_pair_kernel<OUT_BF16>, &cfg) != cudaSuccess)
        d.pair_clusters = 0;
      cudaGetLastError();
    }
    d.sms = sms;
    d.err = static_cast<unsigned *>(errp);
    d.ready = true;
  }
  *out = &d;
  return NVFP4_OK;
}

nvfp4_status launched() {
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return cudaGetLastError() == cudaSuccess ? NVFP4_OK : NVFP4_ERR_CUDA;
}

bool make_codes_map(CUtensorMap *map, const void *base, int64_t rows, int64_t K, int box_rows) {
  cuuint64_t dims[2] = {(cuuint64_t)(K / 2), (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)(K / 2)};
  cuuint32_t box[2] = {128u, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1u, 1u};
  CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(base), dims, strides, box,
                        estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// The swizzled scale buffer viewed as uint64 [pad128(rows)/128][K]: one
// "row" per 128-row block holds its K/64 atoms of 512 bytes; a box of 256
// elements is the 2 KB (four atoms) of one 256-deep K stage.  Boxes past the
// last row block or past K read zeros.
bool make_sf_map(CUtensorMap *map, const void *sf, int64_t rows, int64_t K, int box_rows) {
  cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)(pad128(rows) / 128)};
  cuuint64_t strides[1] = {(cuuint64_t)(K * 8)};
  cuuint32_t box[2] = {256u, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1u, 1u};
  CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT64, 2, const_cast<void *>(sf), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Y as bf16 [M][N] (row stride ld_y) for the CTA-pair GEMM's TMA stores: a
// box of 32 columns (64 bytes) x 32 rows with the 64-byte swizzle the
// epilogue writes its staging boxes in.  Needs a 16-byte-aligned y and a row
// stride that is a multiple of 8 elements (16 bytes).
bool make_y_map(CUtensorMap *map, void *y, int64_t M, int64_t N, int64_t ld_y) {
  cuuint64_t dims[2] = {(cuuint64_t)N, (cuuint64_t)M};
  cuuint64_t strides[1] = {(cuuint64_t)(ld_y * 2)};
  cuuint32_t box[2] = {32u, 32u};
  cuuint32_t estr[2] = {1u, 1u};
  CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, y, dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// GEMM plan: which kernel, which operand drives the 128-row MMA dimension,
// the tile width, split-K and the grid.
struct Plan {
  enum Kind { SINGLE, PAIR, CLUSTER } kind;
  bool swap;       // A operand = weight (rows N), B operand = activation (rows M)
  int bn;
  int tiles_a, tiles_b, splits, kstages;
  int grid;
};

inline int narrow_bn(int64_t rows) { return rows <= 32 ? 32 : (rows <= 64 ? 64 : 128); }
// largest split-K cluster a configuration's reduction slots hold (ClusterCfg::MAX_SPLITS)
inline int max_splits_for_bn(int bn) { return bn >= 128 ? 5 : kMaxSplitCluster; }
inline int bn_index(int bn) { return bn == 32 ? 0 : (bn == 64 ? 1 : 2); }

Plan make_plan(int64_t M, int64_t N, int64_t K, const DeviceState &d) {
  Plan pl{};
  pl.kstages = (int)((K / 64 + 3) / 4);
  const int sms = d.sms > 0 ? d.sms : 148;
  if (M > 128 && N > 128 && d.pair_clusters > 0 &&
      ((M + 255) / 256) * ((N + 255) / 256) >= d.pair_clusters) {
    // large products: CTA pairs on 256 x 256 tiles, one wave of resident pairs
    pl.kind = Plan::PAIR;
    pl.bn = 256;
    pl.tiles_a = (int)((M + 255) / 256);
    pl.tiles_b = (int)((N + 255) / 256);
    pl.splits = 1;
    const int units = pl.tiles_a * pl.tiles_b;
    pl.grid = 2 * (units < d.pair_clusters ? units : d.pair_clusters);
    return pl;
  }
  if (M <= 128 || N <= 128) {
    // one narrow operand: it becomes the MMA's N (decode: the activation;
    // small-N projections: the weight), the other streams through the
    // 128-row side, and K is split over the CTAs of a cluster.  The cluster
    // size minimises waves x (stages per CTA + 1), the +1 standing for the
    // per-CTA fill and reduction.
    pl.swap = M <= 128 && (M <= N || N > 128);
    pl.bn = narrow_bn(pl.swap ? M : N);
    pl.tiles_a = (int)(((pl.swap ? N : M) + 127) / 128);
    pl.tiles_b = 1;
    int best = 0;
    int64_t best_cost = 0;
    for (int c = 1; c <= max_splits_for_bn(pl.bn) && c <= pl.kstages; ++c) {
      const int fit = d.split_clusters[bn_index(pl.bn)][c];
      if (fit <= 0) continue;
      const int64_t waves = (pl.tiles_a + fit - 1) / fit;
      const int64_t cost = waves * ((pl.kstages + c - 1) / c + 1);
      if (best == 0 || cost < best_cost) { best = c; best_cost = cost; }
    }
    if (best > 0) {
      pl.kind = Plan::CLUSTER;
      pl.splits = best;
      pl.grid = pl.tiles_a * best;
      return pl;
    }
  }
  pl.kind = Plan::SINGLE;
  if (M <= 64) {
    // decode-shaped without cluster support: split-K with a separate reduction
    pl.swap = true;
    pl.bn = M <= 32 ? 32 : 64;
    pl.tiles_a = (int)((N + 127) / 128);
    pl.tiles_b = 1;
    int s = (2 * sms) / pl.tiles_a;
    pl.splits = s < 1 ? 1 : (s > pl.kstages ? pl.kstages : s);
  } else {
    pl.swap = false;
    pl.bn = N <= 128 ? 128 : 256;
    pl.tiles_a = (int)((M + 127) / 128);
    pl.tiles_b = (int)((N + pl.bn - 1) / pl.bn);
    const int units = pl.tiles_a * pl.tiles_b;
    int s = units < sms ? sms / units : 1;
    if (s > pl.kstages / 2) s = pl.kstages / 2;
    pl.splits = s < 1 ? 1 : s;
  }
  const int units = pl.tiles_a * pl.tiles_b * pl.splits;
  const int per_sm = pl.bn <= 64 ? 2 : 1;
  pl.grid = units < per_sm * sms ? units : per_sm * sms;
  return pl;
}

size_t gemm_partial_bytes(int64_t M, int64_t N, int64_t K, const DeviceState &d) {
  const Plan pl = make_plan(M, N, K, d);
  return pl.kind == Plan::SINGLE && pl.splits > 1 ? (size_t)pl.splits * (size_t)M * (size_t)N * sizeof(float) : 0;
}

size_t current_partial_bytes(int64_t M, int64_t N, int64_t K) {
  DeviceState *d = nullptr;
  if (device_state(&d) != NVFP4_OK) {
    const DeviceState none{};      // no device: the conservative single-CTA plan
    return gemm_partial_bytes(M, N, K, none);
  }
  return gemm_partial_bytes(M, N, K, *d);
}

// cudaLaunchKernelEx with an optional cluster shape and programmatic
// stream serialization (the kernel may start while the preceding one in the
// stream finishes; it waits for it with griddepcontrol.wait).
template <typename... KArgs, typename... Args>
cudaError_t launch_ex(void (*kernel)(KArgs...), unsigned grid, unsigned block, size_t smem, cudaStream_t s,
                      int cluster, bool pdl, Args &&...args) {
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  int n = 0;
  if (cluster > 0) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = (unsigned)cluster;
    attr[n].val.clusterDim.y = 1;
    attr[n].val.clusterDim.z = 1;
    ++n;
  }
  if (pdl) {
    attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
  }
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(block);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = (unsigned)n;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

template <int BN>
nvfp4_status launch_gemm_bn(const CUtensorMap &ma, const CUtensorMap &mb, const GemmParams &p, int mode,
                            int grid, cudaStream_t s) {
  using C = GemmCfg<BN>;
  if (mode == OUT_BF16)
    nvfp4_gemm_kernel<BN, OUT_BF16><<<grid, C::THREADS, C::SMEM_BYTES, s>>>(ma, mb, p);
  else if (mode == OUT_F32)
    nvfp4_gemm_kernel<BN, OUT_F32><<<grid, C::THREADS, C::SMEM_BYTES, s>>>(ma, mb, p);
  else
    nvfp4_gemm_kernel<BN, OUT_PARTIAL><<<grid, C::THREADS, C::SMEM_BYTES, s>>>(ma, mb, p);
  return launched();
}

template <int BN>
cudaError_t launch_cluster(int mode, unsigned grid, int splits, bool pdl, const CUtensorMap &ma,
                           const CUtensorMap &mb, const GemmParams &p, cudaStream_t stream) {
  using C = ClusterCfg<BN>;
  if (mode == OUT_BF16)
    return launch_ex(nvfp4_gemm_cluster_kernel<BN, OUT_BF16>, grid, C::THREADS, C::SMEM_BYTES, stream, splits, pdl,
                     ma, mb, p);
  if (mode == OUT_GATES)
    return launch_ex(nvfp4_gemm_cluster_kernel<BN, OUT_GATES>, grid, C::THREADS, C::SMEM_BYTES, stream, splits, pdl,
                     ma, mb, p);
  return launch_ex(nvfp4_gemm_cluster_kernel<BN, OUT_F32>, grid, C::THREADS, C::SMEM_BYTES, stream, splits, pdl,
                   ma, mb, p);
}

template <int BN, typename XT>
cudaError_t launch_cluster_fused(int mode, unsigned grid, int splits, const CUtensorMap &ma, const GemmParams &p,
                                 cudaStream_t stream) {
  using C = ClusterCfg<BN, true>;
  if (mode == OUT_BF16)
    return launch_ex(nvfp4_gemm_cluster_kernel<BN, OUT_BF16, XT>, grid, C::THREADS, C::SMEM_BYTES, stream, splits,
                     true, ma, ma, p);
  if (mode == OUT_GATES)
    return launch_ex(nvfp4_gemm_cluster_kernel<BN, OUT_GATES, XT>, grid, C::THREADS, C::SMEM_BYTES, stream, splits,
                     true, ma, ma, p);
  return launch_ex(nvfp4_gemm_cluster_kernel<BN, OUT_F32, XT>, grid, C::THREADS, C::SMEM_BYTES, stream, splits, true,
                   ma, ma, p);
}

// Plan of the one-kernel layer (activation encoded inside the split-K
// cluster GEMM, on the MMA's N side): decode-shaped products (M <= 128
// activation rows, one narrow tile) take the two-kernel layer's plan; products
// with a narrow weight (N <= 128, the gate projections) put the weight on the
// 128-row side and the activation on the N side in tiles of 128 rows, and
// split K over the largest cluster that keeps all tiles in one wave.
// kind SINGLE means there is no such plan.
Plan fused_plan(int64_t M, int64_t N, int64_t K, const DeviceState &d) {
  if (M <= 128) {
    Plan pl = make_plan(M, N, K, d);
    if (pl.kind != Plan::CLUSTER || !pl.swap) pl.kind = Plan::SINGLE;
    return pl;
  }
  Plan pl{};
  pl.kind = Plan::SINGLE;
  if (N > 128) return pl;
  pl.kstages = (int)((K / 64 + 3) / 4);
  pl.swap = true;
  pl.bn = 128;
  pl.tiles_a = 1;
  pl.tiles_b = (int)((M + 127) / 128);
  int best = 0;
  int64_t best_cost = 0;
  for (int c = 1; c <= max_splits_for_bn(128) && c <= pl.kstages; ++c) {
    const int fit = d.fused128_clusters[c];
    if (fit <= 0) continue;
    const int64_t waves = (pl.tiles_b + fit - 1) / fit;
    const int64_t cost = waves * ((pl.kstages + c - 1) / c + 1);
    if (best == 0 || cost < best_cost) { best = c; best_cost = cost; }
  }
  if (best == 0) return pl;
  pl.kind = Plan::CLUSTER;
  pl.splits = best;
  pl.grid = pl.tiles_b * best;
  return pl;
}

// The layer in one kernel: the activation x is quantized inside the cluster
// GEMM (row a9), for decode-shaped products and for narrow weights (the gate
// projections, optionally with their activations in the epilogue:
// gates_n_a >= 0).  Returns UNSUPPORTED when there is no such plan.
nvfp4_status w4a4_fused_impl(const void *x, nvfp4_in_dtype x_dt, int64_t ld_x, const float *x_gscale,
                             const uint8_t *w_codes, const uint8_t *w_sf, const float *w_gscale, void *y,
                             nvfp4_out_dtype y_dt, int64_t ld_y, int64_t M, int64_t N, int64_t K,
                             const DeviceState &dev, cudaStream_t stream, int64_t gates_n_a = -1) {
  const Plan pl = fused_plan(M, N, K, dev);
  if (pl.kind != Plan::CLUSTER) return NVFP4_ERR_UNSUPPORTED;
  GemmParams p{};
  p.sfa = w_sf;
  p.ga = x_gscale;
  p.gb = w_gscale;
  p.rows_a = (int)N;
  p.rows_b = (int)M;
  p.K = (int)K;
  p.kblocks = (int)(K / 64);
  p.kstages = pl.kstages;
  p.tiles_a = pl.tiles_a;
  p.tiles_b = pl.tiles_b;
  p.splits = pl.splits;
  p.group = 1;
  p.err = dev.err;
  p.out = y;
  p.out_si = 1;
  p.out_sj = ld_y;
  p.x = x;
  p.ld_x = ld_x;
  p.x_gscale = x_gscale;
  p.n_split = (int)(gates_n_a >= 0 ? gates_n_a : 0);
  CUtensorMap ma;
  if (!make_codes_map(&ma, w_codes, N, K, 128)) return NVFP4_ERR_CUDA;
  const int mode = gates_n_a >= 0 ? OUT_GATES : (y_dt == NVFP4_OUT_BF16 ? OUT_BF16 : OUT_F32);
  const bool xb = x_dt == NVFP4_IN_BF16;
  const unsigned g = (unsigned)pl.grid;
  cudaError_t e;
  switch (pl.bn) {
    case 32:
      e = xb ? launch_cluster_fused<32, __nv_bfloat16>(mode, g, pl.splits, ma, p, stream)
             : launch_cluster_fused<32, float>(mode, g, pl.splits, ma, p, stream);
      break;
    case 64:
      e = xb ? launch_cluster_fused<64, __nv_bfloat16>(mode, g, pl.splits, ma, p, stream)
             : launch_cluster_fused<64, float>(mode, g, pl.splits, ma, p, stream);
      break;
    default:
      e = xb ? launch_cluster_fused<128, __nv_bfloat16>(mode, g, pl.splits, ma, p, stream)
             : launch_cluster_fused<128, float>(mode, g, pl.splits, ma, p, stream);
      break;
  }
  if (e != cudaSuccess) return NVFP4_ERR_CUDA;
  return launched();
}

// `pdl`: launched right after this library's activation quantize, which
// lets the GEMM start early and stream the weight while the quantize ends.
nvfp4_status gemm_impl(const uint8_t *a_codes, const uint8_t *a_sf, const float *a_gscale,
                       const uint8_t *b_codes, const uint8_t *b_sf, const float *b_gscale, void *y,
                       nvfp4_out_dtype y_dt, int64_t ld_y, int64_t M, int64_t N, int64_t K, void *ws,
                       size_t ws_bytes, cudaStream_t stream, bool pdl, int64_t gates_n_a = -1) {
  DeviceState *dev = nullptr;
  nvfp4_status st = device_state(&dev);
  if (st != NVFP4_OK) return st;
  if (M == 0 || N == 0) return NVFP4_OK;
  const Plan pl = make_plan(M, N, K, *dev);
  if (gates_n_a >= 0 && pl.kind != Plan::CLUSTER) return NVFP4_ERR_UNSUPPORTED;
  const size_t need = gemm_partial_bytes(M, N, K, *dev);
  if (need > 0 && (ws == nullptr || ws_bytes < need)) return NVFP4_ERR_WORKSPACE;
  if (need > 0 && !aligned16(ws)) return NVFP4_ERR_ALIGN;

  if (pl.kind == Plan::PAIR) {
    GemmParams p{};
    p.ga = a_gscale;
    p.gb = b_gscale;
    p.rows_a = (int)M;
    p.rows_b = (int)N;
    p.K = (int)K;
    p.kblocks = (int)(K / 64);
    p.kstages = pl.kstages;
    p.tiles_a = pl.tiles_a;
    p.tiles_b = pl.tiles_b;
    p.splits = 1;
    p.group = kPairRasterGroup;
    p.err = dev->err;
    p.out = y;
    p.out_si = ld_y;
    p.out_sj = 1;
    CUtensorMap ma, mb, msa, msb, my;
    if (!make_codes_map(&ma, a_codes, M, K, 128) || !make_codes_map(&mb, b_codes, N, K, 128) ||
        !make_sf_map(&msa, a_sf, M, K, 1) || !make_sf_map(&msb, b_sf, N, K, 2))
      return NVFP4_ERR_CUDA;
    // BF16 output goes out through TMA stores when Y's layout allows it (the
    // register-store epilogue serves the rest, and FP32 output)
    p.tma_store = y_dt == NVFP4_OUT_BF16 && aligned16(y) && ld_y % 8 == 0 ? 1 : 0;
    if (p.tma_store) {
      if (!make_y_map(&my, y, M, N, ld_y)) return NVFP4_ERR_CUDA;
    } else {
      my = ma;                       // unused
    }
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3(pl.grid);
    cfg.blockDim = dim3(PairCfg::THREADS);
    cfg.dynamicSmemBytes = PairCfg::SMEM_BYTES;
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = y_dt == NVFP4_OUT_BF16
                        ? cudaLaunchKernelEx(&cfg, nvfp4_gemm_pair_kernel<OUT_BF16>, ma, mb, msa, msb, my, p)
                        : cudaLaunchKernelEx(&cfg, nvfp4_gemm_pair_kernel<OUT_F32>, ma, mb, msa, msb, my, p);
    if (e != cudaSuccess) return NVFP4_ERR_CUDA;
    return launched();
  }

  if (pl.kind == Plan::CLUSTER) {
    GemmParams p{};
    const uint8_t *op_a = pl.swap ? b_codes : a_codes;   // A = 128-row MMA operand
    const uint8_t *op_b = pl.swap ? a_codes : b_codes;
    p.sfa = pl.swap ? b_sf : a_sf;
    p.sfb = pl.swap ? a_sf : b_sf;
    p.ga = a_gscale;
    p.gb = b_gscale;
    p.rows_a = (int)(pl.swap ? N : M);
    p.rows_b = (int)(pl.swap ? M : N);
    p.K = (int)K;
    p.kblocks = (int)(K / 64);
    p.kstages = pl.kstages;
    p.tiles_a = pl.tiles_a;
    p.tiles_b = pl.tiles_b;
    p.splits = pl.splits;
    p.group = pl.swap ? 1 : 0;       // which operand is the weight (loaded before the wait)
    p.err = dev->err;
    p.out = y;
    p.out_si = pl.swap ? 1 : ld_y;
    p.out_sj = pl.swap ? ld_y : 1;
    CUtensorMap ma, mb;
    if (!make_codes_map(&ma, op_a, p.rows_a, K, 128) || !make_codes_map(&mb, op_b, p.rows_b, K, pl.bn))
      return NVFP4_ERR_CUDA;
    p.n_split = (int)(gates_n_a >= 0 ? gates_n_a : 0);
    const int mode = gates_n_a >= 0 ? OUT_GATES : (y_dt == NVFP4_OUT_BF16 ? OUT_BF16 : OUT_F32);
    const unsigned g = (unsigned)pl.grid;
    cudaError_t e;
    switch (pl.bn) {
      case 32: e = launch_cluster<32>(mode, g, pl.splits, pdl, ma, mb, p, stream); break;
      case 64: e = launch_cluster<64>(mode, g, pl.splits, pdl, ma, mb, p, stream); break;
      default: e = launch_cluster<128>(mode, g, pl.splits, pdl, ma, mb, p, stream); break;
    }
    if (e != cudaSuccess) return NVFP4_ERR_CUDA;
    return launched();
  }

  GemmParams p{};
  const uint8_t *op_a = pl.swap ? b_codes : a_codes;   // A = 128-row MMA operand
  const uint8_t *op_b = pl.swap ? a_codes : b_codes;
  p.sfa = pl.swap ? b_sf : a_sf;
  p.sfb = pl.swap ? a_sf : b_sf;
  p.ga = a_gscale;
  p.gb = b_gscale;
  p.rows_a = (int)(pl.swap ? N : M);
  p.rows_b = (int)(pl.swap ? M : N);
  p.K = (int)K;
  p.kblocks = (int)(K / 64);
  p.kstages = pl.kstages;
  p.tiles_a = pl.tiles_a;
  p.tiles_b = pl.tiles_b;
  p.splits = pl.splits;
  p.group = 16;
  p.err = dev->err;
  int mode;
  if (pl.splits > 1) {
    mode = OUT_PARTIAL;
    p.out = ws;
    p.part_stride = M * N;
    p.out_si = pl.swap ? 1 : N;      // partials in output coordinates [m][n]
    p.out_sj = pl.swap ? N : 1;
  } else {
    mode = y_dt == NVFP4_OUT_BF16 ? OUT_BF16 : OUT_F32;
    p.out = y;
    p.out_si = pl.swap ? 1 : ld_y;
    p.out_sj = pl.swap ? ld_y : 1;
  }
  CUtensorMap ma, mb;
  if (!make_codes_map(&ma, op_a, p.rows_a, K, 128) || !make_codes_map(&mb, op_b, p.rows_b, K, pl.bn))
    return NVFP4_ERR_CUDA;
  switch (pl.bn) {
    case 256: st = launch_gemm_bn<256>(ma, mb, p, mode, pl.grid, stream); break;
    case 128: st = launch_gemm_bn<128>(ma, mb, p, mode, pl.grid, stream); break;
    case 64: st = launch_gemm_bn<64>(ma, mb, p, mode, pl.grid, stream); break;
    default: st = launch_gemm_bn<32>(ma, mb, p, mode, pl.grid, stream); break;
  }
  if (st != NVFP4_OK || pl.splits == 1) return st;
  const int64_t MN = M * N;
  int grid = (int)((MN + 255) / 256);
  if (grid > 8 * dev->sms) grid = 8 * dev->sms;
  if (y_dt == NVFP4_OUT_BF16)
    splitk_reduce_kernel<OUT_BF16><<<grid, 256, 0, stream>>>(static_cast<const float *>(ws), pl.splits, MN,
                                                             (int)N, a_gscale, b_gscale, y, ld_y);
  else
    splitk_reduce_kernel<OUT_F32><<<grid, 256, 0, stream>>>(static_cast<const float *>(ws), pl.splits, MN,
                                                            (int)N, a_gscale, b_gscale, y, ld_y);
  return launched();
}

nvfp4_status check_gemm_args(const uint8_t *a_codes, const uint8_t *a_sf, const float *a_gscale,
                             const uint8_t *b_codes, const uint8_t *b_sf, const float *b_gscale,
                             const void *y, int y_dt, int64_t ld_y, int64_t M, int64_t N, int64_t K) {
  if (M < 0 || N < 0 || K <= 0 || K % 64 != 0 || M > INT32_MAX / 2 || N > INT32_MAX / 2 || K > (1 << 30))
    return NVFP4_ERR_SHAPE;
  if (y_dt != NVFP4_OUT_BF16 && y_dt != NVFP4_OUT_F32) return NVFP4_ERR_DTYPE;
  if (M == 0 || N == 0) return NVFP4_OK;
  if (!a_codes || !a_sf || !a_gscale || !b_codes || !b_sf || !b_gscale || !y) return NVFP4_ERR_NULL;
  if (ld_y < N) return NVFP4_ERR_SHAPE;
  if (!aligned16(a_codes) || !aligned16(b_codes) || !aligned16(a_sf) || !aligned16(b_sf) || !aligned16(y))
    return NVFP4_ERR_ALIGN;
  return NVFP4_OK;
}

// X viewed as T [rows][K] (row stride ld_x) for the streaming quantize: a
// box of COLS columns x 128 rows, no swizzle, zeros outside the tensor.
template <typename T>
bool make_x_map(CUtensorMap *map, const void *x, int64_t rows, int64_t K, int64_t ld_x) {
  cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)(ld_x * (int64_t)sizeof(T))};
  cuuint32_t box[2] = {(cuuint32_t)QTmaCfg<T>::COLS, 128u};
  cuuint32_t estr[2] = {1u, 1u};
  CUresult r = g_encode(map, sizeof(T) == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2,
                        const_cast<void *>(x), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <typename T>
nvfp4_status launch_quantize(const QuantizeParams &p, const DeviceState &dev, cudaStream_t s, bool pdl) {
  const bool tile_ok = (p.sf_row0 % 128) == 0 && ((p.rows % 128) == 0 || p.pad_rows > 0);
  if (tile_ok && p.rows >= 256) {
    // streaming kernel: one CTA per SM over 128-row units
    CUtensorMap mx;
    if (!make_x_map<T>(&mx, p.x, p.rows, p.K, p.ld_x)) return NVFP4_ERR_CUDA;
    using C = QTmaCfg<T>;
    const int64_t units = ((p.rows + 127) / 128) * ((p.K + C::COLS - 1) / C::COLS);
    const unsigned grid = (unsigned)(units < dev.sms ? units : dev.sms);
    if (launch_ex(quantize_tma_kernel<T>, grid, C::THREADS, C::SMEM_BYTES, s, 0, pdl, mx, p) != cudaSuccess)
      return NVFP4_ERR_CUDA;
    return launched();
  }
  // generic kernel: one warp per 512-column row segment; few rows (decode)
  // get one segment per warp so that the kernel is as short as possible
  const int64_t units = p.rows * ((p.K + 511) / 512);
  cudaError_t e;
  if (units >= 32LL * dev.sms) {
    int64_t blocks = (units / 4 + 7) / 8;
    if (blocks > 8LL * dev.sms) blocks = 8LL * dev.sms;
    e = launch_ex(quantize_rows_kernel<T, 4>, (unsigned)blocks, 256u, 0, s, 0, pdl, p);
  } else {
    int64_t blocks = (units + 7) / 8;
    if (blocks < 1) blocks = 1;
    e = launch_ex(quantize_rows_kernel<T, 1>, (unsigned)blocks, 256u, 0, s, 0, pdl, p);
  }
  if (e != cudaSuccess) return NVFP4_ERR_CUDA;
  return launched();
}

nvfp4_status quantize_impl(const void *x, nvfp4_in_dtype dt, int64_t rows, int64_t K, int64_t ld_x,
                           const float *gscale, uint8_t *codes, uint8_t *sf, int64_t sf_row0, int64_t sf_rows_total,
                           cudaStream_t s, bool pdl) {
  if (dt != NVFP4_IN_BF16 && dt != NVFP4_IN_F32) return NVFP4_ERR_DTYPE;
  if (rows < 0 || K <= 0 || K % 64 != 0 || ld_x < K || sf_row0 < 0 || sf_rows_total < sf_row0 + rows ||
      rows * ((K + 255) / 256) >= (int64_t)UINT32_MAX)
    return NVFP4_ERR_SHAPE;
  const bool owns_pad = sf_row0 + rows == sf_rows_total;
  const int64_t pad_rows = owns_pad ? pad128(sf_rows_total) - sf_rows_total : 0;
  if (rows == 0 && pad_rows == 0) return NVFP4_OK;
  if (!sf || !gscale || (rows > 0 && (!x || !codes))) return NVFP4_ERR_NULL;
  const int esz = dt == NVFP4_IN_BF16 ? 2 : 4;
  if ((rows > 0 && (!aligned16(x) || !aligned16(codes))) || (ld_x * esz) % 16 != 0 || !aligned16(sf))
    return NVFP4_ERR_ALIGN;
  DeviceState *dev = nullptr;
  nvfp4_status st = device_state(&dev);
  if (st != NVFP4_OK) return st;
  QuantizeParams p{x, rows, K, ld_x, gscale, codes, sf, sf_row0, pad_rows, dev->err};
  return dt == NVFP4_IN_BF16 ? launch_quantize<__nv_bfloat16>(p, *dev, s, pdl)
                             : launch_quantize<float>(p, *dev, s, pdl);
}

// mbar_wait with a caller-chosen limit (the self-test of the timeout path).
__device__ __forceinline__ bool mbar_wait_limit(uint64_t *bar, uint32_t parity, unsigned *err, unsigned code,
                                                unsigned long long limit_ns) {
  const uint32_t a = smem_u32(bar);
  const unsigned long long t0 = globaltimer();
  while (true) {
    if (mbar_try_wait(a, parity)) return true;
    if (globaltimer() - t0 > limit_ns) {
      atomicOr(err, code);
      return false;
    }
  }
}

// Failure-detection self-test: one thread waits on an mbarrier that nothing
// arrives on, so the bounded wait runs out, records ERR_SELFTEST in the
// error word and the kernel returns normally (no fault, no trap).
__global__ void wait_timeout_selftest_kernel(unsigned *err, unsigned long long limit_ns, int *result) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_barrier_init();
    const bool ok = mbar_wait_limit(&bar, 0, err, ERR_SELFTEST, limit_ns);
    *result = ok ? 1 : 0;
  }
}

// Reads and clears the error word in one atomic exchange.
__global__ void error_take_kernel(unsigned *err) { g_nvfp4_error_snapshot = atomicExch(err, 0u); }

}  // namespace

extern "C" {

size_t nvfp4_codes_bytes(int64_t rows, int64_t K) {
  if (rows < 0 || K <= 0) return 0;
  return (size_t)rows * (size_t)(K / 2);
}

size_t nvfp4_sf_bytes(int64_t rows, int64_t K) {
  if (rows < 0 || K <= 0) return 0;
  return (size_t)pad128(rows) * (size_t)((K / 16 + 3) / 4 * 4);
}

nvfp4_status nvfp4_amax_gscale(const void *x, nvfp4_in_dtype dt, int64_t rows, int64_t K, int64_t ld_x,
                               float *gscale_out, nvfp4_stream_t stream) {
  if (dt != NVFP4_IN_BF16 && dt != NVFP4_IN_F32) return NVFP4_ERR_DTYPE;
  if (rows < 0 || K <= 0 || K % 64 != 0 || ld_x < K) return NVFP4_ERR_SHAPE;
  if (!gscale_out || (rows > 0 && !x)) return NVFP4_ERR_NULL;
  const int esz = dt == NVFP4_IN_BF16 ? 2 : 4;
  if ((rows > 0 && !aligned16(x)) || (ld_x * esz) % 16 != 0 || (reinterpret_cast<uintptr_t>(gscale_out) & 3))
    return NVFP4_ERR_ALIGN;
  DeviceState *dev = nullptr;
  nvfp4_status st = device_state(&dev);
  if (st != NVFP4_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(gscale_out, 0, sizeof(float), s) != cudaSuccess) return NVFP4_ERR_CUDA;
  if (rows > 0) {
    int64_t n = rows * (K / 8);
    int64_t blocks = (n + 255) / 256;
    if (blocks > 8LL * dev->sms) blocks = 8LL * dev->sms;
    unsigned *acc = reinterpret_cast<unsigned *>(gscale_out);
    if (dt == NVFP4_IN_BF16)
      amax_kernel<__nv_bfloat16><<<(unsigned)blocks, 256, 0, s>>>(static_cast<const __nv_bfloat16 *>(x), rows, K,
                                                                  ld_x, acc);
    else
      amax_kernel<float><<<(unsigned)blocks, 256, 0, s>>>(static_cast<const float *>(x), rows, K, ld_x, acc);
    if ((st = launched()) != NVFP4_OK) return st;
  }
  gscale_finalize_kernel<<<1, 1, 0, s>>>(reinterpret_cast<unsigned *>(gscale_out));
  return launched();
}

nvfp4_status nvfp4_quantize(const void *x, nvfp4_in_dtype dt, int64_t rows, int64_t K, int64_t ld_x,
                            const float *gscale, uint8_t *codes, uint8_t *sf, int64_t sf_row0,
                            int64_t sf_rows_total, nvfp4_stream_t stream) {
  return quantize_impl(x, dt, rows, K, ld_x, gscale, codes, sf, sf_row0, sf_rows_total,
                       reinterpret_cast<cudaStream_t>(stream), false);
}

nvfp4_status nvfp4_harmonize_group(uint8_t *sf, int64_t rows_total, int64_t K, int n_modules,
                                   const int64_t *row_offsets, const float *gscales, float *shared_gscale_out,
                                   nvfp4_stream_t stream) {
  if (!sf || !row_offsets || !gscales || !shared_gscale_out) return NVFP4_ERR_NULL;
  if (n_modules < 1 || n_modules > kMaxModules || rows_total <= 0 || K <= 0 || K % 64 != 0)
    return NVFP4_ERR_SHAPE;
  if (row_offsets[0] != 0 || row_offsets[n_modules] != rows_total) return NVFP4_ERR_SHAPE;
  for (int m = 0; m < n_modules; ++m)
    if (row_offsets[m + 1] <= row_offsets[m]) return NVFP4_ERR_SHAPE;
  if (!aligned16(sf)) return NVFP4_ERR_ALIGN;
  DeviceState *dev = nullptr;
  nvfp4_status st = device_state(&dev);
  if (st != NVFP4_OK) return st;
  HarmonizeParams p{};
  p.sf = sf;
  p.rows_total = rows_total;
  p.K = K;
  p.n = n_modules;
  for (int m = 0; m <= n_modules; ++m) p.offs[m] = row_offsets[m];
  p.gs = gscales;
  p.gstar_out = shared_gscale_out;
  const int64_t total = rows_total * (K / 64);
  int64_t blocks = (total + 255) / 256;
  if (blocks > 8LL * dev->sms) blocks = 8LL * dev->sms;
  if (blocks < 1) blocks = 1;
  harmonize_kernel<<<(unsigned)blocks, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(p);
  return launched();
}

size_t nvfp4_gemm_workspace_bytes(int64_t M, int64_t N, int64_t K) {
  if (M <= 0 || N <= 0 || K <= 0 || K % 64 != 0) return 0;
  return current_partial_bytes(M, N, K);
}

nvfp4_status nvfp4_gemm(const uint8_t *a_codes, const uint8_t *a_sf, const float *a_gscale,
                        const uint8_t *b_codes, const uint8_t *b_sf, const float *b_gscale, void *y,
                        nvfp4_out_dtype y_dt, int64_t ld_y, int64_t M, int64_t N, int64_t K, void *workspace,
                        size_t workspace_bytes, nvfp4_stream_t stream) {
  nvfp4_status st = check_gemm_args(a_codes, a_sf, a_gscale, b_codes, b_sf, b_gscale, y, y_dt, ld_y, M, N, K);
  if (st != NVFP4_OK || M == 0 || N == 0) return st;
  return gemm_impl(a_codes, a_sf, a_gscale, b_codes, b_sf, b_gscale, y, y_dt, ld_y, M, N, K, workspace,
                   workspace_bytes, reinterpret_cast<cudaStream_t>(stream), false);
}

size_t w4a4_gemm_workspace_bytes(int64_t M, int64_t N, int64_t K) {
  if (M <= 0 || N <= 0 || K <= 0 || K % 64 != 0) return 0;
  return align256(nvfp4_codes_bytes(M, K)) + align256(nvfp4_sf_bytes(M, K)) +
         current_partial_bytes(M, N, K);
}

nvfp4_status w4a4_gemm(const void *x, nvfp4_in_dtype x_dt, int64_t ld_x, const float *x_gscale,
                       const uint8_t *w_codes, const uint8_t *w_sf, const float *w_gscale, void *y,
                       nvfp4_out_dtype y_dt, int64_t ld_y, int64_t M, int64_t N, int64_t K, void *workspace,
                       size_t workspace_bytes, nvfp4_stream_t stream) {
  if (x_dt != NVFP4_IN_BF16 && x_dt != NVFP4_IN_F32) return NVFP4_ERR_DTYPE;
  if (M < 0 || N < 0 || K <= 0 || K % 64 != 0 || ld_x < K) return NVFP4_ERR_SHAPE;
  if (M == 0 || N == 0) return NVFP4_OK;
  if (!x || !x_gscale) return NVFP4_ERR_NULL;
  const int esz = x_dt == NVFP4_IN_BF16 ? 2 : 4;
  if (!aligned16(x) || (ld_x * esz) % 16 != 0) return NVFP4_ERR_ALIGN;
  if (!workspace) return NVFP4_ERR_WORKSPACE;
  if (!aligned16(workspace)) return NVFP4_ERR_ALIGN;
  const size_t codes_b = align256(nvfp4_codes_bytes(M, K));
  const size_t sf_b = align256(nvfp4_sf_bytes(M, K));
  if (workspace_bytes < codes_b + sf_b) return NVFP4_ERR_WORKSPACE;
  uint8_t *a_codes = static_cast<uint8_t *>(workspace);
  uint8_t *a_sf = a_codes + codes_b;
  nvfp4_status st = check_gemm_args(a_codes, a_sf, x_gscale, w_codes, w_sf, w_gscale, y, y_dt, ld_y, M, N, K);
  if (st != NVFP4_OK) return st;
  DeviceState *dev = nullptr;
  if ((st = device_state(&dev)) != NVFP4_OK) return st;
  if (workspace_bytes < codes_b + sf_b + gemm_partial_bytes(M, N, K, *dev)) return NVFP4_ERR_WORKSPACE;
  const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  st = quantize_impl(x, x_dt, M, K, ld_x, x_gscale, a_codes, a_sf, 0, M, s, true);
  if (st != NVFP4_OK) return st;
  return gemm_impl(a_codes, a_sf, x_gscale, w_codes, w_sf, w_gscale, y, y_dt, ld_y, M, N, K, a_sf + sf_b,
                   workspace_bytes - codes_b - sf_b, s, true);
}

nvfp4_status w4a4_gemm_noalloc(const void *x, nvfp4_in_dtype x_dt, int64_t ld_x, const float *x_gscale,
                               const uint8_t *w_codes, const uint8_t *w_sf, const float *w_gscale, void *y,
                               nvfp4_out_dtype y_dt, int64_t ld_y, int64_t M, int64_t N, int64_t K,
                               nvfp4_stream_t stream) {
  // per-device address of the fixed scratch, looked up once with the device current
  static std::mutex mu;
  static void *scratch[kMaxDevices] = {};
  if (x_dt != NVFP4_IN_BF16 && x_dt != NVFP4_IN_F32) return NVFP4_ERR_DTYPE;
  if (M < 0 || N < 0 || K <= 0 || K % 64 != 0 || ld_x < K) return NVFP4_ERR_SHAPE;
  if (M == 0 || N == 0) return NVFP4_OK;
  // the device checks first, so that an unsupported GPU reports UNSUPPORTED
  DeviceState *state = nullptr;
  nvfp4_status st = device_state(&state);
  if (st != NVFP4_OK) return st;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return NVFP4_ERR_CUDA;
  void *buf = nullptr;
  {
    std::lock_guard<std::mutex> lock(mu);
    if (!scratch[dev]) {
      void *p = nullptr;
      if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) {
        cudaGetLastError();      // leave no stale error for the next call's launch check
        return NVFP4_ERR_CUDA;
      }
      scratch[dev] = p;
    }
    buf = scratch[dev];
  }
  if (w4a4_gemm_workspace_bytes(M, N, K) > kNoAllocScratchBytes) return NVFP4_ERR_SCRATCH_LIMIT;
  return w4a4_gemm(x, x_dt, ld_x, x_gscale, w_codes, w_sf, w_gscale, y, y_dt, ld_y, M, N, K, buf,
                   kNoAllocScratchBytes, stream);
}

nvfp4_status w4a4_gemm_fused(const void *x, nvfp4_in_dtype x_dt, int64_t ld_x, const float *x_gscale,
                             const uint8_t *w_codes, const uint8_t *w_sf, const float *w_gscale, void *y,
                             nvfp4_out_dtype y_dt, int64_t ld_y, int64_t M, int64_t N, int64_t K,
                             nvfp4_stream_t stream) {
  if (x_dt != NVFP4_IN_BF16 && x_dt != NVFP4_IN_F32) return NVFP4_ERR_DTYPE;
  if (M < 0 || N < 0 || K <= 0 || K % 64 != 0 || ld_x < K) return NVFP4_ERR_SHAPE;
  if (M > 128 && N > 128) return NVFP4_ERR_UNSUPPORTED;
  if (M == 0 || N == 0) return NVFP4_OK;
  if (!x || !x_gscale) return NVFP4_ERR_NULL;
  const int esz = x_dt == NVFP4_IN_BF16 ? 2 : 4;
  if (!aligned16(x) || (ld_x * esz) % 16 != 0) return NVFP4_ERR_ALIGN;
  // the activation-side arguments stand in for the codes the kernel makes itself
  nvfp4_status st = check_gemm_args(w_codes, w_sf, x_gscale, w_codes, w_sf, w_gscale, y, y_dt, ld_y, M, N, K);
  if (st != NVFP4_OK) return st;
  DeviceState *dev = nullptr;
  if ((st = device_state(&dev)) != NVFP4_OK) return st;
  return w4a4_fused_impl(x, x_dt, ld_x, x_gscale, w_codes, w_sf, w_gscale, y, y_dt, ld_y, M, N, K, *dev,
                         reinterpret_cast<cudaStream_t>(stream));
}

nvfp4_status w4a4_gdn_gates(const void *x, nvfp4_in_dtype x_dt, int64_t ld_x, const float *x_gscale,
                            const uint8_t *w_codes, const uint8_t *w_sf, const float *w_gscale, float *gates,
                            int64_t ld_g, int64_t M, int64_t N, int64_t n_a, int64_t K, void *workspace,
                            size_t workspace_bytes, nvfp4_stream_t stream) {
  if (x_dt != NVFP4_IN_BF16 && x_dt != NVFP4_IN_F32) return NVFP4_ERR_DTYPE;
  if (M < 0 || N < 0 || K <= 0 || K % 64 != 0 || ld_x < K || n_a < 0 || n_a > N) return NVFP4_ERR_SHAPE;
  if (N > 128) return NVFP4_ERR_UNSUPPORTED;        // the gate projections are narrow (N = 2 x heads)
  if (M == 0 || N == 0) return NVFP4_OK;
  if (!x || !x_gscale) return NVFP4_ERR_NULL;
  const int esz = x_dt == NVFP4_IN_BF16 ? 2 : 4;
  if (!aligned16(x) || (ld_x * esz) % 16 != 0) return NVFP4_ERR_ALIGN;
  if (!workspace) return NVFP4_ERR_WORKSPACE;
  if (!aligned16(workspace)) return NVFP4_ERR_ALIGN;
  const size_t codes_b = align256(nvfp4_codes_bytes(M, K));
  const size_t sf_b = align256(nvfp4_sf_bytes(M, K));
  if (workspace_bytes < codes_b + sf_b) return NVFP4_ERR_WORKSPACE;
  uint8_t *a_codes = static_cast<uint8_t *>(workspace);
  uint8_t *a_sf = a_codes + codes_b;
  nvfp4_status st = check_gemm_args(a_codes, a_sf, x_gscale, w_codes, w_sf, w_gscale, gates, NVFP4_OUT_F32, ld_g,
                                    M, N, K);
  if (st != NVFP4_OK) return st;
  const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  st = quantize_impl(x, x_dt, M, K, ld_x, x_gscale, a_codes, a_sf, 0, M, s, true);
  if (st != NVFP4_OK) return st;
  return gemm_impl(a_codes, a_sf, x_gscale, w_codes, w_sf, w_gscale, gates, NVFP4_OUT_F32, ld_g, M, N, K,
                   a_sf + sf_b, workspace_bytes - codes_b - sf_b, s, true, n_a);
}

nvfp4_status nvfp4_fake_quant(const void *x, nvfp4_in_dtype dt, int64_t rows, int64_t K, int64_t ld_x,
                              const float *gscale, void *out, nvfp4_out_dtype out_dt, int64_t ld_out,
                              double *err_stats, nvfp4_stream_t stream) {
  if (dt != NVFP4_IN_BF16 && dt != NVFP4_IN_F32) return NVFP4_ERR_DTYPE;
  if (out_dt != NVFP4_OUT_BF16 && out_dt != NVFP4_OUT_F32) return NVFP4_ERR_DTYPE;
  if (rows < 0 || K <= 0 || K % 64 != 0 || ld_x < K || ld_out < K || rows * ((K + 511) / 512) >= (int64_t)UINT32_MAX)
    return NVFP4_ERR_SHAPE;
  if (!gscale || (rows > 0 && (!x || !out))) return NVFP4_ERR_NULL;
  const int esz = dt == NVFP4_IN_BF16 ? 2 : 4, osz = out_dt == NVFP4_OUT_BF16 ? 2 : 4;
  if ((rows > 0 && (!aligned16(x) || !aligned16(out))) || (ld_x * esz) % 16 != 0 || (ld_out * osz) % 16 != 0 ||
      (err_stats && (reinterpret_cast<uintptr_t>(err_stats) & 7)))
    return NVFP4_ERR_ALIGN;
  DeviceState *dev = nullptr;
  nvfp4_status st = device_state(&dev);
  if (st != NVFP4_OK) return st;
  const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (err_stats && cudaMemsetAsync(err_stats, 0, 2 * sizeof(double), s) != cudaSuccess) return NVFP4_ERR_CUDA;
  if (rows == 0) return NVFP4_OK;
  FakeQuantParams p{x, rows, K, ld_x, gscale, out, ld_out, err_stats};
  const int64_t units = rows * ((K + 511) / 512);
  int64_t blocks = (units + 7) / 8;
  if (blocks > 16LL * dev->sms) blocks = 16LL * dev->sms;
  const unsigned g = (unsigned)blocks;
  cudaError_t e;
  if (dt == NVFP4_IN_BF16)
    e = out_dt == NVFP4_OUT_F32 ? launch_ex(fake_quant_kernel<__nv_bfloat16, float>, g, 256u, 0, s, 0, false, p)
                                : launch_ex(fake_quant_kernel<__nv_bfloat16, __nv_bfloat16>, g, 256u, 0, s, 0, false, p);
  else
    e = out_dt == NVFP4_OUT_F32 ? launch_ex(fake_quant_kernel<float, float>, g, 256u, 0, s, 0, false, p)
                                : launch_ex(fake_quant_kernel<float, __nv_bfloat16>, g, 256u, 0, s, 0, false, p);
  if (e != cudaSuccess) return NVFP4_ERR_CUDA;
  return launched();
}

nvfp4_status nvfp4_fp8_quantize(const void *x, nvfp4_in_dtype dt, int64_t n, const float *scale, uint8_t *q,
                                nvfp4_stream_t stream) {
  if (dt != NVFP4_IN_BF16 && dt != NVFP4_IN_F32) return NVFP4_ERR_DTYPE;
  if (n < 0 || n % 8 != 0) return NVFP4_ERR_SHAPE;
  if (n == 0) return NVFP4_OK;
  if (!x || !scale || !q) return NVFP4_ERR_NULL;
  if (!aligned16(x) || (reinterpret_cast<uintptr_t>(q) & 7) || (reinterpret_cast<uintptr_t>(scale) & 3))
    return NVFP4_ERR_ALIGN;
  DeviceState *dev = nullptr;
  nvfp4_status st = device_state(&dev);
  if (st != NVFP4_OK) return st;
  const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  Fp8Params p{x, n, scale, q};
  int64_t blocks = (n / 8 + 255) / 256;
  if (blocks > 8LL * dev->sms) blocks = 8LL * dev->sms;
  const cudaError_t e = dt == NVFP4_IN_BF16
                            ? launch_ex(fp8_quantize_kernel<__nv_bfloat16>, (unsigned)blocks, 256u, 0, s, 0, false, p)
                            : launch_ex(fp8_quantize_kernel<float>, (unsigned)blocks, 256u, 0, s, 0, false, p);
  if (e != cudaSuccess) return NVFP4_ERR_CUDA;
  return launched();
}

nvfp4_status nvfp4_harmonize_requant(uint8_t *codes, uint8_t *sf, int64_t rows_total, int64_t K, int n_modules,
                                     const int64_t *row_offsets, const float *gscales, float *shared_gscale_out,
                                     nvfp4_stream_t stream) {
  if (!codes || !sf || !row_offsets || !gscales || !shared_gscale_out) return NVFP4_ERR_NULL;
  if (n_modules < 1 || n_modules > kMaxModules || rows_total <= 0 || K <= 0 || K % 64 != 0)
    return NVFP4_ERR_SHAPE;
  if (row_offsets[0] != 0 || row_offsets[n_modules] != rows_total) return NVFP4_ERR_SHAPE;
  for (int m = 0; m < n_modules; ++m)
    if (row_offsets[m + 1] <= row_offsets[m]) return NVFP4_ERR_SHAPE;
  if (!aligned16(sf) || (reinterpret_cast<uintptr_t>(codes) & 7)) return NVFP4_ERR_ALIGN;
  DeviceState *dev = nullptr;
  nvfp4_status st = device_state(&dev);
  if (st != NVFP4_OK) return st;
  HarmonizeParams p{};
  p.sf = sf;
  p.rows_total = rows_total;
  p.K = K;
  p.n = n_modules;
  for (int m = 0; m <= n_modules; ++m) p.offs[m] = row_offsets[m];
  p.gs = gscales;
  p.gstar_out = shared_gscale_out;
  const int64_t total = rows_total * (K / 16);
  int64_t blocks = (total + 255) / 256;
  if (blocks > 8LL * dev->sms) blocks = 8LL * dev->sms;
  harmonize_requant_kernel<<<(unsigned)blocks, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(p, codes);
  return launched();
}

nvfp4_status nvfp4_rmsnorm_quantize(const void *x, nvfp4_in_dtype dt, int64_t rows, int64_t K, int64_t ld_x,
                                    const uint16_t *w, int zero_centered, float eps, const float *gscale,
                                    uint8_t *codes, uint8_t *sf, float *inv_out, nvfp4_stream_t stream) {
  if (dt != NVFP4_IN_BF16 && dt != NVFP4_IN_F32) return NVFP4_ERR_DTYPE;
  if (rows < 0 || K <= 0 || K % 64 != 0 || ld_x < K || !(eps > 0.0f) || !(eps <= 3.4028235e38f))
    return NVFP4_ERR_SHAPE;
  if (!sf || !gscale || !w || (rows > 0 && (!x || !codes))) return NVFP4_ERR_NULL;
  const int esz = dt == NVFP4_IN_BF16 ? 2 : 4;
  if ((rows > 0 && (!aligned16(x) || (reinterpret_cast<uintptr_t>(codes) & 7))) || (ld_x * esz) % 16 != 0 ||
      !aligned16(sf) || !aligned16(w) || (inv_out && (reinterpret_cast<uintptr_t>(inv_out) & 3)))
    return NVFP4_ERR_ALIGN;
  // the norm weight is staged in one CTA's shared memory
  if (rms_warp_smem_bytes(K) > kSmemOptin) return NVFP4_ERR_UNSUPPORTED;
  DeviceState *dev = nullptr;
  nvfp4_status st = device_state(&dev);
  if (st != NVFP4_OK) return st;
  const int64_t pad_rows = pad128(rows) - rows;
  if (rows == 0 && pad_rows == 0) return NVFP4_OK;
  const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  RmsQuantParams p{x, rows, K, ld_x, reinterpret_cast<const __nv_bfloat16 *>(w), zero_centered ? 1 : 0, eps,
                   gscale, codes, sf, inv_out, pad_rows};
  // one warp per row (no CTA barrier per row)
  const size_t wsmem = (size_t)rms_warp_smem_bytes(K);
  int per_sm = 0;
  cudaError_t e = dt == NVFP4_IN_BF16
                      ? cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, rmsnorm_quantize_warp_kernel<__nv_bfloat16>,
                                                                      kRmsWarpThreads, wsmem)
                      : cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, rmsnorm_quantize_warp_kernel<float>,
                                                                      kRmsWarpThreads, wsmem);
  if (e != cudaSuccess || per_sm < 1) return NVFP4_ERR_CUDA;
  int64_t grid = (int64_t)per_sm * dev->sms;
  const int64_t need = (rows + kRmsWarpThreads / 32 - 1) / (kRmsWarpThreads / 32);
  if (grid > need) grid = need;
  if (grid < 1) grid = 1;
  e = dt == NVFP4_IN_BF16
          ? launch_ex(rmsnorm_quantize_warp_kernel<__nv_bfloat16>, (unsigned)grid, (unsigned)kRmsWarpThreads, wsmem, s,
                      0, false, p)
          : launch_ex(rmsnorm_quantize_warp_kernel<float>, (unsigned)grid, (unsigned)kRmsWarpThreads, wsmem, s, 0, false,
                      p);
  if (e != cudaSuccess) return NVFP4_ERR_CUDA;
  return launched();
}

nvfp4_status nvfp4_plan_for(int64_t M, int64_t N, int64_t K, int sms, int pair_clusters, const int *split_clusters,
                            int *out) {
  if (!out) return NVFP4_ERR_NULL;
  if (M <= 0 || N <= 0 || K <= 0 || K % 64 != 0 || sms <= 0 || pair_clusters < 0) return NVFP4_ERR_SHAPE;
  DeviceState d{};
  d.sms = sms;
  d.pair_clusters = pair_clusters;
  if (split_clusters)
    for (int b = 0; b < 3; ++b)
      for (int c = 0; c <= kMaxSplitCluster; ++c) d.split_clusters[b][c] = split_clusters[b * (kMaxSplitCluster + 1) + c];
  const Plan pl = make_plan(M, N, K, d);
  out[0] = (int)pl.kind;
  out[1] = pl.bn;
  out[2] = pl.swap ? 1 : 0;
  out[3] = pl.splits;
  out[4] = pl.grid;
  out[5] = pl.tiles_a;
  out[6] = pl.tiles_b;
  out[7] = pl.kstages;
  return NVFP4_OK;
}

nvfp4_status nvfp4_selftest_wait_timeout(int64_t limit_ns, int *result_dev, nvfp4_stream_t stream) {
  if (!result_dev) return NVFP4_ERR_NULL;
  if (limit_ns <= 0 || limit_ns > 2000000000LL) return NVFP4_ERR_SHAPE;
  DeviceState *dev = nullptr;
  nvfp4_status st = device_state(&dev);
  if (st != NVFP4_OK) return st;
  wait_timeout_selftest_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      dev->err, (unsigned long long)limit_ns, result_dev);
  return launched();
}

nvfp4_status nvfp4_last_device_status(nvfp4_stream_t stream, int *flags) {
  if (!flags) return NVFP4_ERR_NULL;
  *flags = 0;
  DeviceState *dev = nullptr;
  nvfp4_status st = device_state(&dev);
  if (st != NVFP4_OK) return st;
  const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  // take the word and clear it in one atomic step on the stream, so a flag
  // that a kernel on another stream sets meanwhile is never lost
  error_take_kernel<<<1, 1, 0, s>>>(dev->err);
  if (launched() != NVFP4_OK) return NVFP4_ERR_CUDA;
  unsigned v = 0;
  if (cudaMemcpyFromSymbolAsync(&v, g_nvfp4_error_snapshot, sizeof(v), 0, cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return NVFP4_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return NVFP4_ERR_CUDA;
  *flags = (int)v;
  return v ? NVFP4_ERR_TIMEOUT : NVFP4_OK;
}

const char *nvfp4_status_string(nvfp4_status s) {
  switch (s) {
    case NVFP4_OK: return "ok";
    case NVFP4_ERR_NULL: return "null pointer";
    case NVFP4_ERR_SHAPE: return "bad shape";
    case NVFP4_ERR_ALIGN: return "misaligned pointer or stride";
    case NVFP4_ERR_DTYPE: return "unknown dtype";
    case NVFP4_ERR_UNSUPPORTED: return "unsupported (needs an sm_100 device)";
    case NVFP4_ERR_TIMEOUT: return "a kernel wait ran out";
    case NVFP4_ERR_CUDA: return "CUDA error";
    case NVFP4_ERR_WORKSPACE: return "workspace missing or too small";
    case NVFP4_ERR_SCRATCH_LIMIT: return "problem needs more scratch than the 8 MiB built-in buffer of w4a4_gemm_noalloc";
  }
  return "unknown status";
}

uint64_t nvfp4_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

}  // extern "C"
