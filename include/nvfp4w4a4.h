/*
 * nvfp4w4a4.h -- C ABI of the NVFP4 W4A4 linear layer for NVIDIA B200 (sm_100a).
 *
 * The operation (from the web pages on arXiv 2609.04098, "Why Gated DeltaNet
 * Survives 4-Bit Quantization: NVFP4 W4A4 for the Recurrent Half of a Hybrid
 * 27B LLM"):
 *   - NVFP4 stores 4-bit E2M1 values with one E4M3 scale per 16 consecutive
 *     elements (the block maximum divided by 6) and one FP32 scale per tensor
 *     (ta-paperlens page, section "前提1"; arxiv-wiki page, "접근 방법").
 *   - W4A4: weights and activations are both NVFP4 and the matrix product runs
 *     on the 4-bit tensor cores (ta-paperlens page, "前提1").
 *   - Modules that a serving kernel fuses into one GEMM (GDN in_proj_qkv with
 *     in_proj_z, in_proj_b with in_proj_a) must share one global scale; the
 *     per-module ratios are folded into the block scales (arxiv-wiki page,
 *     "접근 방법" and "개발자 관점"; abstract on the shd-paper page).
 *
 * Arithmetic (the readings this library implements, bit for bit):
 *   g       : per-tensor FP32 dequantization scale, g = amax / (6*448)
 *   g6      = fl32(6 * g)
 *   s_b     = E4M3_RNE_SATFINITE(fl32(amax_b / g6))     per 16-element block b
 *   d_b     = fl32(dec(s_b) * g)
 *   q_i     = E2M1_RNE_SATFINITE(fl32(x_i / d_b))        (+0 codes if dec(s_b)==0 or d_b==0)
 *   Y[m,n]  = fl32(acc[m,n] * fl32(g_x * g_w)),  acc = sum_k dec(qx)dec(sx)dec(qw)dec(sw)
 *             accumulated in FP32 by the tensor cores, then rounded to BF16
 *             (round to nearest even) or kept as FP32.
 *
 * Data layouts (all device memory unless stated):
 *   codes : [rows, K/2] bytes, row stride K/2; element 2j of a row in the low
 *           nibble of byte j, element 2j+1 in the high nibble.
 *   sf    : swizzled E4M3 scale bytes of a tensor with R rows:
 *           nvfp4_sf_bytes(R, K) bytes = pad128(R) * (K/16); the scale of (row r,
 *           block column c) is at byte
 *             ((r/128)*(K/64) + c/4)*512 + (r%32)*16 + ((r%128)/32)*4 + c%4
 *           (128-row x 4-column atoms of 512 bytes, the layout the sm_100
 *           block-scaled tensor-core instructions read).  Rows in
 *           [R, pad128(R)) are padding and hold zero.
 *   x, y  : row-major with a leading dimension in elements.
 *
 * Conventions for every entry point:
 *   - The caller allocates every buffer (PyTorch in the bundled binding); the
 *     library never calls cudaMalloc/cudaFree.
 *   - All work is enqueued on `stream`; nothing synchronizes the host except
 *     nvfp4_last_device_status(), which synchronizes the stream it is given.
 *   - Preconditions: K % 64 == 0, K > 0, rows >= 0; device pointers 16-byte
 *     aligned; ld_x >= K with ld_x * element size a multiple of 16 bytes;
 *     ld_y >= N (any value); inputs finite; global scales finite and > 0.
 *   - Validation failures return a status code before anything is enqueued;
 *     nothing throws across the ABI.  A CUDA launch error is returned as
 *     NVFP4_ERR_CUDA.  Kernels bound every wait; a wait that runs out records a
 *     flag that nvfp4_last_device_status() reports.
 *   - Calls on one stream are ordered; calls that write the same buffers from
 *     different streams must be ordered by the caller.
 */
#ifndef NVFP4W4A4_H
#define NVFP4W4A4_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *nvfp4_stream_t;   /* same object as cudaStream_t; NULL = legacy stream */

typedef enum {
    NVFP4_OK = 0,
    NVFP4_ERR_NULL = 1,        /* a required pointer is NULL */
    NVFP4_ERR_SHAPE = 2,       /* bad rows/K/M/N/ld or K % 64 != 0 */
    NVFP4_ERR_ALIGN = 3,       /* a pointer or row stride is not 16-byte aligned */
    NVFP4_ERR_DTYPE = 4,       /* unknown dtype enum */
    NVFP4_ERR_UNSUPPORTED = 5, /* valid request this build does not serve */
    NVFP4_ERR_TIMEOUT = 6,     /* a kernel wait ran out (see nvfp4_last_device_status) */
    NVFP4_ERR_CUDA = 7,        /* a CUDA runtime/driver call failed */
    NVFP4_ERR_WORKSPACE = 8,   /* workspace NULL or smaller than the size helper says */
    NVFP4_ERR_SCRATCH_LIMIT = 9 /* w4a4_gemm_noalloc: the problem needs more scratch than its built-in buffer */
} nvfp4_status;

typedef enum { NVFP4_IN_BF16 = 0, NVFP4_IN_F32 = 1 } nvfp4_in_dtype;
typedef enum { NVFP4_OUT_BF16 = 0, NVFP4_OUT_F32 = 1 } nvfp4_out_dtype;

/* Bytes of the packed codes of a [rows, K] tensor: rows * K / 2. */
size_t nvfp4_codes_bytes(int64_t rows, int64_t K);

/* Bytes of the swizzled scale buffer of a [rows, K] tensor: pad128(rows) * K/16. */
size_t nvfp4_sf_bytes(int64_t rows, int64_t K);

/*
 * Per-tensor global scale (row a1 of the layer): *gscale_out = amax(|x|)/(6*448),
 * or 1.0f for an all-zero tensor, where 6 is the largest E2M1 value and 448 the
 * largest E4M3 value (the pages calibrate this scale offline per module,
 * arxiv-wiki page "접근 방법"; this call computes it from the tensor itself).
 *   x          : [rows, K] of dtype dt, row stride ld_x elements (device).
 *   gscale_out : 1 float (device); also used as the reduction accumulator, so
 *                it must not alias x.
 */
nvfp4_status nvfp4_amax_gscale(const void *x, nvfp4_in_dtype dt, int64_t rows, int64_t K,
                               int64_t ld_x, float *gscale_out, nvfp4_stream_t stream);

/*
 * Quantize a [rows, K] tensor to NVFP4 (rows a2, a3 and a5 of the layer;
 * ta-paperlens page "前提1").
 *   x         : [rows, K] bf16 or fp32 (dt), row stride ld_x elements (device).
 *   gscale    : 1 float, the tensor's global scale g (device).
 *   codes     : [rows, K/2] bytes for THIS call's rows (device, written).
 *   sf        : base of the swizzled scale buffer of a tensor with
 *               sf_rows_total rows (device, nvfp4_sf_bytes(sf_rows_total, K)
 *               bytes); this call writes the scales of rows
 *               [sf_row0, sf_row0 + rows).  When sf_row0 + rows == sf_rows_total
 *               it also zeroes the padding rows [sf_rows_total, pad128(sf_rows_total)).
 *   sf_row0, sf_rows_total : place the tensor inside a fused (concatenated
 *               along rows) weight, so each module is quantized with its own g
 *               and then harmonized (nvfp4_harmonize_group).
 */
nvfp4_status nvfp4_quantize(const void *x, nvfp4_in_dtype dt, int64_t rows, int64_t K,
                            int64_t ld_x, const float *gscale, uint8_t *codes, uint8_t *sf,
                            int64_t sf_row0, int64_t sf_rows_total, nvfp4_stream_t stream);

/*
 * Fused-group global-scale repair (row a6; arxiv-wiki page "접근 방법", last
 * bullet, and "개발자 관점": per-module-calibrated checkpoints served by a
 * kernel that fuses the modules into one GEMM need one shared global scale,
 * with the ratios folded into the block scales).
 *   sf            : fused swizzled scale buffer, rows_total rows (device, in place).
 *   row_offsets   : n_modules + 1 HOST integers, 0 = row_offsets[0] < ... <
 *                   row_offsets[n_modules] = rows_total; module m owns rows
 *                   [row_offsets[m], row_offsets[m+1]).
 *   gscales       : n_modules floats, each module's own global scale (device).
 *   shared_gscale_out : 1 float (device): g* = max_m gscales[m].  Must not
 *                   alias gscales.
 * Every scale byte s of module m becomes E4M3_RNE_SATFINITE(fl32(dec(s) *
 * fl32(g_m / g*))); the codes are unchanged.  1 <= n_modules <= 16.
 */
nvfp4_status nvfp4_harmonize_group(uint8_t *sf, int64_t rows_total, int64_t K, int n_modules,
                                   const int64_t *row_offsets, const float *gscales,
                                   float *shared_gscale_out, nvfp4_stream_t stream);

/*
 * Block-scaled W4A4 GEMM on pre-quantized operands (rows a7, a8):
 *   y[m, n] = fl32(acc * fl32(a_gscale * b_gscale)),
 *   acc[m, n] = sum_k dec(a)[m,k] * dec(b)[n,k]  (tcgen05 kind::mxf4nvf4, FP32 in TMEM)
 *   a_codes/a_sf : activation, M rows (device); a_sf has nvfp4_sf_bytes(M, K) bytes.
 *   b_codes/b_sf : weight, N rows (device); b_sf has nvfp4_sf_bytes(N, K) bytes.
 *   a_gscale, b_gscale : 1 float each (device).
 *   y            : [M, N] bf16 or fp32 (y_dt), row stride ld_y elements (device).
 *   workspace    : device scratch of at least nvfp4_gemm_workspace_bytes(M, N, K)
 *                  bytes (may be NULL when that is 0).
 */
size_t nvfp4_gemm_workspace_bytes(int64_t M, int64_t N, int64_t K);
nvfp4_status nvfp4_gemm(const uint8_t *a_codes, const uint8_t *a_sf, const float *a_gscale,
                        const uint8_t *b_codes, const uint8_t *b_sf, const float *b_gscale,
                        void *y, nvfp4_out_dtype y_dt, int64_t ld_y, int64_t M, int64_t N,
                        int64_t K, void *workspace, size_t workspace_bytes,
                        nvfp4_stream_t stream);

/*
 * The W4A4 linear layer (all rows a2-a9): quantize the activation x on the
 * fly with its global scale, then the block-scaled GEMM against pre-quantized
 * NVFP4 weights (ta-paperlens page "前提1": both operands 4-bit, product on
 * 4-bit tensor cores).
 *   x        : [M, K] bf16 or fp32 (x_dt), row stride ld_x elements (device).
 *   x_gscale : 1 float (device).
 *   w_codes, w_sf, w_gscale : the weight as written by nvfp4_quantize (and,
 *              for a fused group, nvfp4_harmonize_group's shared scale).
 *   y        : [M, N] (y_dt), row stride ld_y (device).
 *   workspace: device scratch, >= w4a4_gemm_workspace_bytes(M, N, K) bytes;
 *              holds the quantized activation and any split-K partial sums.
 * Launch behaviour: the quantize and the GEMM are enqueued with programmatic
 * stream serialization.  The quantize waits for the stream's preceding work
 * before it reads x; the GEMM may start while the quantize runs and loads
 * the weight (w_codes, w_sf) before it waits for the quantize.  Weights
 * written by earlier work on the stream are therefore safe, since that work
 * finishes before the quantize lets the GEMM start.  Do not rewrite the
 * weight with a kernel that is still running when w4a4_gemm is enqueued (a
 * kernel that itself let later grids start early); use an event between
 * the two instead.
 */
size_t w4a4_gemm_workspace_bytes(int64_t M, int64_t N, int64_t K);
nvfp4_status w4a4_gemm(const void *x, nvfp4_in_dtype x_dt, int64_t ld_x, const float *x_gscale,
                       const uint8_t *w_codes, const uint8_t *w_sf, const float *w_gscale,
                       void *y, nvfp4_out_dtype y_dt, int64_t ld_y, int64_t M, int64_t N,
                       int64_t K, void *workspace, size_t workspace_bytes,
                       nvfp4_stream_t stream);

/*
 * The W4A4 linear layer for callers that cannot allocate device memory: the
 * same computation and kernels as w4a4_gemm, but the scratch it needs (the
 * quantized activation and any split-K partial sums) lives in a fixed buffer
 * inside the library instead of a caller-provided workspace.  No counterpart
 * exists on the pages; this is a deployment convenience.
 *
 * Who needs it: host code that must not call cudaMalloc at the point of use,
 * for example an inference runtime whose memory plan is fixed before serving
 * starts (every device byte is owned by the framework's arena), a plugin that
 * the host framework gives only input and output pointers, or code that has
 * to stay free of allocation calls because an allocation can synchronize the
 * device or fail under memory pressure in the middle of a step.
 *
 * The buffer is a file-scope 8 MiB (8,388,608-byte) __device__ array; every
 * GPU that loads the library holds it until the process exits.  The arguments
 * mean what they mean for w4a4_gemm; the caller still provides x, the
 * weights, the scales and y.
 *   - Problems whose w4a4_gemm_workspace_bytes(M, N, K) exceeds 8 MiB return
 *     NVFP4_ERR_SCRATCH_LIMIT before anything is enqueued.  That size is what
 *     decides; as an example, on a B200 (where narrow products reduce inside a
 *     thread-block cluster and need no partial sums) the decode products with
 *     M <= 64 and N*K up to 5120 x 17408 fit, while on a device without
 *     cluster support the same M = 64 products need split-K partial sums and
 *     can exceed the buffer.
 *   - The first call on a device looks the buffer's device address up
 *     (cudaGetSymbolAddress) with that device current; make that first call
 *     before any stream capture on the device.
 *   - All calls share the one buffer, which keeps the last call's contents;
 *     nothing in it has to start at zero.  Calls that can overlap on the GPU
 *     (different streams, or different host threads) race on it: order them.
 *   - Calls no cudaMalloc, cudaFree or allocating library routine.
 */
nvfp4_status w4a4_gemm_noalloc(const void *x, nvfp4_in_dtype x_dt, int64_t ld_x, const float *x_gscale,
                               const uint8_t *w_codes, const uint8_t *w_sf, const float *w_gscale,
                               void *y, nvfp4_out_dtype y_dt, int64_t ld_y, int64_t M, int64_t N,
                               int64_t K, nvfp4_stream_t stream);

/*
 * The layer with the activation quantize inside the GEMM (row a9 of the
 * layer, "quantize in the producer"): one kernel, whose extra warps encode
 * each K stage of x straight into the MMA's operand tiles on the MMA's N side;
 * the codes are bit-identical to nvfp4_quantize's.  Two shapes are served:
 *   - decode-shaped products, M <= 128 activation rows (one narrow tile);
 *   - narrow weights, N <= 128 rows with any M (the GDN gate projections):
 *     the weight is the 128-row MMA operand and the activation is encoded in
 *     tiles of 128 rows.
 * NVFP4_ERR_UNSUPPORTED when M > 128 and N > 128, and when the device offers
 * no cluster plan for the shape.  No workspace.  y agrees with w4a4_gemm's
 * within the GEMM tolerance; it is bit-identical on the decode configurations
 * and on the 4096 x 96 x 5120 gate product (same K split, same reduction
 * order).  On B200
 * w4a4_gemm is as fast or faster for these shapes (decode: every weight
 * tile's CTAs re-encode the same activation slice; gates: both about
 * 27.7 us, the encoder's own throughput), so w4a4_gemm does not use it; it
 * is kept as the in-producer form of the layer.  It may start before the
 * stream's preceding work has finished (programmatic launch) but reads
 * nothing, the weight included, until that work has completed.
 */
nvfp4_status w4a4_gemm_fused(const void *x, nvfp4_in_dtype x_dt, int64_t ld_x, const float *x_gscale,
                             const uint8_t *w_codes, const uint8_t *w_sf, const float *w_gscale, void *y,
                             nvfp4_out_dtype y_dt, int64_t ld_y, int64_t M, int64_t N, int64_t K,
                             nvfp4_stream_t stream);

/*
 * Failure-detection self-test: launches one thread that waits, bounded by
 * limit_ns of %globaltimer (0 < limit_ns <= 2e9), on a barrier nothing ever
 * completes.  The wait runs out, sets bit 4 (value 16) of the device error
 * word (read and cleared by nvfp4_last_device_status, which then returns
 * NVFP4_ERR_TIMEOUT) and writes 0 to *result_dev (device int); the kernel
 * returns normally and the context stays usable.  Every wait in the library's
 * kernels is bounded the same way (2 s), so a lost producer or consumer shows
 * up as this status instead of a hang.
 */
nvfp4_status nvfp4_selftest_wait_timeout(int64_t limit_ns, int *result_dev, nvfp4_stream_t stream);

/*
 * ------------------------------------------------------------------------
 * Rows beyond the layer itself, built on the same encoder and GEMM.
 * ------------------------------------------------------------------------
 *
 * GDN gate projections with the gate activations fused into the GEMM
 * epilogue (ta-paperlens page, "前提2": the raw projections a_t and b_t become
 * alpha_t = exp(-softplus(a_t)), how much of the state is kept, and
 * beta_t = sigmoid(b_t), the write strength; the model's per-head decay scale
 * and bias are not part of this call: unit scale, zero bias).
 *   x, x_gscale, w_codes, w_sf, w_gscale, workspace : as for w4a4_gemm; the
 *              weight is the fused [a; b] gate projection (N <= 128 rows,
 *              harmonized to one global scale when a and b were calibrated
 *              apart).
 *   gates    : [M, N] float32 (device), row stride ld_g: columns [0, n_a)
 *              hold alpha, columns [n_a, N) hold beta.
 * Errors: NVFP4_ERR_UNSUPPORTED when N > 128; otherwise as w4a4_gemm.  Same
 * launch ordering as w4a4_gemm.
 */
nvfp4_status w4a4_gdn_gates(const void *x, nvfp4_in_dtype x_dt, int64_t ld_x, const float *x_gscale,
                            const uint8_t *w_codes, const uint8_t *w_sf, const float *w_gscale, float *gates,
                            int64_t ld_g, int64_t M, int64_t N, int64_t n_a, int64_t K, void *workspace,
                            size_t workspace_bytes, nvfp4_stream_t stream);

/*
 * Fake-quant: every element of x replaced by the NVFP4 value it quantizes to,
 * dec(q) * dec(s) * g (the values the W4A4 product sees; the pages measure
 * the relative activation error this introduces, arxiv-wiki page, "주요 결과").
 *   x        : [rows, K] bf16 or fp32, row stride ld_x (device).
 *   gscale   : 1 float (device).
 *   out      : [rows, K] bf16 or fp32 (out_dt), row stride ld_out (device);
 *              FP32 output is the exact value rounded once to fp32, BF16 output
 *              is that fp32 value rounded to bf16.
 *   err_stats: NULL or 2 doubles (device, 8-byte aligned), overwritten with
 *              [sum of (x - q)^2, sum of x^2], q the exact NVFP4 value of x;
 *              the relative error is sqrt(err_stats[0] / err_stats[1]).  Each
 *              16-element block is summed in fp32 and the blocks in float64,
 *              so each sum is within a relative 18 * 2^-24 (about 1.1e-6) of
 *              the exact one; the blocks are added with atomics, so the last
 *              bits depend on timing.
 * Preconditions: K % 64 == 0; 16-byte aligned pointers and row strides.
 */
nvfp4_status nvfp4_fake_quant(const void *x, nvfp4_in_dtype dt, int64_t rows, int64_t K, int64_t ld_x,
                              const float *gscale, void *out, nvfp4_out_dtype out_dt, int64_t ld_out,
                              double *err_stats, nvfp4_stream_t stream);

/*
 * FP8 (E4M3) quantization with a static per-tensor scale, as used for the KV
 * cache (arxiv-wiki page, "주요 결과": a static per-tensor FP8 KV scale shipped
 * with the checkpoint recovers most of the FP8 KV penalty):
 *   q[i] = E4M3_RNE_SATFINITE(fl32(x[i] / scale)), sign in bit 7
 *   (dequantize as dec(q) * scale).
 *   x     : n contiguous bf16 or fp32 values (device, 16-byte aligned), n % 8 == 0.
 *   scale : 1 float (device), finite and > 0.
 *   q     : n bytes (device, 8-byte aligned).
 */
nvfp4_status nvfp4_fp8_quantize(const void *x, nvfp4_in_dtype dt, int64_t n, const float *scale, uint8_t *q,
                                nvfp4_stream_t stream);

/*
 * Re-quantizing variant of the fused-group repair (arxiv-wiki page,
 * "접근 방법", last bullet: the modules of a fused GEMM must share one global
 * scale).  Instead of rewriting only the scale bytes (nvfp4_harmonize_group),
 * every block of module m is dequantized to fp32, v = fl32(dec(q) * dec(s) *
 * g_m) (the fake-quant value), and encoded again against g* = max_m g_m with
 * the same arithmetic as nvfp4_quantize.  Codes and scales both change where
 * that moves them: wherever the new scale is a normal E4M3 value the codes
 * come out unchanged and only the scale can differ from the scale-only
 * rewrite; blocks pushed to subnormal scales get re-rounded codes.
 *   codes, sf     : the fused group's codes [rows_total, K/2] and swizzled
 *                   scales (device, both rewritten in place; padding rows
 *                   untouched).
 *   row_offsets, gscales, shared_gscale_out : as for nvfp4_harmonize_group.
 * Errors: as nvfp4_harmonize_group; codes must be 8-byte aligned.
 */
nvfp4_status nvfp4_harmonize_requant(uint8_t *codes, uint8_t *sf, int64_t rows_total, int64_t K, int n_modules,
                                     const int64_t *row_offsets, const float *gscales, float *shared_gscale_out,
                                     nvfp4_stream_t stream);

/*
 * Quantize fused into the RMSNorm that produces a layer's input (the norms
 * stay in BF16 and the GDN layer feeds the normalized residual stream to its
 * projections: ta-paperlens page, "前提2"), so the normalized activation is
 * never written out:
 *   inv_r = the fp32 nearest to 1/sqrt(mean_k x[r,k]^2 + eps)
 *   y     = bf16(fl32(fl32(x * inv_r) * gamma)),
 *           gamma = w, or fl32(1 + w) when zero_centered != 0
 *   codes, sf = nvfp4_quantize(y, gscale)            (bit for bit)
 * The mean square is evaluated to ~2^-48 relative: inv_r is the correctly
 * rounded value except when the exact value lies that close to the midpoint
 * of two floats.
 *   x        : [rows, K] bf16 or fp32 (dt), row stride ld_x (device); the
 *              residual stream.
 *   w        : [K] bf16 norm weight (device, 16-byte aligned).
 *   eps      : finite and > 0.
 *   gscale   : 1 float (device), the static global scale of y.
 *   codes    : [rows, K/2] bytes (device).
 *   sf       : nvfp4_sf_bytes(rows, K) bytes (device); padding rows zeroed.
 *   inv_out  : NULL or [rows] floats (device): inv_r.
 * Errors: NVFP4_ERR_SHAPE for eps <= 0 or not finite; NVFP4_ERR_UNSUPPORTED
 * when the norm weight does not fit in one CTA's shared memory beside the
 * encoder's staging (K above 111872).
 */
nvfp4_status nvfp4_rmsnorm_quantize(const void *x, nvfp4_in_dtype dt, int64_t rows, int64_t K, int64_t ld_x,
                                    const uint16_t *w, int zero_centered, float eps, const float *gscale,
                                    uint8_t *codes, uint8_t *sf, float *inv_out, nvfp4_stream_t stream);

/*
 * Diagnostic: the launch plan the GEMM entry points choose for an M x N x K
 * product on a device with `sms` SMs, `pair_clusters` co-resident CTA pairs of
 * the pair GEMM and split_clusters[bn][c] co-resident split-K clusters of c
 * CTAs (bn index 0, 1, 2 for an MMA N of 32, 64, 128; c = 0..8; NULL = no
 * cluster support).  The entry points take these numbers from the CUDA
 * occupancy calculator once per device; this call takes them as arguments
 * and touches no device, so the planning can be checked anywhere.
 *   out[8] (host): kind (0 single-CTA kernel, 1 CTA pairs, 2 split-K over a
 *          cluster), MMA N, swap (1: the activation is the MMA's N operand),
 *          K splits, grid CTAs, tiles of the 128/256-row operand, tiles of the
 *          other operand, K stages of 256 elements.
 */
nvfp4_status nvfp4_plan_for(int64_t M, int64_t N, int64_t K, int sms, int pair_clusters,
                            const int *split_clusters, int *out);

/*
 * Reports and clears the library's device error word of the current device:
 * a one-thread kernel enqueued on `stream` takes the word and zeroes it in one
 * atomic exchange, then this call synchronizes `stream` only (not the whole
 * device) and stores the taken word in *flags (host int).  The word is the OR
 * of the flags recorded by every library kernel that finished before that
 * exchange, on any stream (flags of kernels still running on other streams
 * are kept for the next call):
 *   bit 0 (1)  : a producer wait ran out
 *   bit 1 (2)  : an MMA-issue wait ran out
 *   bit 2 (4)  : an epilogue or encoder wait ran out
 *   bit 3 (8)  : a TMEM allocation wait ran out
 *   bit 4 (16) : the self-test's wait ran out (nvfp4_selftest_wait_timeout)
 * Returns NVFP4_ERR_TIMEOUT if any flag was set, NVFP4_ERR_CUDA on a CUDA
 * error (including an earlier asynchronous fault that the synchronization
 * surfaces), NVFP4_ERR_UNSUPPORTED on a device that is not sm_100.
 */
nvfp4_status nvfp4_last_device_status(nvfp4_stream_t stream, int *flags);

/* Static string for a status code. */
const char *nvfp4_status_string(nvfp4_status status);

/* Number of kernel launches this library has enqueued in this process. */
uint64_t nvfp4_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* NVFP4W4A4_H */
