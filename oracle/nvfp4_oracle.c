/*
 * nvfp4_oracle.c -- plain, slow, CPU reference of the NVFP4 W4A4 linear layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path links, loads or calls
 * this file; only the tests, the smoke check and the benchmark's CPU-baseline
 * leg do.  It shares no code, header, table or constant generator with the
 * CUDA library.
 *
 * What it follows (the web pages summarising "Why Gated DeltaNet Survives
 * 4-Bit Quantization: NVFP4 W4A4 for the Recurrent Half of a Hybrid 27B LLM",
 * arXiv 2609.04098):
 *   - format: E2M1 4-bit values, one E4M3 scale per 16-element block, one FP32
 *     global scale per tensor (arxiv-wiki page, "접근 방법" first bullet;
 *     ta-paperlens page, "前提1");
 *   - block scale = block max / 6 (ta-paperlens page, "前提1");
 *   - fused-group repair: per-module global scales rewritten to one shared
 *     global scale with the ratios folded into the block scales (arxiv-wiki
 *     page, "접근 방법" last bullet and "개발자 관점" second bullet; abstract on
 *     the shd-paper page);
 *   - W4A4 product: both operands NVFP4, FP32 accumulation on 4-bit tensor
 *     cores (ta-paperlens page, "前提1").
 * The pages leave the arithmetic order, the rounding mode, the zero-block case
 * and the scale layout open; the readings taken here are:
 *   g6 = fl32(6*g);  t = fl32(amax/g6);  s = E4M3_RNE_SATFINITE(t);
 *   d  = fl32(dec(s)*g);  y = fl32(x/d);  q = E2M1_RNE_SATFINITE(y);
 *   if dec(s)==0 or d==0 every code of the block is +0 (0x0).
 * All fp32 steps are single IEEE operations (compile with -ffp-contract=off).
 *
 * Encoders are written as nearest-point searches over the code tables, the
 * plainest definition of "round to nearest, ties to even" onto a finite grid:
 * the nearest representable magnitude wins; on an exact tie the code whose
 * least significant bit is 0 wins; a magnitude beyond the largest finite
 * value maps to that value (satfinite).
 *
 * Parity pins live in tests/test_oracle_*.py.  The arithmetic order (6*g
 * first, true division by d) is a reading, since the pages do not fix it; the
 * pins hold this file to that reading at non-power-of-two global scales: an
 * exact rational evaluation of the steps above, rounded to binary32 after
 * each one, on inputs a few ulps from the E4M3 midpoints and the E2M1
 * decision boundaries, where the other plausible orders (amax/6/g, x*(1/d),
 * x/dec(s)/g) give different bytes.
 */
#include <math.h>
#include <stdint.h>
#include <stddef.h>
#include <string.h>

#define ORACLE_BLOCK 16

/* ---------------------------------------------------------------- codecs */

/* E2M1: 1 sign bit (bit 3), 2 exponent bits (bias 1), 1 mantissa bit.
 * exponent 0 is subnormal: m*0.5.  Magnitudes: 0 .5 1 1.5 2 3 4 6. */
double oracle_e2m1_decode(int code)
{
    int s = (code >> 3) & 1, e = (code >> 1) & 3, m = code & 1;
    double v = (e == 0) ? 0.5 * m : ldexp(1.0 + 0.5 * m, e - 1);
    return s ? -v : v;
}

/* E4M3 ("fn" flavour): 1 sign bit, 4 exponent bits (bias 7), 3 mantissa bits,
 * no infinities, S.1111.111 is NaN, max finite 448, exponent 0 subnormal m*2^-9. */
double oracle_e4m3_decode(int code)
{
    int s = (code >> 7) & 1, e = (code >> 3) & 15, m = code & 7;
    double v;
    if (e == 15 && m == 7) return NAN;
    v = (e == 0) ? ldexp((double)m, -9) : ldexp(1.0 + m / 8.0, e - 7);
    return s ? -v : v;
}

/* nearest-point search over magnitude codes 0..maxcode, ties to even code */
static int nearest_code(double a, int maxcode, double (*dec)(int))
{
    int best = 0, c;
    double bestd = fabs(a - dec(0));
    /* at or beyond the largest magnitude the nearest code is the largest one
     * (satfinite); deciding it here also keeps huge |a| away from distances
     * that float64 can no longer tell apart */
    if (a >= dec(maxcode)) return maxcode;
    for (c = 1; c <= maxcode; ++c) {
        double dist = fabs(a - dec(c));
        if (dist < bestd || (dist == bestd && (c & 1) == 0)) {
            best = c;
            bestd = dist;
        }
    }
    return best;
}

int oracle_e2m1_encode(float y)
{
    int sign = signbit(y) ? 0x8 : 0x0;
    return sign | nearest_code(fabs((double)y), 7, oracle_e2m1_decode);
}

int oracle_e4m3_encode(float t)
{
    int sign = signbit(t) ? 0x80 : 0x00;
    return sign | nearest_code(fabs((double)t), 0x7E, oracle_e4m3_decode);
}

/* ------------------------------------------------------------- layout (a5) */

/* Byte offset of the scale of (row r, scale column c) in the swizzled
 * scale-factor buffer: 128-row x 4-column atoms of 512 bytes, atoms ordered
 * row-block major then column-block; inside an atom, row r%32 selects a
 * 16-byte line, (r%128)/32 a 4-byte word, c%4 the byte.  Scale columns are
 * padded to a multiple of 4 and rows to a multiple of 128.  (The pages give
 * no layout; this is the layout the sm_100 block-scaled tensor-core path
 * reads, stated in the public PTX ISA and cuBLAS documentation.) */
int64_t oracle_sf_offset(int64_t r, int64_t c, int64_t K)
{
    int64_t c4 = ((K / ORACLE_BLOCK) + 3) / 4 * 4;
    return ((r / 128) * (c4 / 4) + c / 4) * 512 + (r % 32) * 16 + ((r % 128) / 32) * 4 + (c % 4);
}

int64_t oracle_sf_bytes(int64_t rows, int64_t K)
{
    int64_t c4 = ((K / ORACLE_BLOCK) + 3) / 4 * 4;
    return (rows + 127) / 128 * 128 * c4;
}

/* ------------------------------------------------------ global scale (a1) */

/* g = amax / (6*448): the per-tensor FP32 scale that maps the tensor's
 * largest magnitude onto the largest E2M1 value times the largest E4M3
 * value.  An all-zero tensor gets g = 1. */
float oracle_global_scale(const float *x, int64_t n)
{
    float amax = 0.0f;
    int64_t i;
    for (i = 0; i < n; ++i) {
        float a = fabsf(x[i]);
        if (a > amax) amax = a;
    }
    if (amax == 0.0f) return 1.0f;
    return amax / 2688.0f;
}

/* ------------------------------------------------------- quantize (a2-a5) */

/* Quantize rows x K (row stride ld) with global scale g.  codes: rows*K/2
 * bytes, row stride K/2, element 2j in the low nibble of byte j.  sf: the
 * swizzled buffer of a (possibly fused) tensor with sf_rows_total rows; this
 * call writes rows [sf_row0, sf_row0 + rows).  Padding rows are not touched
 * (callers zero the buffer first). */
void oracle_quantize(const float *x, int64_t rows, int64_t K, int64_t ld, float g,
                     uint8_t *codes, uint8_t *sf, int64_t sf_row0)
{
    int64_t r;
    float g6 = 6.0f * g;
#ifdef _OPENMP
#pragma omp parallel for schedule(static)
#endif
    for (r = 0; r < rows; ++r) {
        int64_t b;
        for (b = 0; b < K / ORACLE_BLOCK; ++b) {
            const float *xb = x + r * ld + b * ORACLE_BLOCK;
            float amax = 0.0f, t, decs, d;
            int s, i, q[ORACLE_BLOCK];
            for (i = 0; i < ORACLE_BLOCK; ++i) {
                float a = fabsf(xb[i]);
                if (a > amax) amax = a;
            }
            t = amax / g6;
            s = oracle_e4m3_encode(t);
            decs = (float)oracle_e4m3_decode(s);
            d = decs * g;
            for (i = 0; i < ORACLE_BLOCK; ++i) {
                if (decs == 0.0f || d == 0.0f) {
                    q[i] = 0;
                } else {
                    float y = xb[i] / d;
                    q[i] = oracle_e2m1_encode(y);
                }
            }
            for (i = 0; i < ORACLE_BLOCK / 2; ++i)
                codes[r * (K / 2) + b * (ORACLE_BLOCK / 2) + i] =
                    (uint8_t)(q[2 * i] | (q[2 * i + 1] << 4));
            sf[oracle_sf_offset(sf_row0 + r, b, K)] = (uint8_t)s;
        }
    }
}

/* ------------------------------------------------------ harmonize (a6) */

/* Rewrite the scales of a fused group of n modules (module m owns fused rows
 * [row_offsets[m], row_offsets[m+1])) from per-module global scales gs[m] to
 * one shared scale g* = max_m gs[m]: every scale byte s of module m becomes
 * E4M3_RNE_SATFINITE(fl32(dec(s) * fl32(gs[m] / g*))).  Codes are untouched.
 * Returns g*. */
float oracle_harmonize(uint8_t *sf, int64_t K, int n, const int64_t *row_offsets,
                       const float *gs)
{
    float gstar = gs[0];
    int m;
    for (m = 1; m < n; ++m)
        if (gs[m] > gstar) gstar = gs[m];
    for (m = 0; m < n; ++m) {
        float ratio = gs[m] / gstar;
        int64_t r, c;
        for (r = row_offsets[m]; r < row_offsets[m + 1]; ++r)
            for (c = 0; c < K / ORACLE_BLOCK; ++c) {
                uint8_t *p = sf + oracle_sf_offset(r, c, K);
                float v = (float)oracle_e4m3_decode(*p) * ratio;
                *p = (uint8_t)oracle_e4m3_encode(v);
            }
    }
    return gstar;
}

/* ------------------------------------------------------ dequantize (a7) */

/* out[r*K + k] = dec(q) * dec(s) * g in float64 (exact: 2 x 4 x 24 bits). */
void oracle_dequantize(const uint8_t *codes, const uint8_t *sf, int64_t rows, int64_t K,
                       float g, int64_t sf_row0, double *out)
{
    int64_t r;
#ifdef _OPENMP
#pragma omp parallel for schedule(static)
#endif
    for (r = 0; r < rows; ++r) {
        int64_t k;
        for (k = 0; k < K; ++k) {
            uint8_t byte = codes[r * (K / 2) + k / 2];
            int q = (k & 1) ? (byte >> 4) : (byte & 15);
            int s = sf[oracle_sf_offset(sf_row0 + r, k / ORACLE_BLOCK, K)];
            out[r * K + k] = oracle_e2m1_decode(q) * oracle_e4m3_decode(s) * (double)g;
        }
    }
}

/* ------------------------------------------------- brute-force GEMM (a7-a8) */

/* y[m*N+n] = alpha * sum_k a[m*K+k]*b[n*K+k] and yabs = alpha * sum |.|,
 * in float64, plain triple loop (the pinned definition for small shapes). */
void oracle_gemm_f64(const double *a, const double *b, int64_t M, int64_t N, int64_t K,
                     double alpha, double *y, double *yabs)
{
    int64_t m;
#ifdef _OPENMP
#pragma omp parallel for schedule(static)
#endif
    for (m = 0; m < M; ++m) {
        int64_t n;
        for (n = 0; n < N; ++n) {
            double acc = 0.0, accabs = 0.0;
            int64_t k;
            for (k = 0; k < K; ++k) {
                double p = a[m * K + k] * b[n * K + k];
                acc += p;
                accabs += fabs(p);
            }
            y[m * N + n] = alpha * acc;
            if (yabs) yabs[m * N + n] = fabs(alpha) * accabs;
        }
    }
}

int oracle_num_threads(void)
{
#ifdef _OPENMP
    extern int omp_get_max_threads(void);
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Gather the scale bytes of the given rows out of a swizzled buffer into a
 * plain [nrows, K/16] row-major array (used to compare sampled rows). */
void oracle_sf_gather(const uint8_t *sf, const int64_t *rows, int64_t nrows, int64_t K,
                      uint8_t *out)
{
    int64_t i, c;
    for (i = 0; i < nrows; ++i)
        for (c = 0; c < K / ORACLE_BLOCK; ++c)
            out[i * (K / ORACLE_BLOCK) + c] = sf[oracle_sf_offset(rows[i], c, K)];
}

/* ---------------------------------------------- GDN gate activations (next) */

/* The two gate projections of a GDN layer feed log-space gates (ta-paperlens
 * page, "前提2"): the raw projection a_t goes through softplus and then the
 * exponential to give alpha_t, how much of the state is kept (close to 1 =
 * forget little), and b_t through the logistic sigmoid to give beta_t, the
 * write strength.  The per-head decay scale and bias the model multiplies
 * in are not on the pages, so this reading uses 1 and 0:
 *   alpha = exp(-softplus(a)),  beta = 1 / (1 + exp(-b)),
 * columns [0, n_a) of the fused gate GEMM output are a, the rest b.  float64. */
static double softplus(double y)
{
    return y > 0.0 ? y + log1p(exp(-y)) : log1p(exp(y));
}

void oracle_gdn_gates(const double *y, int64_t rows, int64_t N, int64_t n_a, double *out)
{
    int64_t i;
    for (i = 0; i < rows * N; ++i) {
        double v = y[i];
        out[i] = (i % N) < n_a ? exp(-softplus(v)) : 1.0 / (1.0 + exp(-v));
    }
}

/* ------------------------------------------------ FP8 KV quantize (next) */

/* Static per-tensor FP8 (E4M3) quantization of the KV cache (arxiv-wiki page,
 * "주요 결과": a static per-tensor FP8 scale shipped with the checkpoint
 * recovers most of the FP8 KV penalty): q = E4M3_RNE_SATFINITE(fl32(x / s))
 * with the sign in bit 7; dequantization is dec(q) * s. */
void oracle_fp8_quantize(const float *x, int64_t n, float s, uint8_t *q)
{
    int64_t i;
    for (i = 0; i < n; ++i) {
        float t = x[i] / s;      /* one IEEE fp32 division */
        q[i] = (uint8_t)oracle_e4m3_encode(t);
    }
}
