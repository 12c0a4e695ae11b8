// quantize.cuh -- NVFP4 encoder kernels for sm_100a: per-tensor global scale,
// activation/weight quantize (E2M1 codes + swizzled E4M3 block scales; a
// TMA-fed streaming kernel and a generic per-row kernel), fused-group
// global-scale harmonization, and the rows built on the same encoder:
// fake-quant (quantize then dequantize, with error sums), static-scale FP8
// E4M3 quantize, the re-quantizing harmonize, and the quantize fused into
// the RMSNorm that produces an activation.
//
// Format (web pages on arXiv 2609.04098; ta-paperlens page, section "前提1";
// arxiv-wiki page, "접근 방법"): 4-bit E2M1 values, one E4M3 scale per 16
// consecutive elements equal to the block maximum / 6, and one FP32 scale per
// tensor.  Arithmetic per block (each step one IEEE fp32 operation):
//   g6 = 6*g;  s = E4M3(amax/g6);  d = dec(s)*g;  q_i = E2M1(x_i/d)
// with round-to-nearest-even and saturation at 448 / 6; a block whose scale
// or d is zero gets +0 codes.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cstdint>

#include "ptx.cuh"

namespace nvfp4 {

// byte offset of the scale of (row r, block column c) in the swizzled buffer
// (128-row x 4-column atoms of 512 bytes; K % 64 == 0 so K/64 atoms per row block)
__device__ __forceinline__ int64_t sf_index(int64_t r, int64_t c, int64_t K) {
  return ((r >> 7) * (K >> 6) + (c >> 2)) * 512 + (r & 31) * 16 + ((r >> 5) & 3) * 4 + (c & 3);
}

// ------------------------------------------------------------ input blocks
// One 16-element scale block of the input as loaded: bf16 as eight packed
// pairs (element 2i in the low half of word i), fp32 as sixteen floats.
template <typename T>
struct Block16;

template <>
struct Block16<__nv_bfloat16> {
  uint32_t w[8];
  __device__ __forceinline__ void zero() {
#pragma unroll
    for (int i = 0; i < 8; ++i) w[i] = 0u;
  }
  __device__ __forceinline__ void set(uint4 a, uint4 b) {
    w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w; w[4] = b.x; w[5] = b.y; w[6] = b.z; w[7] = b.w;
  }
  __device__ __forceinline__ void load(const __nv_bfloat16 *p) {
    set(__ldg(reinterpret_cast<const uint4 *>(p)), __ldg(reinterpret_cast<const uint4 *>(p) + 1));
  }
  __device__ __forceinline__ void load_shared(const __nv_bfloat16 *p) {
    const uint4 *q = reinterpret_cast<const uint4 *>(p);
    set(q[0], q[1]);
  }
  __device__ __forceinline__ float elem(int e) const {      // e a compile-time index
    return __uint_as_float((e & 1) ? (w[e >> 1] & 0xFFFF0000u) : (w[e >> 1] << 16));
  }
  // max |x| of the block: a tree of bf16x2 max-of-magnitudes, then the two halves
  __device__ __forceinline__ float amax() const {
    uint32_t a = bmax2(bmax2(bmax2(w[0], w[1]), bmax2(w[2], w[3])), bmax2(bmax2(w[4], w[5]), bmax2(w[6], w[7])));
    a &= 0x7FFF7FFFu;
    return fmaxf(__uint_as_float(a << 16), __uint_as_float(a & 0xFFFF0000u));
  }
  static __device__ __forceinline__ uint32_t bmax2(uint32_t x, uint32_t y) {
    uint32_t m;
    asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(m) : "r"(x), "r"(y));
    return m;
  }
};

template <>
struct Block16<float> {
  float v[16];
  __device__ __forceinline__ void zero() {
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = 0.0f;
  }
  __device__ __forceinline__ void set4(int i, float4 a) {
    v[4 * i] = a.x; v[4 * i + 1] = a.y; v[4 * i + 2] = a.z; v[4 * i + 3] = a.w;
  }
  __device__ __forceinline__ void load(const float *p) {
#pragma unroll
    for (int i = 0; i < 4; ++i) set4(i, __ldg(reinterpret_cast<const float4 *>(p) + i));
  }
  __device__ __forceinline__ void load_shared(const float *p) {
#pragma unroll
    for (int i = 0; i < 4; ++i) set4(i, reinterpret_cast<const float4 *>(p)[i]);
  }
  __device__ __forceinline__ float elem(int e) const { return v[e]; }
  __device__ __forceinline__ float amax() const {
    float m = 0.0f;
#pragma unroll
    for (int i = 0; i < 16; ++i) m = fmaxf(m, fabsf(v[i]));
    return m;
  }
};

__device__ __forceinline__ float to_f32(__nv_bfloat16 h) { return __bfloat162float(h); }
__device__ __forceinline__ float to_f32(float f) { return f; }

// --------------------------------------------------------------- the encoder
// The definition (each step one IEEE fp32 operation, round to nearest even):
//   s = E4M3(fl32(amax / fl32(6g))),  d = fl32(dec(s) * g),  q_i = E2M1(fl32(x_i / d)).
// The encoder reaches the same codes without a division.  With
// r = fl32(fl32(1/dec(s)) * fl32(1/g)) (relative error <= 3u, u = 2^-24), the
// products y- = fl32(x * fl32(r(1 - 2^-21))) and y+ = fl32(x * fl32(r(1 + 2^-21)))
// bracket the exact quotient fl32(x/d) in magnitude (margin >= u after all
// roundings), and E2M1 rounding is monotone in |y|: where the hardware
// conversion gives the same code for y- and y+, that is the code of
// fl32(x/d).  Where the two codes differ (the bracket is far narrower than the
// grid, so they are neighbours and the bracket holds exactly one rounding
// boundary T, one of 0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5), the side of T on
// which fl32(x/d) falls is decided exactly (see quotient_vs).  The scale
// byte is decided the same way from amax * fl32(1/g6) widened by 2^-21 both
// ways, with the midpoint between the two candidate E4M3 values as T.  With
// bf16 inputs, quotients land on or next to a boundary for a few elements
// in a thousand (exact ties included), so this path must stay cheap.
constexpr float kWidenLo = 0.999999523162841796875f;   // 1 - 2^-21
constexpr float kWidenHi = 1.000000476837158203125f;   // 1 + 2^-21

struct EncodeConsts {
  float g, g6, rg;          // g, fl32(6g), fl32(1/g)
  float rg6_lo, rg6_hi;     // fl32(1/g6) widened down and up by 2^-21
  bool fast;                // g well inside the normal range: products neither overflow nor underflow
};

__device__ __forceinline__ EncodeConsts encode_consts_of(float g) {
  EncodeConsts k;
  k.g = g;
  k.g6 = __fmul_rn(6.0f, k.g);
  k.rg = __frcp_rn(k.g);
  const float rg6 = __frcp_rn(k.g6);
  k.rg6_lo = __fmul_rn(rg6, kWidenLo);
  k.rg6_hi = __fmul_rn(rg6, kWidenHi);
  k.fast = k.g >= 8.67361738e-19f && k.g <= 1.15292150e18f;   // 2^-60 .. 2^60
  return k;
}

__device__ __forceinline__ EncodeConsts encode_consts(const float *gscale) { return encode_consts_of(__ldg(gscale)); }

// Shared table of fl32(1/dec(s)) for every finite non-negative E4M3 byte s;
// entry 0 is unused (a zero scale short-circuits to zero codes).
__device__ __forceinline__ void fill_rcp_table(float *tab) {
  for (int i = threadIdx.x; i < 128; i += blockDim.x)
    tab[i] = i == 0 || i == 127 ? 0.0f : __frcp_rn(e4m3_to_f32((uint32_t)i));
}

__device__ __noinline__ float div_rn_slow(float a, float b) { return __fdiv_rn(a, b); }

// Sign of fl32(a / b) - T for a >= 0 and b > 0 normal, T > 0 a normal float
// with at most five significant bits (an E2M1 boundary or an E4M3 midpoint).
// With h+ and h- half the float spacing above and below T, RNE gives
// fl32(a/b) > T exactly when a/b > T + h+, and fl32(a/b) < T exactly when
// a/b < T - h- (at either bound the tie goes to T, whose last significand bit
// is 0); that is, when D = a - T*b is above h+ * b or below -h- * b.  One FMA
// gives D: T*b has at most 29 significant bits and a at most 24, so wherever
// a/b lies within 2^-17 of T the exact difference is a multiple of
// 2^(e - 28) below 2^(e - 16) (e the exponent of T*b), i.e. it fits in 24
// bits and the FMA returns it exactly; farther from T the rounded D keeps its
// sign and stays far from h+-*b, so the comparison still decides correctly.
// h+-*b are exact (powers of two times b, far above the subnormal range for
// the scales this library accepts).
__device__ __forceinline__ int quotient_vs(float a, float b, float T) {
  const uint32_t tb = __float_as_uint(T);
  const float hp = __uint_as_float((tb & 0x7F800000u) - (24u << 23));     // 2^(e_T - 24)
  const float hm = (tb & 0x7FFFFFu) == 0u ? __fmul_rn(hp, 0.5f) : hp;    // below a power of two the spacing halves
  const float D = __fmaf_rn(-T, b, a);
  if (D > __fmul_rn(hp, b)) return 1;
  if (D < -__fmul_rn(hm, b)) return -1;
  return 0;
}

// The E2M1 rounding boundary between magnitudes m and m + 1 (m = 0..6):
// 0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.  Their fp32 patterns have zero low 21
// bits; shifted right by 21 they are 0x1F4 plus 0, 6, 9, 11, 13, 15, 17.
__device__ __forceinline__ float e2m1_boundary(uint32_t m) {
  constexpr unsigned long long kOff =
      (6ull << 5) | (9ull << 10) | (11ull << 15) | (13ull << 20) | (15ull << 25) | (17ull << 30);
  return __uint_as_float((0x1F4u + (uint32_t)((kOff >> (5u * m)) & 31u)) << 21);
}

// E2M1 codes of eight values under the two bracketing multipliers: the code
// word from r- and the code word from r+ (element 2j in the low nibble of byte j).
__device__ __forceinline__ void e2m1x8_bracket(float x0, float x1, float x2, float x3, float x4, float x5,
                                               float x6, float x7, float rlo, float rhi, uint32_t &wlo,
                                               uint32_t &whi) {
  asm("{\n\t"
      ".reg .b64 a0, a1, a2, a3, bl, bh, d;\n\t"
      ".reg .f32 p0, p1;\n\t"
      ".reg .b8 l0, l1, l2, l3, h0, h1, h2, h3;\n\t"
      "mov.b64 bl, {%10, %10};\n\t"
      "mov.b64 bh, {%11, %11};\n\t"
      "mov.b64 a0, {%2, %3};\n\t"
      "mov.b64 a1, {%4, %5};\n\t"
      "mov.b64 a2, {%6, %7};\n\t"
      "mov.b64 a3, {%8, %9};\n\t"
      "mul.rn.f32x2 d, a0, bl;\n\t mov.b64 {p0, p1}, d;\n\t cvt.rn.satfinite.e2m1x2.f32 l0, p1, p0;\n\t"
      "mul.rn.f32x2 d, a1, bl;\n\t mov.b64 {p0, p1}, d;\n\t cvt.rn.satfinite.e2m1x2.f32 l1, p1, p0;\n\t"
      "mul.rn.f32x2 d, a2, bl;\n\t mov.b64 {p0, p1}, d;\n\t cvt.rn.satfinite.e2m1x2.f32 l2, p1, p0;\n\t"
      "mul.rn.f32x2 d, a3, bl;\n\t mov.b64 {p0, p1}, d;\n\t cvt.rn.satfinite.e2m1x2.f32 l3, p1, p0;\n\t"
      "mul.rn.f32x2 d, a0, bh;\n\t mov.b64 {p0, p1}, d;\n\t cvt.rn.satfinite.e2m1x2.f32 h0, p1, p0;\n\t"
      "mul.rn.f32x2 d, a1, bh;\n\t mov.b64 {p0, p1}, d;\n\t cvt.rn.satfinite.e2m1x2.f32 h1, p1, p0;\n\t"
      "mul.rn.f32x2 d, a2, bh;\n\t mov.b64 {p0, p1}, d;\n\t cvt.rn.satfinite.e2m1x2.f32 h2, p1, p0;\n\t"
      "mul.rn.f32x2 d, a3, bh;\n\t mov.b64 {p0, p1}, d;\n\t cvt.rn.satfinite.e2m1x2.f32 h3, p1, p0;\n\t"
      "mov.b32 %0, {l0, l1, l2, l3};\n\t"
      "mov.b32 %1, {h0, h1, h2, h3};\n\t"
      "}"
      : "=r"(wlo), "=r"(whi)
      : "f"(x0), "f"(x1), "f"(x2), "f"(x3), "f"(x4), "f"(x5), "f"(x6), "f"(x7), "f"(rlo), "f"(rhi));
}

// E2M1 code (nibble) of one value, satfinite, round to nearest even.
__device__ __forceinline__ uint32_t e2m1_code(float y) {
  uint16_t b;
  asm("{\n\t.reg .b8 c;\n\tcvt.rn.satfinite.e2m1x2.f32 c, %1, %1;\n\tcvt.u16.u8 %0, c;\n\t}" : "=h"(b) : "f"(y));
  return b & 0xFu;
}

// Settle the elements whose bracket codes differ (nonzero nibbles of
// lo ^ hi, elements 8w..8w+7 in word w): the lower candidate magnitude m
// fixes the boundary T between m and m + 1; the element takes m + 1 above T,
// m below, the even one of the two on T.  `src` is the block in memory
// (elements re-read by index).  32-bit words throughout.
template <typename T>
__device__ __forceinline__ uint32_t settle_word(const T *src, uint32_t lo, uint32_t hi, float d) {
  uint32_t m = lo ^ hi;
  while (m != 0u) {
    const int sh = (__ffs(m) - 1) & ~3;
    m &= ~(0xFu << sh);
    const uint32_t mlow = min((lo >> sh) & 7u, (hi >> sh) & 7u);
    const float xv = to_f32(src[sh >> 2]);
    const int c = quotient_vs(fabsf(xv), d, e2m1_boundary(mlow));
    const uint32_t mag = c > 0 ? mlow + 1u : (c < 0 ? mlow : ((mlow & 1u) ? mlow + 1u : mlow));
    lo = (lo & ~(0xFu << sh)) | ((mag | ((__float_as_uint(xv) >> 28) & 8u)) << sh);
  }
  return lo;
}

template <typename T>
__device__ __forceinline__ uint2 settle_codes(const T *src, uint32_t lo0, uint32_t hi0, uint32_t lo1, uint32_t hi1,
                                              float d) {
  if (lo0 != hi0) lo0 = settle_word(src, lo0, hi0, d);
  if (lo1 != hi1) lo1 = settle_word(src + 8, lo1, hi1, d);
  return make_uint2(lo0, lo1);
}

// The whole block by the definition (extreme global scales only).
template <typename T>
__device__ __noinline__ uint2 encode16_ieee(const T *src, uint32_t s, float g) {
  const float d = __fmul_rn(e4m3_to_f32(s), g);
  if (d == 0.0f) return make_uint2(0u, 0u);
  uint32_t w[2] = {0u, 0u};
  for (int e = 0; e < 16; ++e) w[e >> 3] |= e2m1_code(__fdiv_rn(to_f32(src[e]), d)) << ((e & 7) * 4);
  return make_uint2(w[0], w[1]);
}

// Encode one 16-element block held in registers (`src` is the same block in
// memory, read only on the rare settling paths).  Returns the two code
// words; the scale byte goes to *s_out.
template <typename T>
__device__ __forceinline__ uint2 encode16(const Block16<T> &b, const EncodeConsts &k, const float *rcp_tab,
                                          const T *src, uint32_t *s_out) {
  const float amax = b.amax();
  uint16_t pr;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(pr) : "f"(__fmul_rn(amax, k.rg6_hi)),
      "f"(__fmul_rn(amax, k.rg6_lo)));
  uint32_t s = pr & 0xFFu;
  const uint32_t s_up = (uint32_t)(pr >> 8);
  if (!k.fast) {
    s = f32_to_e4m3(div_rn_slow(amax, k.g6));
  } else if (s != s_up) {
    // neighbouring E4M3 values: decide against their midpoint
    const float mid = __fmul_rn(__fadd_rn(e4m3_to_f32(s), e4m3_to_f32(s_up)), 0.5f);
    const int c = quotient_vs(amax, k.g6, mid);
    s = c > 0 ? s_up : (c < 0 ? s : ((s & 1u) ? s_up : s));
  }
  *s_out = s;
  if (s == 0u) return make_uint2(0u, 0u);
  if (!k.fast) return encode16_ieee(src, s, k.g);
  const float r = __fmul_rn(rcp_tab[s], k.rg);
  const float rlo = __fmul_rn(r, kWidenLo), rhi = __fmul_rn(r, kWidenHi);
  uint32_t lo0, hi0, lo1, hi1;
  e2m1x8_bracket(b.elem(0), b.elem(1), b.elem(2), b.elem(3), b.elem(4), b.elem(5), b.elem(6), b.elem(7), rlo, rhi,
                 lo0, hi0);
  e2m1x8_bracket(b.elem(8), b.elem(9), b.elem(10), b.elem(11), b.elem(12), b.elem(13), b.elem(14), b.elem(15), rlo,
                 rhi, lo1, hi1);
  if (((lo0 ^ hi0) | (lo1 ^ hi1)) != 0u) return settle_codes(src, lo0, hi0, lo1, hi1, __fmul_rn(e4m3_to_f32(s), k.g));
  return make_uint2(lo0, lo1);
}

struct QuantizeParams {
  const void *x;
  int64_t rows, K, ld_x;
  const float *gscale;
  uint8_t *codes;
  uint8_t *sf;
  int64_t sf_row0;
  int64_t pad_rows;  // padding rows (zeroed) after this call's rows, or 0
  unsigned *err;
};

// Programmatic-dependent-launch prologue of every kernel that reads what an
// earlier kernel wrote: wait for the stream's preceding grid, then let the
// next one be scheduled (it in turn waits for this grid where it must).
__device__ __forceinline__ void pdl_prologue() {
  griddep_wait();
  if (threadIdx.x == 0) griddep_launch_dependents();
}

// Zero the scale bytes of `pad_rows` padding rows starting at scale row
// `first` (fewer than 128 rows of K/16 columns: 32-bit index arithmetic
// unless K is huge), spread over the whole grid.
__device__ __forceinline__ void zero_pad_scales(uint8_t *sf, int64_t first, int64_t pad_rows, int64_t K) {
  const int64_t ncols = K >> 4;
  const int64_t pad_bytes = pad_rows * ncols;
  const int64_t tid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t nthreads = static_cast<int64_t>(gridDim.x) * blockDim.x;
  if (pad_bytes < (int64_t(1) << 31)) {
    const uint32_t nc = (uint32_t)ncols;
    for (uint32_t i = (uint32_t)tid; i < (uint32_t)pad_bytes; i += (uint32_t)nthreads) {
      const uint32_t rr = i / nc, c = i - rr * nc;
      sf[sf_index(first + rr, c, K)] = 0;
    }
  } else {
    for (int64_t i = tid; i < pad_bytes; i += nthreads) sf[sf_index(first + i / ncols, i % ncols, K)] = 0;
  }
}

// Generic path (any row offset inside a fused buffer, any row count): one
// warp per 512-column segment of a row, lane l encodes block l of it (32
// bytes of bf16 per lane, 1 KB contiguous per warp), UNROLL segments loaded
// before any is encoded.  Codes are 8-byte stores, each scale byte is stored
// on its own.
template <typename T, int UNROLL>
__global__ void __launch_bounds__(256) quantize_rows_kernel(QuantizeParams p) {
  __shared__ float rcp_tab[128];
  fill_rcp_table(rcp_tab);
  pdl_prologue();
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const uint32_t warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const uint32_t nwarps = (gridDim.x * blockDim.x) >> 5;
  const uint32_t nseg = (uint32_t)((p.K + 511) >> 9);
  const uint32_t units = (uint32_t)p.rows * nseg;
  const T *x = static_cast<const T *>(p.x);
  // the encoder constants are read after the first loads are in flight, so
  // the two round trips overlap (few-row calls run a single iteration)
  EncodeConsts kc;
  bool have_kc = false;

  for (uint32_t u0 = warp * UNROLL; u0 < units; u0 += nwarps * UNROLL) {
    Block16<T> in[UNROLL];
    int64_t row[UNROLL];
    int col[UNROLL];
#pragma unroll
    for (int j = 0; j < UNROLL; ++j) {
      const uint32_t u = u0 + j;
      row[j] = u / nseg;
      col[j] = (int)(u - (uint32_t)row[j] * nseg) * 512 + lane * 16;
      in[j].zero();
      if (u < units && col[j] < p.K) in[j].load(x + row[j] * p.ld_x + col[j]);
    }
    if (!have_kc) {
      kc = encode_consts(p.gscale);
      have_kc = true;
    }
#pragma unroll
    for (int j = 0; j < UNROLL; ++j) {
      if (u0 + j < units && col[j] < p.K) {
        uint32_t s;
        const uint2 word = encode16(in[j], kc, rcp_tab, x + row[j] * p.ld_x + col[j], &s);
        *reinterpret_cast<uint2 *>(p.codes + row[j] * (p.K >> 1) + (col[j] >> 1)) = word;
        p.sf[sf_index(p.sf_row0 + row[j], col[j] >> 4, p.K)] = static_cast<uint8_t>(s);
      }
    }
  }
  zero_pad_scales(p.sf, p.sf_row0 + p.rows, p.pad_rows, p.K);
}

// Streaming path for calls whose scale rows start on a 128-row boundary and
// that own every row of their last 128-row block (the activation quantize
// always does).  One CTA of 32 warps per SM, persistent over units of 128
// rows x COLS columns (64 KB of input; COLS = 256 bf16 / 128 fp32) that
// stream through a ring of shared-memory stages by 2D TMA (rows past `rows`
// and columns past K read as zeros, so padding rows get zero scales).  Every
// warp encodes: lane l takes block l % (COLS/16) of row l / (COLS/16) of
// each step and writes its 8 code bytes and its scale byte straight to
// global memory (a warp's scale bytes fill 4-byte runs of the swizzled atoms,
// which the L2 merges).  Each warp hands a stage back on its own; lane 0 of
// warp 0 also refills it, once all 32 warps have, with the unit STAGES
// ahead.  No warp is set aside for loading, so all 32 warps issue encoder
// work (the encoder is issue-bound).
template <typename T>
struct QTmaCfg {
  static constexpr int ROWS = 128;
  static constexpr int COLS = sizeof(T) == 2 ? 256 : 128;
  static constexpr int BPR = COLS / 16;                 // blocks per row
  static constexpr int RPS = 32 / BPR;                  // rows per warp step
  static constexpr int WARPS = 32;
  static constexpr int SPW = ROWS / RPS / WARPS;        // steps per warp per unit
  static constexpr int STAGE_BYTES = ROWS * COLS * (int)sizeof(T);
  static constexpr int STAGES = 3;
  static constexpr int THREADS = 32 * WARPS;
  static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + 2 * STAGES * 8 + 512 + 16;
  static_assert(ROWS % (RPS * WARPS) == 0 && SPW >= 1, "unit split");
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

template <typename T>
__global__ void __launch_bounds__(QTmaCfg<T>::THREADS, 1)
    quantize_tma_kernel(const __grid_constant__ CUtensorMap tmx, const QuantizeParams p) {
  using C = QTmaCfg<T>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *ring = smem;
  uint64_t *full = reinterpret_cast<uint64_t *>(ring + C::STAGES * C::STAGE_BYTES);
  uint64_t *empty = full + C::STAGES;
  float *rcp_tab = reinterpret_cast<float *>(empty + C::STAGES);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(rcp_tab + 128);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t nseg = (uint32_t)((p.K + C::COLS - 1) / C::COLS);
  const uint32_t units = (uint32_t)((p.rows + 127) >> 7) * nseg;
  const bool loader = threadIdx.x == 0;
  auto issue = [&](int st, uint32_t u) {
    const uint32_t rb = u / nseg, seg = u - rb * nseg;
    mbar_arrive_expect_tx(&full[st], C::STAGE_BYTES);
    tma_load_2d(ring + st * C::STAGE_BYTES, &tmx, &full[st], (int32_t)(seg * C::COLS), (int32_t)(rb * 128));
  };
  if (loader) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], C::WARPS);
    }
    *abort_flag = 0;
    fence_barrier_init();
    prefetch_tmap(&tmx);
  }
  fill_rcp_table(rcp_tab);
  pdl_prologue();
  __syncthreads();
  // loader only: stages with a copy issued (bit s) and the parity of the
  // phase that copy completes (bit s), for draining after a timeout
  uint32_t pend = 0u, par = 0u;
  if (loader) {
    // the first round of the ring (x is readable: the prologue has waited)
    for (int s = 0; s < C::STAGES; ++s) {
      const uint32_t u = blockIdx.x + (uint32_t)s * gridDim.x;
      if (u < units) {
        issue(s, u);
        pend |= 1u << s;
      }
    }
  }

  const int cb = lane % C::BPR, rsub = lane / C::BPR;
  const EncodeConsts kc = encode_consts(p.gscale);
  // per-lane offsets that do not change from unit to unit: this lane's rows
  // of the unit (codes: row * K/2) and their places in the scale atoms
  int64_t code_off[C::SPW];
  int sf_off[C::SPW];
#pragma unroll
  for (int j = 0; j < C::SPW; ++j) {
    const int r = (warp * C::SPW + j) * C::RPS + rsub;
    code_off[j] = (int64_t)r * (p.K >> 1);
    sf_off[j] = (r & 31) * 16 + (r >> 5) * 4 + (cb & 3);
  }
  const int64_t atoms_per_rb = p.K >> 6;
  int st = 0;
  uint32_t ph = 0;
  // (row block, segment) of unit u, advanced by gridDim.x units per step
  // without a division in the loop
  const uint32_t step_rb = gridDim.x / nseg, step_seg = gridDim.x - step_rb * nseg;
  uint32_t rb = blockIdx.x / nseg, seg = blockIdx.x - rb * nseg;
  for (uint32_t u = blockIdx.x; u < units; u += gridDim.x) {
    if (!mbar_wait_warp(&full[st], ph, p.err, ERR_EPILOGUE, abort_flag)) break;
    const T *sx = reinterpret_cast<const T *>(ring + st * C::STAGE_BYTES) + rsub * C::COLS + cb * 16;
    const int64_t gcol = (int64_t)seg * C::COLS + cb * 16;
    const bool col_ok = gcol < p.K;
    const int64_t row0 = (int64_t)rb * 128;
    uint8_t *codes_u = p.codes + row0 * (p.K >> 1) + (gcol >> 1);
    uint8_t *sf_u = p.sf + (((p.sf_row0 >> 7) + rb) * atoms_per_rb + (gcol >> 6)) * 512;
    Block16<T> in[C::SPW];
#pragma unroll
    for (int j = 0; j < C::SPW; ++j) in[j].load_shared(sx + (warp * C::SPW + j) * C::RPS * C::COLS);
#pragma unroll
    for (int j = 0; j < C::SPW; ++j) {
      const int r = (warp * C::SPW + j) * C::RPS + rsub;
      uint32_t s;
      const uint2 word = encode16(in[j], kc, rcp_tab, sx + (warp * C::SPW + j) * C::RPS * C::COLS, &s);
      if (col_ok) {
        if (row0 + r < p.rows) *reinterpret_cast<uint2 *>(codes_u + code_off[j]) = word;
        sf_u[sf_off[j]] = (uint8_t)s;
      }
    }
    // this warp is done with the stage (its reads happen-before the arrive)
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[st]);
    bool stop = false;
    if (loader) {
      // refill the stage with this CTA's unit STAGES ahead once every warp
      // has released it
      const uint32_t un = u + (uint32_t)C::STAGES * gridDim.x;
      if (un < units) {
        if (mbar_wait(&empty[st], ph, p.err, ERR_PRODUCER, abort_flag)) {
          issue(st, un);
          pend |= 1u << st;
          par = (par & ~(1u << st)) | ((ph ^ 1u) << st);
        } else {
          stop = true;
        }
      }
    }
    if (__any_sync(0xFFFFFFFFu, stop)) break;       // the whole warp leaves together
    if (++st == C::STAGES) { st = 0; ph ^= 1; }
    rb += step_rb;
    seg += step_seg;
    if (seg >= nseg) { seg -= nseg; ++rb; }
  }
  if (loader && *abort_flag) {
    // a wait ran out: let the copies still in flight land before the CTA's
    // shared memory goes away (a consumed copy's phase has completed already)
    volatile int never = 0;
    for (int s = 0; s < C::STAGES; ++s)
      if ((pend >> s) & 1u) mbar_wait(&full[s], (par >> s) & 1u, p.err, ERR_PRODUCER, &never);
  }
}

// ------------------------------------------------------ fake-quant (Q -> DQ)
// Value of an E2M1 code: magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6, sign in bit 3.
__device__ __forceinline__ float e2m1_to_f32(uint32_t c) {
  const uint32_t m = c & 7u;
  const uint32_t bits = m >= 2u ? ((126u + (m >> 1)) << 23) | ((m & 1u) << 22) : (m == 1u ? 0x3F000000u : 0u);
  return __uint_as_float(bits | ((c & 8u) << 28));
}

// Sixteen E2M1 codes (w.x holds elements 0-7, element 2j in the low nibble of
// byte j) times an E4M3 scale value ds, as floats: the conversion instruction
// takes one byte (two codes) to two halves, one half-precision multiply by ds
// (exact: the products have at most 6 significant bits and stay in the normal
// half range), then the widening to fp32 (exact).
__device__ __forceinline__ void e2m1x16_times_scale(uint2 w, float ds, float (&out)[16]) {
  const __half2 s2 = __float2half2_rn(ds);
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    uint32_t p[4];
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "mov.b32 {b0, b1, b2, b3}, %4;\n\t"
        "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t"
        "cvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
        "cvt.rn.f16x2.e2m1x2 %2, b2;\n\t"
        "cvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
        : "=r"(p[0]), "=r"(p[1]), "=r"(p[2]), "=r"(p[3])
        : "r"(h ? w.y : w.x));
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const __half2 q = __hmul2(*reinterpret_cast<const __half2 *>(&p[j]), s2);
      out[8 * h + 2 * j] = __low2float(q);
      out[8 * h + 2 * j + 1] = __high2float(q);
    }
  }
}

struct FakeQuantParams {
  const void *x;
  int64_t rows, K, ld_x;
  const float *gscale;
  void *out;
  int64_t ld_out;
  double *stats;     // [sum of squared error, sum of squared input], or null
};

template <typename OUT>
__device__ __forceinline__ void store16(OUT *dst, const float (&v)[16]);
template <>
__device__ __forceinline__ void store16<float>(float *dst, const float (&v)[16]) {
#pragma unroll
  for (int i = 0; i < 4; ++i) reinterpret_cast<float4 *>(dst)[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
}
template <>
__device__ __forceinline__ void store16<__nv_bfloat16>(__nv_bfloat16 *dst, const float (&v)[16]) {
  uint32_t w[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
    w[i] = *reinterpret_cast<uint32_t *>(&h);
  }
  reinterpret_cast<uint4 *>(dst)[0] = make_uint4(w[0], w[1], w[2], w[3]);
  reinterpret_cast<uint4 *>(dst)[1] = make_uint4(w[4], w[5], w[6], w[7]);
}

// Every element replaced by the NVFP4 value it quantizes to (the same
// encoder as the quantize kernels, then dec(q) * dec(s) * g: the first
// product is exact, so the result is fl32 of the exact value), plus the
// sums of the squared error against the exact value and of the squared
// input.  One warp per 512-column row segment, lane l owning block l, like
// quantize_rows_kernel.
// The sums are taken in fp32 over each 16-element block and in float64
// across blocks, so that no element needs a float64 conversion (those ran
// on the conversion pipe, which set the kernel's time).  The error of an
// element, x - q with q = dec(q)*dec(s)*g, is formed from p = fl32(q) and
// its remainder r = q - p (one FMA, exact): x - p is exact wherever q is
// non-zero and unsaturated (x and p within a factor of two), so d = x - p - r
// carries one rounding.  A block's sums of non-negative fp32 terms then
// carry a relative error below 18 * 2^-24 (about 1.1e-6); the float64 sum
// across blocks adds nothing visible at that level.
template <typename T, typename OUT>
__global__ void __launch_bounds__(256, 4) fake_quant_kernel(FakeQuantParams p) {
  __shared__ float rcp_tab[128];
  fill_rcp_table(rcp_tab);
  pdl_prologue();
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const uint32_t warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const uint32_t nwarps = (gridDim.x * blockDim.x) >> 5;
  const uint32_t nseg = (uint32_t)((p.K + 511) >> 9);
  const uint32_t units = (uint32_t)p.rows * nseg;
  const EncodeConsts kc = encode_consts(p.gscale);
  const T *x = static_cast<const T *>(p.x);
  OUT *out = static_cast<OUT *>(p.out);
  double se = 0.0, sx = 0.0;
  for (uint32_t u0 = warp * 2; u0 < units; u0 += nwarps * 2) {
    // two row segments per warp: both loads in flight before either is encoded
    Block16<T> bb[2];
    int64_t rr[2];
    int cc[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const uint32_t u = u0 + h;
      rr[h] = u / nseg;
      cc[h] = (int)(u - (uint32_t)rr[h] * nseg) * 512 + lane * 16;
      bb[h].zero();
      if (u < units && cc[h] < p.K) bb[h].load(x + rr[h] * p.ld_x + cc[h]);
    }
#pragma unroll
    for (int h = 0; h < 2; ++h) {
    if (u0 + h >= units || cc[h] >= p.K) continue;
    const int64_t row = rr[h];
    const int col = cc[h];
    const T *src = x + row * p.ld_x + col;
    const Block16<T> &b = bb[h];
    uint32_t s;
    const uint2 w = encode16(b, kc, rcp_tab, src, &s);
    // dec(q) * dec(s): the hardware turns two codes into two halves, and their
    // product with the scale is exact in f16 (at most 6 significant bits,
    // magnitudes from 2^-10 to 2688)
    float qv[16];
    e2m1x16_times_scale(w, e4m3_to_f32(s), qv);
    float v[16];
    float se_b = 0.0f, sx_b = 0.0f;
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      const float qs = qv[e];
      const float pv = __fmul_rn(qs, kc.g);
      v[e] = pv;
      const float xe = b.elem(e);
      const float d = __fsub_rn(__fsub_rn(xe, pv), __fmaf_rn(qs, kc.g, -pv));
      se_b = __fmaf_rn(d, d, se_b);
      sx_b = __fmaf_rn(xe, xe, sx_b);
    }
    se += (double)se_b;
    sx += (double)sx_b;
    store16<OUT>(out + row * p.ld_out + col, v);
    }
  }
  if (p.stats) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      se += __shfl_xor_sync(0xFFFFFFFFu, se, o);
      sx += __shfl_xor_sync(0xFFFFFFFFu, sx, o);
    }
    if (lane == 0) {
      atomicAdd(p.stats, se);
      atomicAdd(p.stats + 1, sx);
    }
  }
}

// ------------------------------------------------- FP8 (E4M3) KV quantize
// q = E4M3_RNE_SATFINITE(fl32(x / s)) with a static per-tensor scale s (sign
// in bit 7).  Decided like the block scales: x * fl32(1/s) widened by 2^-21
// both ways brackets fl32(x/s); equal hardware conversions are the answer,
// otherwise the two neighbouring codes' midpoint is compared exactly.
struct Fp8Params {
  const void *x;
  int64_t n;            // elements, a multiple of 8
  const float *scale;
  uint8_t *q;
};

// Midpoints between neighbouring E4M3 magnitudes: mid[m] = (dec(m) + dec(m + 1)) / 2
// for m = 0..125 (exact in fp32: at most five significant bits).
__device__ __forceinline__ void fill_e4m3_mid_table(float *tab) {
  for (int i = threadIdx.x; i < 128; i += blockDim.x)
    tab[i] = i < 126 ? __fmul_rn(__fadd_rn(e4m3_to_f32((uint32_t)i), e4m3_to_f32((uint32_t)i + 1u)), 0.5f) : 0.0f;
}

// The code of x where the two bracketing conversions disagree (neighbouring
// magnitudes m0 < m1): above their midpoint m1, below m0, on it the even one.
__device__ __forceinline__ uint32_t fp8_settle(float x, float s, uint32_t lo, uint32_t hi, const float *mid_tab) {
  const uint32_t ml = lo & 0x7Fu, mh = hi & 0x7Fu;
  const uint32_t m0 = min(ml, mh), m1 = max(ml, mh);
  const int c = quotient_vs(fabsf(x), s, mid_tab[m0]);
  const uint32_t m = c > 0 ? m1 : (c < 0 ? m0 : ((m0 & 1u) ? m1 : m0));
  return m | (__float_as_uint(x) >> 24 & 0x80u);
}

// Eight values to eight E4M3 codes (byte j = element j).  Each conversion
// instruction takes two elements; the words from the two bracketing
// multipliers are compared whole, and only bytes that differ are settled.
__device__ __forceinline__ uint2 fp8x8(const float (&v)[8], float s, float rlo, float rhi, const float *mid_tab) {
  uint32_t lo[2], hi[2];
#pragma unroll
  for (int w = 0; w < 2; ++w) {
    uint16_t l0, l1, h0, h1;
    const float *e = v + 4 * w;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(l0) : "f"(__fmul_rn(e[1], rlo)), "f"(__fmul_rn(e[0], rlo)));
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(l1) : "f"(__fmul_rn(e[3], rlo)), "f"(__fmul_rn(e[2], rlo)));
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(h0) : "f"(__fmul_rn(e[1], rhi)), "f"(__fmul_rn(e[0], rhi)));
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(h1) : "f"(__fmul_rn(e[3], rhi)), "f"(__fmul_rn(e[2], rhi)));
    lo[w] = (uint32_t)l0 | ((uint32_t)l1 << 16);
    hi[w] = (uint32_t)h0 | ((uint32_t)h1 << 16);
  }
  // differing bytes are settled one per lane per round: the warp runs as
  // many rounds as its lane with the most of them (mostly one), not one
  // round per byte position that any lane has
  uint32_t d0 = lo[0] ^ hi[0], d1 = lo[1] ^ hi[1];
  while ((d0 | d1) != 0u) {
    const bool w = d0 == 0u;
    const uint32_t d = w ? d1 : d0;
    const int sh = (__ffs(d) - 1) & ~7;
    const int k = (w ? 4 : 0) + (sh >> 3);
    if (w) d1 &= ~(0xFFu << sh); else d0 &= ~(0xFFu << sh);
    float xv = v[0];
#pragma unroll
    for (int j = 1; j < 8; ++j) xv = k == j ? v[j] : xv;
    const uint32_t lw = w ? lo[1] : lo[0], hw = w ? hi[1] : hi[0];
    const uint32_t code = fp8_settle(xv, s, lw >> sh & 0xFFu, hw >> sh & 0xFFu, mid_tab);
    const uint32_t nw = (lw & ~(0xFFu << sh)) | (code << sh);
    if (w) lo[1] = nw; else lo[0] = nw;
  }
  return make_uint2(lo[0], lo[1]);
}

template <typename T>
__global__ void __launch_bounds__(256) fp8_quantize_kernel(Fp8Params p) {
  __shared__ float mid_tab[128];
  fill_e4m3_mid_table(mid_tab);
  pdl_prologue();
  __syncthreads();
  const float s = __ldg(p.scale);
  const bool fast = s >= 8.67361738e-19f && s <= 1.15292150e18f;   // 2^-60 .. 2^60
  const float rs = __frcp_rn(s);
  const float rlo = __fmul_rn(rs, kWidenLo), rhi = __fmul_rn(rs, kWidenHi);
  const T *x = static_cast<const T *>(p.x);
  const int64_t chunks = p.n >> 3;
  const int64_t nthreads = static_cast<int64_t>(gridDim.x) * blockDim.x;
  constexpr int U = 4;      // chunks loaded before any is converted
  for (int64_t base = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; base < chunks;
       base += U * nthreads) {
    float v[U][8];
#pragma unroll
    for (int c = 0; c < U; ++c) {
      const int64_t i = base + c * nthreads;
      if (i >= chunks) {
#pragma unroll
        for (int k = 0; k < 8; ++k) v[c][k] = 0.0f;
        continue;
      }
      if constexpr (sizeof(T) == 2) {
        const uint4 r = __ldg(reinterpret_cast<const uint4 *>(x) + i);
        const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          v[c][2 * k] = __uint_as_float(w[k] << 16);
          v[c][2 * k + 1] = __uint_as_float(w[k] & 0xFFFF0000u);
        }
      } else {
        const float4 a4 = __ldg(reinterpret_cast<const float4 *>(x) + 2 * i);
        const float4 b4 = __ldg(reinterpret_cast<const float4 *>(x) + 2 * i + 1);
        v[c][0] = a4.x; v[c][1] = a4.y; v[c][2] = a4.z; v[c][3] = a4.w;
        v[c][4] = b4.x; v[c][5] = b4.y; v[c][6] = b4.z; v[c][7] = b4.w;
      }
    }
#pragma unroll
    for (int c = 0; c < U; ++c) {
      const int64_t i = base + c * nthreads;
      if (i >= chunks) continue;
      uint2 out;
      if (fast) {
        out = fp8x8(v[c], s, rlo, rhi, mid_tab);
      } else {
        uint32_t o[2] = {0u, 0u};
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          uint16_t pr;
          asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(pr) : "f"(0.0f), "f"(div_rn_slow(v[c][k], s)));
          o[k >> 2] |= (uint32_t)(pr & 0xFFu) << ((k & 3) * 8);
        }
        out = make_uint2(o[0], o[1]);
      }
      reinterpret_cast<uint2 *>(p.q)[i] = out;
    }
  }
}

// ------------------------------------------------------------- global scale
template <typename T>
__global__ void __launch_bounds__(256) amax_kernel(const T *x, int64_t rows, int64_t K, int64_t ld,
                                                   unsigned *amax_bits) {
  pdl_prologue();
  const int64_t chunks_per_row = K >> 4;
  const int64_t n = rows * chunks_per_row;
  float m = 0.0f;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t r = i / chunks_per_row, c = (i - r * chunks_per_row) * 16;
    Block16<T> b;
    b.load(x + r * ld + c);
    m = fmaxf(m, b.amax());
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
  __shared__ float wmax[8];
  if ((threadIdx.x & 31) == 0) wmax[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int w = 1; w < (int)(blockDim.x >> 5); ++w) m = fmaxf(m, wmax[w]);
    // non-negative floats order like their bit patterns
    atomicMax(amax_bits, __float_as_uint(m));
  }
}

// g = amax / (6*448), or 1 for an all-zero tensor; rewrites the word in place
__global__ void gscale_finalize_kernel(unsigned *amax_bits) {
  const float a = __uint_as_float(*amax_bits);
  const float g = (a == 0.0f) ? 1.0f : __fdiv_rn(a, 2688.0f);
  *reinterpret_cast<float *>(amax_bits) = g;
}

// ---------------------------------------------------------------- harmonize
constexpr int kMaxModules = 16;

struct HarmonizeParams {
  uint8_t *sf;
  int64_t rows_total, K;
  int n;
  int64_t offs[kMaxModules + 1];
  const float *gs;
  float *gstar_out;
};

// One thread per (row, 4 block columns) = one 32-bit word of the swizzled
// buffer.  g* = max_m g_m; each scale byte of module m becomes
// E4M3(dec(s) * (g_m / g*)).
__global__ void __launch_bounds__(256) harmonize_kernel(HarmonizeParams p) {
  __shared__ float ratio[kMaxModules];
  __shared__ float gstar_s;
  if (threadIdx.x == 0) {
    float gstar = __ldg(p.gs);
    for (int m = 1; m < p.n; ++m) gstar = fmaxf(gstar, __ldg(p.gs + m));
    gstar_s = gstar;
    for (int m = 0; m < p.n; ++m) ratio[m] = __fdiv_rn(__ldg(p.gs + m), gstar);
  }
  __syncthreads();
  if (blockIdx.x == 0 && threadIdx.x == 0) *p.gstar_out = gstar_s;
  const int64_t words_per_row = p.K >> 6;
  const int64_t total = p.rows_total * words_per_row;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t r = i / words_per_row, cw = i - r * words_per_row;
    int m = 0;
    while (m + 1 < p.n && r >= p.offs[m + 1]) ++m;
    const float rt = ratio[m];
    uint32_t *w = reinterpret_cast<uint32_t *>(p.sf + sf_index(r, cw * 4, p.K));
    const uint32_t in = *w;
    uint32_t out = 0;
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      const float v = __fmul_rn(e4m3_to_f32((in >> (8 * b)) & 0xFFu), rt);
      out |= f32_to_e4m3(v) << (8 * b);
    }
    *w = out;
  }
}

// Re-quantizing harmonize of a fused group, in place.  Every block of module
// m is dequantized to fp32 (dec(q) * dec(s) is exact, so fl32(that * g_m) is
// the exact NVFP4 value rounded once, as the fake-quant kernel writes it) and
// encoded again against g* = max g_m with the quantize kernels' encoder.
// Codes and scale bytes both change; padding rows are left as they are.
// One thread per 16-element block; the decoded values also go to shared
// memory, where the encoder's rare settling path re-reads them.
__global__ void __launch_bounds__(256) harmonize_requant_kernel(HarmonizeParams p, uint8_t *codes) {
  __shared__ float rcp_tab[128];
  __shared__ float gs[kMaxModules];
  __shared__ float gstar_s;
  __shared__ __align__(16) float vals[256][16];
  fill_rcp_table(rcp_tab);
  if (threadIdx.x == 0) {
    float gstar = __ldg(p.gs);
    for (int m = 0; m < p.n; ++m) {
      gs[m] = __ldg(p.gs + m);
      gstar = fmaxf(gstar, gs[m]);
    }
    gstar_s = gstar;
  }
  __syncthreads();
  if (blockIdx.x == 0 && threadIdx.x == 0) *p.gstar_out = gstar_s;
  const EncodeConsts kc = encode_consts_of(gstar_s);
  float *src = vals[threadIdx.x];
  const int64_t nb = p.K >> 4;
  const int64_t total = p.rows_total * nb;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t r = i / nb, c = i - r * nb;
    int m = 0;
    while (m + 1 < p.n && r >= p.offs[m + 1]) ++m;
    uint8_t *sfp = p.sf + sf_index(r, c, p.K);
    uint2 *cp = reinterpret_cast<uint2 *>(codes + r * (p.K >> 1) + c * 8);
    const uint2 cw = *cp;
    const float ds = e4m3_to_f32(*sfp), g = gs[m];
    Block16<float> b;
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      const uint32_t q = ((e < 8 ? cw.x : cw.y) >> ((e & 7) * 4)) & 0xFu;
      b.v[e] = __fmul_rn(__fmul_rn(e2m1_to_f32(q), ds), g);
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) reinterpret_cast<float4 *>(src)[k] = make_float4(b.v[4 * k], b.v[4 * k + 1], b.v[4 * k + 2], b.v[4 * k + 3]);
    uint32_t s;
    *cp = encode16(b, kc, rcp_tab, src, &s);
    *sfp = static_cast<uint8_t>(s);
  }
}

// ------------------------------------------- quantize fused into RMSNorm
// The BF16 RMSNorm of the residual stream, quantized in the same pass:
//   inv = the fp32 nearest to 1/sqrt(mean_k x_k^2 + eps)
//   y_k = bf16(fl32(fl32(x_k * inv) * gamma_k)),  gamma = w or fl32(1 + w)
// then y quantized like any activation (codes, swizzled scales).  The mean
// square is accumulated in fp64 (each square exact; relative error of the
// sum below 2^-46 for rows up to 36K columns), scaled by fl64(1/K), plus
// eps, and rsqrt (at most one ulp) gives 1/sqrt to ~2^-48: the fp32 rounding
// then agrees with the exact one except when the exact value lies within
// that distance of a midpoint between two floats.
struct RmsQuantParams {
  const void *x;
  int64_t rows, K, ld_x;
  const __nv_bfloat16 *w;   // norm weight [K]
  int zero_centered;        // gamma = fl32(1 + w) instead of w
  float eps;
  const float *gscale;
  uint8_t *codes;
  uint8_t *sf;
  float *inv_out;           // per-row factor [rows], or null
  int64_t pad_rows;
};

// The same RMSNorm-fused quantize with one warp per row: lane l owns blocks
// l, l + 32, ... of its row.  Phase 1 sums their squares in fp64 and the warp
// reduces the sum with shuffles (no CTA barrier); phase 2 reads the blocks
// again (from L2), forms y and encodes it.  Each lane keeps its current block
// of y in a 32-byte shared slot, where the encoder's settling path re-reads
// elements.  The norm weight is staged once per CTA.
constexpr int kRmsWarpThreads = 256;

__host__ __device__ constexpr int64_t rms_warp_smem_bytes(int64_t K) {
  return K * 2 + kRmsWarpThreads * 32 + 128 * 4;
}

template <typename T>
__global__ void __launch_bounds__(kRmsWarpThreads, 4) rmsnorm_quantize_warp_kernel(const RmsQuantParams p) {
  extern __shared__ __align__(16) uint8_t smem[];
  __nv_bfloat16 *wsm = reinterpret_cast<__nv_bfloat16 *>(smem);
  __nv_bfloat16 *ystage = reinterpret_cast<__nv_bfloat16 *>(smem + p.K * 2) + threadIdx.x * 16;
  float *rcp_tab = reinterpret_cast<float *>(smem + p.K * 2 + kRmsWarpThreads * 32);
  fill_rcp_table(rcp_tab);
  pdl_prologue();
  for (int64_t i = threadIdx.x; i < (p.K >> 3); i += kRmsWarpThreads)
    reinterpret_cast<uint4 *>(wsm)[i] = __ldg(reinterpret_cast<const uint4 *>(p.w) + i);
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int64_t nwarps = (int64_t)gridDim.x * (kRmsWarpThreads / 32);
  const T *x = static_cast<const T *>(p.x);
  const EncodeConsts kc = encode_consts(p.gscale);
  const int nb = (int)(p.K >> 4);
  const double rk = __drcp_rn((double)p.K);
  const double eps = (double)p.eps;
  for (int64_t row = (int64_t)blockIdx.x * (kRmsWarpThreads / 32) + (threadIdx.x >> 5); row < p.rows; row += nwarps) {
    const T *xr = x + row * p.ld_x;
    double acc = 0.0;
#pragma unroll 2
    for (int c = lane; c < nb; c += 32) {
      Block16<T> b;
      b.load(xr + c * 16);
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        const double v = (double)b.elem(e);
        acc = fma(v, v, acc);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xFFFFFFFFu, acc, o);
    const float inv = __double2float_rn(rsqrt(fma(acc, rk, eps)));
    if (lane == 0 && p.inv_out) p.inv_out[row] = inv;
    uint8_t *crow = p.codes + row * (p.K >> 1);
    for (int c = lane; c < nb; c += 32) {
      Block16<T> xb;
      xb.load(xr + c * 16);
      const uint4 w0 = reinterpret_cast<const uint4 *>(wsm)[2 * c], w1 = reinterpret_cast<const uint4 *>(wsm)[2 * c + 1];
      const uint32_t ww[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
      Block16<__nv_bfloat16> yb;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        float g0 = __uint_as_float(ww[i] << 16), g1 = __uint_as_float(ww[i] & 0xFFFF0000u);
        if (p.zero_centered) {
          g0 = __fadd_rn(1.0f, g0);
          g1 = __fadd_rn(1.0f, g1);
        }
        const float y0 = __fmul_rn(__fmul_rn(xb.elem(2 * i), inv), g0);
        const float y1 = __fmul_rn(__fmul_rn(xb.elem(2 * i + 1), inv), g1);
        __nv_bfloat162 h = __floats2bfloat162_rn(y0, y1);
        yb.w[i] = *reinterpret_cast<uint32_t *>(&h);
      }
      reinterpret_cast<uint4 *>(ystage)[0] = make_uint4(yb.w[0], yb.w[1], yb.w[2], yb.w[3]);
      reinterpret_cast<uint4 *>(ystage)[1] = make_uint4(yb.w[4], yb.w[5], yb.w[6], yb.w[7]);
      uint32_t s;
      const uint2 word = encode16(yb, kc, rcp_tab, ystage, &s);
      *reinterpret_cast<uint2 *>(crow + c * 8) = word;
      p.sf[sf_index(row, c, p.K)] = static_cast<uint8_t>(s);
    }
  }
  zero_pad_scales(p.sf, p.rows, p.pad_rows, p.K);
}

}  // namespace nvfp4
