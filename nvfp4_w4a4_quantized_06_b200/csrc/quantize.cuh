// quantize.cuh -- NVFP4 encoder kernels for sm_100a: per-tensor global scale,
// activation/weight quantize (E2M1 codes + swizzled E4M3 block scales) and
// fused-group global-scale harmonization.
//
// Format (web pages on arXiv 2609.04098; ta-paperlens page, section "前提1";
// arxiv-wiki page, "접근 방법"): 4-bit E2M1 values, one E4M3 scale per 16
// consecutive elements equal to the block maximum / 6, and one FP32 scale per
// tensor.  Arithmetic per block (each step one IEEE fp32 operation):
//   g6 = 6*g;  s = E4M3(amax/g6);  d = dec(s)*g;  q_i = E2M1(x_i/d)
// with round-to-nearest-even and saturation at 448 / 6; a block whose scale
// or d is zero gets +0 codes.
#pragma once
#include <cuda_bf16.h>
#include <cstdint>

#include "ptx.cuh"

namespace nvfp4 {

// byte offset of the scale of (row r, block column c) in the swizzled buffer
// (128-row x 4-column atoms of 512 bytes; K % 64 == 0 so K/64 atoms per row block)
__device__ __forceinline__ int64_t sf_index(int64_t r, int64_t c, int64_t K) {
  return ((r >> 7) * (K >> 6) + (c >> 2)) * 512 + (r & 31) * 16 + ((r >> 5) & 3) * 4 + (c & 3);
}

template <typename T>
struct Vec8;  // eight consecutive input elements as fp32

template <>
struct Vec8<__nv_bfloat16> {
  uint4 raw;
  __device__ __forceinline__ void zero() { raw = make_uint4(0u, 0u, 0u, 0u); }
  __device__ __forceinline__ void load(const __nv_bfloat16 *p) {
    raw = __ldg(reinterpret_cast<const uint4 *>(p));
  }
  __device__ __forceinline__ void to_f32(float (&v)[8]) const {
    const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      v[2 * i] = __uint_as_float(w[i] << 16);
      v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
  }
};

template <>
struct Vec8<float> {
  float4 a, b;
  __device__ __forceinline__ void zero() {
    a = make_float4(0.f, 0.f, 0.f, 0.f);
    b = a;
  }
  __device__ __forceinline__ void load(const float *p) {
    a = __ldg(reinterpret_cast<const float4 *>(p));
    b = __ldg(reinterpret_cast<const float4 *>(p) + 1);
  }
  __device__ __forceinline__ void to_f32(float (&v)[8]) const {
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  }
};

template <typename T>
struct Vec16;  // sixteen consecutive input elements (one scale block)

template <>
struct Vec16<__nv_bfloat16> {
  uint4 a, b;
  __device__ __forceinline__ void zero() { a = b = make_uint4(0u, 0u, 0u, 0u); }
  __device__ __forceinline__ void load(const __nv_bfloat16 *p) {
    a = __ldg(reinterpret_cast<const uint4 *>(p));
    b = __ldg(reinterpret_cast<const uint4 *>(p) + 1);
  }
  __device__ __forceinline__ void to_f32(float (&v)[16]) const {
    const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      v[2 * i] = __uint_as_float(w[i] << 16);
      v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
  }
};

template <>
struct Vec16<float> {
  float4 q[4];
  __device__ __forceinline__ void zero() {
#pragma unroll
    for (int i = 0; i < 4; ++i) q[i] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
  __device__ __forceinline__ void load(const float *p) {
#pragma unroll
    for (int i = 0; i < 4; ++i) q[i] = __ldg(reinterpret_cast<const float4 *>(p) + i);
  }
  __device__ __forceinline__ void to_f32(float (&v)[16]) const {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      v[4 * i] = q[i].x; v[4 * i + 1] = q[i].y; v[4 * i + 2] = q[i].z; v[4 * i + 3] = q[i].w;
    }
  }
};

// Per-tensor constants of the encoder.
struct EncodeConsts {
  float g, g6;      // global scale and fl32(6*g)
  float rg, rg6;    // fl32(1/g), fl32(1/g6)
  bool fast;        // the multiply-by-reciprocal path is usable (g well inside the normal range)
};

__device__ __forceinline__ EncodeConsts encode_consts(const float *gscale) {
  EncodeConsts k;
  k.g = __ldg(gscale);
  k.g6 = __fmul_rn(6.0f, k.g);
  k.rg = __frcp_rn(k.g);
  k.rg6 = __frcp_rn(k.g6);
  k.fast = k.g >= 8.67361738e-19f && k.g <= 1.15292150e18f;   // 2^-60 .. 2^60
  return k;
}

// Shared table of fl32(1/dec(s)) for every finite non-negative E4M3 byte s;
// entry 0 is unused (a zero scale short-circuits to zero codes).
__device__ __forceinline__ void fill_rcp_table(float *tab) {
  for (int i = threadIdx.x; i < 128; i += blockDim.x)
    tab[i] = i == 0 || i == 127 ? 0.0f : __frcp_rn(e4m3_to_f32((uint32_t)i));
}

// IEEE reference path of one half-block: t = amax / g6, y = x / (dec(s)*g).
__device__ __noinline__ uint32_t encode8_ieee(const float *v, float amax, float g, float g6, uint32_t *s_out) {
  const uint32_t s = f32_to_e4m3(__fdiv_rn(amax, g6));
  *s_out = s;
  const float d = __fmul_rn(e4m3_to_f32(s), g);
  if (s == 0u || d == 0.0f) return 0u;
  float y[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) y[i] = __fdiv_rn(v[i], d);
  return f32x8_to_e2m1(y);
}

// Encode eight values of one half-block given the block's amax; returns the
// packed code word and (through *s_out) the E4M3 scale byte.  The result is
// bit-identical to the IEEE definition
//   s = E4M3(fl32(amax / fl32(6g))),  q_i = E2M1(fl32(x_i / fl32(dec(s) g))).
// Fast path: t' = fl32(amax * fl32(1/g6)) is within 2 ulps of fl32(amax/g6)
// and y' = fl32(fl32(x * fl32(1/dec(s))) * fl32(1/g)) within 6 ulps of
// fl32(x/d).  A rounding decision can only differ if a decision point lies
// between the two values: every E4M3 midpoint has 19 and every E2M1 decision
// threshold (0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5) 21 trailing zero bits in its
// fp32 encoding, so a value whose bit pattern is not within 8 of such a
// multiple is decided exactly.  Otherwise (and for extreme g) the IEEE path
// recomputes the group.
__device__ __forceinline__ uint32_t encode8(const float (&v)[8], float amax, const EncodeConsts &k,
                                            const float *rcp_tab, uint32_t *s_out) {
  if (!k.fast) return encode8_ieee(v, amax, k.g, k.g6, s_out);
  const float t = __fmul_rn(amax, k.rg6);
  if (((__float_as_uint(t) + 8u) & 0x7FFF0u) == 0u) return encode8_ieee(v, amax, k.g, k.g6, s_out);
  const uint32_t s = f32_to_e4m3(t);
  *s_out = s;
  if (s == 0u) return 0u;
  const float rs = rcp_tab[s];
  float y[8];
  uint32_t near = 0xFFFFFFFFu;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    y[i] = __fmul_rn(__fmul_rn(v[i], rs), k.rg);
    const uint32_t b = __float_as_uint(y[i]) & 0x7FFFFFFFu;
    near = min(near, ((b + 8u) & 0x1FFFF0u) | (b < 0x3E000000u ? 1u : 0u));
  }
  if (near == 0u) return encode8_ieee(v, amax, k.g, k.g6, s_out);
  return f32x8_to_e2m1(y);
}

__device__ __noinline__ float div_rn_slow(float a, float b) { return __fdiv_rn(a, b); }

// One whole 16-element block.  Same definition and exactness argument as
// encode8, applied per value: t' = fl32(amax * fl32(1/g6)) and
// y' = fl32(x * fl32(fl32(1/dec(s)) * fl32(1/g))) are within 2 and 6 ulps of
// the IEEE results; only a value whose bit pattern lies within 8 of a multiple
// of 2^19 (t) or 2^21 (y) -- a superset of the decision points -- is
// recomputed with IEEE division, one value at a time.  (With bf16 inputs and
// block scales built from them, values land next to round numbers far more
// often than chance, so recomputing whole blocks would be costly.)
__device__ __forceinline__ uint2 encode16(const float (&v)[16], float amax, const EncodeConsts &k,
                                          const float *rcp_tab, uint32_t *s_out) {
  float t = __fmul_rn(amax, k.rg6);
  if (!k.fast || ((__float_as_uint(t) + 8u) & 0x7FFF0u) == 0u) t = div_rn_slow(amax, k.g6);
  const uint32_t s = f32_to_e4m3(t);
  *s_out = s;
  if (s == 0u) return make_uint2(0u, 0u);
  float y[16];
  if (k.fast) {
    const float r = __fmul_rn(rcp_tab[s], k.rg);
    uint32_t near = 0xFFFFFFFFu;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      y[i] = __fmul_rn(v[i], r);
      near = min(near, (__float_as_uint(y[i]) + 8u) & 0x1FFFF0u);
    }
    if (near == 0u) {
      const float d = __fmul_rn(e4m3_to_f32(s), k.g);
#pragma unroll
      for (int i = 0; i < 16; ++i)
        if (((__float_as_uint(y[i]) + 8u) & 0x1FFFF0u) == 0u) y[i] = div_rn_slow(v[i], d);
    }
  } else {
    const float d = __fmul_rn(e4m3_to_f32(s), k.g);
    if (d == 0.0f) return make_uint2(0u, 0u);
#pragma unroll
    for (int i = 0; i < 16; ++i) y[i] = div_rn_slow(v[i], d);
  }
  uint2 out;
  out.x = f32x8_to_e2m1(*reinterpret_cast<const float(*)[8]>(&y[0]));
  out.y = f32x8_to_e2m1(*reinterpret_cast<const float(*)[8]>(&y[8]));
  return out;
}

struct QuantizeParams {
  const void *x;
  int64_t rows, K, ld_x;
  const float *gscale;
  uint8_t *codes;
  uint8_t *sf;
  int64_t sf_row0;
  int64_t pad_rows;  // padding rows (zeroed) after this call's rows, or 0
};

// Generic path (any row offset inside a fused buffer): one warp handles a
// 256-element segment of one row per unit; lane l owns elements [8l, 8l+8),
// lanes 2i and 2i+1 form 16-element block i and exchange their half-maxima
// with one shuffle.  Loads are 16-byte vectors, code words 4-byte stores, and
// every scale byte is stored on its own.  UNROLL units are loaded before any
// is encoded.
template <typename T, int UNROLL>
__global__ void __launch_bounds__(256) quantize_kernel(QuantizeParams p) {
  const int lane = threadIdx.x & 31;
  const uint32_t warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const uint32_t nwarps = (gridDim.x * blockDim.x) >> 5;
  const uint32_t nseg = (uint32_t)((p.K + 255) >> 8);
  const uint32_t units = (uint32_t)p.rows * nseg;
  const int64_t ncols = p.K >> 4;
  __shared__ float rcp_tab[128];
  fill_rcp_table(rcp_tab);
  __syncthreads();
  const EncodeConsts kc = encode_consts(p.gscale);
  const T *x = static_cast<const T *>(p.x);

  for (uint32_t u0 = warp * UNROLL; u0 < units; u0 += nwarps * UNROLL) {
    Vec8<T> in[UNROLL];
    int64_t row[UNROLL];
    int col[UNROLL];
#pragma unroll
    for (int j = 0; j < UNROLL; ++j) {
      const uint32_t u = u0 + j;
      row[j] = u / nseg;
      col[j] = (int)(u - (uint32_t)row[j] * nseg) * 256 + lane * 8;
      in[j].zero();
      if (u < units && col[j] < p.K) in[j].load(x + row[j] * p.ld_x + col[j]);
    }
#pragma unroll
    for (int j = 0; j < UNROLL; ++j) {
      const bool active = u0 + j < units && col[j] < p.K;
      float v[8];
      in[j].to_f32(v);
      float amax = 0.0f;
#pragma unroll
      for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(v[i]));
      amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, 1));
      if (active) {
        uint32_t s;
        const uint32_t word = encode8(v, amax, kc, rcp_tab, &s);
        *reinterpret_cast<uint32_t *>(p.codes + row[j] * (p.K >> 1) + (col[j] >> 1)) = word;
        if ((lane & 1) == 0) p.sf[sf_index(p.sf_row0 + row[j], col[j] >> 4, p.K)] = static_cast<uint8_t>(s);
      }
    }
  }
  // zero the scale bytes of the padding rows this call owns
  const int64_t pad_bytes = p.pad_rows * ncols;
  const int64_t tid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t nthreads = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = tid; i < pad_bytes; i += nthreads) {
    const int64_t r = p.sf_row0 + p.rows + i / ncols, c = i % ncols;
    p.sf[sf_index(r, c, p.K)] = 0;
  }
}

// Tile path, used when this call's scale rows start on a 128-row boundary and
// it owns every row of its last 128-row block (the activation quantize always
// does).  A CTA of 8 warps handles a 128-row x 512-column tile; lane l of a
// warp encodes 16-element block l of a row segment (32 contiguous bytes of
// bf16 per lane, 1 KB per warp-row), warp w takes rows w, w+8, ..., w+120.
// The tile's 32 scale columns -- exactly eight 512-byte atoms, contiguous in
// the swizzled buffer -- are collected in shared memory and written with
// 16-byte stores.  Rows past `rows` (padding) get zero scales.
template <typename T, int UNROLL>
__global__ void __launch_bounds__(256) quantize_tile_kernel(QuantizeParams p) {
  __shared__ __align__(16) uint8_t sf_tile[4096];
  __shared__ float rcp_tab[128];
  fill_rcp_table(rcp_tab);
  __syncthreads();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const uint32_t nseg = (uint32_t)((p.K + 511) >> 9);
  const uint32_t nrb = (uint32_t)((p.rows + 127) >> 7);
  const uint32_t units = nrb * nseg;
  const uint32_t atoms_per_rb = (uint32_t)(p.K >> 6);
  const EncodeConsts kc = encode_consts(p.gscale);
  const T *x = static_cast<const T *>(p.x);
  const int sf_off = (lane >> 2) * 512 + (lane & 3);     // this lane's block column inside the tile

  for (uint32_t u = blockIdx.x; u < units; u += gridDim.x) {
    const uint32_t rb = u / nseg, seg = u - rb * nseg;
    const int col = (int)seg * 512 + lane * 16;
    const bool col_ok = col < p.K;
    const int64_t row0 = (int64_t)rb * 128 + warp;
    const T *xp = x + row0 * p.ld_x + col;
    uint8_t *cp = p.codes + row0 * (p.K >> 1) + (col >> 1);
#pragma unroll 1
    for (int i0 = 0; i0 < 16; i0 += UNROLL) {
      Vec16<T> in[UNROLL];
#pragma unroll
      for (int j = 0; j < UNROLL; ++j) {
        in[j].zero();
        if (col_ok && row0 + 8 * (i0 + j) < p.rows) in[j].load(xp + (int64_t)(8 * (i0 + j)) * p.ld_x);
      }
#pragma unroll
      for (int j = 0; j < UNROLL; ++j) {
        const int rl = warp + 8 * (i0 + j);
        float v[16];
        in[j].to_f32(v);
        float amax = 0.0f;
#pragma unroll
        for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(v[i]));
        uint32_t s = 0;
        if (col_ok && row0 + 8 * (i0 + j) < p.rows) {
          const uint2 word = encode16(v, amax, kc, rcp_tab, &s);
          *reinterpret_cast<uint2 *>(cp + (int64_t)(8 * (i0 + j)) * (p.K >> 1)) = word;
        }
        sf_tile[sf_off + (rl & 31) * 16 + (rl >> 5) * 4] = (uint8_t)s;
      }
    }
    __syncthreads();
    const uint32_t natoms = min(8u, atoms_per_rb - seg * 8);
    uint8_t *dst = p.sf + ((int64_t)((p.sf_row0 >> 7) + rb) * atoms_per_rb + seg * 8) * 512;
    for (uint32_t t = threadIdx.x; t < natoms * 32; t += blockDim.x)
      reinterpret_cast<uint4 *>(dst)[t] = reinterpret_cast<const uint4 *>(sf_tile)[t];
    __syncthreads();
  }
}

// ------------------------------------------------------------- global scale
template <typename T>
__global__ void __launch_bounds__(256) amax_kernel(const T *x, int64_t rows, int64_t K, int64_t ld,
                                                   unsigned *amax_bits) {
  const int64_t chunks_per_row = K >> 3;
  const int64_t n = rows * chunks_per_row;
  float m = 0.0f;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t r = i / chunks_per_row, c = (i - r * chunks_per_row) * 8;
    Vec8<T> v8;
    v8.load(x + r * ld + c);
    float v[8];
    v8.to_f32(v);
#pragma unroll
    for (int j = 0; j < 8; ++j) m = fmaxf(m, fabsf(v[j]));
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

}  // namespace nvfp4
