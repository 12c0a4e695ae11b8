"""CPU oracle of the NVFP4 W4A4 linear layer -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` import this package.  The CUDA library never loads it, and it
shares no code, header, table or constant generator with the CUDA library:
the arithmetic lives in ``nvfp4_oracle.c`` (plain C, fp32 steps as single IEEE
operations, float64 for dequantization and the GEMM reference) and this module
only marshals numpy arrays into it.

Sources (web pages on arXiv 2609.04098, "Why Gated DeltaNet Survives 4-Bit
Quantization"): the NVFP4 format and the W4A4 product on the ta-paperlens page
("前提1") and the arxiv-wiki page ("접근 방법"); the fused-group global-scale
repair on the arxiv-wiki page ("접근 방법", "개발자 관점") and the abstract on the
shd-paper page.  Readings the pages leave open are listed in the C file's
header.  Every step is pinned by tests/test_oracle_*.py; the arithmetic order
for non-power-of-two global scales (a reading: the pages do not fix it) is
pinned against an exact rational evaluation of that reading on inputs at the
rounding boundaries, where other orders give different bytes.
The rows marked "next" (GDN gate activations, fake-quant, FP8 KV quantize,
the re-quantizing harmonize and the quantize fused into the preceding
RMSNorm) follow the same pages (ta-paperlens "前提2": the GDN layer feeds the
residual stream through its projections and every norm stays in BF16;
arxiv-wiki "주요 결과", "접근 방법") and are pinned in tests/test_oracle_next.py.
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess
from fractions import Fraction

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "nvfp4_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libnvfp4_oracle.so")
_lib = None

BLOCK = 16


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (IEEE fp32, no contraction, OpenMP rows)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-ffp-contract=off", "-fno-fast-math",
               "-fopenmp", "-o", _LIB_PATH + ".tmp", _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(_LIB_PATH + ".tmp", _LIB_PATH)
    return _LIB_PATH


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB_PATH)
        i64, f32, f64, vp, i32 = ctypes.c_int64, ctypes.c_float, ctypes.c_double, ctypes.c_void_p, ctypes.c_int
        L.oracle_e2m1_decode.argtypes, L.oracle_e2m1_decode.restype = [i32], f64
        L.oracle_e4m3_decode.argtypes, L.oracle_e4m3_decode.restype = [i32], f64
        L.oracle_e2m1_encode.argtypes, L.oracle_e2m1_encode.restype = [f32], i32
        L.oracle_e4m3_encode.argtypes, L.oracle_e4m3_encode.restype = [f32], i32
        L.oracle_sf_offset.argtypes, L.oracle_sf_offset.restype = [i64, i64, i64], i64
        L.oracle_sf_bytes.argtypes, L.oracle_sf_bytes.restype = [i64, i64], i64
        L.oracle_global_scale.argtypes, L.oracle_global_scale.restype = [vp, i64], f32
        L.oracle_quantize.argtypes, L.oracle_quantize.restype = [vp, i64, i64, i64, f32, vp, vp, i64], None
        L.oracle_harmonize.argtypes, L.oracle_harmonize.restype = [vp, i64, i32, vp, vp], f32
        L.oracle_dequantize.argtypes, L.oracle_dequantize.restype = [vp, vp, i64, i64, f32, i64, vp], None
        L.oracle_gemm_f64.argtypes, L.oracle_gemm_f64.restype = [vp, vp, i64, i64, i64, f64, vp, vp], None
        L.oracle_sf_gather.argtypes, L.oracle_sf_gather.restype = [vp, vp, i64, i64, vp], None
        L.oracle_num_threads.argtypes, L.oracle_num_threads.restype = [], i32
        L.oracle_gdn_gates.argtypes, L.oracle_gdn_gates.restype = [vp, i64, i64, i64, vp], None
        L.oracle_fp8_quantize.argtypes, L.oracle_fp8_quantize.restype = [vp, i64, f32, vp], None
        _lib = L
    return _lib


def _ptr(a: np.ndarray) -> int:
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data


# ------------------------------------------------------------------ codecs
def e2m1_decode(code: int) -> float:
    return lib().oracle_e2m1_decode(int(code))


def e4m3_decode(code: int) -> float:
    return lib().oracle_e4m3_decode(int(code))


def e2m1_encode(y) -> int:
    return lib().oracle_e2m1_encode(float(np.float32(y)))


def e4m3_encode(t) -> int:
    return lib().oracle_e4m3_encode(float(np.float32(t)))


# ------------------------------------------------------------------ layout
def sf_bytes(rows: int, K: int) -> int:
    return int(lib().oracle_sf_bytes(rows, K))


def sf_offset(r: int, c: int, K: int) -> int:
    return int(lib().oracle_sf_offset(r, c, K))


def sf_gather(sf: np.ndarray, rows, K: int) -> np.ndarray:
    """Scale bytes of `rows` as a plain [len(rows), K/16] uint8 array."""
    rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    out = np.zeros((rows.size, K // BLOCK), dtype=np.uint8)
    sf = np.ascontiguousarray(sf, dtype=np.uint8)
    lib().oracle_sf_gather(_ptr(sf), _ptr(rows), rows.size, K, _ptr(out))
    return out


# ---------------------------------------------------------------- steps
def global_scale(x: np.ndarray) -> np.float32:
    x = np.ascontiguousarray(x, dtype=np.float32)
    return np.float32(lib().oracle_global_scale(_ptr(x), x.size))


def quantize(x: np.ndarray, g, sf: np.ndarray | None = None, sf_row0: int = 0,
             sf_rows_total: int | None = None):
    """Quantize x [rows, K] (float32; bf16 callers convert exactly first).

    Returns (codes [rows, K/2] uint8, sf flat uint8 swizzled buffer)."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    rows, K = x.shape
    assert K % 64 == 0
    if sf is None:
        total = rows if sf_rows_total is None else sf_rows_total
        sf = np.zeros(sf_bytes(total, K), dtype=np.uint8)
    codes = np.zeros((rows, K // 2), dtype=np.uint8)
    lib().oracle_quantize(_ptr(x), rows, K, K, float(np.float32(g)), _ptr(codes), _ptr(sf), sf_row0)
    return codes, sf


def harmonize(sf: np.ndarray, K: int, row_offsets, gscales) -> np.float32:
    """In-place rewrite of a fused group's scales to g* = max(gscales); returns g*."""
    offs = np.ascontiguousarray(np.asarray(row_offsets, dtype=np.int64))
    gs = np.ascontiguousarray(np.asarray(gscales, dtype=np.float32))
    assert offs.size == gs.size + 1
    return np.float32(lib().oracle_harmonize(_ptr(sf), K, gs.size, _ptr(offs), _ptr(gs)))


def dequantize(codes: np.ndarray, sf: np.ndarray, g, sf_row0: int = 0) -> np.ndarray:
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    rows, K = codes.shape[0], codes.shape[1] * 2
    out = np.empty((rows, K), dtype=np.float64)
    lib().oracle_dequantize(_ptr(codes), _ptr(np.ascontiguousarray(sf)), rows, K,
                            float(np.float32(g)), sf_row0, _ptr(out))
    return out


def gemm_f64(a: np.ndarray, b: np.ndarray, alpha: float, brute: bool = False):
    """Y = alpha * a @ b.T and Yabs = |alpha| * |a| @ |b|.T in float64.

    brute=True runs the plain C triple loop; otherwise numpy's float64 matmul
    (a library primitive) computes the same sums."""
    a = np.ascontiguousarray(a, dtype=np.float64)
    b = np.ascontiguousarray(b, dtype=np.float64)
    M, K = a.shape
    N = b.shape[0]
    if brute:
        y = np.empty((M, N)); yabs = np.empty((M, N))
        lib().oracle_gemm_f64(_ptr(a), _ptr(b), M, N, K, float(alpha), _ptr(y), _ptr(yabs))
        return y, yabs
    y = (a @ b.T) * alpha
    yabs = (np.abs(a) @ np.abs(b).T) * abs(alpha)
    return y, yabs


def linear_reference(x: np.ndarray, gx, w_codes: np.ndarray, w_sf: np.ndarray, gw,
                     brute: bool = False):
    """The whole W4A4 linear on the CPU: quantize x, dequantize both operands,
    float64 GEMM with alpha = gx*gw.  Returns (y, yabs, x_codes, x_sf)."""
    xc, xs = quantize(x, gx)
    # unit-scale operands: every product dec(q)dec(s)dec(q')dec(s') has at most
    # 12 significant bits, so the float64 sums are exact for these ranges; the
    # two global scales are applied once, in float64, at the end
    a = dequantize(xc, xs, 1.0)
    b = dequantize(w_codes, w_sf, 1.0)
    y, yabs = gemm_f64(a, b, float(np.float64(gx) * np.float64(gw)), brute=brute)
    return y, yabs, xc, xs


# --------------------------------------------------- rows marked "next"
def gdn_gates(y: np.ndarray, n_a: int) -> np.ndarray:
    """alpha = exp(-softplus(y)) on columns [0, n_a), beta = sigmoid(y) on the
    rest (float64; the gate-projection epilogue of a GDN layer)."""
    y = np.ascontiguousarray(y, dtype=np.float64)
    rows, N = y.shape
    out = np.empty_like(y)
    lib().oracle_gdn_gates(_ptr(y), rows, N, int(n_a), _ptr(out))
    return out


def fake_quant(x: np.ndarray, g):
    """Quantize then dequantize (Q -> DQ): the NVFP4 value every element of x
    is replaced by (float64, exact), and the error statistics
    (sum of squared error, sum of squared input)."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    codes, sf = quantize(x, g)
    dq = dequantize(codes, sf, g)
    x64 = x.astype(np.float64)
    return dq, float(np.sum((x64 - dq) ** 2)), float(np.sum(x64 ** 2))


def fp8_quantize(x: np.ndarray, s) -> np.ndarray:
    """FP8 E4M3 codes (sign in bit 7) of fl32(x / s), static per-tensor scale s."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    q = np.empty(x.shape, dtype=np.uint8)
    lib().oracle_fp8_quantize(_ptr(x), x.size, float(np.float32(s)), _ptr(q))
    return q


def harmonize_requant(codes: np.ndarray, sf: np.ndarray, K: int, row_offsets, gscales):
    """Re-quantizing harmonize of a fused group: every module's weights, taken
    as their NVFP4 values rounded once to fp32 (the fake-quant value,
    dec(q)*dec(s)*g_m), are quantized again against g* = max(g_m).  Codes and
    scales both change.  Returns (codes', sf', g*); the inputs are not touched."""
    offs = [int(o) for o in row_offsets]
    gs = [np.float32(g) for g in gscales]
    assert len(offs) == len(gs) + 1 and offs[0] == 0
    gstar = max(gs)
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    out_codes = np.empty_like(codes)
    out_sf = np.zeros_like(sf)
    for m, g in enumerate(gs):
        r0, r1 = offs[m], offs[m + 1]
        xhat = dequantize(codes[r0:r1], sf, g, sf_row0=r0).astype(np.float32)   # one rounding of an exact value
        out_codes[r0:r1], _ = quantize(xhat, gstar, sf=out_sf, sf_row0=r0)
    return out_codes, out_sf, gstar


# ---------------------------------------- quantize fused into RMSNorm
RMS_NEAR_TIE = 2.0 ** -44   # |m^2 V - 1| below this: 1/sqrt(V) lies within ~2^-45 of an fp32 midpoint


def _exact_sum_squares(row: np.ndarray) -> Fraction:
    """Sum of x^2 over a row of float32 values, exactly: x = m * 2^(e-24) with
    m an integer below 2^24, so x^2 = m^2 * 2^(2e-48); the m^2 of equal
    exponents are added as integers and the groups shifted into one."""
    mant, ex = np.frexp(row.astype(np.float64))
    mi = np.ldexp(mant, 24).astype(np.int64)
    assert np.array_equal(mi.astype(np.float64), np.ldexp(mant, 24)), "float32 input expected"
    sq = mi * mi                                   # < 2^48, exact
    e2 = 2 * (ex.astype(np.int64) - 24)
    nz = mi != 0
    if not np.any(nz):
        return Fraction(0)
    e0 = int(e2[nz].min())
    total = 0
    for k in np.unique(e2[nz]):
        part = sq[nz & (e2 == k)]
        s = (int((part >> 32).sum()) << 32) + int((part & 0xFFFFFFFF).sum())   # two halves: no int64 overflow
        total += s << (int(k) - e0)
    return Fraction(total) * Fraction(2) ** e0


def rsqrt_rn32(V: Fraction):
    """The float32 nearest to 1/sqrt(V) (ties to the even significand), for a
    positive rational V, decided exactly: 1/sqrt(V) > m  <=>  m^2 V < 1 for a
    midpoint m between neighbouring floats.  Also returns how close
    1/sqrt(V) comes to either midpoint, as min |m^2 V - 1|."""
    assert V > 0
    f = np.float32(1.0 / math.sqrt(float(V)))
    inf, zero = np.float32(np.inf), np.float32(0.0)
    while True:
        up, dn = np.nextafter(f, inf), np.nextafter(f, zero)
        mh = (Fraction(float(f)) + Fraction(float(up))) / 2
        ml = (Fraction(float(dn)) + Fraction(float(f))) / 2
        th, tl = mh * mh * V, ml * ml * V
        if th < 1:
            f = up
            continue
        if tl > 1:
            f = dn
            continue
        odd = int(np.array(f).view(np.uint32)) & 1
        if th == 1 and odd:
            f = up
        elif tl == 1 and odd:
            f = dn
        return f, float(min(abs(th - 1), abs(tl - 1)))


def rms_inv(x: np.ndarray, eps):
    """Per row: inv = the float32 nearest to 1/sqrt(mean(x^2) + eps), with the
    mean taken exactly (eps a positive float32), and whether the exact value
    lies within ~2^-45 of a rounding midpoint (then a kernel that evaluates it
    to ~2^-48 may round either way)."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    e = Fraction(float(np.float32(eps)))
    assert e > 0
    rows, K = x.shape
    inv = np.empty(rows, np.float32)
    near = np.zeros(rows, bool)
    for r in range(rows):
        V = _exact_sum_squares(x[r]) / K + e
        inv[r], close = rsqrt_rn32(V)
        near[r] = close < RMS_NEAR_TIE
    return inv, near


def _bf16_rne(v: np.ndarray) -> np.ndarray:
    import torch
    return torch.from_numpy(np.ascontiguousarray(v, dtype=np.float32)).to(torch.bfloat16).to(torch.float32).numpy()


def rmsnorm(x: np.ndarray, w: np.ndarray, eps, zero_centered: bool = False, inv=None):
    """RMSNorm of the residual stream as the BF16 input of the projections
    that read it (the norms stay in BF16): h = fl32(x * inv),
    y = bf16(fl32(h * gamma)) with gamma = w (or fl32(1 + w) for the
    zero-centred form), w the norm weight (bf16 values).  Returns
    (y as float32 [rows, K], inv [rows], near-tie flags [rows]); `inv`
    overrides the per-row factor (for rows flagged near a tie)."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    w = np.asarray(w, dtype=np.float32)
    assert np.array_equal(_bf16_rne(w), w), "norm weight must hold bf16 values"
    inv_rn, near = rms_inv(x, eps)
    if inv is not None:
        inv_rn = np.asarray(inv, dtype=np.float32)
    h = x * inv_rn[:, None]                                   # float32 products, each rounded once
    gamma = (np.float32(1.0) + w) if zero_centered else w
    y = _bf16_rne(h * gamma[None, :])
    return y, inv_rn, near


def rmsnorm_quantize(x: np.ndarray, w: np.ndarray, eps, g, zero_centered: bool = False, inv=None):
    """NVFP4 quantize of the RMSNorm output: (codes, sf, y, inv, near-tie)."""
    y, inv_rn, near = rmsnorm(x, w, eps, zero_centered, inv)
    codes, sf = quantize(y, g)
    return codes, sf, y, inv_rn, near


def num_threads() -> int:
    return int(lib().oracle_num_threads())
