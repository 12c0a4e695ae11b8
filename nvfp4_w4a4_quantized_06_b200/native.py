"""ctypes binding of libnvfp4w4a4.so (the C ABI in include/nvfp4w4a4.h).

Argument marshalling only: torch allocates the outputs and supplies the
current CUDA stream; every step of the layer runs in the library's kernels.
There is no fallback: if the library is missing or the call fails, this
module raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libnvfp4w4a4.so")

IN_BF16, IN_F32 = 0, 1
OUT_BF16, OUT_F32 = 0, 1
STATUS = {0: "ok", 1: "null pointer", 2: "bad shape", 3: "misaligned", 4: "bad dtype",
          5: "unsupported", 6: "timeout", 7: "CUDA error", 8: "workspace", 9: "scratch limit"}

_lib = None


class Nvfp4Error(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn} failed: {STATUS.get(status, status)} ({status})")
        self.status = status


def lib() -> ctypes.CDLL:
    """Load the in-tree library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: run `python -m nvfp4_w4a4_quantized_06_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, i64, i32, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t
        L.nvfp4_codes_bytes.argtypes, L.nvfp4_codes_bytes.restype = [i64, i64], sz
        L.nvfp4_sf_bytes.argtypes, L.nvfp4_sf_bytes.restype = [i64, i64], sz
        L.nvfp4_amax_gscale.argtypes = [vp, i32, i64, i64, i64, vp, vp]
        L.nvfp4_quantize.argtypes = [vp, i32, i64, i64, i64, vp, vp, vp, i64, i64, vp]
        L.nvfp4_harmonize_group.argtypes = [vp, i64, i64, i32, vp, vp, vp, vp]
        L.nvfp4_gemm_workspace_bytes.argtypes, L.nvfp4_gemm_workspace_bytes.restype = [i64, i64, i64], sz
        L.nvfp4_gemm.argtypes = [vp, vp, vp, vp, vp, vp, vp, i32, i64, i64, i64, i64, vp, sz, vp]
        L.w4a4_gemm_workspace_bytes.argtypes, L.w4a4_gemm_workspace_bytes.restype = [i64, i64, i64], sz
        L.w4a4_gemm.argtypes = [vp, i32, i64, vp, vp, vp, vp, vp, i32, i64, i64, i64, i64, vp, sz, vp]
        L.w4a4_gemm_noalloc.argtypes = [vp, i32, i64, vp, vp, vp, vp, vp, i32, i64, i64, i64, i64, vp]
        L.w4a4_gemm_fused.argtypes = [vp, i32, i64, vp, vp, vp, vp, vp, i32, i64, i64, i64, i64, vp]
        L.w4a4_gdn_gates.argtypes = [vp, i32, i64, vp, vp, vp, vp, vp, i64, i64, i64, i64, i64, vp, sz, vp]
        L.nvfp4_fake_quant.argtypes = [vp, i32, i64, i64, i64, vp, vp, i32, i64, vp, vp]
        L.nvfp4_fp8_quantize.argtypes = [vp, i32, i64, vp, vp, vp]
        L.nvfp4_harmonize_requant.argtypes = [vp, vp, i64, i64, i32, vp, vp, vp, vp]
        L.nvfp4_rmsnorm_quantize.argtypes = [vp, i32, i64, i64, i64, vp, i32, ctypes.c_float, vp, vp, vp, vp, vp]
        L.nvfp4_selftest_wait_timeout.argtypes = [i64, vp, vp]
        L.nvfp4_plan_for.argtypes = [i64, i64, i64, i32, i32, vp, vp]
        L.nvfp4_last_device_status.argtypes = [vp, ctypes.POINTER(ctypes.c_int)]
        L.nvfp4_status_string.argtypes, L.nvfp4_status_string.restype = [i32], ctypes.c_char_p
        L.nvfp4_launch_count.argtypes, L.nvfp4_launch_count.restype = [], ctypes.c_uint64
        for f in ("nvfp4_amax_gscale", "nvfp4_quantize", "nvfp4_harmonize_group", "nvfp4_gemm",
                  "w4a4_gemm", "w4a4_gemm_noalloc", "w4a4_gemm_fused", "w4a4_gdn_gates", "nvfp4_fake_quant", "nvfp4_fp8_quantize",
                  "nvfp4_harmonize_requant", "nvfp4_rmsnorm_quantize", "nvfp4_selftest_wait_timeout", "nvfp4_plan_for", "nvfp4_last_device_status"):
            getattr(L, f).restype = i32
        _lib = L
    return _lib


# NVFP4_DEBUG=1: after every call, synchronize and read the device error word,
# so that a kernel whose bounded wait ran out is reported by the call that
# launched it (off by default: it serializes the host with the GPU, and it
# cannot be used while a CUDA graph is being captured).
DEBUG = os.environ.get("NVFP4_DEBUG", "0") not in ("", "0")


def _check(fn: str, status: int) -> None:
    if status != 0:
        raise Nvfp4Error(fn, status)
    if DEBUG:
        flags = last_device_status()
        if flags:
            raise Nvfp4Error(f"{fn} (device error flags {flags:#x})", 6)


def _stream() -> int:
    return torch.cuda.current_stream().cuda_stream


def _ptr(t: torch.Tensor | None) -> int | None:
    return None if t is None else t.data_ptr()


def _in_dtype(x: torch.Tensor) -> int:
    if x.dtype == torch.bfloat16:
        return IN_BF16
    if x.dtype == torch.float32:
        return IN_F32
    raise TypeError(f"unsupported input dtype {x.dtype}")


def _out_dtype(dt: torch.dtype) -> int:
    if dt == torch.bfloat16:
        return OUT_BF16
    if dt == torch.float32:
        return OUT_F32
    raise TypeError(f"unsupported output dtype {dt}")


def _require_cuda(*ts: torch.Tensor) -> None:
    for t in ts:
        if t is not None and not t.is_cuda:
            raise ValueError("tensors must live on the GPU")


# Layout checks: the C ABI takes bare pointers and sizes, so the binding
# makes sure every tensor really has the layout and size those imply before
# any pointer reaches the library (a short buffer would be written past its end).
def _mat(name: str, t: torch.Tensor, rows: int | None = None, cols: int | None = None) -> None:
    """A row-major matrix view: 2-D, unit column stride, any row stride."""
    if t.dim() != 2:
        raise ValueError(f"{name} must be 2-D, got shape {tuple(t.shape)}")
    if (rows is not None and t.shape[0] != rows) or (cols is not None and t.shape[1] != cols):
        raise ValueError(f"{name} must be [{rows}, {cols}], got {tuple(t.shape)}")
    if t.numel() and t.stride(1) != 1:
        raise ValueError(f"{name} must have unit column stride")


def _codes(name: str, t: torch.Tensor, rows: int, K: int) -> None:
    """Packed NVFP4 codes of a [rows, K] tensor: uint8 [rows, K/2], row stride K/2."""
    if t.dtype != torch.uint8:
        raise TypeError(f"{name} must be uint8, got {t.dtype}")
    _mat(name, t, rows, K // 2)
    if rows > 1 and t.stride(0) != K // 2:
        raise ValueError(f"{name} must have row stride K/2 = {K // 2}")


def _buf(name: str, t: torch.Tensor, dtype: torch.dtype, n: int) -> None:
    """A contiguous buffer of at least n elements of dtype."""
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if t.numel() < n:
        raise ValueError(f"{name} holds {t.numel()} elements, needs {n}")


def _offsets(row_offsets) -> list[int]:
    offs = [int(o) for o in row_offsets]
    if len(offs) < 2:
        raise ValueError("row_offsets needs at least two entries")
    return offs


def codes_bytes(rows: int, K: int) -> int:
    return int(lib().nvfp4_codes_bytes(rows, K))


def sf_bytes(rows: int, K: int) -> int:
    return int(lib().nvfp4_sf_bytes(rows, K))


def amax_gscale(x: torch.Tensor, out: torch.Tensor | None = None) -> torch.Tensor:
    """Per-tensor global scale amax/(6*448) as a 1-element fp32 device tensor."""
    _mat("x", x)
    if out is not None:
        _buf("out", out, torch.float32, 1)
    _require_cuda(x, out)
    rows, K = x.shape
    out = torch.empty(1, dtype=torch.float32, device=x.device) if out is None else out
    _check("nvfp4_amax_gscale", lib().nvfp4_amax_gscale(_ptr(x), _in_dtype(x), rows, K, x.stride(0),
                                                         _ptr(out), _stream()))
    return out


def quantize(x: torch.Tensor, gscale: torch.Tensor, codes: torch.Tensor | None = None,
             sf: torch.Tensor | None = None, sf_row0: int = 0, sf_rows_total: int | None = None):
    """NVFP4-quantize x [rows, K]; returns (codes [rows, K/2] uint8, sf uint8 swizzled)."""
    _mat("x", x)
    rows, K = x.shape
    total = rows if sf_rows_total is None else sf_rows_total
    _buf("gscale", gscale, torch.float32, 1)
    if codes is not None:
        _codes("codes", codes, rows, K)
    if sf is not None:
        _buf("sf", sf, torch.uint8, sf_bytes(total, K))
    _require_cuda(x, gscale, codes, sf)
    if codes is None:
        codes = torch.empty((rows, K // 2), dtype=torch.uint8, device=x.device)
    if sf is None:
        sf = torch.empty(sf_bytes(total, K), dtype=torch.uint8, device=x.device)
    _check("nvfp4_quantize", lib().nvfp4_quantize(_ptr(x), _in_dtype(x), rows, K, x.stride(0), _ptr(gscale),
                                                   _ptr(codes), _ptr(sf), sf_row0, total, _stream()))
    return codes, sf


def harmonize(sf: torch.Tensor, rows_total: int, K: int, row_offsets, gscales: torch.Tensor,
              out: torch.Tensor | None = None) -> torch.Tensor:
    """Rewrite a fused group's scales to one shared global scale; returns g*."""
    row_offsets = _offsets(row_offsets)
    _buf("sf", sf, torch.uint8, sf_bytes(rows_total, K))
    _buf("gscales", gscales, torch.float32, len(row_offsets) - 1)
    if out is not None:
        _buf("out", out, torch.float32, 1)
    _require_cuda(sf, gscales, out)
    offs = (ctypes.c_int64 * len(row_offsets))(*row_offsets)
    out = torch.empty(1, dtype=torch.float32, device=sf.device) if out is None else out
    _check("nvfp4_harmonize_group", lib().nvfp4_harmonize_group(
        _ptr(sf), rows_total, K, len(row_offsets) - 1, ctypes.cast(offs, ctypes.c_void_p),
        _ptr(gscales), _ptr(out), _stream()))
    return out


def gemm(a_codes, a_sf, a_gscale, b_codes, b_sf, b_gscale, out_dtype=torch.bfloat16,
         out: torch.Tensor | None = None, workspace: torch.Tensor | None = None) -> torch.Tensor:
    """Y[M, N] = (ga*gb) * dec(A) @ dec(B)^T on pre-quantized NVFP4 operands."""
    _mat("a_codes", a_codes)
    _mat("b_codes", b_codes)
    M, K = a_codes.shape[0], a_codes.shape[1] * 2
    N = b_codes.shape[0]
    _codes("a_codes", a_codes, M, K)
    _codes("b_codes", b_codes, N, K)
    _buf("a_sf", a_sf, torch.uint8, sf_bytes(M, K))
    _buf("b_sf", b_sf, torch.uint8, sf_bytes(N, K))
    _buf("a_gscale", a_gscale, torch.float32, 1)
    _buf("b_gscale", b_gscale, torch.float32, 1)
    if out is not None:
        _mat("out", out, M, N)
    if workspace is not None:
        _buf("workspace", workspace, torch.uint8, 0)
    _require_cuda(a_codes, a_sf, a_gscale, b_codes, b_sf, b_gscale, out, workspace)
    if out is None:
        out = torch.empty((M, N), dtype=out_dtype, device=a_codes.device)
    need = int(lib().nvfp4_gemm_workspace_bytes(M, N, K))
    if workspace is None and need:
        workspace = torch.empty(need, dtype=torch.uint8, device=a_codes.device)
    _check("nvfp4_gemm", lib().nvfp4_gemm(
        _ptr(a_codes), _ptr(a_sf), _ptr(a_gscale), _ptr(b_codes), _ptr(b_sf), _ptr(b_gscale),
        _ptr(out), _out_dtype(out.dtype), out.stride(0), M, N, K, _ptr(workspace),
        0 if workspace is None else workspace.numel(), _stream()))
    return out


def _linear_args(x, x_gscale, w_codes, w_sf, w_gscale, out, workspace=None):
    """Check the operands of a linear-type call; returns (M, K, N)."""
    _mat("x", x)
    M, K = x.shape
    _mat("w_codes", w_codes)
    N = w_codes.shape[0]
    _codes("w_codes", w_codes, N, K)
    _buf("w_sf", w_sf, torch.uint8, sf_bytes(N, K))
    _buf("x_gscale", x_gscale, torch.float32, 1)
    _buf("w_gscale", w_gscale, torch.float32, 1)
    if out is not None:
        _mat("out", out, M, N)
    if workspace is not None:
        _buf("workspace", workspace, torch.uint8, 0)
    _require_cuda(x, x_gscale, w_codes, w_sf, w_gscale, out, workspace)
    return M, K, N


def linear_workspace_bytes(M: int, N: int, K: int) -> int:
    return int(lib().w4a4_gemm_workspace_bytes(M, N, K))


def linear(x: torch.Tensor, x_gscale: torch.Tensor, w_codes: torch.Tensor, w_sf: torch.Tensor,
           w_gscale: torch.Tensor, out_dtype=torch.bfloat16, out: torch.Tensor | None = None,
           workspace: torch.Tensor | None = None) -> torch.Tensor:
    """The W4A4 linear: on-the-fly NVFP4 quantize of x, then the block-scaled GEMM."""
    M, K, N = _linear_args(x, x_gscale, w_codes, w_sf, w_gscale, out, workspace)
    if out is None:
        out = torch.empty((M, N), dtype=out_dtype, device=x.device)
    if workspace is None:
        workspace = torch.empty(linear_workspace_bytes(M, N, K), dtype=torch.uint8, device=x.device)
    _check("w4a4_gemm", lib().w4a4_gemm(
        _ptr(x), _in_dtype(x), x.stride(0), _ptr(x_gscale), _ptr(w_codes), _ptr(w_sf), _ptr(w_gscale),
        _ptr(out), _out_dtype(out.dtype), out.stride(0), M, N, K, _ptr(workspace), workspace.numel(),
        _stream()))
    return out


def linear_noalloc(x: torch.Tensor, x_gscale: torch.Tensor, w_codes: torch.Tensor, w_sf: torch.Tensor,
                   w_gscale: torch.Tensor, out_dtype=torch.bfloat16,
                   out: torch.Tensor | None = None) -> torch.Tensor:
    """The W4A4 linear without a caller workspace: the library's fixed 8 MiB
    scratch buffer holds the quantized activation and split-K partials (for
    callers that cannot allocate device memory at the point of use)."""
    M, K, N = _linear_args(x, x_gscale, w_codes, w_sf, w_gscale, out)
    if out is None:
        out = torch.empty((M, N), dtype=out_dtype, device=x.device)
    _check("w4a4_gemm_noalloc", lib().w4a4_gemm_noalloc(
        _ptr(x), _in_dtype(x), x.stride(0), _ptr(x_gscale), _ptr(w_codes), _ptr(w_sf), _ptr(w_gscale),
        _ptr(out), _out_dtype(out.dtype), out.stride(0), M, N, K, _stream()))
    return out


def linear_fused(x: torch.Tensor, x_gscale: torch.Tensor, w_codes: torch.Tensor, w_sf: torch.Tensor,
                 w_gscale: torch.Tensor, out_dtype=torch.bfloat16, out: torch.Tensor | None = None) -> torch.Tensor:
    """The layer with the activation quantized inside the GEMM kernel, for
    decode-shaped products (M <= 128) and narrow weights (N <= 128, e.g. the
    gate projections); bit-identical to linear() on the shapes measured."""
    M, K, N = _linear_args(x, x_gscale, w_codes, w_sf, w_gscale, out)
    if out is None:
        out = torch.empty((M, N), dtype=out_dtype, device=x.device)
    _check("w4a4_gemm_fused", lib().w4a4_gemm_fused(
        _ptr(x), _in_dtype(x), x.stride(0), _ptr(x_gscale), _ptr(w_codes), _ptr(w_sf), _ptr(w_gscale),
        _ptr(out), _out_dtype(out.dtype), out.stride(0), M, N, K, _stream()))
    return out


def gdn_gates(x: torch.Tensor, x_gscale: torch.Tensor, w_codes: torch.Tensor, w_sf: torch.Tensor,
              w_gscale: torch.Tensor, n_a: int, out: torch.Tensor | None = None,
              workspace: torch.Tensor | None = None) -> torch.Tensor:
    """The fused GDN gate projection: [M, N] float32 with alpha = exp(-softplus(a))
    in columns [0, n_a) and beta = sigmoid(b) in the rest."""
    if out is not None and out.dtype != torch.float32:
        raise TypeError(f"out must be float32, got {out.dtype}")
    M, K, N = _linear_args(x, x_gscale, w_codes, w_sf, w_gscale, out, workspace)
    if out is None:
        out = torch.empty((M, N), dtype=torch.float32, device=x.device)
    if workspace is None:
        workspace = torch.empty(linear_workspace_bytes(M, N, K), dtype=torch.uint8, device=x.device)
    _check("w4a4_gdn_gates", lib().w4a4_gdn_gates(
        _ptr(x), _in_dtype(x), x.stride(0), _ptr(x_gscale), _ptr(w_codes), _ptr(w_sf), _ptr(w_gscale),
        _ptr(out), out.stride(0), M, N, int(n_a), K, _ptr(workspace), workspace.numel(), _stream()))
    return out


def fake_quant(x: torch.Tensor, gscale: torch.Tensor, out_dtype=torch.float32,
               stats: torch.Tensor | None = None) -> tuple[torch.Tensor, torch.Tensor]:
    """Quantize-then-dequantize x; returns (values, [sum sq error, sum sq x] float64)."""
    _mat("x", x)
    _buf("gscale", gscale, torch.float32, 1)
    if stats is not None:
        _buf("stats", stats, torch.float64, 2)
    _require_cuda(x, gscale, stats)
    rows, K = x.shape
    out = torch.empty((rows, K), dtype=out_dtype, device=x.device)
    if stats is None:
        stats = torch.empty(2, dtype=torch.float64, device=x.device)
    _check("nvfp4_fake_quant", lib().nvfp4_fake_quant(
        _ptr(x), _in_dtype(x), rows, K, x.stride(0), _ptr(gscale), _ptr(out), _out_dtype(out_dtype),
        out.stride(0), _ptr(stats), _stream()))
    return out, stats


def fp8_quantize(x: torch.Tensor, scale: torch.Tensor, out: torch.Tensor | None = None) -> torch.Tensor:
    """FP8 E4M3 codes (uint8, sign in bit 7) of x / scale, x contiguous."""
    if not x.is_contiguous():
        raise ValueError("x must be contiguous")
    _buf("scale", scale, torch.float32, 1)
    if out is not None:
        _buf("out", out, torch.uint8, x.numel())
    _require_cuda(x, scale, out)
    if out is None:
        out = torch.empty(x.shape, dtype=torch.uint8, device=x.device)
    _check("nvfp4_fp8_quantize", lib().nvfp4_fp8_quantize(_ptr(x), _in_dtype(x), x.numel(), _ptr(scale),
                                                          _ptr(out), _stream()))
    return out


def harmonize_requant(codes: torch.Tensor, sf: torch.Tensor, K: int, row_offsets, gscales: torch.Tensor,
                      out: torch.Tensor | None = None) -> torch.Tensor:
    """Re-quantize a fused group's codes and scales (in place) against one
    shared global scale; returns g*."""
    row_offsets = _offsets(row_offsets)
    _codes("codes", codes, row_offsets[-1], K)
    _buf("sf", sf, torch.uint8, sf_bytes(row_offsets[-1], K))
    _buf("gscales", gscales, torch.float32, len(row_offsets) - 1)
    if out is not None:
        _buf("out", out, torch.float32, 1)
    _require_cuda(codes, sf, gscales, out)
    offs = (ctypes.c_int64 * len(row_offsets))(*row_offsets)
    out = torch.empty(1, dtype=torch.float32, device=sf.device) if out is None else out
    _check("nvfp4_harmonize_requant", lib().nvfp4_harmonize_requant(
        _ptr(codes), _ptr(sf), int(row_offsets[-1]), K, len(row_offsets) - 1, ctypes.cast(offs, ctypes.c_void_p),
        _ptr(gscales), _ptr(out), _stream()))
    return out


def rmsnorm_quantize(x: torch.Tensor, w: torch.Tensor, eps: float, gscale: torch.Tensor,
                     zero_centered: bool = False, codes: torch.Tensor | None = None,
                     sf: torch.Tensor | None = None, inv: torch.Tensor | None = None):
    """NVFP4 codes and scales of the BF16 RMSNorm of x with weight w (bf16 [K]);
    returns (codes, sf, inv) where inv [rows] fp32 holds each row's 1/rms."""
    _mat("x", x)
    rows, K = x.shape
    if w.dtype != torch.bfloat16 or not w.is_contiguous() or w.numel() != K:
        raise TypeError(f"the norm weight must be a contiguous bf16 vector of {K} elements")
    _buf("gscale", gscale, torch.float32, 1)
    if codes is not None:
        _codes("codes", codes, rows, K)
    if sf is not None:
        _buf("sf", sf, torch.uint8, sf_bytes(rows, K))
    if inv is not None:
        _buf("inv", inv, torch.float32, rows)
    _require_cuda(x, w, gscale, codes, sf, inv)
    if codes is None:
        codes = torch.empty((rows, K // 2), dtype=torch.uint8, device=x.device)
    if sf is None:
        sf = torch.empty(sf_bytes(rows, K), dtype=torch.uint8, device=x.device)
    if inv is None:
        inv = torch.empty(rows, dtype=torch.float32, device=x.device)
    _check("nvfp4_rmsnorm_quantize", lib().nvfp4_rmsnorm_quantize(
        _ptr(x), _in_dtype(x), rows, K, x.stride(0), _ptr(w), 1 if zero_centered else 0, float(eps),
        _ptr(gscale), _ptr(codes), _ptr(sf), _ptr(inv), _stream()))
    return codes, sf, inv


PLAN_KINDS = {0: "single", 1: "pair", 2: "cluster"}


def plan_for(M: int, N: int, K: int, sms: int = 148, pair_clusters: int = 0, split_clusters=None) -> dict:
    """The GEMM launch plan for an M x N x K product given the device's
    occupancy figures (no device is touched); split_clusters[bn][c] for MMA N
    32/64/128 and cluster sizes c = 0..8."""
    table = None
    if split_clusters is not None:
        flat = [int(v) for row in split_clusters for v in row]
        if len(flat) != 27:
            raise ValueError("split_clusters must be 3 rows of 9 counts")
        table = (ctypes.c_int * 27)(*flat)
    out = (ctypes.c_int * 8)()
    _check("nvfp4_plan_for", lib().nvfp4_plan_for(M, N, K, sms, pair_clusters,
                                                  None if table is None else ctypes.cast(table, ctypes.c_void_p),
                                                  ctypes.cast(out, ctypes.c_void_p)))
    keys = ("kind", "bn", "swap", "splits", "grid", "tiles_a", "tiles_b", "kstages")
    d = dict(zip(keys, list(out)))
    d["kind"] = PLAN_KINDS[d["kind"]]
    d["swap"] = bool(d["swap"])
    return d


def selftest_wait_timeout(limit_ns: int = 50_000_000) -> torch.Tensor:
    """Run the bounded-wait self-test; returns the device int the waiter wrote
    (0: the wait ran out, as intended)."""
    res = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    _check("nvfp4_selftest_wait_timeout", lib().nvfp4_selftest_wait_timeout(int(limit_ns), _ptr(res), _stream()))
    return res


def last_device_status() -> int:
    """Take and clear the device error flags on the current stream, wait for
    that stream, and return the flags (0 = clean)."""
    flags = ctypes.c_int(0)
    st = lib().nvfp4_last_device_status(_stream(), ctypes.byref(flags))
    if st not in (0, 6):
        raise Nvfp4Error("nvfp4_last_device_status", st)
    return flags.value


def launch_count() -> int:
    return int(lib().nvfp4_launch_count())
