"""Shared helpers for the GPU parity tests: run a step through the C ABI,
run the same step in the CPU oracle, compare.

Tolerances (derived from the arithmetic, not tuned):
  * codes, scales, global scales: bit-exact;
  * GEMM, FP32 output: every element |Y - Yref| <= 1e-3 * Yabs, where Yabs is
    the float64 sum of |products| (only the FP32 accumulation order differs
    from the float64 reference), and ||Y - Yref||_F <= 1e-3 * ||Yref||_F;
  * GEMM, BF16 output: the same plus BF16's half-ulp, 2^-8 * |Yref|.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
from nvfp4_w4a4_quantized_06_b200 import native

GEMM_RTOL = 1e-3
BF16_HALF_ULP = 2.0 ** -8


def to_f32_numpy(x: torch.Tensor) -> np.ndarray:
    return x.detach().to("cpu", torch.float32).numpy()


def oracle_quantize(x: torch.Tensor, g: np.float32):
    return oracle.quantize(to_f32_numpy(x), g)


def assert_codes_equal(gpu_codes: torch.Tensor, ref_codes: np.ndarray, what: str = "codes"):
    got = gpu_codes.cpu().numpy()
    if not np.array_equal(got, ref_codes):
        bad = np.argwhere(got != ref_codes)
        r, c = bad[0]
        raise AssertionError(f"{what}: {len(bad)} bytes differ; first at {tuple(bad[0])}: "
                             f"gpu {got[r, c]:#04x} oracle {ref_codes[r, c]:#04x}")


def assert_sf_rows_equal(gpu_sf: torch.Tensor, ref_sf: np.ndarray, rows_gpu, rows_ref, K: int):
    got = oracle.sf_gather(gpu_sf.cpu().numpy(), rows_gpu, K)
    want = oracle.sf_gather(ref_sf, rows_ref, K)
    if not np.array_equal(got, want):
        bad = np.argwhere(got != want)
        r, c = bad[0]
        raise AssertionError(f"scales: {len(bad)} differ; first at row {rows_gpu[r]} col {c}: "
                             f"gpu {got[r, c]:#04x} oracle {want[r, c]:#04x}")


def assert_gemm_close(y_gpu: torch.Tensor, y_ref: np.ndarray, yabs: np.ndarray):
    y = y_gpu.detach().to("cpu", torch.float64).numpy()
    tol = GEMM_RTOL * yabs
    if y_gpu.dtype == torch.bfloat16:
        tol = tol + BF16_HALF_ULP * np.abs(y_ref)
    err = np.abs(y - y_ref)
    bad = err > tol
    if bad.any():
        i = np.argwhere(bad)[0]
        raise AssertionError(
            f"{bad.sum()} of {bad.size} outputs outside tolerance; first {tuple(i)}: gpu {y[tuple(i)]!r} "
            f"ref {y_ref[tuple(i)]!r} |.| {yabs[tuple(i)]!r}; max err/Yabs "
            f"{float(np.max(err / np.maximum(yabs, 1e-300))):.3e}")
    if y_gpu.dtype == torch.float32:
        den = np.linalg.norm(y_ref)
        if den > 0:
            assert np.linalg.norm(y - y_ref) <= GEMM_RTOL * den
    return float(np.max(err / np.maximum(yabs, 1e-300)))


def checked_gscale(x_cpu: torch.Tensor, x_dev: torch.Tensor | None = None):
    """The global scale of an input as the oracle computes it on the CPU copy,
    checked bit for bit against the library's nvfp4_amax_gscale on the device
    copy.  Returns (the oracle's value as np.float32, the same value as a
    1-element device tensor): both sides of a parity test then start from the
    oracle's scale, and no oracle input comes from the CUDA path."""
    g_ref = oracle.global_scale(to_f32_numpy(x_cpu))
    if x_dev is None:
        x_dev = x_cpu.to("cuda")
    g_gpu = f32(native.amax_gscale(x_dev))
    assert np.array([g_gpu]).view(np.uint32)[0] == np.array([g_ref]).view(np.uint32)[0], (g_gpu, g_ref)
    return g_ref, torch.tensor([g_ref], dtype=torch.float32, device=x_dev.device)


def f32(t: torch.Tensor) -> np.float32:
    return np.float32(t.item())
