"""GPU parity of the rows marked "next" against the oracle, through the C ABI:
the GDN gate projection with its activations fused into the GEMM epilogue,
fake-quant (Q -> DQ) with its error statistics, and static-scale FP8 E4M3
quantize."""
import numpy as np
import pytest
import torch

import oracle
from nvfp4_w4a4_quantized_06_b200 import native
from nvfp4_w4a4_quantized_06_b200 import workloads as W
from parity import f32, to_f32_numpy

pytestmark = pytest.mark.gpu
DEV = "cuda"
GEMM_RTOL = 1e-3


def _gate_weights(wl):
    K, N = wl.K, wl.N
    offs = np.concatenate([[0], np.cumsum(wl.modules)]).astype(np.int64)
    codes = torch.empty((N, K // 2), dtype=torch.uint8, device=DEV)
    sf = torch.empty(native.sf_bytes(N, K), dtype=torch.uint8, device=DEV)
    mods = []
    for m in range(len(wl.modules)):
        w = W.make_w(wl, m)
        g = native.amax_gscale(w.to(DEV))
        native.quantize(w.to(DEV), g, codes=codes[offs[m]:offs[m + 1]], sf=sf, sf_row0=int(offs[m]), sf_rows_total=N)
        mods.append((w, g))
    gstar = native.harmonize(sf, N, K, offs, torch.cat([g for _, g in mods]))
    # the oracle's copy of the same fused, harmonized weight
    ref_sf = np.zeros(oracle.sf_bytes(N, K), np.uint8)
    ref_codes = []
    for m, (w, g) in enumerate(mods):
        c, _ = oracle.quantize(to_f32_numpy(w), f32(g), sf=ref_sf, sf_row0=int(offs[m]))
        ref_codes.append(c)
    ref_gstar = oracle.harmonize(ref_sf, K, offs, [f32(g) for _, g in mods])
    assert f32(gstar) == ref_gstar
    return codes, sf, gstar, np.concatenate(ref_codes), ref_sf, ref_gstar


@pytest.mark.parametrize("M", [4096, 32])
def test_gdn_gates_fused_epilogue(M):
    """alpha = exp(-softplus(a)) on the 48 a columns, beta = sigmoid(b) on the
    48 b columns.  Both activations have slope at most 1/4, so the bound is a
    quarter of the GEMM's 1e-3 * sum|products|, plus the fp32 evaluation of
    exp / log1p (a few ulps of values <= 1)."""
    wl = W.WORKLOADS["gdn_gates_ab"]
    codes, sf, gw, rcodes, rsf, rg = _gate_weights(wl)
    x_cpu = W.make_x(wl)[:M]
    x = x_cpu.to(DEV)
    gx = native.amax_gscale(x)
    out = native.gdn_gates(x, gx, codes, sf, gw, n_a=wl.modules[0])
    torch.cuda.synchronize()
    assert native.last_device_status() == 0
    rows = W.sample_rows(M, min(M, 384), seed=5)
    y_ref, yabs, _, _ = oracle.linear_reference(to_f32_numpy(x_cpu[torch.from_numpy(rows)]), f32(gx), rcodes, rsf, rg)
    ref = oracle.gdn_gates(y_ref, wl.modules[0])
    got = out[torch.from_numpy(rows).to(DEV)].double().cpu().numpy()
    tol = 0.25 * GEMM_RTOL * yabs + 1e-5 * np.abs(ref) + 1e-7
    err = np.abs(got - ref)
    assert np.all(err <= tol), float((err - tol).max())
    assert np.all((got >= 0) & (got <= 1))


@pytest.mark.parametrize("in_dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("rows,K", [(300, 576), (64, 5120)])
def test_fake_quant_bit_exact(rows, K, in_dtype, out_dtype):
    x_cpu = W.gaussian(rows, K, seed=rows + K, outliers=W.Outliers("scale", 0.03, 35.0), dtype=in_dtype)
    x = x_cpu.to(DEV)
    g = native.amax_gscale(x)
    out, stats = native.fake_quant(x, g, out_dtype=out_dtype)
    torch.cuda.synchronize()
    assert native.last_device_status() == 0
    dq, se, sx = oracle.fake_quant(to_f32_numpy(x_cpu), f32(g))
    ref = torch.from_numpy(dq.astype(np.float32)).to(out_dtype)       # exact value rounded to fp32, then to bf16
    assert torch.equal(out.cpu(), ref)
    st = stats.cpu().numpy()
    assert st[0] == pytest.approx(se, rel=1e-9) and st[1] == pytest.approx(sx, rel=1e-9)


def test_fake_quant_relative_error_workload():
    """The relative activation error of the prefill activation stays in the
    same band as the pages' A4 error (about 7.5-9.2% on real activations)."""
    wl = W.WORKLOADS["prefill_mlp_gate_up"]
    x = W.make_x(wl).to(DEV)
    g = native.amax_gscale(x)
    _, stats = native.fake_quant(x, g)
    se, sx = stats.cpu().numpy()
    rel = float(np.sqrt(se / sx))
    assert 0.07 < rel < 0.10, rel


@pytest.mark.parametrize("in_dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("scale", [0.125, 0.0371, 3.7e-3])
def test_fp8_quantize_bit_exact(in_dtype, scale):
    rng = np.random.default_rng(int(scale * 1e4))
    s = np.float32(scale)
    vals = np.array([oracle.e4m3_decode(c) for c in range(0x7F)], np.float64)
    mids = (vals[1:] + vals[:-1]) / 2
    # values on, next to and between the grid points (scaled), beyond the
    # range, zeros, and Gaussian bulk
    parts = [vals, mids, np.nextafter(mids, 0), np.nextafter(mids, 1e9), [500.0, 1e6, 0.0, -0.0]]
    grid = np.concatenate([np.concatenate(parts), -np.concatenate(parts)]) * float(s)
    bulk = rng.standard_normal(40000) * float(s) * 60
    x = np.concatenate([grid, bulk]).astype(np.float32)
    x = x[: x.size // 8 * 8]
    xt = torch.from_numpy(x).to(in_dtype)
    q = native.fp8_quantize(xt.to(DEV), torch.tensor([s], device=DEV))
    torch.cuda.synchronize()
    assert native.last_device_status() == 0
    ref = oracle.fp8_quantize(to_f32_numpy(xt), s)
    assert np.array_equal(q.cpu().numpy(), ref)
