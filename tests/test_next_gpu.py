"""GPU parity of the rows marked "next" against the oracle, through the C ABI:
the GDN gate projection with its activations fused into the GEMM epilogue,
fake-quant (Q -> DQ) with its error statistics, static-scale FP8 E4M3
quantize, the re-quantizing harmonize and the quantize fused into RMSNorm."""
import numpy as np
import pytest
import torch

import oracle
from nvfp4_w4a4_quantized_06_b200 import native
from nvfp4_w4a4_quantized_06_b200 import workloads as W
from parity import assert_codes_equal, assert_sf_rows_equal, checked_gscale, f32, to_f32_numpy

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
        _, g = checked_gscale(w)
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
    48 b columns, every output of the launch checked.  Both activations have slope at most 1/4, so the bound is a
    quarter of the GEMM's 1e-3 * sum|products|, plus the fp32 evaluation of
    1 / (1 + e^{+-y}) (a few ulps of values <= 1)."""
    wl = W.WORKLOADS["gdn_gates_ab"]
    codes, sf, gw, rcodes, rsf, rg = _gate_weights(wl)
    x_cpu = W.make_x(wl)[:M]
    x = x_cpu.to(DEV)
    _, gx = checked_gscale(x_cpu, x)
    out = native.gdn_gates(x, gx, codes, sf, gw, n_a=wl.modules[0])
    torch.cuda.synchronize()
    assert native.last_device_status() == 0
    y_ref, yabs, _, _ = oracle.linear_reference(to_f32_numpy(x_cpu), f32(gx), rcodes, rsf, rg)
    ref = oracle.gdn_gates(y_ref, wl.modules[0])
    got = out.double().cpu().numpy()
    tol = 0.25 * GEMM_RTOL * yabs + 1e-5 * np.abs(ref) + 1e-7
    err = np.abs(got - ref)
    assert np.all(err <= tol), float((err - tol).max())
    assert np.all((got >= 0) & (got <= 1))


def test_gdn_gates_saturate():
    """Pre-activations far past where an fp32 exponential overflows (|y| up
    to about 770): the gates reach their limits 0 and 1, never NaN, and match
    the oracle's float64 activations within the same bound."""
    M, N, n_a, K = 64, 96, 48, 256
    c = torch.linspace(-2.0, 2.0, M).to(torch.bfloat16)
    t = torch.tensor([((j % 12) + 1) / 8.0 * (1 if j % 2 else -1) for j in range(N)]).to(torch.bfloat16)
    x_cpu = c[:, None].expand(M, K).contiguous()
    w_cpu = t[:, None].expand(N, K).contiguous()
    x, w = x_cpu.to(DEV), w_cpu.to(DEV)
    (gx_r, gx), (gw_r, gw) = checked_gscale(x_cpu, x), checked_gscale(w_cpu, w)
    wc, ws = native.quantize(w, gw)
    out = native.gdn_gates(x, gx, wc, ws, gw, n_a=n_a)
    torch.cuda.synchronize()
    assert native.last_device_status() == 0
    rwc, rws = oracle.quantize(to_f32_numpy(w_cpu), gw_r)
    y_ref, yabs, _, _ = oracle.linear_reference(to_f32_numpy(x_cpu), gx_r, rwc, rws, gw_r)
    assert np.abs(y_ref).max() > 600
    ref = oracle.gdn_gates(y_ref, n_a)
    got = out.double().cpu().numpy()
    assert not np.isnan(got).any()
    tol = 0.25 * GEMM_RTOL * yabs + 1e-5 * np.abs(ref) + 1e-7
    assert np.all(np.abs(got - ref) <= tol), float((np.abs(got - ref) - tol).max())
    assert np.all((got >= 0) & (got <= 1))
    assert (got == 0).any() and (got == 1).any()


@pytest.mark.parametrize("in_dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("rows,K", [(300, 576), (64, 5120)])
def test_fake_quant_bit_exact(rows, K, in_dtype, out_dtype):
    x_cpu = W.gaussian(rows, K, seed=rows + K, outliers=W.Outliers("scale", 0.03, 35.0), dtype=in_dtype)
    x = x_cpu.to(DEV)
    g_ref, g = checked_gscale(x_cpu, x)
    out, stats = native.fake_quant(x, g, out_dtype=out_dtype)
    torch.cuda.synchronize()
    assert native.last_device_status() == 0
    dq, se, sx = oracle.fake_quant(to_f32_numpy(x_cpu), g_ref)
    ref = torch.from_numpy(dq.astype(np.float32)).to(out_dtype)       # exact value rounded to fp32, then to bf16
    assert torch.equal(out.cpu(), ref)
    # the kernel sums each 16-element block in fp32 (non-negative terms, one
    # rounding per term and per addition: relative error below 18 * 2^-24)
    # and the blocks in float64
    st = stats.cpu().numpy()
    assert st[0] == pytest.approx(se, rel=18 * 2.0 ** -24) and st[1] == pytest.approx(sx, rel=18 * 2.0 ** -24)


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


# ------------------------------------------------- re-quantizing harmonize
def _quantized_group(mods, K):
    """Quantize each module with its own scale into one fused buffer, on the
    GPU and in the oracle; returns both copies."""
    N = sum(w.shape[0] for w, _ in mods)
    offs = np.concatenate([[0], np.cumsum([w.shape[0] for w, _ in mods])]).astype(np.int64)
    codes = torch.empty((N, K // 2), dtype=torch.uint8, device=DEV)
    sf = torch.empty(native.sf_bytes(N, K), dtype=torch.uint8, device=DEV)
    ref_sf = np.zeros(oracle.sf_bytes(N, K), np.uint8)
    ref_codes = []
    for m, (w, g) in enumerate(mods):
        gd = torch.tensor([g], dtype=torch.float32, device=DEV)
        native.quantize(w.to(DEV), gd, codes=codes[offs[m]:offs[m + 1]], sf=sf, sf_row0=int(offs[m]),
                        sf_rows_total=N)
        c, _ = oracle.quantize(to_f32_numpy(w), np.float32(g), sf=ref_sf, sf_row0=int(offs[m]))
        ref_codes.append(c)
    torch.cuda.synchronize()
    assert_codes_equal(codes, np.concatenate(ref_codes))
    assert np.array_equal(sf.cpu().numpy(), ref_sf)
    return offs, codes, sf, np.concatenate(ref_codes), ref_sf


@pytest.mark.parametrize("case", ["gates_ab", "ragged3", "tiny_ratio"])
def test_harmonize_requant_matches_oracle(case):
    if case == "gates_ab":
        K, specs = 5120, [(48, 1, 0.02), (48, 2, 0.02)]
    elif case == "ragged3":
        K, specs = 320, [(33, 3, 0.02), (100, 4, 0.05), (7, 5, 0.004)]
    else:                                   # one module 2e-5 as large: its scales go subnormal at g*
        K, specs = 256, [(40, 6, 0.02), (24, 7, 0.02 * 2e-5)]
    mods = []
    for rows, seed, std in specs:
        w = W.gaussian(rows, K, seed=seed, std=std)
        mods.append((w, oracle.global_scale(to_f32_numpy(w))))
    offs, codes, sf, rc, rs = _quantized_group(mods, K)
    gs = torch.tensor([g for _, g in mods], dtype=torch.float32, device=DEV)
    gstar = native.harmonize_requant(codes, sf, K, offs, gs)
    ref_codes, ref_sf, ref_gstar = oracle.harmonize_requant(rc, rs, K, offs, [g for _, g in mods])
    torch.cuda.synchronize()
    assert f32(gstar) == ref_gstar
    assert_codes_equal(codes, ref_codes)
    assert np.array_equal(sf.cpu().numpy(), ref_sf), "scale buffer differs"
    if case == "tiny_ratio":
        assert not np.array_equal(ref_codes, rc)        # the case does move codes
    assert native.last_device_status() == 0


def test_harmonize_requant_full_qkv_z_sampled():
    """The fused qkv+z weight (10240 + 6144 rows, K 5120) re-quantized on the
    GPU in one launch; a seeded sample of each module's rows checked against
    the oracle run on just those rows (the operation is row by row)."""
    wl = W.WORKLOADS["gdn_qkv_z"]
    K, N = wl.K, wl.N
    offs = np.concatenate([[0], np.cumsum(wl.modules)]).astype(np.int64)
    codes = torch.empty((N, K // 2), dtype=torch.uint8, device=DEV)
    sf = torch.empty(native.sf_bytes(N, K), dtype=torch.uint8, device=DEV)
    ws, gs = [], []
    for m in range(len(wl.modules)):
        w = W.make_w(wl, m)
        if m == 1:
            w = w * 0.37                    # a ratio that is not a power of two
        ws.append(w)
        gs.append(oracle.global_scale(to_f32_numpy(w)))
        native.quantize(w.to(DEV), torch.tensor([gs[m]], device=DEV), codes=codes[offs[m]:offs[m + 1]], sf=sf,
                        sf_row0=int(offs[m]), sf_rows_total=N)
    gstar = native.harmonize_requant(codes, sf, K, offs, torch.tensor(gs, device=DEV))
    samp = [W.sample_rows(wl.modules[m], 96, seed=m) for m in range(len(wl.modules))]
    sub_offs = np.concatenate([[0], np.cumsum([len(x) for x in samp])])
    sub_sf = np.zeros(oracle.sf_bytes(int(sub_offs[-1]), K), np.uint8)
    sub_codes = np.concatenate([oracle.quantize(to_f32_numpy(ws[m][torch.from_numpy(s)]), gs[m], sf=sub_sf,
                                                sf_row0=int(sub_offs[m]))[0] for m, s in enumerate(samp)])
    ref_codes, ref_sf, ref_gstar = oracle.harmonize_requant(sub_codes, sub_sf, K, sub_offs, gs)
    torch.cuda.synchronize()
    assert f32(gstar) == ref_gstar
    fused_rows = np.concatenate([offs[m] + s for m, s in enumerate(samp)])
    assert_codes_equal(codes[torch.from_numpy(fused_rows).to(DEV)], ref_codes)
    assert_sf_rows_equal(sf, ref_sf, fused_rows, np.arange(len(fused_rows)), K)
    assert native.last_device_status() == 0


# ------------------------------------------ quantize fused into RMSNorm
def _static_scale(x: torch.Tensor, w: torch.Tensor, eps: float, zero_centered: bool) -> np.float32:
    """A calibrated static scale for the normalized activation, from torch's
    own CPU RMSNorm (input preparation only)."""
    gamma = (1 + w.float()) if zero_centered else w.float()
    y = torch.nn.functional.rms_norm(x.float(), (x.shape[1],), weight=gamma, eps=eps)
    return np.float32(y.abs().max().item()) / np.float32(2688.0)


def _check_rmsnorm(x_cpu, w_cpu, eps, zero_centered, rows=None):
    """GPU rmsnorm_quantize of all of x against the oracle on `rows` (all by
    default): per-row factor bit-exact, codes and scales byte for byte."""
    g = _static_scale(x_cpu, w_cpu, eps, zero_centered)
    codes, sf, inv = native.rmsnorm_quantize(x_cpu.to(DEV), w_cpu.to(DEV), eps,
                                             torch.tensor([g], device=DEV), zero_centered)
    R, K = x_cpu.shape
    sel = np.arange(R) if rows is None else rows
    xs = to_f32_numpy(x_cpu[torch.from_numpy(sel)])
    wn = to_f32_numpy(w_cpu)
    rc, rs, _, rinv, near = oracle.rmsnorm_quantize(xs, wn, eps, g, zero_centered)
    torch.cuda.synchronize()
    ginv = inv.cpu().numpy()[sel]
    # The kernel evaluates the mean square to about 2^-48 relative, so it
    # rounds the per-row factor correctly unless the exact value lies within
    # ~2^-45 of a midpoint between two floats; the oracle flags such rows.
    # The seeded inputs are chosen so that no row is that close: every row is
    # then compared with the oracle's correctly rounded factor, bit for bit.
    assert not near.any(), f"rows {np.flatnonzero(near)} sit at a rounding midpoint; change the seed"
    assert np.array_equal(ginv.view(np.uint32), rinv.view(np.uint32)), "per-row factor differs"
    if rows is None:
        assert_codes_equal(codes, rc)
        assert np.array_equal(sf.cpu().numpy(), rs), "swizzled scale buffer differs"
    else:
        assert_codes_equal(codes[torch.from_numpy(sel).to(DEV)], rc)
        assert_sf_rows_equal(sf, rs, sel, np.arange(len(sel)), K)
        if R % 128:
            pad = oracle.sf_gather(sf.cpu().numpy(), np.arange(R, (R + 127) // 128 * 128), K)
            assert np.all(pad == 0)
    assert native.last_device_status() == 0


@pytest.mark.parametrize("rows,K,dtype,zc", [
    (1, 64, torch.bfloat16, False),
    (33, 320, torch.bfloat16, True),
    (300, 5120, torch.bfloat16, False),
    (129, 2048, torch.float32, False),
    (4096, 5120, torch.bfloat16, True),       # several rows per warp
    (2000, 1024, torch.float32, True),
    (64, 17408, torch.bfloat16, False),       # 34 blocks per lane
    (3, 111872, torch.bfloat16, False),       # the widest row the norm weight's shared copy allows
    (2, 111872, torch.float32, True),
])
def test_rmsnorm_quantize_matches_oracle(rows, K, dtype, zc):
    x = W.gaussian(rows, K, seed=rows + K, outliers=W.Outliers("scale", 0.01, 30.0), dtype=dtype)
    w = W.norm_weight(K, seed=K, zero_centered=zc)
    _check_rmsnorm(x, w, 1e-6, zc, rows=None if rows * K <= 2_000_000 else W.sample_rows(rows, 256))


def test_rmsnorm_quantize_degenerate_rows():
    """All-zero rows (inv = 1/sqrt(eps)), constant rows, a lone spike, and
    tiny values next to large ones in one row."""
    K = 256
    x = torch.zeros((6, K), dtype=torch.float32)
    x[1] = 1.875
    x[2, 17] = 8.0
    x[3] = torch.linspace(-3, 3, K)
    x[4, ::2] = 1e-20
    x[4, 1] = 300.0
    x[5] = -2.0
    w = W.norm_weight(K, seed=3)
    _check_rmsnorm(x.to(torch.bfloat16), w, 0.484375, False)
    _check_rmsnorm(x, w, 1e-6, True)


def test_rmsnorm_quantize_full_prefill_sampled():
    """The prefill residual (32768 x 5120 bf16) in one launch; 192 seeded rows
    checked against the oracle, padding rows zero."""
    wl = W.WORKLOADS["prefill_mlp_gate_up"]
    x = W.make_x(wl)
    w = W.norm_weight(wl.K, seed=11)
    _check_rmsnorm(x, w, 1e-6, False, rows=W.sample_rows(wl.M, 192))
