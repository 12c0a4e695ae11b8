"""GPU parity of the global scale, quantize and harmonize kernels against the
CPU oracle, through the C ABI.  Codes and scales must be bit-exact."""
import numpy as np
import pytest
import torch

import oracle
from nvfp4_w4a4_quantized_06_b200 import native
from nvfp4_w4a4_quantized_06_b200 import workloads as W
from parity import assert_codes_equal, assert_sf_rows_equal, checked_gscale, f32, to_f32_numpy

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _quant_check(x_cpu: torch.Tensor, g=None, ld_pad: int = 0):
    """quantize on GPU and in the oracle; compare every code and scale byte
    (including padding rows) and the global scale."""
    rows, K = x_cpu.shape
    if ld_pad:
        big = torch.zeros((rows, K + ld_pad), dtype=x_cpu.dtype)
        big[:, :K] = x_cpu
        x = big.to(DEV)[:, :K]
    else:
        x = x_cpu.to(DEV)
    g_gpu = native.amax_gscale(x)
    g_ref = oracle.global_scale(to_f32_numpy(x_cpu))
    assert f32(g_gpu) == g_ref, (f32(g_gpu), g_ref)
    if g is not None:
        g_gpu = torch.tensor([g], dtype=torch.float32, device=DEV)
        g_ref = np.float32(g)
    codes, sf = native.quantize(x, g_gpu)
    rc, rs = oracle.quantize(to_f32_numpy(x_cpu), g_ref)
    torch.cuda.synchronize()
    assert_codes_equal(codes, rc)
    assert np.array_equal(sf.cpu().numpy(), rs), "swizzled scale buffer differs"
    assert native.last_device_status() == 0
    return codes, sf


def test_tiny_fp32():
    wl = W.WORKLOADS["tiny"]
    _quant_check(W.make_x(wl))
    _quant_check(W.make_w(wl, 0))


@pytest.mark.parametrize("rows,K", [(1, 64), (33, 192), (127, 320), (129, 256), (300, 576), (4096, 2048)])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_ragged_shapes(rows, K, dtype):
    x = W.gaussian(rows, K, seed=rows * 7 + K, outliers=W.Outliers("scale", 0.05, 40.0), dtype=dtype)
    _quant_check(x)


def test_strided_rows():
    x = W.gaussian(65, 320, seed=3)
    _quant_check(x, ld_pad=64)


def test_e2m1_rounding_sweep():
    """g = 1 and one element of every block equal to 6: t = 1, scale 1.0, d = 1,
    so every other element is encoded as itself -- a dense sweep of the
    hardware conversion around all E2M1 midpoints, ties and saturation."""
    vals = [np.float32(v) for v in np.linspace(-7.5, 7.5, 3001)]
    for m in [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0]:
        for sgn in (1, -1):
            v = np.float32(sgn * m)
            vals.append(v)
            for _ in range(3):
                v = np.nextafter(v, np.float32(100 * sgn)); vals.append(v)
            v = np.float32(sgn * m)
            for _ in range(3):
                v = np.nextafter(v, np.float32(0)); vals.append(v)
    vals += [np.float32(-0.0), np.float32(1e-38), np.float32(-1e-38), np.float32(1e-45)]
    vals = np.array(vals, np.float32)
    nb = (len(vals) + 14) // 15
    x = np.zeros((nb, 16), np.float32)
    x[:, 0] = 6.0
    flat = np.zeros(nb * 15, np.float32)
    flat[:len(vals)] = vals
    x[:, 1:] = np.clip(flat.reshape(nb, 15), -6.0, 6.0)
    rows = (nb * 16 + 255) // 256
    X = np.zeros(rows * 256, np.float32)
    X[:nb * 16] = x.reshape(-1)
    _quant_check(torch.from_numpy(X.reshape(rows, 256)), g=1.0)


def test_e4m3_rounding_sweep():
    """g = fl32(1/6) makes fl32(6*g) == 1, so every scale byte is E4M3(amax):
    a sweep of the hardware scale conversion over midpoints, subnormals and
    saturation (amax beyond 464 saturates to 448)."""
    g = np.float32(1.0) / np.float32(6.0)
    assert np.float32(6.0) * g == np.float32(1.0)
    amax = []
    for c in range(0x7E):
        lo, hi = oracle.e4m3_decode(c), oracle.e4m3_decode(c + 1)
        mid = np.float32((lo + hi) / 2)
        for v in (mid, np.nextafter(mid, np.float32(0)), np.nextafter(mid, np.float32(1e9)), np.float32(hi)):
            amax.append(v)
    amax += [np.float32(v) for v in (500.0, 1000.0, 1e6, 2.0 ** -11, 2.0 ** -10, 3e-3)]
    amax = np.array(amax, np.float32)
    x = np.zeros((len(amax), 16), np.float32)
    x[:, 3] = amax
    x[:, 7] = -amax / 3
    rows = (x.size + 255) // 256
    X = np.zeros(rows * 256, np.float32)
    X[:x.size] = x.reshape(-1)
    _quant_check(torch.from_numpy(X.reshape(rows, 256)), g=float(g))


def test_zero_tensor_and_saturation():
    _quant_check(torch.zeros(16, 128))                        # g = 1, all scales and codes 0
    x = W.gaussian(40, 256, seed=8, dtype=torch.float32)
    _quant_check(x, g=float(np.float32(1e-4)))               # static scale far too small


def test_fused_group_offsets_and_padding():
    K = 320
    w0 = W.gaussian(48, K, seed=1, std=0.02)
    w1 = W.gaussian(48, K, seed=2, std=0.02)
    sf = torch.full((native.sf_bytes(96, K),), 0xAB, dtype=torch.uint8, device=DEV)
    codes = torch.empty((96, K // 2), dtype=torch.uint8, device=DEV)
    gs = []
    for i, (w, r0) in enumerate(((w0, 0), (w1, 48))):
        wd = w.to(DEV)
        _, g = checked_gscale(w, wd)
        gs.append(g)
        native.quantize(wd, g, codes=codes[r0:r0 + 48], sf=sf, sf_row0=r0, sf_rows_total=96)
    ref_sf = np.zeros(oracle.sf_bytes(96, K), np.uint8)
    rc0, _ = oracle.quantize(to_f32_numpy(w0), f32(gs[0]), sf=ref_sf, sf_row0=0)
    rc1, _ = oracle.quantize(to_f32_numpy(w1), f32(gs[1]), sf=ref_sf, sf_row0=48)
    torch.cuda.synchronize()
    assert_codes_equal(codes, np.concatenate([rc0, rc1]))
    assert np.array_equal(sf.cpu().numpy(), ref_sf)          # padding rows 96..127 zeroed too
    # harmonize on both sides
    gst = torch.cat(gs)
    gstar = native.harmonize(sf, 96, K, [0, 48, 96], gst)
    ref_gstar = oracle.harmonize(ref_sf, K, [0, 48, 96], [f32(g) for g in gs])
    torch.cuda.synchronize()
    assert f32(gstar) == ref_gstar
    assert np.array_equal(sf.cpu().numpy(), ref_sf)


@pytest.mark.parametrize("name", ["gdn_gates_ab", "decode_out_proj", "decode_down_proj"])
def test_workload_full(name):
    wl = W.WORKLOADS[name]
    _quant_check(W.make_x(wl))
    for m in range(len(wl.modules)):
        _quant_check(W.make_w(wl, m))


@pytest.mark.parametrize("name", ["gdn_qkv_z", "prefill_mlp_gate_up"])
def test_workload_sampled_rows(name):
    """Full-size tensors quantized on the GPU in one launch; a seeded sample of
    rows (first and last included) checked byte for byte."""
    wl = W.WORKLOADS[name]
    tensors = [W.make_x(wl)] + [W.make_w(wl, m) for m in range(len(wl.modules))]
    for t in tensors:
        x = t.to(DEV)
        g_ref, g = checked_gscale(t, x)
        codes, sf = native.quantize(x, g)
        rows = W.sample_rows(t.shape[0], 192)
        rc, rs = oracle.quantize(to_f32_numpy(t[torch.from_numpy(rows)]), g_ref)
        torch.cuda.synchronize()
        assert_codes_equal(codes[torch.from_numpy(rows).to(DEV)], rc)
        assert_sf_rows_equal(sf, rs, rows, np.arange(len(rows)), t.shape[1])
        # padding rows of the last atom are zero
        R = t.shape[0]
        if R % 128:
            pad = oracle.sf_gather(sf.cpu().numpy(), np.arange(R, (R + 127) // 128 * 128), t.shape[1])
            assert np.all(pad == 0)
        del x, codes, sf
    assert native.last_device_status() == 0


def test_harmonize_workload_groups():
    for name in ("gdn_gates_ab", "gdn_qkv_z"):
        wl = W.WORKLOADS[name]
        K, N = wl.K, wl.N
        offs = np.concatenate([[0], np.cumsum(wl.modules)]).astype(np.int64)
        sf = torch.empty(native.sf_bytes(N, K), dtype=torch.uint8, device=DEV)
        codes = torch.empty((N, K // 2), dtype=torch.uint8, device=DEV)
        gs, ws = [], []
        for m in range(len(wl.modules)):
            w = W.make_w(wl, m)
            ws.append(w)
            wd = w.to(DEV)
            _, g = checked_gscale(w, wd)
            gs.append(g)
            native.quantize(wd, g, codes=codes[offs[m]:offs[m + 1]], sf=sf, sf_row0=int(offs[m]),
                            sf_rows_total=N)
        gstar = native.harmonize(sf, N, K, offs, torch.cat(gs))
        # oracle on a row sample of each module, harmonized with the same scales
        samp = [W.sample_rows(wl.modules[m], 96, seed=m) for m in range(len(wl.modules))]
        sub_offs = np.concatenate([[0], np.cumsum([len(s) for s in samp])])
        ref_sf = np.zeros(oracle.sf_bytes(int(sub_offs[-1]), K), np.uint8)
        for m, s in enumerate(samp):
            oracle.quantize(to_f32_numpy(ws[m][torch.from_numpy(s)]), f32(gs[m]), sf=ref_sf,
                            sf_row0=int(sub_offs[m]))
        ref_gstar = oracle.harmonize(ref_sf, K, sub_offs, [f32(g) for g in gs])
        torch.cuda.synchronize()
        assert f32(gstar) == ref_gstar
        fused_rows = np.concatenate([offs[m] + s for m, s in enumerate(samp)])
        assert_sf_rows_equal(sf, ref_sf, fused_rows, np.arange(len(fused_rows)), K)
