"""Guard canaries around every buffer a kernel writes (in place of a memory
sanitizer): each output, workspace and in-place buffer is a view into a
larger allocation whose 4 KB before and after hold a byte pattern.  After
the call the pattern must be intact, and the guarded result must equal the
result of the same call on ordinary allocations, bit for bit.  Small odd
shapes: M = 1, 33, 127 rows; N = 48, 96; K not a multiple of 256."""
import math

import numpy as np
import pytest
import torch

from nvfp4_w4a4_quantized_06_b200 import native
from nvfp4_w4a4_quantized_06_b200 import workloads as W

pytestmark = pytest.mark.gpu
DEV = "cuda"
GUARD = 4096          # bytes on each side
PATTERN = 0xA5


class Guarded:
    """A tensor of `shape` inside a buffer with GUARD pattern bytes on both sides."""

    def __init__(self, shape, dtype):
        esz = torch.empty(0, dtype=dtype).element_size()
        n = math.prod(shape)
        g = GUARD // esz
        self.buf = torch.empty(g + n + g, dtype=dtype, device=DEV)
        self.buf.view(torch.uint8).fill_(PATTERN)
        self.t = self.buf[g:g + n].view(shape)

    def check(self, what):
        b = self.buf.view(torch.uint8)
        head, tail = b[:GUARD], b[-GUARD:]
        assert bool(torch.all(head == PATTERN)), f"{what}: bytes written before the buffer"
        assert bool(torch.all(tail == PATTERN)), f"{what}: bytes written past the end of the buffer"


def _same(a, b, what):
    assert torch.equal(a.view(torch.uint8) if a.dtype != torch.uint8 else a,
                       b.view(torch.uint8) if b.dtype != torch.uint8 else b), f"{what}: guarded result differs"


def _weights(N, K, seed):
    w = W.gaussian(N, K, seed=seed, std=0.02).to(DEV)
    g = native.amax_gscale(w)
    wc, ws = native.quantize(w, g)
    return wc, ws, g


@pytest.mark.parametrize("rows", [1, 33, 127])
@pytest.mark.parametrize("K", [64, 320])
def test_quantize_guards(rows, K):
    x = W.gaussian(rows, K, seed=rows + K).to(DEV)
    g = native.amax_gscale(x)
    codes, sf = native.quantize(x, g)
    gc, gs = Guarded((rows, K // 2), torch.uint8), Guarded((native.sf_bytes(rows, K),), torch.uint8)
    native.quantize(x, g, codes=gc.t, sf=gs.t)
    torch.cuda.synchronize()
    gc.check("codes")
    gs.check("scales")
    _same(gc.t, codes, "codes")
    _same(gs.t, sf, "scales")
    # the same rows as the second module of a fused buffer (scale rows at an offset)
    total = rows + 48
    gs2 = Guarded((native.sf_bytes(total, K),), torch.uint8)
    native.quantize(x, g, codes=gc.t, sf=gs2.t, sf_row0=48, sf_rows_total=total)
    torch.cuda.synchronize()
    gc.check("codes (fused)")
    gs2.check("scales (fused)")
    assert native.last_device_status() == 0


@pytest.mark.parametrize("M", [1, 33, 127])
@pytest.mark.parametrize("N", [48, 96])
@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.float32])
def test_linear_and_gemm_guards(M, N, out_dtype):
    K = 320
    x = W.gaussian(M, K, seed=M * 3 + N).to(DEV)
    gx = native.amax_gscale(x)
    wc, ws, gw = _weights(N, K, N)
    y = native.linear(x, gx, wc, ws, gw, out_dtype=out_dtype)
    gy = Guarded((M, N), out_dtype)
    gw_s = Guarded((native.linear_workspace_bytes(M, N, K),), torch.uint8)
    native.linear(x, gx, wc, ws, gw, out=gy.t, workspace=gw_s.t)
    torch.cuda.synchronize()
    gy.check("linear output")
    gw_s.check("linear workspace")
    _same(gy.t, y, "linear output")
    # the entry point without a workspace, and the one-kernel variant where
    # the activation is the narrow operand (its only supported shapes)
    for fn in (native.linear_noalloc, native.linear_fused) if M <= N else (native.linear_noalloc,):
        ref = fn(x, gx, wc, ws, gw, out_dtype=out_dtype)
        g2 = Guarded((M, N), out_dtype)
        fn(x, gx, wc, ws, gw, out=g2.t)
        torch.cuda.synchronize()
        g2.check(fn.__name__)
        _same(g2.t, ref, fn.__name__)
    ac, asf = native.quantize(x, gx)
    y2 = native.gemm(ac, asf, gx, wc, ws, gw, out_dtype=out_dtype)
    g3 = Guarded((M, N), out_dtype)
    native.gemm(ac, asf, gx, wc, ws, gw, out=g3.t)
    torch.cuda.synchronize()
    g3.check("gemm output")
    _same(g3.t, y2, "gemm output")
    assert native.last_device_status() == 0


@pytest.mark.parametrize("M", [1, 33, 127])
def test_gates_guards(M):
    K, N = 320, 96
    x = W.gaussian(M, K, seed=M).to(DEV)
    gx = native.amax_gscale(x)
    wc, ws, gw = _weights(N, K, 7)
    ref = native.gdn_gates(x, gx, wc, ws, gw, n_a=48)
    go = Guarded((M, N), torch.float32)
    native.gdn_gates(x, gx, wc, ws, gw, n_a=48, out=go.t)
    torch.cuda.synchronize()
    go.check("gates")
    _same(go.t, ref, "gates")
    assert native.last_device_status() == 0


@pytest.mark.parametrize("rows", [1, 33, 127])
def test_next_row_guards(rows):
    K = 320
    x = W.gaussian(rows, K, seed=rows + 1).to(DEV)
    g = native.amax_gscale(x)
    # RMSNorm-fused quantize
    w = W.norm_weight(K, seed=2).to(DEV)
    c, s, inv = native.rmsnorm_quantize(x, w, 1e-6, g)
    gc, gs, gi = (Guarded((rows, K // 2), torch.uint8), Guarded((native.sf_bytes(rows, K),), torch.uint8),
                  Guarded((rows,), torch.float32))
    native.rmsnorm_quantize(x, w, 1e-6, g, codes=gc.t, sf=gs.t, inv=gi.t)
    torch.cuda.synchronize()
    for gd, ref, what in ((gc, c, "rmsnorm codes"), (gs, s, "rmsnorm scales"), (gi, inv, "rmsnorm factors")):
        gd.check(what)
        _same(gd.t, ref, what)
    # fake-quant through the C ABI (the binding allocates its own output)
    ref, _ = native.fake_quant(x, g, out_dtype=torch.bfloat16)
    go, gst = Guarded((rows, K), torch.bfloat16), Guarded((2,), torch.float64)
    st = native.lib().nvfp4_fake_quant(x.data_ptr(), native.IN_BF16, rows, K, K, g.data_ptr(), go.t.data_ptr(),
                                       native.OUT_BF16, K, gst.t.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert st == 0
    torch.cuda.synchronize()
    go.check("fake-quant values")
    gst.check("fake-quant statistics")
    _same(go.t, ref, "fake-quant values")
    # FP8 quantize
    flat = x.reshape(-1)[: (x.numel() // 8) * 8].contiguous()
    sc = (flat.abs().max().float() / 448.0).reshape(1)
    q = native.fp8_quantize(flat, sc)
    gq = Guarded((flat.numel(),), torch.uint8)
    native.fp8_quantize(flat, sc, out=gq.t)
    torch.cuda.synchronize()
    gq.check("fp8 codes")
    _same(gq.t, q, "fp8 codes")
    assert native.last_device_status() == 0


def test_harmonize_guards():
    """Both harmonize variants rewrite a fused group in place: nothing outside
    the group's codes and scales may change."""
    K, rows = 320, (33, 15)
    N = sum(rows)
    offs = np.array([0, rows[0], N], np.int64)
    for requant in (False, True):
        gc, gs = Guarded((N, K // 2), torch.uint8), Guarded((native.sf_bytes(N, K),), torch.uint8)
        gsc = []
        for m, r in enumerate(rows):
            w = W.gaussian(r, K, seed=20 + m, std=0.02 * (m + 1)).to(DEV)
            g = native.amax_gscale(w)
            native.quantize(w, g, codes=gc.t[offs[m]:offs[m + 1]], sf=gs.t, sf_row0=int(offs[m]), sf_rows_total=N)
            gsc.append(g)
        gscales = torch.cat(gsc)
        if requant:
            native.harmonize_requant(gc.t, gs.t, K, offs, gscales)
        else:
            native.harmonize(gs.t, N, K, offs, gscales)
        torch.cuda.synchronize()
        gc.check("group codes")
        gs.check("group scales")
    assert native.last_device_status() == 0
