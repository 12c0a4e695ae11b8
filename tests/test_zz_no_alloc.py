"""GPU check of w4a4_gemm_noalloc, the entry point for callers that cannot
allocate device memory where they run the layer (a runtime with a fixed
memory plan, a plugin that only receives input and output pointers): it
must give the same result as w4a4_gemm, which takes a caller-provided
workspace, while keeping its scratch in the library's own fixed buffer.

The file is named to be collected last, so that a run stopping at the first
failure has already run every other test; it passes on its own in a fresh
process too (the first call looks the buffer's address up).
"""
import numpy as np
import pytest
import torch

from nvfp4_w4a4_quantized_06_b200 import native
from nvfp4_w4a4_quantized_06_b200 import workloads as W

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _weights(N, K, seed):
    w = W.gaussian(N, K, seed=seed, std=0.02).to(DEV)
    gw = native.amax_gscale(w)
    wc, ws = native.quantize(w, gw)
    return wc, ws, gw


@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.float32])
def test_noalloc_matches_workspace_entry_point_twice(out_dtype):
    # Two products one after the other, each called twice, so that later calls
    # run on a buffer an earlier call left filled: a decode-shaped product
    # (the quantized activation in the scratch, reduced inside a cluster) and
    # a ragged one whose plan splits K on single CTAs (split-K partial sums in
    # the scratch too).  The entry points run the same plan and kernels, so
    # the outputs must be identical bit for bit.
    cases = [(32, 5120, 5120, 11), (384, 1000, 1344, 12)]
    # on this device the second product's plan really keeps partial sums (the
    # GEMM's own workspace size is that of the partials, 0 for other plans)
    assert native.lib().nvfp4_gemm_workspace_bytes(384, 1000, 1344) > 0
    assert native.lib().nvfp4_gemm_workspace_bytes(32, 5120, 5120) == 0
    for M, N, K, seed in cases:
        x = W.gaussian(M, K, seed=seed, outliers=W.Outliers("scale", 0.02, 30.0)).to(DEV)
        gx = native.amax_gscale(x)
        wc, ws, gw = _weights(N, K, seed + 100)
        assert native.linear_workspace_bytes(M, N, K) <= 8 << 20
        y_ref = native.linear(x, gx, wc, ws, gw, out_dtype=out_dtype)
        y1 = native.linear_noalloc(x, gx, wc, ws, gw, out_dtype=out_dtype)
        y2 = native.linear_noalloc(x, gx, wc, ws, gw, out_dtype=out_dtype)
        torch.cuda.synchronize()
        assert native.last_device_status() == 0
        assert torch.equal(y1, y_ref)
        assert torch.equal(y2, y_ref)


def test_noalloc_rejects_problems_beyond_its_buffer():
    M, N, K = 4096, 96, 5120          # the activation alone needs ~11 MB of scratch
    assert native.linear_workspace_bytes(M, N, K) > 8 << 20
    x = torch.zeros(M, K, dtype=torch.bfloat16, device=DEV)
    gx = torch.ones(1, dtype=torch.float32, device=DEV)
    wc, ws, gw = _weights(N, K, 5)
    with pytest.raises(native.Nvfp4Error) as e:
        native.linear_noalloc(x, gx, wc, ws, gw)
    assert e.value.status == 9
    assert native.lib().nvfp4_status_string(9).decode().startswith("problem needs more scratch")
    assert np.isfinite(native.linear(x, gx, wc, ws, gw).float().cpu().numpy()).all()
