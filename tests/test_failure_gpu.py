"""Failure detection without a GPU fault: every wait in the library's kernels
is bounded; when one runs out, the kernel records a flag in the device error
word and returns.  The self-test kernel waits on a barrier that nothing ever
completes (a short limit), and the host sees the flag; the context keeps
working afterwards."""
import pytest
import torch

import oracle
from nvfp4_w4a4_quantized_06_b200 import native
from nvfp4_w4a4_quantized_06_b200 import workloads as W
from parity import assert_codes_equal, f32, to_f32_numpy

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_and_context_survives():
    assert native.last_device_status() == 0             # start clean
    res = native.selftest_wait_timeout(50_000_000)       # 50 ms
    torch.cuda.synchronize()
    assert res.item() == 0                               # the wait ran out
    flags = native.last_device_status()
    assert flags & 16                                    # ERR_SELFTEST recorded
    assert native.last_device_status() == 0             # and cleared by the read
    # the context is intact: a quantize afterwards is still bit-exact
    x_cpu = W.gaussian(64, 256, seed=1)
    g = native.amax_gscale(x_cpu.cuda())
    codes, _ = native.quantize(x_cpu.cuda(), g)
    rc, _ = oracle.quantize(to_f32_numpy(x_cpu), f32(g))
    assert_codes_equal(codes, rc)


def test_selftest_argument_checks():
    with pytest.raises(native.Nvfp4Error) as e:
        native.selftest_wait_timeout(0)
    assert e.value.status == 2
