"""Pins of the oracle for the rows marked "next": the GDN gate activations,
fake-quant (quantize then dequantize) and static-scale FP8 KV quantize.
Each check is fixed by mathematics or by the format, not by re-typing the
oracle's own formula."""
import math

import numpy as np
import pytest

import oracle


def test_gate_activations_closed_forms():
    # softplus(ln 3) = ln 4, so alpha = 1/4 and beta = sigmoid(ln 3) = 3/4;
    # at 0 both are 1/2; far out the gates saturate to 1 and 0
    y = np.array([[math.log(3.0), math.log(3.0), 0.0, 0.0, -60.0, 60.0]])
    a = oracle.gdn_gates(y[:, :3], n_a=3)[0]
    b = oracle.gdn_gates(y[:, 3:], n_a=0)[0]
    assert a[0] == pytest.approx(0.25, rel=1e-15) and a[2] == pytest.approx(0.5, rel=1e-15)
    assert b[0] == pytest.approx(0.5, rel=1e-15)
    al = oracle.gdn_gates(np.array([[-60.0, 60.0]]), n_a=2)[0]
    be = oracle.gdn_gates(np.array([[-60.0, 60.0]]), n_a=0)[0]
    assert al[0] == pytest.approx(1.0, abs=1e-25) and al[1] == pytest.approx(math.exp(-60.0), rel=1e-12)
    assert be[0] == pytest.approx(math.exp(-60.0), rel=1e-12) and be[1] == pytest.approx(1.0, abs=1e-25)


def test_gate_activations_complement_and_order():
    # exp(-softplus(y)) = 1/(1+e^y) = sigmoid(-y): the keep gate of y and the
    # write gate of y sum to one, and the columns split at n_a
    y = np.random.default_rng(1).standard_normal((7, 10)) * 6
    alpha = oracle.gdn_gates(y, n_a=10)
    beta = oracle.gdn_gates(y, n_a=0)
    assert np.allclose(alpha + beta, 1.0, rtol=0, atol=1e-15)
    mixed = oracle.gdn_gates(y, n_a=4)
    assert np.array_equal(mixed[:, :4], alpha[:, :4]) and np.array_equal(mixed[:, 4:], beta[:, 4:])
    s = np.sort(y.ravel())
    assert np.all(np.diff(oracle.gdn_gates(s[None, :], n_a=0)[0]) >= 0)      # beta increasing
    assert np.all(np.diff(oracle.gdn_gates(s[None, :], n_a=s.size)[0]) <= 0)  # alpha decreasing


def _grid_tensor(rng, rows, K, g):
    """A tensor whose blocks each hold a +-6 element: its NVFP4 encoding is
    itself (block scale exactly amax/6, every element on the E2M1 grid)."""
    codes = rng.integers(0, 16, size=(rows, K)).astype(np.int64)
    codes[:, ::16] = np.where(rng.random((rows, K // 16)) < 0.5, 7, 15)          # +-6 in every block
    scales = rng.integers(8, 0x70, size=(rows, K // 16))                          # normal E4M3 scales
    val = np.array([oracle.e2m1_decode(c) for c in range(16)])
    sc = np.array([oracle.e4m3_decode(int(c)) for c in range(128)])
    x = val[codes] * np.repeat(sc[scales], 16, axis=1) * float(g)
    return x.astype(np.float32), x


def test_fake_quant_reproduces_grid_values():
    rng = np.random.default_rng(2)
    g = np.float32(0.25)                         # a power of two keeps every product exact
    x32, x64 = _grid_tensor(rng, 12, 128, g)
    assert np.array_equal(x32.astype(np.float64), x64)
    dq, se, sx = oracle.fake_quant(x32, g)
    assert np.array_equal(dq, x64) and se == 0.0 and sx == pytest.approx(np.sum(x64 ** 2))


def test_fake_quant_outlier_stays_in_its_block():
    rng = np.random.default_rng(3)
    x = rng.standard_normal((4, 256)).astype(np.float32)
    g = oracle.global_scale(x * 50)               # a scale that leaves room for the outlier
    base, _, _ = oracle.fake_quant(x, g)
    y = x.copy()
    y[2, 37] = 40.0                               # block 2 of row 2
    dq, _, _ = oracle.fake_quant(y, g)
    changed = np.argwhere(dq != base)
    assert changed.size and np.all(changed[:, 0] == 2) and np.all(changed[:, 1] // 16 == 37 // 16)


def test_fake_quant_error_statistics():
    x = np.random.default_rng(4).standard_normal((64, 512)).astype(np.float32)
    dq, se, sx = oracle.fake_quant(x, oracle.global_scale(x))
    x64 = x.astype(np.float64)
    assert se == pytest.approx(np.sum((x64 - dq) ** 2), rel=1e-12)
    assert sx == pytest.approx(np.sum(x64 ** 2), rel=1e-12)
    # every element moves by at most half the spacing of its block's grid:
    # the grid step is at most 2 * dec(s) * g <= 2 * amax/6 * (1 + 2^-4)
    blocks = np.abs(x64).reshape(64, -1, 16).max(axis=2, keepdims=True)
    err = np.abs(x64 - dq).reshape(64, -1, 16)
    assert np.all(err <= blocks / 6 * (1 + 2.0 ** -4) + 1e-30)


def test_fp8_round_trip_saturation_and_ties():
    s = np.float32(0.125)                          # a power of two: x/s exact
    vals = np.array([oracle.e4m3_decode(c) for c in range(0x7F)], np.float64)
    x = np.concatenate([vals, -vals]).astype(np.float32) * s
    q = oracle.fp8_quantize(x, s)
    assert np.array_equal(q[:0x7F], np.arange(0x7F, dtype=np.uint8))
    assert np.array_equal(q[0x7F:], np.arange(0x7F, dtype=np.uint8) | 0x80)
    # midpoints between neighbours go to the even code; beyond 448 saturates
    mid = ((vals[1:] + vals[:-1]) / 2).astype(np.float32) * s
    qm = oracle.fp8_quantize(mid, s)
    lo = np.arange(0x7E)
    assert np.array_equal(qm, np.where(lo % 2 == 0, lo, lo + 1).astype(np.uint8))
    big = oracle.fp8_quantize(np.array([500.0, 1e30, -1e30], np.float32) * s, s)
    assert list(big) == [0x7E, 0x7E, 0xFE]
    assert oracle.fp8_quantize(np.array([-0.0], np.float32), s)[0] == 0x80
