"""Pins of the oracle for the rows marked "next": the GDN gate activations,
fake-quant (quantize then dequantize), static-scale FP8 KV quantize, the
re-quantizing harmonize and the quantize fused into the preceding RMSNorm.
Each check is fixed by mathematics or by the format, not by re-typing the
oracle's own formula."""
import math
from decimal import Decimal, localcontext

import numpy as np
import pytest
import torch

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


# ------------------------------------------------- re-quantizing harmonize
def _weights(seed, rows, K, std):
    w = np.random.default_rng(seed).standard_normal((rows, K)).astype(np.float32) * np.float32(std)
    return torch.from_numpy(w).to(torch.bfloat16).float().numpy()


def test_requant_is_identity_at_the_same_scale():
    # one module (g* = g): every block's values dequantized and encoded again
    # land on the same scale (amax within 2^-23 of 6 dec(s) g) and the same
    # codes (each within 2^-23 of its grid point) -- normal scales only
    w = _weights(5, 96, 320, 0.02)
    g = oracle.global_scale(w)
    codes, sf = oracle.quantize(w, g)
    assert np.all(oracle.sf_gather(sf, np.arange(96), 320) >= 0x08)
    c2, s2, gstar = oracle.harmonize_requant(codes, sf, 320, [0, 96], [g])
    assert gstar == g and np.array_equal(c2, codes) and np.array_equal(s2, sf)


def test_requant_power_of_two_ratio_equals_scale_rewrite():
    # g_1 = g_0 / 4: re-quantizing module 1 against g* = g_0 only divides its
    # scales by 4 (exact while they stay normal), which is what the
    # scale-only harmonize does; module 0 is unchanged
    K = 256
    w0, w1 = _weights(6, 40, K, 0.02), _weights(7, 24, K, 0.02)
    g0 = oracle.global_scale(w0)
    g1 = np.float32(g0 / np.float32(4.0))
    sf = np.zeros(oracle.sf_bytes(64, K), np.uint8)
    c0, _ = oracle.quantize(w0, g0, sf=sf, sf_row0=0)
    c1, _ = oracle.quantize(w1 / 8, g1, sf=sf, sf_row0=40)      # small weights keep module 1's scales in range
    codes = np.concatenate([c0, c1])
    s1 = oracle.sf_gather(sf, np.arange(40, 64), K)
    assert np.all(s1 >= 0x18)                                     # dec(s)/4 stays normal
    c2, s2, gstar = oracle.harmonize_requant(codes, sf, K, [0, 40, 64], [g0, g1])
    rewritten = sf.copy()
    assert oracle.harmonize(rewritten, K, [0, 40, 64], [g0, g1]) == gstar == g0
    assert np.array_equal(c2, codes) and np.array_equal(s2, rewritten)


def test_requant_generic_ratio():
    # A ratio that is not a power of two.  (1) The output is a valid NVFP4
    # encoding of the fp32 dequantized weights at g*: each element is within
    # half a grid step of its block's normal scale.  (2) Where the new scale
    # is normal, the codes are the old ones: the block's values move by the
    # scale's rounding, at most 1/16 relative, less than any E2M1 half-gap.
    # (3) A tiny ratio pushes scales into the subnormal E4M3 range; there the
    # codes change, and wherever both variants chose the same scale byte,
    # re-quantizing is at least as close to the dequantized weights as the
    # scale-only rewrite, element by element (RNE picks the nearest code).
    K = 320
    w0, w1 = _weights(8, 48, K, 0.02), _weights(9, 48, K, 0.013)
    for ratio in (None, np.float32(2e-5)):
        g0 = oracle.global_scale(w0)
        g1 = oracle.global_scale(w1) if ratio is None else np.float32(g0 * ratio)
        x1 = w1 if ratio is None else w1 * ratio / 0.013 * 0.02
        sf = np.zeros(oracle.sf_bytes(96, K), np.uint8)
        c0, _ = oracle.quantize(w0, g0, sf=sf, sf_row0=0)
        c1, _ = oracle.quantize(x1, g1, sf=sf, sf_row0=48)
        codes = np.concatenate([c0, c1])
        c2, s2, gstar = oracle.harmonize_requant(codes, sf, K, [0, 48, 96], [g0, g1])
        assert gstar == max(g0, g1)
        xhat = np.concatenate([oracle.dequantize(c0, sf, g0), oracle.dequantize(c1, sf, g1, sf_row0=48)])
        xhat = xhat.astype(np.float32).astype(np.float64)
        dq = oracle.dequantize(c2, s2, gstar)
        new_s = oracle.sf_gather(s2, np.arange(96), K)
        normal = np.repeat(new_s >= 0x08, 16, axis=1)
        amax = np.repeat(np.abs(xhat).reshape(96, -1, 16).max(axis=2), 16, axis=1)
        err = np.abs(xhat - dq)
        assert np.all(err[normal] <= (amax / 6 * (1 + 2.0 ** -4))[normal] + 1e-30)
        nib = lambda c: np.stack([c & 15, c >> 4], axis=2).reshape(96, K)
        assert np.array_equal(nib(c2)[normal], nib(codes)[normal])
        if ratio is not None:
            assert not normal[48:].all() and not np.array_equal(c2[48:], codes[48:])
            rewritten = sf.copy()
            oracle.harmonize(rewritten, K, [0, 48, 96], [g0, g1])
            same = np.repeat(oracle.sf_gather(rewritten, np.arange(96), K) == new_s, 16, axis=1)
            err_rw = np.abs(xhat - oracle.dequantize(codes, rewritten, gstar))
            assert same[48:].any() and np.all(err[same] <= err_rw[same])


# ------------------------------------------ quantize fused into RMSNorm
def test_rms_inv_closed_forms():
    # all elements 1.875: mean 3.515625, + eps 0.484375 = 4, so inv = 1/2;
    # one element 8 in 64: mean 1, + eps 3 = 4; signs do not matter
    x = np.full((1, 64), 1.875, np.float32)
    assert oracle.rms_inv(x, 0.484375)[0][0] == np.float32(0.5)
    x = np.where(np.arange(64) % 3 == 0, -1.875, 1.875).astype(np.float32)[None, :]
    assert oracle.rms_inv(x, 0.484375)[0][0] == np.float32(0.5)
    x = np.zeros((1, 64), np.float32)
    x[0, 17] = 8.0
    assert oracle.rms_inv(x, 3.0)[0][0] == np.float32(0.5)
    # the all-zero row: 1/sqrt(eps)
    assert oracle.rms_inv(np.zeros((1, 64), np.float32), 0.25)[0][0] == np.float32(2.0)


def test_rms_inv_is_correctly_rounded():
    # independent evaluation: the sum of squares and 1/sqrt in 90-digit
    # decimal arithmetic; the oracle's float must be the nearest one
    rng = np.random.default_rng(10)
    x = rng.standard_normal((24, 640)).astype(np.float32) * np.float32(3.0)
    x[3] *= np.float32(1e-3)
    x[4, :600] = 0.0
    eps = np.float32(1e-6)
    inv, near = oracle.rms_inv(x, eps)
    assert not near.any()
    with localcontext() as ctx:
        ctx.prec = 90
        for r in range(x.shape[0]):
            s = sum(Decimal(float(v)) * Decimal(float(v)) for v in x[r])
            exact = 1 / (s / Decimal(x.shape[1]) + Decimal(float(eps))).sqrt()
            f = inv[r]
            up = np.nextafter(f, np.float32(np.inf))
            dn = np.nextafter(f, np.float32(0))
            assert (Decimal(float(dn)) + Decimal(float(f))) / 2 < exact < (Decimal(float(f)) + Decimal(float(up))) / 2


def test_rmsnorm_against_library_rms_norm():
    # torch's own RMSNorm (float32, its own reduction order and rsqrt) lands
    # within one bf16 step of the oracle everywhere and on it almost always
    rng = np.random.default_rng(11)
    x = torch.from_numpy(rng.standard_normal((64, 1024)).astype(np.float32) * 2).to(torch.bfloat16).float()
    w = torch.from_numpy(1 + 0.1 * rng.standard_normal(1024).astype(np.float32)).to(torch.bfloat16).float()
    y, _, _ = oracle.rmsnorm(x.numpy(), w.numpy(), 1e-6)
    ref = torch.nn.functional.rms_norm(x, (1024,), weight=w, eps=1e-6).to(torch.bfloat16).float().numpy()
    step = np.abs(ref) * 2.0 ** -7 + 1e-30
    assert np.all(np.abs(y - ref) <= step)
    assert np.mean(y == ref) > 0.99
    # zero-centred form with w = 0 is the standard form with w = 1
    yz, _, _ = oracle.rmsnorm(x.numpy(), np.zeros(1024, np.float32), 1e-6, zero_centered=True)
    y1, _, _ = oracle.rmsnorm(x.numpy(), np.ones(1024, np.float32), 1e-6)
    assert np.array_equal(yz, y1)


def test_rmsnorm_quantize_scale_invariance():
    # x -> 2^k x with eps -> 4^k eps scales the mean square by 4^k exactly and
    # the correctly rounded inv by 2^-k, so y, codes and scales are identical
    rng = np.random.default_rng(12)
    x = torch.from_numpy(rng.standard_normal((8, 512)).astype(np.float32)).to(torch.bfloat16).float().numpy()
    w = torch.from_numpy(1 + 0.1 * rng.standard_normal(512).astype(np.float32)).to(torch.bfloat16).float().numpy()
    c0, s0, y0, i0, _ = oracle.rmsnorm_quantize(x, w, 1e-6, 0.01)
    c1, s1, y1, i1, _ = oracle.rmsnorm_quantize(x * 8, w, np.float32(1e-6) * 64, 0.01)
    assert np.array_equal(i1 * 8, i0) and np.array_equal(y0, y1)
    assert np.array_equal(c0, c1) and np.array_equal(s0, s1)


def test_rmsnorm_quantize_constant_row():
    # x = 1.875 everywhere, eps = 0.484375, w = 1: inv = 1/2 and y = 0.9375;
    # with g = 0.9375/2688 every block's scale is 448 and every code is +6
    x = np.full((4, 128), 1.875, np.float32)
    g = np.float32(0.9375) / np.float32(2688.0)
    codes, sf, y, inv, _ = oracle.rmsnorm_quantize(x, np.ones(128, np.float32), 0.484375, g)
    assert np.all(y == 0.9375) and np.all(inv == 0.5)
    assert np.all(codes == 0x77)
    assert np.all(oracle.sf_gather(sf, np.arange(4), 128) == 0x7E)
