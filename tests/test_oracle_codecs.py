"""Pins for the oracle's E2M1 / E4M3 codecs (CPU only).

The oracle encodes by nearest-point search over its code tables.  These tests
hold it against things other than itself: the format facts the pages state
(tests/golden/nvfp4_format.txt), hand-derived tie cases, a textbook
round-to-nearest-even at a fixed number of mantissa bits written with
numpy.rint, and two independent library casts (ml_dtypes and torch).
"""
import math
import os

import ml_dtypes
import numpy as np
import pytest
import torch

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "nvfp4_format.txt")


def golden():
    out = {}
    for line in open(GOLDEN):
        line = line.split("#", 1)[0].strip()
        if line:
            k, v = line.split(":", 1)
            out[k.strip()] = [float(t) for t in v.split()]
    return out


def test_e2m1_decode_matches_format_table(oracle):
    mags = golden()["e2m1_magnitudes"]
    for c in range(8):
        assert oracle.e2m1_decode(c) == mags[c]
        neg = oracle.e2m1_decode(c | 8)
        assert neg == -mags[c] and math.copysign(1.0, neg) == -1.0


def test_e2m1_roundtrip_all_codes(oracle):
    for c in range(16):
        assert oracle.e2m1_encode(oracle.e2m1_decode(c)) == c


def test_e2m1_ties_go_to_even_code(oracle):
    # hand-derived: each midpoint sits between an even and an odd code index
    expected = {0.25: 0, 0.75: 2, 1.25: 2, 1.75: 4, 2.5: 4, 3.5: 6, 5.0: 6}
    for y, c in expected.items():
        assert oracle.e2m1_encode(y) == c, y
        assert oracle.e2m1_encode(-y) == c | 8, -y


def test_e2m1_neighbours_of_midpoints(oracle):
    mids = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0]
    for i, m in enumerate(mids):
        below = np.nextafter(np.float32(m), np.float32(0))
        above = np.nextafter(np.float32(m), np.float32(10))
        assert oracle.e2m1_encode(below) == i
        assert oracle.e2m1_encode(above) == i + 1


def test_e2m1_saturation_and_sign(oracle):
    for y in [6.0, 6.5, 7.0, 100.0, 3.0e38, float("inf")]:
        assert oracle.e2m1_encode(y) == 7
        assert oracle.e2m1_encode(-y) == 15
    assert oracle.e2m1_encode(-0.0) == 8
    assert oracle.e2m1_encode(-0.1) == 8
    assert oracle.e2m1_encode(0.1) == 0
    assert oracle.e2m1_encode(1e-45) == 0


def _rne_e2m1_textbook(y: np.ndarray) -> np.ndarray:
    """Round |y| to 1 mantissa bit (exponent range 0..2, subnormal step 0.5),
    half to even with numpy.rint, saturate at 6; return code index."""
    a = np.abs(y.astype(np.float64))
    e = np.floor(np.log2(np.maximum(a, 1.0)))      # exponent >= 0 (subnormal region uses step .5)
    e = np.minimum(e, 2.0)
    step = np.where(a < 1.0, 0.5, 2.0 ** (e - 1))
    r = np.rint(a / step) * step
    r = np.minimum(r, 6.0)
    mags = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6])
    idx = np.searchsorted(mags, r)
    return idx | np.where(np.signbit(y), 8, 0)


def test_e2m1_dense_sweep_vs_textbook_and_ml_dtypes(oracle):
    rng = np.random.default_rng(7)
    ys = [np.float32(v) for v in np.linspace(-8, 8, 4001)]
    for m in [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0]:
        v = np.float32(m)
        for _ in range(5):
            ys += [v, -v]
            v = np.nextafter(v, np.float32(10))
        v = np.float32(m)
        for _ in range(5):
            v = np.nextafter(v, np.float32(0))
            ys += [v, -v]
    ys += list(rng.standard_normal(3000).astype(np.float32) * 3)
    ys = np.array(ys, dtype=np.float32)
    got = np.array([oracle.e2m1_encode(y) for y in ys])
    assert np.array_equal(got, _rne_e2m1_textbook(ys))
    lib = ys.astype(ml_dtypes.float4_e2m1fn).view(np.uint8) & 0xF
    assert np.array_equal(got, lib)


def test_e4m3_decode_all_codes_vs_libraries(oracle):
    codes = np.arange(256, dtype=np.uint8)
    ref_t = torch.from_numpy(codes.copy()).view(torch.float8_e4m3fn).float().numpy()
    ref_m = codes.view(ml_dtypes.float8_e4m3fn).astype(np.float32)
    for c in range(256):
        v = oracle.e4m3_decode(c)
        if (c & 0x7F) == 0x7F:
            assert math.isnan(v) and math.isnan(ref_t[c]) and math.isnan(ref_m[c])
        else:
            assert v == ref_t[c] == ref_m[c], c
    assert oracle.e4m3_decode(0x7E) == golden()["e4m3_max"][0]


def test_e4m3_roundtrip_all_finite_codes(oracle):
    for c in range(256):
        if (c & 0x7F) != 0x7F:
            assert oracle.e4m3_encode(oracle.e4m3_decode(c)) == c


def test_e4m3_encode_sweep_vs_libraries(oracle):
    # every midpoint between adjacent finite codes (ties), +-2 ulps around it,
    # and a log-uniform random sweep over the whole range up to 464
    vals = []
    for c in range(0x7E):
        lo, hi = oracle.e4m3_decode(c), oracle.e4m3_decode(c + 1)
        mid = np.float32((lo + hi) / 2)
        assert float(mid) == (lo + hi) / 2           # the midpoint is exact in fp32
        v = mid
        for _ in range(3):
            vals.append(v)
            v = np.nextafter(v, np.float32(1e9))
        v = mid
        for _ in range(2):
            v = np.nextafter(v, np.float32(0))
            vals.append(v)
    rng = np.random.default_rng(3)
    vals += list((2.0 ** rng.uniform(-14, math.log2(464), 20000)).astype(np.float32))
    vals += [np.float32(0), np.float32(464.0), np.float32(2.0 ** -10), np.float32(1e-30)]
    vals = np.array(vals, dtype=np.float32)
    vals = vals[vals <= 464]
    got = np.array([oracle.e4m3_encode(v) for v in vals], dtype=np.uint8)
    ref_t = torch.from_numpy(vals).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    ref_m = vals.astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
    assert np.array_equal(got, ref_t)
    assert np.array_equal(got, ref_m)


def test_e4m3_saturates_instead_of_nan(oracle):
    for t in [464.0001, 480.0, 1000.0, 3e38, float("inf")]:
        assert oracle.e4m3_encode(t) == 0x7E
    assert oracle.e4m3_encode(2.0 ** -10) == 0x00       # tie between 0 and 2^-9 -> even (0)
    assert oracle.e4m3_encode(1.5 * 2.0 ** -9) == 0x02  # tie between 1 and 2 (x 2^-9) -> even


@pytest.mark.parametrize("code", [0x08, 0x38, 0x40, 0x7E])
def test_e4m3_known_values(oracle, code):
    # hand-derived from the bit layout: 0x08 = 2^-6, 0x38 = 1.0, 0x40 = 2.0, 0x7E = 448
    expected = {0x08: 2.0 ** -6, 0x38: 1.0, 0x40: 2.0, 0x7E: 448.0}[code]
    assert oracle.e4m3_decode(code) == expected
