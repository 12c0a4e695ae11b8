"""The GPU encoder's arithmetic, modelled step by step in numpy and checked
exhaustively against the definition (no GPU needed).

The quantize kernels never divide.  Per block they take
  r = fl32(fl32(1/dec(s)) * fl32(1/g)),  r- = fl32(r (1 - 2^-21)),  r+ = fl32(r (1 + 2^-21)),
convert fl32(x r-) and fl32(x r+) to E2M1 with round-to-nearest-even and
saturation, and where the two codes differ they settle the element by
comparing D = fma(-T, d, |x|) (exact near T) with +-half an ulp of T times d,
T the E2M1 boundary between the two codes, d = fl32(dec(s) g).  The scale byte is chosen the same
way from amax * fl32(1/fl32(6 g)) widened both ways, settled against the
midpoint of its two E4M3 candidates.

This file checks, for every finite non-negative bf16 value, every E4M3 block
scale and a spread of global scales, that the two products bracket the
quotient's code, that equal codes are the definition's code, that different
codes are neighbours, and that the settling rule then gives the definition's
code -- i.e. that the kernels' encoder equals E2M1(fl32(x / d)) and
E4M3(fl32(amax / fl32(6 g))) on every input, not only on the tested tensors.
(Sign is symmetric: round-to-nearest-even and saturation commute with it.)
"""
import numpy as np

import oracle

F32 = np.float32
WIDEN_LO = F32(1.0 - 2.0 ** -21)
WIDEN_HI = F32(1.0 + 2.0 ** -21)
E2M1_BOUNDARY = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])
E4M3_VALUES = np.array([oracle.e4m3_decode(c) for c in range(0x7F)])          # 0 .. 448
E4M3_MID = (E4M3_VALUES[1:] + E4M3_VALUES[:-1]) / 2


def e2m1_mag(a):
    """E2M1 magnitude index (0..7) of a >= 0: round to nearest, ties to the
    even index, saturate at 6."""
    a = np.asarray(a, np.float64)
    m = np.searchsorted(E2M1_BOUNDARY, a, side="left")
    tie = (m < 7) & (a == E2M1_BOUNDARY[np.minimum(m, 6)])
    return np.where(tie & (m % 2 == 1), m + 1, m)


def e4m3_code(t):
    """E4M3 byte of t >= 0: round to nearest, ties to even, saturate at 448."""
    t = np.asarray(t, np.float64)
    c = np.searchsorted(E4M3_MID, t, side="left")
    tie = (c < 126) & (t == E4M3_MID[np.minimum(c, 125)])
    return np.where(tie & (c % 2 == 1), c + 1, c)


def fma32(x, y, z):
    """fl32(x * y + z) for fp32 x (at most 5 significant bits), y and z: the
    product is exact in fp64 and so is the sum whenever the exponents of the
    two terms are within 24 of each other (the only case the rule below needs
    exactly); farther apart the fp64 sum rounds only bits far below the fp32
    result."""
    return (np.asarray(x, np.float64) * np.asarray(y, np.float64) + np.asarray(z, np.float64)).astype(np.float32)


def settle(a, b, T):
    """Sign of fl32(a / b) - T as the kernels decide it: D = fma(-T, b, a) in
    fp32, then above h+ * b rounds above T, below -h- * b rounds below, in
    between is T (h+- half the float spacing above and below T)."""
    T = np.asarray(T, np.float32)
    bits = T.view(np.uint32).astype(np.int64)
    hp = np.ldexp(np.float32(1.0), (((bits >> 23) & 0xFF) - 127 - 24).astype(np.int32)).astype(np.float32)
    hm = np.where((bits & 0x7FFFFF) == 0, hp / F32(2), hp).astype(np.float32)
    D = fma32(-T, np.asarray(b, np.float32), np.asarray(a, np.float32))
    up = (hp * np.asarray(b, np.float32)).astype(np.float32)
    dn = (hm * np.asarray(b, np.float32)).astype(np.float32)
    return np.where(D > up, 1, np.where(D < -dn, -1, 0))


def pick(lo, hi, c):
    """Neighbouring candidates lo < hi and the settled side c."""
    return np.where(c > 0, hi, np.where(c < 0, lo, np.where(lo % 2 == 1, hi, lo)))


BF16_POS = np.arange(0, 0x7F80, dtype=np.uint32)                                # +0 .. largest finite
X_ALL = (BF16_POS << 16).view(np.float32)
GLOBAL_SCALES = np.concatenate([
    np.array([1.0 / 2688, 1.0 / 6, 1.0, 0.0371, 3.7e-3, 448.0, 2.0 ** -40, 2.0 ** 40], np.float32),
    np.exp(np.random.default_rng(0).uniform(np.log(1e-15), np.log(1e12), 12)).astype(np.float32)])


def test_model_helpers_match_the_oracle_codecs():
    ys = np.concatenate([np.linspace(0, 7, 2801), E2M1_BOUNDARY, np.nextafter(E2M1_BOUNDARY, 0),
                         np.nextafter(E2M1_BOUNDARY, 9)]).astype(np.float32)
    assert all(int(e2m1_mag(y)) == oracle.e2m1_encode(y) & 7 for y in ys)
    ts = np.concatenate([E4M3_VALUES, E4M3_MID, np.nextafter(E4M3_MID, 0), np.nextafter(E4M3_MID, 1e9),
                         [500.0, 1e9, 2.0 ** -11, 2.0 ** -10]]).astype(np.float32)
    assert all(int(e4m3_code(t)) == oracle.e4m3_encode(t) for t in ts)


def test_element_encoder_equals_the_division_for_every_bf16_value():
    checked = settled = 0
    for g in GLOBAL_SCALES:
        rg = F32(1) / g
        for s in range(1, 0x7F):
            ds = F32(E4M3_VALUES[s])
            d = ds * g
            if not (d > 0 and np.isfinite(d)):
                continue
            x = X_ALL[X_ALL <= F32(8) * d]                                     # larger values saturate on both sides
            r = (F32(1) / ds) * rg
            lo = e2m1_mag(x * (r * WIDEN_LO))
            hi = e2m1_mag(x * (r * WIDEN_HI))
            want = e2m1_mag(x / d)
            assert np.all(lo <= want) and np.all(want <= hi), (g, s)
            assert np.all(hi - lo <= 1), (g, s)
            diff = lo != hi
            got = np.where(diff, pick(lo, hi, settle(x, np.full_like(x, d), E2M1_BOUNDARY[np.minimum(lo, 6)].astype(np.float32))), lo)
            assert np.array_equal(got, want), (g, s)
            checked += x.size
            settled += int(diff.sum())
    assert checked > 10_000_000 and settled > 0


def test_scale_encoder_equals_the_division_for_every_bf16_amax():
    settled = 0
    for g in GLOBAL_SCALES:
        g6 = F32(6) * g
        rg6 = F32(1) / g6
        with np.errstate(over="ignore"):                 # huge amax: inf on both sides, saturates to 448
            lo = e4m3_code(X_ALL * (rg6 * WIDEN_LO))
            hi = e4m3_code(X_ALL * (rg6 * WIDEN_HI))
            want = e4m3_code(X_ALL / g6)
        assert np.all(lo <= want) and np.all(want <= hi) and np.all(hi - lo <= 1), g
        diff = lo != hi
        mid = ((E4M3_VALUES[lo].astype(np.float32) + E4M3_VALUES[np.minimum(hi, 126)].astype(np.float32))
               * F32(0.5)).astype(np.float32)
        c = settle(X_ALL[diff], np.full(int(diff.sum()), g6, np.float32), mid[diff])
        got = lo.copy()
        got[diff] = pick(lo[diff], hi[diff], c)
        assert np.array_equal(got, want), g
        settled += int(diff.sum())
    assert settled > 0


def test_fp8_encoder_equals_the_division_for_every_bf16_value():
    """The FP8 KV quantize uses the same scheme: E4M3 of x * fl32(1/s) widened
    both ways, settled against the midpoint of the two candidates."""
    settled = 0
    for s in GLOBAL_SCALES:
        rs = F32(1) / s
        with np.errstate(over="ignore"):
            lo = e4m3_code(X_ALL * (rs * WIDEN_LO))
            hi = e4m3_code(X_ALL * (rs * WIDEN_HI))
            want = e4m3_code(X_ALL / s)
        assert np.all(lo <= want) and np.all(want <= hi) and np.all(hi - lo <= 1), s
        diff = lo != hi
        mid = ((E4M3_VALUES[lo].astype(np.float32) + E4M3_VALUES[np.minimum(hi, 126)].astype(np.float32))
               * F32(0.5)).astype(np.float32)
        got = lo.copy()
        got[diff] = pick(lo[diff], hi[diff], settle(X_ALL[diff], np.full(int(diff.sum()), s, np.float32), mid[diff]))
        assert np.array_equal(got, want), s
        settled += int(diff.sum())
    assert settled > 0
