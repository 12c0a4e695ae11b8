"""Pins for the oracle's quantize / layout / harmonize steps (CPU only)."""
import numpy as np
import pytest

from nvfp4_w4a4_quantized_06_b200 import workloads as W

E2M1 = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6])


# ------------------------------------------------------------------ layout
def test_sf_offset_literal_positions(oracle):
    K = 512                     # 32 scale columns -> 8 atoms per 128-row block
    assert oracle.sf_offset(0, 0, K) == 0
    assert oracle.sf_offset(0, 1, K) == 1
    assert oracle.sf_offset(0, 3, K) == 3
    assert oracle.sf_offset(1, 0, K) == 16
    assert oracle.sf_offset(31, 0, K) == 31 * 16
    assert oracle.sf_offset(32, 0, K) == 4
    assert oracle.sf_offset(96, 2, K) == 12 + 2
    assert oracle.sf_offset(0, 4, K) == 512
    assert oracle.sf_offset(128, 0, K) == 8 * 512
    assert oracle.sf_offset(130, 5, K) == 8 * 512 + 512 + 2 * 16 + 1
    assert oracle.sf_bytes(1, K) == 128 * 32
    assert oracle.sf_bytes(129, K) == 256 * 32


@pytest.mark.parametrize("rows,K", [(128, 64), (200, 320), (32, 256)])
def test_sf_layout_is_a_bijection(oracle, rows, K):
    pad = (rows + 127) // 128 * 128
    offs = sorted(oracle.sf_offset(r, c, K) for r in range(pad) for c in range(K // 16))
    assert offs == list(range(oracle.sf_bytes(rows, K)))


# ------------------------------------------------------------ global scale
def test_global_scale(oracle):
    x = np.zeros((4, 64), np.float32)
    assert oracle.global_scale(x) == np.float32(1.0)
    x[2, 5] = -2688.0
    assert oracle.global_scale(x) == np.float32(1.0)
    x[1, 1] = 5376.0
    assert oracle.global_scale(x) == np.float32(2.0)


# ---------------------------------------------------------------- quantize
def test_hand_worked_block(oracle):
    # g = 1: amax = 12 -> t = 12/6 = 2 -> scale code 0x40 (2.0) -> d = 2
    # y = x/2 -> E2M1 nearest (ties to even)
    x = np.zeros((1, 64), np.float32)
    blk = [12, 1, -2.9, 0.4, 0.5, 2.5, -7, 5, 0, -0.0, 3, -1, 8, 10, 11, 0.2]
    x[0, :16] = blk
    # y = [6, .5, -1.45, .2, .25, 1.25, -3.5, 2.5, 0, -0, 1.5, -.5, 4, 5, 5.5, .1]
    want = [7, 1, 8 | 3, 0, 0, 2, 8 | 6, 4, 0, 8, 3, 8 | 1, 6, 6, 7, 0]
    codes, sf = oracle.quantize(x, 1.0)
    got = [(codes[0, i // 2] >> (4 * (i % 2))) & 15 for i in range(16)]
    assert got == want
    assert sf[oracle.sf_offset(0, 0, 64)] == 0x40
    # nibble order: element 0 in the low nibble of byte 0
    assert codes[0, 0] == (7 | (1 << 4))
    # an all-zero block: scale 0 and +0 codes
    assert sf[oracle.sf_offset(0, 1, 64)] == 0 and np.all(codes[0, 8:16] == 0)


def test_hand_worked_scale_rounding(oracle):
    # g = 1, amax = 7 -> t = 7/6 = 1.1666.. -> E4M3 1.125 (0x39) -> d = 1.125
    # y(7) = 6.222 -> saturates to 6; y(-3.4) = -3.0222 -> -3
    x = np.zeros((1, 64), np.float32)
    x[0, 0], x[0, 1] = 7.0, -3.4
    codes, sf = oracle.quantize(x, 1.0)
    assert sf[0] == 0x39
    assert codes[0, 0] == (7 | ((8 | 5) << 4))


def _random_exact_tensor(rng, rows, K, g):
    """x = dec(q) * dec(s) * g with one +-6 per block, so that quantize must
    return exactly (q, s) when g is a power of two."""
    nb = K // 16
    s_codes = rng.integers(0x08, 0x7F, size=(rows, nb))          # normal scales
    s_codes[s_codes == 0x7F] = 0x7E
    q = rng.integers(0, 16, size=(rows, K))
    pos = rng.integers(0, 16, size=(rows, nb))
    for r in range(rows):
        for b in range(nb):
            q[r, b * 16 + pos[r, b]] = 7 | (8 * rng.integers(0, 2))
    from oracle import e4m3_decode
    sdec = np.vectorize(e4m3_decode)(s_codes)
    qdec = np.where(q & 8, -1, 1) * E2M1[q & 7]
    x = qdec * np.repeat(sdec, 16, axis=1) * g
    return x.astype(np.float32), q, s_codes


@pytest.mark.parametrize("g", [1.0, 2.0 ** -7, 2.0 ** 5])
def test_exact_round_trip(oracle, g):
    rng = np.random.default_rng(11)
    rows, K = 40, 256
    x, q, s_codes = _random_exact_tensor(rng, rows, K, g)
    codes, sf = oracle.quantize(x, g)
    got_q = np.stack([codes & 15, codes >> 4], axis=-1).reshape(rows, K)
    # +-0 codes: the value 0 can come back with either sign code; compare values
    assert np.array_equal(np.where(got_q & 7 == 0, 0, got_q), np.where(q & 7 == 0, 0, q))
    assert np.array_equal(oracle.sf_gather(sf, np.arange(rows), K), s_codes.astype(np.uint8))


def test_error_bound_and_block_invariants(oracle):
    x = W.gaussian(48, 512, seed=5, outliers=W.Outliers("scale", 0.05, 40.0),
                   dtype=__import__("torch").float32).numpy()
    g = oracle.global_scale(x)
    codes, sf = oracle.quantize(x, g)
    deq = oracle.dequantize(codes, sf, g)
    sdec = np.vectorize(oracle.e4m3_decode)(oracle.sf_gather(sf, np.arange(48), 512))
    unit = np.repeat(sdec, 16, axis=1) * float(g)            # value of one E2M1 step of 1.0
    y = x / unit
    gap = np.where(np.abs(y) < 2, 0.5, np.where(np.abs(y) < 4, 1.0, 2.0))
    inside = np.abs(y) <= 6
    err = np.abs(x - deq)
    # half a grid step, plus fp32 rounding slack of the scale arithmetic
    assert np.all(err[inside] <= 0.5 * gap[inside] * unit[inside] * (1 + 1e-6) + 1e-30)
    # saturated elements: error is what exceeds 6 steps
    sat = ~inside
    assert np.all(err[sat] <= (np.abs(y[sat]) - 6) * unit[sat] * (1 + 1e-6) + 1e-30)
    # block facts: max/RMS <= 4 holds for every 16-block of inputs and outputs
    for arr in (x.astype(np.float64), deq):
        b = arr.reshape(-1, 16)
        rms = np.sqrt(np.mean(b * b, axis=1))
        mx = np.max(np.abs(b), axis=1)
        ok = rms > 0
        assert np.all(mx[ok] / rms[ok] <= 4.0 + 1e-12)
    # the largest element of each non-zero block lands within one E4M3 rounding of 6
    big = np.max(np.abs(y).reshape(-1, 16), axis=1)
    assert np.all((big >= 6 / 1.0625 - 1e-6) & (big <= 6 * 1.0625 + 1e-6))


def test_outlier_damages_only_its_block(oracle):
    x = W.gaussian(8, 256, seed=9, dtype=__import__("torch").float32).numpy()
    g = np.float32(np.abs(x).max() * 40 / 2688)   # held fixed across both calls
    c0, s0 = oracle.quantize(x, g)
    x2 = x.copy()
    x2[3, 37] *= 40                              # block (row 3, block 2)
    c1, s1 = oracle.quantize(x2, g)
    changed_codes = np.argwhere(c0 != c1)
    assert len(changed_codes) > 0
    assert np.all(changed_codes[:, 0] == 3) and np.all(changed_codes[:, 1] // 8 == 2)
    d = np.nonzero(s0 != s1)[0]
    assert list(d) == [oracle.sf_offset(3, 2, 256)]
    # with g recomputed from the new amax every block may move (stated, not pinned)


def test_zero_and_tiny_scales(oracle):
    x = np.zeros((2, 64), np.float32)
    x[0, :16] = 1e-30          # t underflows below 2^-10 -> scale 0 -> codes +0
    x[1, 16:32] = -1e-30
    codes, sf = oracle.quantize(x, 1.0)
    assert np.all(codes == 0) and np.all(sf == 0)


def test_sampled_rows_match_full(oracle):
    x = W.gaussian(300, 320, seed=4).float().numpy()
    g = oracle.global_scale(x)
    c_full, s_full = oracle.quantize(x, g)
    rows = W.sample_rows(300, 17)
    c_s, s_s = oracle.quantize(x[rows], g)
    assert np.array_equal(c_full[rows], c_s)
    assert np.array_equal(oracle.sf_gather(s_full, rows, 320),
                          oracle.sf_gather(s_s, np.arange(len(rows)), 320))


def test_fused_group_rows_offset(oracle):
    K = 256
    w0 = W.gaussian(48, K, seed=1, std=0.02).float().numpy()
    w1 = W.gaussian(48, K, seed=2, std=0.02).float().numpy()
    g0, g1 = oracle.global_scale(w0), oracle.global_scale(w1)
    sf = np.zeros(oracle.sf_bytes(96, K), np.uint8)
    c0, _ = oracle.quantize(w0, g0, sf=sf, sf_row0=0)
    c1, _ = oracle.quantize(w1, g1, sf=sf, sf_row0=48)
    _, s_alone = oracle.quantize(w1, g1)
    assert np.array_equal(oracle.sf_gather(sf, np.arange(48, 96), K),
                          oracle.sf_gather(s_alone, np.arange(48), K))
    # padding rows 96..127 stay zero
    assert np.all(oracle.sf_gather(sf, np.arange(96, 128), K) == 0)


# --------------------------------------------------------------- harmonize
def _fused(oracle, K=256, stds=(0.02, 0.02), rows=(48, 48)):
    ws = [W.gaussian(r, K, seed=i + 1, std=s).float().numpy() for i, (r, s) in enumerate(zip(rows, stds))]
    gs = [oracle.global_scale(w) for w in ws]
    offs = np.concatenate([[0], np.cumsum(rows)])
    sf = np.zeros(oracle.sf_bytes(int(offs[-1]), K), np.uint8)
    codes = [oracle.quantize(w, g, sf=sf, sf_row0=int(o))[0] for w, g, o in zip(ws, gs, offs)]
    return ws, gs, offs, sf, np.concatenate(codes)


def test_harmonize_identity_when_scales_equal(oracle):
    ws, gs, offs, sf, codes = _fused(oracle)
    before = sf.copy()
    gstar = oracle.harmonize(sf, 256, offs, [gs[0], gs[0]])
    assert gstar == gs[0] and np.array_equal(sf, before)


def test_harmonize_power_of_two_ratio_is_exact(oracle):
    ws, gs, offs, sf, codes = _fused(oracle)
    before = sf.copy()
    gstar = oracle.harmonize(sf, 256, offs, [np.float32(2.0), np.float32(8.0)])
    assert gstar == 8.0
    b = oracle.sf_gather(before, np.arange(48), 256)
    a = oracle.sf_gather(sf, np.arange(48), 256)
    dec = np.vectorize(oracle.e4m3_decode)
    ok = dec(b) >= 2.0 ** -6 * 4          # quarter of a normal stays normal
    assert np.all(dec(a)[ok] == dec(b)[ok] / 4)
    assert np.array_equal(oracle.sf_gather(sf, np.arange(48, 96), 256),
                          oracle.sf_gather(before, np.arange(48, 96), 256))


def test_harmonize_preserves_dequantized_weights(oracle):
    K = 256
    ws, gs, offs, sf, codes = _fused(oracle, K, stds=(0.02, 0.031), rows=(48, 80))
    assert gs[0] != gs[1]
    deq_before = np.concatenate([oracle.dequantize(codes[o0:o1], sf, g, sf_row0=o0)
                                 for g, o0, o1 in zip(gs, offs[:-1], offs[1:])])
    gstar = oracle.harmonize(sf, K, offs, gs)
    assert gstar == max(gs)
    deq_after = oracle.dequantize(codes, sf, gstar)
    # per element: |after - before| <= 2^-4 * |scale step| (normal) or 2^-10 * g* (subnormal)
    rows = np.arange(int(offs[-1]))
    unit_after = np.repeat(np.vectorize(oracle.e4m3_decode)(oracle.sf_gather(sf, rows, K)), 16, 1) * float(gstar)
    q = np.abs(deq_after) / np.where(unit_after > 0, unit_after, 1)
    bound = np.maximum(np.abs(deq_before) * (2 ** -4 + 1e-6), q * 2.0 ** -10 * float(gstar))
    assert np.all(np.abs(deq_after - deq_before) <= bound + 1e-30)
    rel = np.linalg.norm(deq_after - deq_before) / np.linalg.norm(deq_before)
    assert rel < 2 ** -4


def test_unharmonized_fused_gemm_shows_scale_mismatch(oracle):
    """The serving bug the pages repair: a fused kernel that applies one module's
    global scale to all rows mis-scales the others by g_m/g_0; after
    harmonization the shared scale is right for every row."""
    K = 256
    ws, gs, offs, sf, codes = _fused(oracle, K, stds=(0.02, 0.05), rows=(48, 48))
    wrong = oracle.dequantize(codes, sf, gs[0])                      # g_0 for all rows
    right = np.concatenate([oracle.dequantize(codes[o0:o1], sf, g, sf_row0=o0)
                            for g, o0, o1 in zip(gs, offs[:-1], offs[1:])])
    ratio = np.linalg.norm(wrong[48:]) / np.linalg.norm(right[48:])
    assert abs(ratio - gs[0] / gs[1]) < 1e-6
    gstar = oracle.harmonize(sf, K, offs, gs)
    fixed = oracle.dequantize(codes, sf, gstar)
    assert np.linalg.norm(fixed - right) / np.linalg.norm(right) < 2 ** -4


# ------------------------------------------------ arithmetic order, exactly
# The pages fix the block scale as "block maximum / 6" relative to a per-tensor
# FP32 scale (ta-paperlens page, 前提1) but not the order of the fp32 steps.
# The reading the oracle states is
#   g6 = fl32(6 g), t = fl32(amax / g6), s = E4M3(t), d = fl32(dec(s) g), y = fl32(x / d).
# The checks below evaluate that reading in exact rational arithmetic, with an
# explicit round-to-nearest-even onto binary32 after each step, at global
# scales that are not powers of two, on inputs placed within a few ulps of the
# E4M3 midpoints and the E2M1 decision boundaries, where a different order of
# operations changes the result.
from fractions import Fraction as Fr  # noqa: E402

E2M1_MAG = [Fr(0), Fr(1, 2), Fr(1), Fr(3, 2), Fr(2), Fr(3), Fr(4), Fr(6)]


def _e4m3_mag(c):
    e, m = c >> 3, c & 7
    return Fr(m, 512) if e == 0 else (1 + Fr(m, 8)) * Fr(2) ** (e - 7)


E4M3_MAG = [_e4m3_mag(c) for c in range(0x7F)]          # codes 0 .. 0x7E (448)


def _fl32(q: Fr) -> Fr:
    """The binary32 value nearest to the rational q (ties to even), subnormals
    included; |q| stays far below the overflow threshold in these tests."""
    if q == 0:
        return Fr(0)
    a = abs(q)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    while Fr(2) ** e > a:
        e -= 1
    while Fr(2) ** (e + 1) <= a:
        e += 1
    quantum = Fr(2) ** (max(e, -126) - 23)
    m = a / quantum
    n = m.numerator // m.denominator
    rem = m - n
    if rem > Fr(1, 2) or (rem == Fr(1, 2) and n % 2 == 1):
        n += 1
    return (n * quantum) if q > 0 else -(n * quantum)


def _nearest(a: Fr, grid):
    """Index of the grid magnitude nearest to a >= 0; ties to the even index;
    beyond the top the top index (satfinite)."""
    if a >= grid[-1]:
        return len(grid) - 1
    best = 0
    for c in range(1, len(grid)):
        d, db = abs(a - grid[c]), abs(a - grid[best])
        if d < db or (d == db and c % 2 == 0):
            best = c
    return best


def _exact_block(xb, g, order="reading"):
    """Scale byte and 16 codes of one block by the stated reading (or by one of
    the plausible wrong orders, which the test shows the inputs can tell apart)."""
    g = Fr(float(g))
    xs = [Fr(float(v)) for v in xb]
    amax = max(abs(v) for v in xs)
    if order == "amax/6/g":
        t = _fl32(_fl32(amax / 6) / g)
    elif order == "6g exact":
        t = _fl32(amax / (6 * g))
    else:
        t = _fl32(amax / _fl32(6 * g))
    s = _nearest(t, E4M3_MAG)
    decs = E4M3_MAG[s]
    if decs == 0:
        return s, [0] * 16
    d = _fl32(decs * g)
    codes = []
    for v in xs:
        if order == "x*(1/d)":
            y = _fl32(v * _fl32(1 / d))
        elif order == "x/dec(s)/g":
            y = _fl32(_fl32(v / decs) / g)
        else:
            y = _fl32(v / d)
        c = _nearest(abs(y), E2M1_MAG)
        codes.append(c | (8 if y < 0 or (y == 0 and v < 0) else 0))
    return s, codes


def _ulps(v: np.float32, k: int) -> np.float32:
    return (np.array([v], np.float32).view(np.int32) + k).view(np.float32)[0]


def _order_probe_blocks(g: np.float32) -> np.ndarray:
    """Blocks whose maximum lands within 3 ulps of an E4M3 midpoint (after the
    division by fl32(6g)), and blocks whose other 15 elements land within 2
    ulps of an E2M1 decision boundary (after the division by d)."""
    g6 = np.float32(6) * g
    blocks = []
    mids = [(E4M3_MAG[c] + E4M3_MAG[c + 1]) / 2 for c in range(8, 0x7E, 5)]     # normal range
    for mid in mids:
        centre = np.float32(float(mid) * float(g6))
        for k in range(-3, 4):
            b = np.zeros(16, np.float32)
            b[0] = _ulps(centre, k)
            b[1:] = b[0] * np.float32(0.25)
            blocks.append(b)
    bounds = [Fr(1, 4), Fr(3, 4), Fr(5, 4), Fr(7, 4), Fr(5, 2), Fr(7, 2), Fr(5)]
    for sc in (0x2B, 0x3D, 0x46, 0x59, 0x6A):                # scale codes to aim at
        amax = np.float32(6 * float(E4M3_MAG[sc]) * float(g6))
        decs = Fr(float(E4M3_MAG[_nearest(_fl32(Fr(float(amax)) / _fl32(6 * Fr(float(g)))), E4M3_MAG)]))
        d = _fl32(decs * Fr(float(g)))
        vals = [np.float32(float(T * d)) for T in bounds]
        probes = [_ulps(v, k) for v in vals for k in (-2, -1, 0, 1, 2)]
        for i in range(0, len(probes), 15):
            b = np.zeros(16, np.float32)
            b[0] = amax
            chunk = probes[i:i + 15]
            b[1:1 + len(chunk)] = [p if j % 2 else -p for j, p in enumerate(chunk)]
            blocks.append(b)
    n = len(blocks) + (-len(blocks)) % 4                     # whole 64-element rows
    blocks += [np.zeros(16, np.float32)] * (n - len(blocks))
    return np.stack(blocks).reshape(-1, 64)


ORDER_GSCALES = [np.float32(0.37 / 2688), np.float32(3.3 / 2688), np.float32(0.0123), np.float32(0.7 / 2688)]


def test_arithmetic_order_matches_the_exact_reading(oracle):
    detected = {alt: 0 for alt in ("amax/6/g", "x*(1/d)", "x/dec(s)/g", "6g exact")}
    for g in ORDER_GSCALES:
        x = _order_probe_blocks(g)
        rows = x.shape[0]
        codes, sf = oracle.quantize(x, g)
        got_s = oracle.sf_gather(sf, np.arange(rows), 64).reshape(-1)
        got_q = np.stack([codes & 15, codes >> 4], axis=-1).reshape(-1, 16)
        blocks = x.reshape(-1, 16)
        want = [_exact_block(b, g) for b in blocks]
        for i, (s, q) in enumerate(want):
            assert got_s[i] == s, (float(g), i, got_s[i], s)
            assert list(got_q[i]) == q, (float(g), i, list(got_q[i]), q)
        for alt in detected:
            detected[alt] += sum(_exact_block(b, g, alt) != w for b, w in zip(blocks, want))
    # the probes are sharp enough to tell the stated order from the plausible
    # alternatives: each of them changes scales or codes on these inputs
    assert all(n > 0 for n in detected.values()), detected


def test_exact_reading_helpers():
    """The rational helpers against plain facts: binary32 rounding at a tie,
    a subnormal, and the E4M3 / E2M1 grids' ends and ties."""
    assert _fl32(Fr(1) + Fr(2) ** -24) == 1                          # tie -> even
    assert _fl32(Fr(1) + Fr(3, 2 ** 25)) == 1 + Fr(2) ** -23          # above the tie
    assert _fl32(Fr(3, 2 ** 151)) == Fr(1, 2 ** 149)                  # subnormal quantum
    assert _fl32(Fr(1, 3)) == Fr(float(np.float32(1 / 3)))
    assert _nearest(Fr(1, 4), E2M1_MAG) == 0 and _nearest(Fr(3, 4), E2M1_MAG) == 2
    assert _nearest(Fr(5), E2M1_MAG) == 6 and _nearest(Fr(100), E2M1_MAG) == 7
    assert E4M3_MAG[0x7E] == 448 and E4M3_MAG[1] == Fr(1, 512) and E4M3_MAG[8] == Fr(1, 64)
    assert _nearest(Fr(17, 16), E4M3_MAG) == 0x38                     # 1.0625: tie -> 1.0 (even)
