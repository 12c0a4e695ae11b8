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
