"""The GEMM launch planning, checked on the host (no GPU needed) through the
diagnostic entry point nvfp4_plan_for, with occupancy figures of a 148-SM
part given as arguments."""
import math

import pytest

from nvfp4_w4a4_quantized_06_b200 import build, native
from nvfp4_w4a4_quantized_06_b200 import workloads as W

SMS = 148
PAIRS = 74
# co-resident split-K clusters of c CTAs, one CTA per SM: floor(148 / c)
SPLITS = [[SMS // c if c else 0 for c in range(9)] for _ in range(3)]


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    native.lib()


def best_split(tiles, kstages, fit, bn=32):
    """Cluster size minimising waves x (stages per CTA + 1), first on ties;
    a 128-wide MMA N allows clusters of up to 5 CTAs (its reduction slots)."""
    best, cost = 0, None
    for c in range(1, min(5 if bn >= 128 else 8, kstages) + 1):
        if fit[c] <= 0:
            continue
        k = math.ceil(tiles / fit[c]) * (math.ceil(kstages / c) + 1)
        if cost is None or k < cost:
            best, cost = c, k
    return best


def test_every_configuration_gets_its_kernel():
    for name, wl in W.WORKLOADS.items():
        M, N, K = wl.M, wl.N, wl.K
        p = native.plan_for(M, N, K, SMS, PAIRS, SPLITS)
        assert p["kstages"] == math.ceil(K / 256)
        if M > 128 and N > 128:
            # large products: CTA pairs on 256 x 256 tiles, one wave of resident pairs
            assert p["kind"] == "pair" and p["bn"] == 256 and p["splits"] == 1, name
            assert (p["tiles_a"], p["tiles_b"]) == (math.ceil(M / 256), math.ceil(N / 256))
            assert p["grid"] == 2 * min(p["tiles_a"] * p["tiles_b"], PAIRS)
        else:
            # one narrow operand becomes the MMA's N; K is split over a cluster
            narrow = min(M, N) if M <= 128 and N <= 128 else (M if M <= 128 else N)
            swap = M <= 128 and (M <= N or N > 128)
            assert p["kind"] == "cluster" and p["swap"] == swap, name
            assert p["bn"] == (32 if narrow <= 32 else 64 if narrow <= 64 else 128)
            tiles = math.ceil((N if swap else M) / 128)
            assert p["tiles_a"] == tiles
            assert p["splits"] == best_split(tiles, p["kstages"], SPLITS[0], p["bn"])
            assert p["grid"] == tiles * p["splits"]


def test_decode_and_gate_plans():
    # the decode projection: the 32 activation rows are the MMA's N, 40 weight
    # tiles, K split three ways (one wave, 7 of the 20 K stages per CTA)
    p = native.plan_for(32, 5120, 5120, SMS, PAIRS, SPLITS)
    assert (p["kind"], p["bn"], p["swap"], p["splits"], p["grid"]) == ("cluster", 32, True, 3, 120)
    # the gate projection: the 96 weight rows are the MMA's N
    p = native.plan_for(4096, 96, 5120, SMS, PAIRS, SPLITS)
    assert (p["kind"], p["bn"], p["swap"], p["splits"], p["grid"]) == ("cluster", 128, False, 4, 128)


def test_fallbacks():
    # no cluster support: the single-CTA kernel with split-K partials
    p = native.plan_for(32, 5120, 5120, SMS, PAIRS, None)
    assert p["kind"] == "single" and p["swap"] and p["bn"] == 32 and p["splits"] >= 1
    # a large product with fewer tiles than resident pairs still gets pairs only
    # when it fills them; otherwise the single-CTA kernel spreads K
    p = native.plan_for(256, 256, 5120, SMS, PAIRS, SPLITS)
    assert p["kind"] == "single" and p["splits"] >= 1
    p = native.plan_for(256 * 8, 256 * 10, 5120, SMS, PAIRS, SPLITS)
    assert p["kind"] == "pair" and p["grid"] == 2 * PAIRS


def test_validation():
    with pytest.raises(native.Nvfp4Error, match="bad shape"):
        native.plan_for(32, 64, 100, SMS, PAIRS, SPLITS)
    with pytest.raises(native.Nvfp4Error, match="bad shape"):
        native.plan_for(32, 64, 256, 0, PAIRS, SPLITS)
    with pytest.raises(ValueError, match="3 rows"):
        native.plan_for(32, 64, 256, SMS, PAIRS, [[1, 2]])
    assert native.lib().nvfp4_plan_for(32, 64, 256, SMS, PAIRS, None, None) == 1
