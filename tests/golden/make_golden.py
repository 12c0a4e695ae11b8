"""Writes tests/golden/tiny_oracle_digest.txt from the CPU oracle alone.

Run:  python tests/golden/make_golden.py
The digest pins the oracle's output on the tiny 64x128x256 workload (the layer
and the rows beyond it) so that an accidental change to its arithmetic shows
up; a deliberate change regenerates it and names, in the commit message, the
page passage or reading behind it.
"""
import hashlib
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from nvfp4_w4a4_quantized_06_b200 import workloads as W  # noqa: E402


def digest():
    wl = W.WORKLOADS["tiny"]
    x = W.make_x(wl).numpy()
    w = W.make_w(wl, 0).numpy()
    gx, gw = oracle.global_scale(x), oracle.global_scale(w)
    xc, xs = oracle.quantize(x, gx)
    wc, ws = oracle.quantize(w, gw)
    y, _, _, _ = oracle.linear_reference(x, gx, wc, ws, gw)
    h = lambda a: hashlib.sha256(np.ascontiguousarray(a).tobytes()).hexdigest()
    return {
        "x_gscale_hex": np.float32(gx).view(np.uint32).item().to_bytes(4, "big").hex(),
        "w_gscale_hex": np.float32(gw).view(np.uint32).item().to_bytes(4, "big").hex(),
        "x_codes_sha256": h(xc), "x_sf_sha256": h(xs),
        "w_codes_sha256": h(wc), "w_sf_sha256": h(ws),
        "y00_f64": repr(float(y[0, 0])), "y_sum_f64": repr(float(y.sum())),
        **next_rows(x, w, gx, y, h),
    }


def next_rows(x, w, gx, y, h):
    """The rows beyond the layer on the same tiny inputs: gate activations of
    the product, fake-quant, FP8 codes, the re-quantizing harmonize of the
    weight split into two modules with their own scales, and the quantize
    fused into RMSNorm (norm weight seed 11)."""
    gates = oracle.gdn_gates(y, n_a=64)
    dq, se, sx = oracle.fake_quant(x, gx)
    fp8 = oracle.fp8_quantize(x, np.float32(np.abs(x).max()) / np.float32(448.0))
    w0, w1 = w[:64], w[64:] * np.float32(0.37)
    g0, g1 = oracle.global_scale(w0), oracle.global_scale(w1)
    K = w.shape[1]
    sf = np.zeros(oracle.sf_bytes(128, K), np.uint8)
    c0, _ = oracle.quantize(w0, g0, sf=sf, sf_row0=0)
    c1, _ = oracle.quantize(w1, g1, sf=sf, sf_row0=64)
    rc, rs, gstar = oracle.harmonize_requant(np.concatenate([c0, c1]), sf, K, [0, 64, 128], [g0, g1])
    nw = W.norm_weight(K, seed=11).float().numpy()
    nc, ns, ny, inv, near = oracle.rmsnorm_quantize(x, nw, 1e-6, gx)
    return {
        "gates_sum_f64": repr(float(gates.sum())),
        "fake_quant_sha256": h(dq), "fake_quant_rel_err": repr(float(np.sqrt(se / sx))),
        "fp8_codes_sha256": h(fp8),
        "requant_gstar_hex": np.float32(gstar).view(np.uint32).item().to_bytes(4, "big").hex(),
        "requant_codes_sha256": h(rc), "requant_sf_sha256": h(rs),
        "rmsnorm_inv_sha256": h(inv), "rmsnorm_codes_sha256": h(nc), "rmsnorm_sf_sha256": h(ns),
        "rmsnorm_near_ties": str(int(near.sum())),
    }


if __name__ == "__main__":
    out = os.path.join(os.path.dirname(os.path.abspath(__file__)), "tiny_oracle_digest.txt")
    with open(out, "w") as f:
        f.write("# written by tests/golden/make_golden.py from oracle/ only (tiny 64x128x256 workload)\n")
        for k, v in digest().items():
            f.write(f"{k}: {v}\n")
    print(open(out).read())
