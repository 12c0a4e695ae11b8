"""Writes tests/golden/tiny_oracle_digest.txt from the CPU oracle alone.

Run:  python tests/golden/make_golden.py
The digest pins the oracle's output on the tiny 64x128x256 workload so that an
accidental change to its arithmetic shows up; a deliberate change regenerates
it and names, in the commit message, the page passage or reading behind it.
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
    }


if __name__ == "__main__":
    out = os.path.join(os.path.dirname(os.path.abspath(__file__)), "tiny_oracle_digest.txt")
    with open(out, "w") as f:
        f.write("# written by tests/golden/make_golden.py from oracle/ only (tiny 64x128x256 workload)\n")
        for k, v in digest().items():
            f.write(f"{k}: {v}\n")
    print(open(out).read())
