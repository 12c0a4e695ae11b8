"""Save/load of the shipped artefacts (no GPU needed): NVFP4 weights from the
CPU oracle's quantize, a harmonized fused group, and static FP8 KV scales
round-trip byte for byte; damaged files are refused with a clear error."""
import os

import numpy as np
import pytest
import torch

import oracle
from nvfp4_w4a4_quantized_06_b200 import checkpoint as ck
from nvfp4_w4a4_quantized_06_b200 import workloads as W


def _layer(rows, K, seed):
    w = W.gaussian(rows, K, seed=seed, std=0.02).float().numpy()
    g = oracle.global_scale(w)
    codes, sf = oracle.quantize(w, g)
    return ck.QuantizedLinear(torch.from_numpy(codes), torch.from_numpy(sf), torch.tensor([g], dtype=torch.float32))


def _group(K=256):
    offs = [0, 48, 96]
    sf = np.zeros(oracle.sf_bytes(96, K), np.uint8)
    codes, gs = [], []
    for m in range(2):
        w = W.gaussian(48, K, seed=10 + m, std=0.02 * (m + 1)).float().numpy()
        g = oracle.global_scale(w)
        codes.append(oracle.quantize(w, g, sf=sf, sf_row0=offs[m])[0])
        gs.append(g)
    gstar = oracle.harmonize(sf, K, offs, gs)
    return ck.QuantizedLinear(torch.from_numpy(np.concatenate(codes)), torch.from_numpy(sf),
                              torch.tensor([gstar], dtype=torch.float32), (48, 48))


def test_round_trip(work_dir):
    layers = {"mlp.gate_up": _layer(130, 320, 1), "gdn.in_proj_ba": _group()}
    kv = {"layer3.k": 0.0125, "layer3.v": 0.031}
    p = os.path.join(work_dir, "model.nvfp4")
    ck.save(p, layers, kv)
    got, kv2 = ck.load(p)
    assert set(got) == set(layers) and kv2 == pytest.approx(kv, rel=0, abs=1e-9)
    for name, q in layers.items():
        r = got[name]
        assert torch.equal(r.codes, q.codes) and torch.equal(r.sf, q.sf) and torch.equal(r.gscale, q.gscale)
        assert r.module_rows == q.module_rows and (r.N, r.K) == (q.N, q.K)


def test_damaged_files_are_refused(work_dir):
    q = _layer(64, 256, 3)
    p = os.path.join(work_dir, "m.nvfp4")
    with pytest.raises(ValueError, match="scales"):
        ck.save(p, {"a": ck.QuantizedLinear(q.codes, q.sf[:-1], q.gscale)})
    with pytest.raises(ValueError, match="multiple of 64"):
        ck.save(p, {"a": ck.QuantizedLinear(q.codes[:, :100], q.sf, q.gscale)})
    with pytest.raises(ValueError, match="global scale"):
        ck.save(p, {"a": ck.QuantizedLinear(q.codes, q.sf, torch.tensor([0.0]))})
    with pytest.raises(ValueError, match="add up"):
        ck.save(p, {"a": ck.QuantizedLinear(q.codes, q.sf, q.gscale, (32, 16))})
    with pytest.raises(ValueError, match="KV scale"):
        ck.save(p, {"a": q}, {"k": float("nan")})
    ck.save(p, {"a": q})
    d = torch.load(p, weights_only=True)
    d["version"] = 99
    torch.save(d, p)
    with pytest.raises(ValueError, match="version"):
        ck.load(p)
    d["version"] = ck.VERSION
    d["layers"]["a"]["sf"] = d["layers"]["a"]["sf"][:100]
    torch.save(d, p)
    with pytest.raises(ValueError, match="scales"):
        ck.load(p)
    torch.save({"something": 1}, p)
    with pytest.raises(ValueError, match="not an"):
        ck.load(p)


def test_layout_matches_the_oracle():
    # the checkpoint's own size rule agrees with the scale layout the oracle writes
    for rows, K in ((1, 64), (129, 320), (256, 5120)):
        assert ck._sf_bytes(rows, K) == oracle.sf_bytes(rows, K)
