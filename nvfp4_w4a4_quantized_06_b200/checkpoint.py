"""Save and load the shipped artefacts of a quantized model: every linear
layer's NVFP4 weight (packed E2M1 codes, swizzled E4M3 block scales, the FP32
global scale; for a fused group, the rows of each module) and the static
per-tensor FP8 KV-cache scales.  The pages' recipe ships exactly these:
every linear layer quantized, with calibrated FP8 KV scales alongside
(arxiv-wiki page, "주요 결과"; abstract on the shd-paper page).

The file is a `torch.save` dictionary of CPU tensors; `load` reads it with
`weights_only=True` and checks every layer's shapes and dtypes against the
layout the library reads, so a truncated or mislabelled tensor fails here and
not inside a kernel.
"""
from __future__ import annotations

import os
from dataclasses import dataclass, field

import torch

FORMAT = "nvfp4-w4a4-linear"
VERSION = 1


def _sf_bytes(rows: int, K: int) -> int:
    """Bytes of the swizzled scale buffer: rows padded to 128, K/16 columns."""
    return (rows + 127) // 128 * 128 * (K // 16)


@dataclass
class QuantizedLinear:
    codes: torch.Tensor                 # uint8 [N, K/2]
    sf: torch.Tensor                    # uint8 [pad128(N) * K/16], swizzled
    gscale: torch.Tensor                # float32 [1]; g* for a harmonized fused group
    module_rows: tuple = field(default=())   # rows of each fused module (sum N), () if one module

    @property
    def N(self) -> int:
        return int(self.codes.shape[0])

    @property
    def K(self) -> int:
        return int(self.codes.shape[1]) * 2

    def validate(self, name: str = "layer") -> None:
        c, s, g = self.codes, self.sf, self.gscale
        if c.dtype != torch.uint8 or c.dim() != 2:
            raise ValueError(f"{name}: codes must be a 2-D uint8 tensor")
        if self.K % 64 != 0 or self.N <= 0:
            raise ValueError(f"{name}: K = {self.K} must be a positive multiple of 64")
        if s.dtype != torch.uint8 or s.dim() != 1 or s.numel() != _sf_bytes(self.N, self.K):
            raise ValueError(f"{name}: scales must be {_sf_bytes(self.N, self.K)} uint8 bytes")
        if g.dtype != torch.float32 or g.numel() != 1:
            raise ValueError(f"{name}: the global scale must be one float32")
        gv = float(g.reshape(-1)[0])
        if not (gv > 0.0 and gv < float("inf")):
            raise ValueError(f"{name}: the global scale must be finite and > 0")
        if self.module_rows and (sum(self.module_rows) != self.N or min(self.module_rows) <= 0):
            raise ValueError(f"{name}: module rows {self.module_rows} do not add up to N = {self.N}")

    def to(self, device) -> "QuantizedLinear":
        return QuantizedLinear(self.codes.to(device), self.sf.to(device), self.gscale.to(device),
                               tuple(self.module_rows))


def save(path: str, layers: dict, kv_scales: dict | None = None) -> None:
    """Write `layers` (name -> QuantizedLinear) and `kv_scales` (name -> float)."""
    out = {"format": FORMAT, "version": VERSION, "layers": {}, "kv_scales": {}}
    for name, q in layers.items():
        q.validate(name)
        out["layers"][name] = {"codes": q.codes.detach().cpu().contiguous(), "sf": q.sf.detach().cpu().contiguous(),
                               "gscale": q.gscale.detach().cpu().reshape(1).contiguous(),
                               "module_rows": torch.tensor(list(q.module_rows), dtype=torch.int64)}
    for name, s in (kv_scales or {}).items():
        v = float(s)
        if not (v > 0.0 and v < float("inf")):
            raise ValueError(f"KV scale {name}: must be finite and > 0")
        out["kv_scales"][name] = torch.tensor([v], dtype=torch.float32)
    tmp = path + ".tmp"
    torch.save(out, tmp)
    os.replace(tmp, path)


def load(path: str, device="cpu"):
    """Read a file written by `save`; returns (layers, kv_scales) with the
    tensors on `device`."""
    d = torch.load(path, map_location="cpu", weights_only=True)
    if not isinstance(d, dict) or d.get("format") != FORMAT:
        raise ValueError(f"{path}: not an {FORMAT} checkpoint")
    if d.get("version") != VERSION:
        raise ValueError(f"{path}: version {d.get('version')}, this library reads {VERSION}")
    layers = {}
    for name, e in d["layers"].items():
        q = QuantizedLinear(e["codes"], e["sf"], e["gscale"], tuple(int(r) for r in e["module_rows"].tolist()))
        q.validate(name)
        layers[name] = q.to(device)
    kv = {name: float(t.reshape(-1)[0]) for name, t in d["kv_scales"].items()}
    return layers, kv
