"""Seeded synthetic workloads for the NVFP4 W4A4 linear layer.

This module only draws random numbers and shapes them; it holds none of the
layer's arithmetic (no scales, no rounding, no layout), so the CUDA path and
the CPU oracle can both be fed from it.

The shapes stand in for the layers of the hybrid 27B model the pages study
(hidden size 5120, MLP 17408, GDN in_proj_qkv 10240, in_proj_z 6144 and two
48-wide per-head gate projections; prefill of a 32K-token prompt and decode at
32 concurrent sequences).  The outlier recipes follow the input statistics the
pages report for GDN inputs (a mid-layer max/RMS of about 63.5 with 10.6% of
16-element blocks one-hot; arxiv-wiki page, "주요 결과", Table 2).

Recipe (all numpy PCG64):
  * Gaussians: ``standard_normal`` in float32, times the stated sigma in
    float32, then cast to bfloat16 by torch (round to nearest even).
  * Outliers are drawn from the same generator after the Gaussians: blocks
    chosen without replacement, a position uniform inside the block.
    ``scale``: that element is multiplied by the factor (sign kept).
    ``onehot``: that element is set to +-value with a random sign.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np
import torch

BLOCK = 16


@dataclass(frozen=True)
class Outliers:
    kind: str          # "scale" | "onehot" | "none"
    frac: float        # fraction of 16-element blocks hit
    value: float       # multiplier ("scale") or magnitude ("onehot")


@dataclass(frozen=True)
class Workload:
    name: str
    M: int
    K: int
    modules: tuple            # output rows of each weight module, fused along N
    x_dtype: torch.dtype
    x_outliers: Outliers
    w_std: float = 0.02
    x_seed: int = 0
    w_seeds: tuple = field(default=())

    @property
    def N(self) -> int:
        return int(sum(self.modules))

    @property
    def flops(self) -> int:
        return 2 * self.M * self.N * self.K


NONE = Outliers("none", 0.0, 0.0)

WORKLOADS = {
    # 64x128x256 fp32: the small case the oracle finishes in well under a second
    "tiny": Workload("tiny", 64, 256, (128,), torch.float32, Outliers("scale", 0.02, 40.0),
                     w_seeds=(1,)),
    # GDN gate projections a and b served as one GEMM (N = 48 + 48)
    "gdn_gates_ab": Workload("gdn_gates_ab", 4096, 5120, (48, 48), torch.bfloat16,
                             Outliers("onehot", 0.106, 63.5), w_seeds=(1, 2)),
    # GDN in_proj_qkv and in_proj_z served as one GEMM (N = 10240 + 6144)
    "gdn_qkv_z": Workload("gdn_qkv_z", 8192, 5120, (10240, 6144), torch.bfloat16,
                          Outliers("onehot", 0.106, 63.5), w_seeds=(1, 2)),
    # prefill of a 32K-token prompt through the MLP gate/up projection
    "prefill_mlp_gate_up": Workload("prefill_mlp_gate_up", 32768, 5120, (34816,), torch.bfloat16,
                                    Outliers("scale", 0.01, 30.0), w_seeds=(1,)),
    # decode at 32 concurrent sequences
    "decode_out_proj": Workload("decode_out_proj", 32, 5120, (5120,), torch.bfloat16, NONE,
                                w_seeds=(1,)),
    "decode_down_proj": Workload("decode_down_proj", 32, 17408, (5120,), torch.bfloat16, NONE,
                                 w_seeds=(2,)),
}


def _inject(rng: np.random.Generator, x: np.ndarray, out: Outliers) -> None:
    if out.kind == "none" or out.frac <= 0:
        return
    rows, K = x.shape
    nblocks = rows * (K // BLOCK)
    n_hit = int(round(out.frac * nblocks))
    if n_hit == 0:
        return
    blocks = rng.choice(nblocks, size=n_hit, replace=False)
    pos = rng.integers(0, BLOCK, size=n_hit)
    flat = x.reshape(-1)
    idx = blocks.astype(np.int64) * BLOCK + pos
    if out.kind == "scale":
        flat[idx] = flat[idx] * np.float32(out.value)
    elif out.kind == "onehot":
        sign = np.where(rng.integers(0, 2, size=n_hit) == 1, np.float32(1), np.float32(-1))
        flat[idx] = sign * np.float32(out.value)
    else:
        raise ValueError(out.kind)


def gaussian(rows: int, K: int, seed: int, std: float = 1.0,
             outliers: Outliers = NONE, dtype: torch.dtype = torch.bfloat16) -> torch.Tensor:
    """Seeded [rows, K] CPU tensor: N(0, std^2) with optional block outliers."""
    rng = np.random.Generator(np.random.PCG64(seed))
    x = rng.standard_normal((rows, K), dtype=np.float32)
    if std != 1.0:
        x *= np.float32(std)
    _inject(rng, x, outliers)
    t = torch.from_numpy(x)
    return t if dtype == torch.float32 else t.to(dtype)


def make_x(wl: Workload) -> torch.Tensor:
    return gaussian(wl.M, wl.K, wl.x_seed, 1.0, wl.x_outliers, wl.x_dtype)


def make_w(wl: Workload, module: int) -> torch.Tensor:
    return gaussian(wl.modules[module], wl.K, wl.w_seeds[module], wl.w_std, NONE, wl.x_dtype)


def norm_weight(K: int, seed: int, zero_centered: bool = False) -> torch.Tensor:
    """Seeded random-init RMSNorm weight [K] in bf16: 1 + 0.1 N(0,1), or the
    0.1 N(0,1) offset of the zero-centred form (gamma = 1 + w)."""
    rng = np.random.Generator(np.random.PCG64(seed))
    w = rng.standard_normal(K, dtype=np.float32) * np.float32(0.1)
    if not zero_centered:
        w += np.float32(1.0)
    return torch.from_numpy(w).to(torch.bfloat16)


def sample_rows(M: int, n: int, seed: int = 1234) -> np.ndarray:
    """Sorted seeded row sample that always includes the first and last row."""
    if n >= M:
        return np.arange(M, dtype=np.int64)
    rng = np.random.Generator(np.random.PCG64(seed))
    rows = rng.choice(M, size=n, replace=False)
    rows[0], rows[-1] = 0, M - 1
    return np.unique(rows).astype(np.int64)
