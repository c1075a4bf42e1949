"""Seeded synthetic workloads for the DualQuant solver and activation path.

This module only draws random inputs; it holds none of the method's arithmetic. Both the
oracle-side tests and the CUDA-side tests/bench take their inputs from here.

The real workloads on the DualQuant pages are Llama/Qwen weights and activations, which
are not available; these generators stand in for them with the matrix shapes of the
Llama-3.2-1B, Llama-3.1-8B and Llama-2-7B projections and the value distributions below.

Recipe (shared by host and device generators):
  * seed = 1000 * config + 16 * block + proj_idx  (proj order q, k, v, o, gate, up, down)
  * values drawn in float64 (host, NumPy PCG64) or float32 (device, torch Philox), then
    rounded to float32 and to bfloat16 (round to nearest even) unless the config is fp32
  * outlier count = round-half-even(fraction * dim), at least 1, drawn without replacement
  * Student-t(4) scaled to std s uses scale s / sqrt(2) (Var t4 = 2); it is drawn as
    Z * sqrt(4 / V) with V = -2 log(U1 U2) (a chi-square with 4 degrees of freedom)
  * Laplace(b) is drawn as b * (E1 - E2), E = -ln(1 - U) with U uniform in [0, 1) (both
    exponentials are finite: 1 - U is in (0, 1])
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np
import torch

PROJ = ("q", "k", "v", "o", "gate", "up", "down")


@dataclass(frozen=True)
class FormatSpec:
    kind: str          # "INT4" | "MXINT4" | "MXFP4" | "NVFP4"
    group: int         # block length B along a row (INT4: 64/128; MX: 32; NV: 16)


INT4_G128 = FormatSpec("INT4", 128)
INT4_G64 = FormatSpec("INT4", 64)
MXINT4 = FormatSpec("MXINT4", 32)
MXFP4 = FormatSpec("MXFP4", 32)
NVFP4 = FormatSpec("NVFP4", 16)
FORMATS = {"INT4": INT4_G128, "INT4_G64": INT4_G64, "MXINT4": MXINT4, "MXFP4": MXFP4,
           "NVFP4": NVFP4}


@dataclass(frozen=True)
class WeightConfig:
    cid: int
    name: str
    blocks: int
    shapes: dict           # proj -> (m, n)
    dist: str              # "normal" | "t4" | "laplace"
    scale: float           # std (normal / t4) or Laplace b
    outlier_axis: str      # "col" | "row" | "entries"
    outlier_frac: float
    outlier_gain: float
    fmt: FormatSpec
    iters: int
    dtype: str             # "bf16" | "f32"

    def layer_set(self):
        """[(block, proj_idx, m, n)] in block-major, projection-minor order."""
        out = []
        for b in range(self.blocks):
            for p, name in enumerate(PROJ):
                if name in self.shapes:
                    m, n = self.shapes[name]
                    out.append((b, p, m, n))
        return out

    def elements(self):
        return sum(m * n for _, _, m, n in self.layer_set())


def _llama(q, kv, ffn):
    return {"q": (q, q), "k": (kv, q), "v": (kv, q), "o": (q, q),
            "gate": (ffn, q), "up": (ffn, q), "down": (q, ffn)}


CONFIGS = {
    1: WeightConfig(1, "single 512x512 fp32 tile", 1, {"q": (512, 512)}, "normal", 0.02,
                    "entries", 0.005, 20.0, INT4_G128, 20, "f32"),
    2: WeightConfig(2, "Llama-3.2-1B-shaped layer set", 16, _llama(2048, 512, 8192), "t4",
                    0.02, "col", 0.01, 8.0, MXFP4, 16, "bf16"),
    3: WeightConfig(3, "Llama-3.1-8B-shaped layer set", 32, _llama(4096, 1024, 14336),
                    "normal", 0.015, "col", 0.005, 10.0, NVFP4, 16, "bf16"),
    4: WeightConfig(4, "Llama-2-7B-shaped layer set", 32,
                    {"q": (4096, 4096), "k": (4096, 4096), "v": (4096, 4096),
                     "o": (4096, 4096), "gate": (11008, 4096), "up": (11008, 4096),
                     "down": (4096, 11008)}, "laplace", 0.01, "row", 0.02, 5.0, MXINT4, 16,
                    "bf16"),
}

# Activation workload: 8192 tokens x 4096 channels, N(0,1), 6 channels x50. Its column
# scales come from a k_proj of the 8B shape (1024 x 4096) drawn with the 1B layer set's
# recipe (Student-t(4), std 0.02, 1% of columns x8) and solved in MXFP4 for 16 iterations.
ACT_TOKENS, ACT_CHANNELS, ACT_OUTLIERS, ACT_GAIN = 8192, 4096, 6, 50.0
ACT_SEED = 5000
ACT_KPROJ = WeightConfig(5, "k_proj for activation rescaling", 1, {"k": (1024, 4096)}, "t4",
                         0.02, "col", 0.01, 8.0, MXFP4, 16, "bf16")
ACT_FORMATS = (NVFP4, INT4_G128)


def seed_of(cid: int, block: int, proj_idx: int) -> int:
    return 1000 * cid + 16 * block + proj_idx


def outlier_count(frac: float, dim: int) -> int:
    return max(1, int(round(frac * dim)))   # Python round() is round-half-even


# ----------------------------------------------------------------------------- host side
def _host_base(rng: np.random.Generator, dist: str, scale: float, shape) -> np.ndarray:
    if dist == "normal":
        return rng.standard_normal(shape) * scale
    if dist == "t4":
        z = rng.standard_normal(shape)
        u1 = 1.0 - rng.random(shape)        # (0, 1]
        u2 = 1.0 - rng.random(shape)
        v = -2.0 * np.log(u1 * u2)
        return z * np.sqrt(4.0 / v) * (scale / math.sqrt(2.0))
    if dist == "laplace":
        e1 = -np.log(1.0 - rng.random(shape))
        e2 = -np.log(1.0 - rng.random(shape))
        return scale * (e1 - e2)
    raise ValueError(dist)


def round_to_bf16(x: np.ndarray) -> np.ndarray:
    """float64 -> float32 -> bfloat16 (both round to nearest even); returns a torch tensor."""
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16)


def weight_host(cfg: WeightConfig, block: int, proj_idx: int, m: int = None,
                n: int = None) -> torch.Tensor:
    """One weight matrix of a config, drawn on the host (CPU torch tensor)."""
    if m is None:
        m, n = cfg.shapes[PROJ[proj_idx]]
    rng = np.random.Generator(np.random.PCG64(seed_of(cfg.cid, block, proj_idx)))
    w = _host_base(rng, cfg.dist, cfg.scale, (m, n))
    if cfg.outlier_axis == "col":
        cols = rng.choice(n, outlier_count(cfg.outlier_frac, n), replace=False)
        w[:, cols] *= cfg.outlier_gain
    elif cfg.outlier_axis == "row":
        rows = rng.choice(m, outlier_count(cfg.outlier_frac, m), replace=False)
        w[rows, :] *= cfg.outlier_gain
    elif cfg.outlier_axis == "entries":
        # 4 random columns carry the outlier entries
        cols = rng.choice(n, 4, replace=False)
        k = outlier_count(cfg.outlier_frac, m * n)
        flat = rng.choice(4 * m, k, replace=False)
        w[flat % m, cols[flat // m]] *= cfg.outlier_gain
    if cfg.dtype == "f32":
        return torch.from_numpy(w.astype(np.float32))
    return round_to_bf16(w)


def act_host(seed: int = ACT_SEED, tokens: int = ACT_TOKENS,
             channels: int = ACT_CHANNELS) -> torch.Tensor:
    rng = np.random.Generator(np.random.PCG64(seed))
    x = rng.standard_normal((tokens, channels))
    ch = rng.permutation(channels)[:ACT_OUTLIERS]
    x[:, ch] *= ACT_GAIN
    return round_to_bf16(x)


# --------------------------------------------------------------------------- device side
def _dev_base(g: torch.Generator, dist: str, scale: float, shape, device) -> torch.Tensor:
    if dist == "normal":
        return torch.randn(shape, generator=g, device=device) * scale
    if dist == "t4":
        z = torch.randn(shape, generator=g, device=device)
        u1 = 1.0 - torch.rand(shape, generator=g, device=device)
        u2 = 1.0 - torch.rand(shape, generator=g, device=device)
        v = -2.0 * torch.log(u1 * u2)
        return z * torch.sqrt(4.0 / v) * (scale / math.sqrt(2.0))
    if dist == "laplace":
        e1 = -torch.log(1.0 - torch.rand(shape, generator=g, device=device))
        e2 = -torch.log(1.0 - torch.rand(shape, generator=g, device=device))
        return scale * (e1 - e2)
    raise ValueError(dist)


def weight_device(cfg: WeightConfig, block: int, proj_idx: int, device="cuda",
                  seed_offset: int = 0) -> torch.Tensor:
    """Same recipe drawn on the device (torch Philox stream, so values differ from host)."""
    m, n = cfg.shapes[PROJ[proj_idx]]
    g = torch.Generator(device=device)
    g.manual_seed(seed_of(cfg.cid, block, proj_idx) + 1_000_000 * seed_offset)
    w = _dev_base(g, cfg.dist, cfg.scale, (m, n), device)
    if cfg.outlier_axis == "col":
        k = outlier_count(cfg.outlier_frac, n)
        cols = torch.randperm(n, generator=g, device=device)[:k]
        w[:, cols] *= cfg.outlier_gain
    elif cfg.outlier_axis == "row":
        k = outlier_count(cfg.outlier_frac, m)
        rows = torch.randperm(m, generator=g, device=device)[:k]
        w[rows, :] *= cfg.outlier_gain
    elif cfg.outlier_axis == "entries":
        cols = torch.randperm(n, generator=g, device=device)[:4]
        k = outlier_count(cfg.outlier_frac, m * n)
        flat = torch.randperm(4 * m, generator=g, device=device)[:k]
        w[flat % m, cols[flat // m]] *= cfg.outlier_gain
    if cfg.dtype == "f32":
        return w.contiguous()
    return w.to(torch.bfloat16).contiguous()


def act_device(seed: int = ACT_SEED, tokens: int = ACT_TOKENS, channels: int = ACT_CHANNELS,
               device="cuda") -> torch.Tensor:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    x = torch.randn((tokens, channels), generator=g, device=device)
    ch = torch.randperm(channels, generator=g, device=device)[:ACT_OUTLIERS]
    x[:, ch] *= ACT_GAIN
    return x.to(torch.bfloat16).contiguous()
