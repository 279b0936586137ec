"""Seeded synthetic inputs for the MLP block, shared by the tests, the bench
and the smoke check.

This module draws random numbers and rounds them to the storage dtype; it
holds none of the block's arithmetic. Each tensor has its own CPU generator
seed (X: 0, A: 1, a: 2, B: 3, b: 4, dZ: 5, plus `seed_offset`), values are
drawn as float32 N(0, std²) and then rounded to bfloat16 (round to nearest
even) for the bf16 dtype. The oracle reads the same rounded host arrays the
GPU receives.
"""
from __future__ import annotations

import torch

from .configs import MLPConfig

SEEDS = {"X": 0, "A": 1, "a": 2, "B": 3, "b": 4, "dZ": 5}


def _normal(shape, std: float, seed: int) -> torch.Tensor:
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    if std == 0.0:
        return torch.zeros(shape, dtype=torch.float32)
    return torch.randn(shape, generator=g, dtype=torch.float32) * std


def torch_dtype(name: str) -> torch.dtype:
    return {"bf16": torch.bfloat16, "fp32": torch.float32}[name]


def make_inputs(cfg: MLPConfig, seed_offset: int = 0, T: int | None = None) -> dict:
    """CPU tensors X (T×h), A (h×F), a (F), B (F×h), b (h), dZ (T×h) in the
    config's dtype. `T` overrides the config's token count."""
    T = cfg.T if T is None else T
    dt = torch_dtype(cfg.dtype)
    s = {k: v + seed_offset for k, v in SEEDS.items()}
    out = {
        "X": _normal((T, cfg.h), cfg.std_X, s["X"]),
        "A": _normal((cfg.h, cfg.F), cfg.std_A, s["A"]),
        "a": _normal((cfg.F,), cfg.std_a, s["a"]),
        "B": _normal((cfg.F, cfg.h), cfg.std_B, s["B"]),
        "b": _normal((cfg.h,), cfg.std_b, s["b"]),
        "dZ": _normal((T, cfg.h), cfg.std_dZ, s["dZ"]),
    }
    return {k: v.to(dt).contiguous() for k, v in out.items()}


def make_shape(T: int, h: int, F: int, dtype: str = "bf16", seed_offset: int = 0,
               std_w: float = 0.05, std_bias: float = 0.1) -> dict:
    """Inputs of an arbitrary shape with O(1) pre-activations, for parity
    cases that are not one of the named presets."""
    from .configs import MLPConfig
    cfg = MLPConfig("custom", T, h, F, 1, dtype, 1.0, std_w, std_w, std_bias, std_bias)
    return make_inputs(cfg, seed_offset)


def sample_indices(n_total: int, n_pick: int, seed: int = 1234) -> torch.Tensor:
    """Sorted distinct indices in [0, n_total), seeded, always including the
    first and last index (tile edges and ragged tails)."""
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    n_pick = min(n_pick, n_total)
    idx = torch.randperm(n_total, generator=g)[:n_pick]
    idx = torch.unique(torch.cat([idx, torch.tensor([0, n_total - 1])]))
    return idx.sort().values
