"""Seeded synthetic inputs for the routed-branch forward.

This module only draws random tensors; it holds none of the method's
arithmetic, so both the CUDA path and the CPU oracle can be fed from it.

Recipe (per tensor, its own generator seeded with seed * 16 + tensor index):
  x   [L, d]    ~ N(0, 1), cast to bf16 (round to nearest even)
  W   [N, d]    ~ N(0, 1/d): drawn in fp32, scaled by d**-0.5, cast to bf16
  V   [N, d]    ~ N(0, 1/d)
  W_r [N_r, d]  ~ N(0, 1/d)   (one routing vector per grid row)
  W_c [N_c, d]  ~ N(0, 1/d)
Shared dense MLP weights (make_mlp_weights), hidden width F:
  W_g [F, d]    ~ N(0, 1/d)   (gate projection, one row per hidden unit)
  W_u [F, d]    ~ N(0, 1/d)   (up projection)
  W_d [d, F]    ~ N(0, 1/F)   (down projection, one row per output feature)
Large tensors are drawn in row chunks of CHUNK_ROWS from the same generator.
With zipf=True (skewed routing), feature d-1 of every token is set to 1 and
W_r[i, d-1] = -1.1 * ln(rank_r(i)), W_c[j, d-1] = -1.1 * ln(rank_c(j)), where
rank_r / rank_c are permutations of 1..N_r / 1..N_c drawn from a CPU generator
seeded with seed * 16 + 5 / + 6: an additive Zipf(s = 1.1) log-bias on the
router logits.
"""
from __future__ import annotations

import math

import numpy as np
import torch

from .configs import LayerConfig

CHUNK_ROWS = 1 << 16
TENSOR_INDEX = {"x": 0, "W": 1, "V": 2, "W_r": 3, "W_c": 4, "W_g": 7, "W_u": 8, "W_d": 9}


def _gen(device: torch.device, seed: int, which: str) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed * 16 + TENSOR_INDEX[which])
    return g


def _normal_bf16(rows: int, d: int, std: float, device, gen) -> torch.Tensor:
    out = torch.empty((rows, d), dtype=torch.bfloat16, device=device)
    for r0 in range(0, rows, CHUNK_ROWS):
        r1 = min(rows, r0 + CHUNK_ROWS)
        blk = torch.randn((r1 - r0, d), generator=gen, device=device, dtype=torch.float32)
        if std != 1.0:
            blk.mul_(std)
        out[r0:r1].copy_(blk)          # fp32 -> bf16, round to nearest even
    return out


def _zipf_bias(n: int, seed: int, which: int) -> torch.Tensor:
    g = torch.Generator()
    g.manual_seed(seed * 16 + which)
    rank = torch.randperm(n, generator=g) + 1            # a permutation of 1..n
    return (-1.1 * torch.log(rank.to(torch.float64))).to(torch.float32)


def make_inputs(cfg: LayerConfig, device="cpu", seed: int = 0, with_experts: bool = True):
    """Return a dict of bf16 tensors x, W, V, W_r, W_c on `device`."""
    device = torch.device(device)
    std = 1.0 / math.sqrt(cfg.d)
    out = {
        "x": _normal_bf16(cfg.L, cfg.d, 1.0, device, _gen(device, seed, "x")),
        "W_r": _normal_bf16(cfg.N_r, cfg.d, std, device, _gen(device, seed, "W_r")),
        "W_c": _normal_bf16(cfg.N_c, cfg.d, std, device, _gen(device, seed, "W_c")),
    }
    if with_experts:
        out["W"] = _normal_bf16(cfg.N, cfg.d, std, device, _gen(device, seed, "W"))
        out["V"] = _normal_bf16(cfg.N, cfg.d, std, device, _gen(device, seed, "V"))
    if cfg.zipf:
        out["x"][:, cfg.d - 1] = 1.0
        out["W_r"][:, cfg.d - 1] = _zipf_bias(cfg.N_r, seed, 5).to(device=device, dtype=torch.bfloat16)
        out["W_c"][:, cfg.d - 1] = _zipf_bias(cfg.N_c, seed, 6).to(device=device, dtype=torch.bfloat16)
    return out


def make_mlp_weights(d: int, F: int, device="cpu", seed: int = 0):
    """Return a dict of bf16 tensors W_g, W_u [F, d] and W_d [d, F] on `device`."""
    device = torch.device(device)
    return {
        "W_g": _normal_bf16(F, d, 1.0 / math.sqrt(d), device, _gen(device, seed, "W_g")),
        "W_u": _normal_bf16(F, d, 1.0 / math.sqrt(d), device, _gen(device, seed, "W_u")),
        "W_d": _normal_bf16(d, F, 1.0 / math.sqrt(F), device, _gen(device, seed, "W_d")),
    }


def to_u16(t: torch.Tensor) -> np.ndarray:
    """bf16 tensor -> numpy uint16 array of its bit patterns (host copy)."""
    assert t.dtype == torch.bfloat16
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def random_logprobs(L: int, n: int, seed: int, quantum: float | None = None) -> np.ndarray:
    """fp32 rows shaped like log-probabilities (N(-8, 2) draws, all negative in
    practice); with `quantum`, rounded to multiples of it to force exact ties."""
    rng = np.random.default_rng(seed)
    s = rng.normal(-8.0, 2.0, size=(L, n))
    if quantum is not None:
        s = np.round(s / quantum) * quantum
    return s.astype(np.float32)
