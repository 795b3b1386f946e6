"""Helpers shared by the GPU parity tests: host copies, the near-tie rule and
the y tolerance.  Only marshalling and comparison -- no method arithmetic."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from atomic_expert_layer_b200 import inputs

# y tolerance for bf16 inputs with fp32 accumulation
Y_MAX_ABS = 2e-2
Y_REL_L2 = 5e-3
# an index may differ from the oracle's only where the cell's score is this
# close to the K-th score (GPU and oracle log-probabilities differ in the last bits)
NEAR_TIE = 1e-5


def host(t: torch.Tensor) -> np.ndarray:
    if t.dtype == torch.bfloat16:
        return inputs.to_u16(t)
    return t.detach().cpu().numpy()


def check_y(y_gpu: np.ndarray, y_ref: np.ndarray, what: str = "y") -> dict:
    y_gpu = y_gpu.astype(np.float64)
    err = np.abs(y_gpu - y_ref)
    rel = float(np.linalg.norm(y_gpu - y_ref) / max(np.linalg.norm(y_ref), 1e-300))
    stats = dict(max_abs=float(err.max()), rel_l2=rel,
                 max_abs_over_max=float(err.max() / max(np.abs(y_ref).max(), 1e-300)))
    assert stats["max_abs"] <= Y_MAX_ABS, (what, stats)
    assert stats["rel_l2"] <= Y_REL_L2, (what, stats)
    return stats


def check_routing_near_ties(idx_gpu, idx_ref, score_ref, p_r, p_c, N_c) -> int:
    """Index sets must match except for cells whose (oracle) score is within
    NEAR_TIE of the K-th score.  Returns the number of tokens that differ."""
    ndiff = 0
    for t in range(idx_gpu.shape[0]):
        a, b = set(idx_gpu[t].tolist()), set(idx_ref[t].tolist())
        if a == b:
            continue
        ndiff += 1
        sK = float(score_ref[t, -1])
        for n in a ^ b:
            s = float(np.float32(p_r[t, n // N_c]) + np.float32(p_c[t, n % N_c]))
            assert abs(s - sK) < NEAR_TIE, (t, n, s, sK)
    return ndiff


def oracle_y_rows(x_gpu, W_gpu, V_gpu, idx_gpu, gate_gpu, tokens) -> np.ndarray:
    """Oracle (fp64, token-centric) y rows for `tokens` with the given routing,
    gathering only the expert rows those tokens use."""
    tok = torch.as_tensor(np.asarray(tokens), device=idx_gpu.device, dtype=torch.long)
    sub_idx = idx_gpu[tok].long()
    uniq, inv = torch.unique(sub_idx, return_inverse=True)
    Wr = host(W_gpu[uniq])
    Vr = host(V_gpu[uniq])
    xr = host(x_gpu[tok])
    idx_local = inv.to(torch.int32).cpu().numpy()
    g = gate_gpu[tok].cpu().numpy()
    return oracle.expert_fwd_token_centric(xr, Wr, Vr, idx_local, g)


def distinct_random_idx(L: int, K: int, N: int, seed: int) -> np.ndarray:
    """L rows of K distinct expert ids in [0, N) (test input for the schedule)."""
    rng = np.random.default_rng(seed)
    out = np.empty((L, K), np.int32)
    for t in range(L):
        out[t] = rng.choice(N, size=K, replace=False)
    return out
