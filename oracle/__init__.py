"""CPU oracle for the routed branch of an OmniMoE layer -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may import this package.  The
library (``atomic_expert_layer_b200``) never does, and this package never
imports the library: the two share no code.  Inputs come from the seeded
generator module, which holds none of the method's arithmetic.

The arithmetic lives in ``omni_oracle.c`` (plain C, fp64, OpenMP over tokens);
this module only builds it with gcc and marshals numpy arrays through ctypes.
Every function follows the formulas of "OmniMoE: An Efficient MoE by
Orchestrating Atomic Experts at Scale" (rainbus review page, method paragraph,
steps 1-3); the readings taken where the page is silent are listed at the top
of ``omni_oracle.c``.

bf16 tensors are passed as ``numpy.uint16`` arrays of their bit patterns.
W_r and W_c are N_r x d and N_c x d (one routing vector per row).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "omni_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile omni_oracle.c into liboracle.so next to it (gcc, -O2, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=c99", "-fopenmp", "-ffp-contract=off", "-fno-fast-math",
               "-shared", "-fPIC", _SRC, "-o", _LIB + ".tmp", "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(_LIB + ".tmp", _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        I = ctypes.c_int
        lib.oracle_router_logprobs.argtypes = [P, P, P, I, I, I, I, P, P, I]
        lib.oracle_topk_from_logprobs.argtypes = [P, P, I, I, I, I, P, P, P, I]
        lib.oracle_schedule.argtypes = [P, P, I, I, I, I, P, P, P, P, P, P, P, P]
        lib.oracle_expert_fwd_token_centric.argtypes = [P, P, P, I, I, P, P, P, I, P, I]
        lib.oracle_expert_fwd_expert_centric.argtypes = [P, P, P, I, I, I, I, P, P, P, P, P, I, P]
        lib.oracle_expert_bwd.argtypes = [P, P, P, I, I, I, I, P, P, P, P, P, P, P]
        lib.oracle_router_bwd.argtypes = [P, P, P, I, I, I, I, I, P, P, P, P, P, P, P, P]
        lib.oracle_shared_mlp.argtypes = [P, P, P, P, I, I, P, I, P, I]
        lib.oracle_max_threads.argtypes = []
        for f in (lib.oracle_router_logprobs, lib.oracle_topk_from_logprobs, lib.oracle_schedule,
                  lib.oracle_expert_fwd_token_centric, lib.oracle_expert_fwd_expert_centric,
                  lib.oracle_max_threads):
            f.restype = ctypes.c_int
        _lib = lib
    return _lib


def _p(a: np.ndarray | None):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=dtype)


def _check(rc: int, what: str) -> None:
    if rc != 0:
        raise ValueError(f"{what} failed with code {rc}")


def max_threads() -> int:
    return int(_load().oracle_max_threads())


def router_logprobs(x, W_r, W_c, nthreads: int = 0):
    """p_r = LogSoftmax(x W_r^T), p_c = LogSoftmax(x W_c^T): fp64, rounded to fp32."""
    x, W_r, W_c = _c(x, np.uint16), _c(W_r, np.uint16), _c(W_c, np.uint16)
    L, d = x.shape
    N_r, N_c = W_r.shape[0], W_c.shape[0]
    assert W_r.shape[1] == d and W_c.shape[1] == d
    p_r = np.empty((L, N_r), np.float32)
    p_c = np.empty((L, N_c), np.float32)
    _check(_load().oracle_router_logprobs(_p(x), _p(W_r), _p(W_c), L, d, N_r, N_c,
                                          _p(p_r), _p(p_c), nthreads), "router_logprobs")
    return p_r, p_c


def topk_from_logprobs(p_r, p_c, K: int, nthreads: int = 0):
    """Exact global top-K over S_ij = fl32(p_r[i] + p_c[j]) and softmax gates."""
    p_r, p_c = _c(p_r, np.float32), _c(p_c, np.float32)
    L, N_r = p_r.shape
    N_c = p_c.shape[1]
    idx = np.empty((L, K), np.int32)
    score = np.empty((L, K), np.float32)
    gate = np.empty((L, K), np.float32)
    _check(_load().oracle_topk_from_logprobs(_p(p_r), _p(p_c), L, N_r, N_c, K,
                                             _p(idx), _p(score), _p(gate), nthreads),
           "topk_from_logprobs")
    return idx, score, gate


def schedule(idx, gate, N: int, B: int):
    """Expert-centric task order (group, token, expert) and group bookkeeping."""
    idx, gate = _c(idx, np.int32), _c(gate, np.float32)
    L, K = idx.shape
    M = L * K
    G = (N + B - 1) // B
    out = dict(
        task_token=np.empty(M, np.int32), task_expert=np.empty(M, np.int32),
        task_gate=np.empty(M, np.float32), group_offsets=np.empty(G + 1, np.int32),
        group_counts=np.empty(G, np.int32), active_groups=np.full(G, -1, np.int32),
        num_active=np.zeros(1, np.int32), num_distinct=np.zeros(1, np.int32))
    _check(_load().oracle_schedule(_p(idx), _p(gate), L, K, N, B, _p(out["task_token"]),
                                   _p(out["task_expert"]), _p(out["task_gate"]),
                                   _p(out["group_offsets"]), _p(out["group_counts"]),
                                   _p(out["active_groups"]), _p(out["num_active"]),
                                   _p(out["num_distinct"])), "schedule")
    out["num_active"] = int(out["num_active"][0])
    out["num_distinct"] = int(out["num_distinct"][0])
    return out


def expert_fwd_token_centric(x, W, V, idx, gate, tokens=None, nthreads: int = 0):
    """fp64 y rows for the given tokens (all tokens if None), token by token."""
    x, W, V = _c(x, np.uint16), _c(W, np.uint16), _c(V, np.uint16)
    idx, gate = _c(idx, np.int32), _c(gate, np.float32)
    d = x.shape[1]
    K = idx.shape[1]
    if tokens is None:
        n = x.shape[0]
        tok = None
    else:
        tok = _c(tokens, np.int32)
        n = tok.shape[0]
    y = np.empty((n, d), np.float64)
    _check(_load().oracle_expert_fwd_token_centric(_p(x), _p(W), _p(V), d, K, _p(idx), _p(gate),
                                                   _p(tok), n, _p(y), nthreads),
           "expert_fwd_token_centric")
    return y


def shared_mlp(x, W_g, W_u, W_d, tokens=None, nthreads: int = 0):
    """fp64 MLP(x) = (SiLU(x W_g^T) * (x W_u^T)) W_d^T for the given tokens
    (all if None).  W_g, W_u: [F, d]; W_d: [d, F]; bf16 bit patterns."""
    x, W_g, W_u, W_d = (_c(a, np.uint16) for a in (x, W_g, W_u, W_d))
    d = x.shape[1]
    F = W_g.shape[0]
    if W_g.shape != (F, d) or W_u.shape != (F, d) or W_d.shape != (d, F):
        raise ValueError("shared_mlp: W_g, W_u must be [F, d] and W_d [d, F]")
    if tokens is None:
        n = x.shape[0]
        tok = None
    else:
        tok = _c(tokens, np.int32)
        n = tok.shape[0]
    out = np.empty((n, d), np.float64)
    _check(_load().oracle_shared_mlp(_p(x), _p(W_g), _p(W_u), _p(W_d), d, F, _p(tok), n, _p(out),
                                     nthreads), "shared_mlp")
    return out


def expert_fwd_expert_centric(x, W, V, sched, B: int):
    """fp64 y from a schedule, group by group (dense G_q per group)."""
    x, W, V = _c(x, np.uint16), _c(W, np.uint16), _c(V, np.uint16)
    L, d = x.shape
    N = W.shape[0]
    y = np.empty((L, d), np.float64)
    _check(_load().oracle_expert_fwd_expert_centric(
        _p(x), _p(W), _p(V), L, d, N, B, _p(_c(sched["task_token"], np.int32)),
        _p(_c(sched["task_expert"], np.int32)), _p(_c(sched["task_gate"], np.float32)),
        _p(_c(sched["group_offsets"], np.int32)), _p(_c(sched["active_groups"], np.int32)),
        int(sched["num_active"]), _p(y)), "expert_fwd_expert_centric")
    return y


def routed_fwd(x, W, V, W_r, W_c, K: int, B: int, tokens=None, nthreads: int = 0):
    """Whole routed branch for the given tokens: router, top-K, gates, y (fp64).

    The schedule does not change y (it is a reordering of the same sum), so the
    per-token rows are computed token-centrically.
    """
    x = _c(x, np.uint16)
    xs = x if tokens is None else x[_c(tokens, np.int64)]
    p_r, p_c = router_logprobs(xs, W_r, W_c, nthreads)
    idx, score, gate = topk_from_logprobs(p_r, p_c, K, nthreads)
    y = expert_fwd_token_centric(xs, W, V, idx, gate, None, nthreads)
    return dict(p_r=p_r, p_c=p_c, idx=idx, score=score, gate=gate, y=y)


# ------------------------------------------------------------------ backward
def expert_bwd(x, W, V, idx, gate, dy):
    """Backward of the expert part with the routing fixed (fp64): returns
    dx [L, d], dW and dV [rows of W, d], dgate [L, K].  W / V may be the
    compacted rows the tokens use, idx then holding row numbers."""
    x, W, V = _c(x, np.uint16), _c(W, np.uint16), _c(V, np.uint16)
    idx, gate, dy = _c(idx, np.int32), _c(gate, np.float32), _c(dy, np.float32)
    L, d = x.shape
    K = idx.shape[1]
    rows = W.shape[0]
    out = dict(dx=np.empty((L, d)), dW=np.empty((rows, d)), dV=np.empty((rows, d)),
               dgate=np.empty((L, K)))
    _check(_load().oracle_expert_bwd(_p(x), _p(W), _p(V), L, d, K, rows, _p(idx), _p(gate),
                                     _p(dy), _p(out["dx"]), _p(out["dW"]), _p(out["dV"]),
                                     _p(out["dgate"])), "expert_bwd")
    return out


def router_bwd(x, W_r, W_c, p_r, p_c, idx, gate, dgate, dx=None):
    """Backward of the router given dgate (fp64): returns dx (added to the
    given dx if any), dW_r [N_r, d], dW_c [N_c, d]."""
    x, W_r, W_c = _c(x, np.uint16), _c(W_r, np.uint16), _c(W_c, np.uint16)
    p_r, p_c = _c(p_r, np.float32), _c(p_c, np.float32)
    idx, gate, dgate = _c(idx, np.int32), _c(gate, np.float32), _c(dgate, np.float64)
    L, d = x.shape
    N_r, N_c = W_r.shape[0], W_c.shape[0]
    K = idx.shape[1]
    dx = np.zeros((L, d)) if dx is None else _c(dx, np.float64).copy()
    dW_r, dW_c = np.empty((N_r, d)), np.empty((N_c, d))
    _check(_load().oracle_router_bwd(_p(x), _p(W_r), _p(W_c), L, d, N_r, N_c, K, _p(p_r), _p(p_c),
                                     _p(idx), _p(gate), _p(dgate), _p(dx), _p(dW_r), _p(dW_c)),
           "router_bwd")
    return dict(dx=dx, dW_r=dW_r, dW_c=dW_c)


def routed_bwd(x, W, V, W_r, W_c, p_r, p_c, idx, gate, dy):
    """Whole routed-branch backward with the forward's routing fixed (fp64)."""
    e = expert_bwd(x, W, V, idx, gate, dy)
    r = router_bwd(x, W_r, W_c, p_r, p_c, idx, gate, e["dgate"], dx=e["dx"])
    return dict(dx=r["dx"], dW=e["dW"], dV=e["dV"], dW_r=r["dW_r"], dW_c=r["dW_c"],
                dgate=e["dgate"])
