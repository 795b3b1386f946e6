"""B200 (sm_100a) routed-branch forward of an OmniMoE layer.

The computation lives in libomni.so (hand-written CUDA, C ABI in
include/omni.h).  This package only loads it and marshals torch tensors:
  - ``omni_*`` functions mirror the C entry points argument for argument;
  - ``router_topk``, ``schedule``, ``grouped_expert_fwd``, ``routed_fwd``,
    ``routed_bwd``, ``shared_mlp_fwd`` and ``layer_fwd`` allocate the output
    tensors and a workspace, then call them.
"""
from __future__ import annotations

import torch

from ._lib import (OMNI_ROUTER_LOGPROBS_IN, OMNI_TOKEN_ORDER, OMNI_TOPK_BLOCKWISE,  # noqa: F401
                   OMNI_Y_ACCUMULATE, OMNI_EXPERT_DENSE, OMNI_EXPERT_SPARSE,
                   omni_workspace_size_flags, omni_expert_workspace_size_flags,
                   OmniError, load,
                   expert_workspace, omni_expert_workspace_size, omni_get_device_status,
                   omni_grouped_expert_fwd, omni_grouped_expert_fwd_noalloc,
                   omni_noalloc_get_device_status, omni_routed_bwd,
                   omni_routed_bwd_workspace_size, omni_routed_fwd,
                   omni_router_topk,
                   omni_router_workspace_size, omni_schedule, omni_schedule_workspace_size,
                   omni_selftest_wait_timeout, omni_shared_mlp_fwd,
                   omni_shared_mlp_workspace_size, shared_mlp_workspace,
                   omni_workspace_size, router_workspace, schedule_workspace, workspace)

__all__ = [
    "load", "OmniError", "OMNI_ROUTER_LOGPROBS_IN", "OMNI_Y_ACCUMULATE", "OMNI_TOKEN_ORDER", "OMNI_TOPK_BLOCKWISE",
    "OMNI_EXPERT_DENSE", "OMNI_EXPERT_SPARSE", "omni_workspace_size_flags",
    "omni_expert_workspace_size_flags",
    "omni_workspace_size", "omni_router_topk", "omni_schedule", "omni_grouped_expert_fwd",
    "omni_routed_fwd", "omni_get_device_status", "workspace", "omni_grouped_expert_fwd_noalloc",
    "omni_noalloc_get_device_status",
    "router_topk", "schedule", "grouped_expert_fwd", "routed_fwd", "omni_routed_bwd", "routed_bwd",
    "omni_routed_bwd_workspace_size",
    "omni_shared_mlp_workspace_size", "omni_shared_mlp_fwd", "shared_mlp_fwd", "layer_fwd",
]


def router_topk(x, W_r, W_c, K, ws=None, p_r=None, p_c=None, logprobs_in=False,
                blockwise=False, stream=None):
    """Top-K experts per token.  With logprobs_in, p_r / p_c are inputs and
    x may be None (then pass W_r / W_c as None too).  blockwise (with
    logprobs_in) selects with the blockwise grid scan instead of the
    row / column pruning; the result is the same."""
    if logprobs_in:
        L, N_r = p_r.shape
        N_c = p_c.shape[1]
        d = 0
        dev = p_r.device
    else:
        L, d = x.shape
        N_r, N_c = W_r.shape[0], W_c.shape[0]
        dev = x.device
        p_r = torch.empty((L, N_r), dtype=torch.float32, device=dev) if p_r is None else p_r
        p_c = torch.empty((L, N_c), dtype=torch.float32, device=dev) if p_c is None else p_c
    idx = torch.empty((L, K), dtype=torch.int32, device=dev)
    score = torch.empty((L, K), dtype=torch.float32, device=dev)
    gate = torch.empty((L, K), dtype=torch.float32, device=dev)
    ws = router_workspace(L, N_r, N_c, K, dev) if ws is None else ws
    flags = (OMNI_ROUTER_LOGPROBS_IN if logprobs_in else 0) | (OMNI_TOPK_BLOCKWISE if blockwise else 0)
    omni_router_topk(x, W_r, W_c, L, d, N_r, N_c, K, p_r, p_c, idx, score, gate, flags, ws, stream)
    return dict(p_r=p_r, p_c=p_c, idx=idx, score=score, gate=gate)


def schedule(idx, gate, N, B, ws=None, stream=None):
    L, K = idx.shape
    dev = idx.device
    M, G = L * K, (N + B - 1) // B
    out = dict(task_token=torch.empty(M, dtype=torch.int32, device=dev),
               task_expert=torch.empty(M, dtype=torch.int32, device=dev),
               task_gate=torch.empty(M, dtype=torch.float32, device=dev),
               group_offsets=torch.empty(G + 1, dtype=torch.int32, device=dev),
               group_counts=torch.empty(G, dtype=torch.int32, device=dev),
               active_groups=torch.empty(G, dtype=torch.int32, device=dev),
               num_active=torch.empty(1, dtype=torch.int32, device=dev),
               num_distinct=torch.empty(1, dtype=torch.int32, device=dev))
    ws = schedule_workspace(L, K, N, B, dev) if ws is None else ws
    omni_schedule(idx, gate, L, K, N, B, out["task_token"], out["task_expert"], out["task_gate"],
                  out["group_offsets"], out["group_counts"], out["active_groups"],
                  out["num_active"], out["num_distinct"], ws, stream)
    return out


_EXPERT_MODE = {"auto": 0, "dense": OMNI_EXPERT_DENSE, "sparse": OMNI_EXPERT_SPARSE}


def grouped_expert_fwd(x, W, V, sched, K, B, y=None, accumulate=False, ws=None, stream=None,
                       expert_mode="auto"):
    """expert_mode: "auto" (the library's size rule), "dense" (always try the
    tensor-core tiles for dense experts) or "sparse" (task by task only)."""
    L, d = x.shape
    N = W.shape[0]
    mode = _EXPERT_MODE[expert_mode]
    y = torch.empty((L, d), dtype=torch.float32, device=x.device) if y is None else y
    ws = expert_workspace(L, d, K, N, B, x.device, mode) if ws is None else ws
    omni_grouped_expert_fwd(x, W, V, L, d, K, N, B, sched["task_token"], sched["task_expert"],
                            sched["task_gate"], sched["group_offsets"], sched["active_groups"],
                            sched["num_active"], y, (OMNI_Y_ACCUMULATE if accumulate else 0) | mode,
                            ws, stream)
    return y


def routed_fwd(x, W, V, W_r, W_c, K, B, y=None, ws=None, want_routing=False, accumulate=False,
               token_order=False, stream=None, expert_mode="auto"):
    L, d = x.shape
    N_r, N_c = W_r.shape[0], W_c.shape[0]
    mode = _EXPERT_MODE[expert_mode]
    flags = (OMNI_Y_ACCUMULATE if accumulate else 0) | (OMNI_TOKEN_ORDER if token_order else 0) | mode
    y = torch.empty((L, d), dtype=torch.float32, device=x.device) if y is None else y
    ws = workspace(L, d, N_r, N_c, K, B, x.device, flags) if ws is None else ws
    idx = gate = None
    if want_routing:
        idx = torch.empty((L, K), dtype=torch.int32, device=x.device)
        gate = torch.empty((L, K), dtype=torch.float32, device=x.device)
    omni_routed_fwd(x, W, V, W_r, W_c, L, d, N_r, N_c, K, B, y, idx, gate, flags, ws, stream)
    return (y, idx, gate) if want_routing else y


def routed_bwd(x, W, V, W_r, W_c, idx, gate, dy, dW=None, dV=None, dW_r=None, dW_c=None,
               ws=None, stream=None):
    """Backward of the routed branch with the forward's routing (idx, gate)
    fixed.  Returns dx (new) and the weight gradients, accumulated into the
    given fp32 buffers (new zeroed ones if None)."""
    L, d = x.shape
    N_r, N_c = W_r.shape[0], W_c.shape[0]
    K = idx.shape[1]
    dev = x.device
    f32 = dict(dtype=torch.float32, device=dev)
    dx = torch.empty((L, d), **f32)
    dW = torch.zeros(W.shape, **f32) if dW is None else dW
    dV = torch.zeros(V.shape, **f32) if dV is None else dV
    dW_r = torch.zeros(W_r.shape, **f32) if dW_r is None else dW_r
    dW_c = torch.zeros(W_c.shape, **f32) if dW_c is None else dW_c
    if ws is None:
        ws = torch.empty(omni_routed_bwd_workspace_size(L, d, N_r, N_c, K), dtype=torch.uint8,
                         device=dev)
    omni_routed_bwd(x, W, V, W_r, W_c, L, d, N_r, N_c, K, idx, gate, dy, dx, dW, dV, dW_r, dW_c,
                    0, ws, stream)
    return dict(dx=dx, dW=dW, dV=dV, dW_r=dW_r, dW_c=dW_c)


def shared_mlp_fwd(x, W_g, W_u, W_d, y=None, accumulate=False, ws=None, stream=None):
    """MLP(x) = (SiLU(x W_g^T) * (x W_u^T)) W_d^T into y (fp32), or added to
    it with accumulate=True.  W_g, W_u: [F, d]; W_d: [d, F]; all bf16."""
    L, d = x.shape
    F = W_g.shape[0]
    y = torch.empty((L, d), dtype=torch.float32, device=x.device) if y is None else y
    ws = shared_mlp_workspace(L, d, F, x.device) if ws is None else ws
    omni_shared_mlp_fwd(x, W_g, W_u, W_d, L, d, F, y, OMNI_Y_ACCUMULATE if accumulate else 0, ws,
                        stream)
    return y


def layer_fwd(x, W, V, W_r, W_c, W_g, W_u, W_d, K, B, y=None, ws=None, mlp_ws=None,
              stream=None):
    """The whole layer: y = routed(x) + MLP(x), as omni_routed_fwd followed by
    omni_shared_mlp_fwd with OMNI_Y_ACCUMULATE on the same stream."""
    y = routed_fwd(x, W, V, W_r, W_c, K, B, y=y, ws=ws, stream=stream)
    return shared_mlp_fwd(x, W_g, W_u, W_d, y=y, accumulate=True, ws=mlp_ws, stream=stream)
