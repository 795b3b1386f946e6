"""ctypes binding of libomni.so -- argument marshalling only.

Every function here forwards to the C entry point of the same name declared
in include/omni.h.  Tensors are torch CUDA tensors; their data pointers and
the current CUDA stream are passed through.  Nothing is computed in Python,
and there is no fallback: if libomni.so is missing or no GPU is present,
calls raise.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libomni.so")

OMNI_ROUTER_LOGPROBS_IN = 1
OMNI_Y_ACCUMULATE = 2
OMNI_TOKEN_ORDER = 4
OMNI_TOPK_BLOCKWISE = 8
OMNI_EXPERT_DENSE = 16
OMNI_EXPERT_SPARSE = 32

STATUS = {0: "OMNI_OK", -1: "OMNI_ERR_INVALID_ARG", -2: "OMNI_ERR_UNSUPPORTED",
          -3: "OMNI_ERR_WORKSPACE", -4: "OMNI_ERR_CUDA", -5: "OMNI_ERR_DEVICE"}

# exported symbols and their ctypes signatures (kept in step with include/omni.h)
_P, _I, _U, _Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_uint, ctypes.c_size_t
SIGNATURES = {
    "omni_version": ([], _I),
    "omni_status_string": ([_I], ctypes.c_char_p),
    "omni_device_status_string": ([_I], ctypes.c_char_p),
    "omni_workspace_size": ([_I, _I, _I, _I, _I, _I], _Z),
    "omni_workspace_size_flags": ([_I, _I, _I, _I, _I, _I, _U], _Z),
    "omni_router_workspace_size": ([_I, _I, _I, _I], _Z),
    "omni_schedule_workspace_size": ([_I, _I, _I, _I], _Z),
    "omni_expert_workspace_size": ([_I, _I, _I, _I, _I], _Z),
    "omni_expert_workspace_size_flags": ([_I, _I, _I, _I, _I, _U], _Z),
    "omni_router_topk": ([_P, _P, _P, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P, _U, _P, _Z, _P], _I),
    "omni_schedule": ([_P, _P, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P, _P, _P, _P, _Z, _P], _I),
    "omni_grouped_expert_fwd": ([_P, _P, _P, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P, _P,
                                 _U, _P, _Z, _P], _I),
    "omni_routed_fwd": ([_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _P, _P, _P, _U, _P, _Z, _P],
                        _I),
    "omni_routed_bwd_workspace_size": ([_I, _I, _I, _I, _I], _Z),
    "omni_routed_bwd": ([_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P, _P, _P,
                         _U, _P, _Z, _P], _I),
    "omni_shared_mlp_workspace_size": ([_I, _I, _I], _Z),
    "omni_shared_mlp_fwd": ([_P, _P, _P, _P, _I, _I, _I, _P, _U, _P, _Z, _P], _I),
    "omni_get_device_status": ([_P, _Z, _P, ctypes.POINTER(ctypes.c_int)], _I),
    "omni_selftest_wait_timeout": ([_P, _Z, _I, _P], _I),
    "omni_grouped_expert_fwd_noalloc": ([_P, _P, _P, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P,
                                         _P, _U, _P], _I),
    "omni_noalloc_get_device_status": ([_P, ctypes.POINTER(ctypes.c_int)], _I),
}

_lib = None


class OmniError(RuntimeError):
    def __init__(self, fn: str, code: int):
        super().__init__(f"{fn} returned {STATUS.get(code, code)}")
        self.code = code


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libomni.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(path):
            raise RuntimeError(f"{path} is missing: build it with "
                               "`python -m atomic_expert_layer_b200.build`")
        lib = ctypes.CDLL(path)
        for name, (args, res) in SIGNATURES.items():
            f = getattr(lib, name)
            f.argtypes = args
            f.restype = res
        _lib = lib
    return _lib


def _ptr(t: torch.Tensor | None):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("libomni takes CUDA tensors")
    if not t.is_contiguous():
        raise ValueError("libomni takes contiguous tensors")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _check(name: str, rc: int) -> None:
    if rc != 0:
        raise OmniError(name, rc)


def _u16(t: torch.Tensor) -> torch.Tensor:
    if t.dtype not in (torch.bfloat16, torch.int16, torch.uint16):
        raise ValueError("bf16 tensors expected")
    return t


def omni_workspace_size(L, d, N_r, N_c, K, B) -> int:
    return int(load().omni_workspace_size(L, d, N_r, N_c, K, B))


def omni_workspace_size_flags(L, d, N_r, N_c, K, B, flags) -> int:
    return int(load().omni_workspace_size_flags(L, d, N_r, N_c, K, B, flags))


def omni_router_workspace_size(L, N_r, N_c, K) -> int:
    return int(load().omni_router_workspace_size(L, N_r, N_c, K))


def omni_schedule_workspace_size(L, K, N, B) -> int:
    return int(load().omni_schedule_workspace_size(L, K, N, B))


def omni_expert_workspace_size(L, d, K, N, B) -> int:
    return int(load().omni_expert_workspace_size(L, d, K, N, B))


def omni_expert_workspace_size_flags(L, d, K, N, B, flags) -> int:
    return int(load().omni_expert_workspace_size_flags(L, d, K, N, B, flags))


def _alloc(n: int, device) -> torch.Tensor:
    if n == 0:
        raise ValueError("invalid sizes")
    return torch.empty(n, dtype=torch.uint8, device=device)


def workspace(L, d, N_r, N_c, K, B, device="cuda", flags=0) -> torch.Tensor:
    """Workspace for omni_routed_fwd (and any of the stage calls) at these
    sizes, for calls made with `flags`."""
    return _alloc(omni_workspace_size_flags(L, d, N_r, N_c, K, B, flags), device)


def router_workspace(L, N_r, N_c, K, device="cuda") -> torch.Tensor:
    return _alloc(omni_router_workspace_size(L, N_r, N_c, K), device)


def schedule_workspace(L, K, N, B, device="cuda") -> torch.Tensor:
    return _alloc(omni_schedule_workspace_size(L, K, N, B), device)


def expert_workspace(L, d, K, N, B, device="cuda", flags=0) -> torch.Tensor:
    return _alloc(omni_expert_workspace_size_flags(L, d, K, N, B, flags), device)


def omni_router_topk(x, W_r, W_c, L, d, N_r, N_c, K, p_r, p_c, idx, score, gate, flags, ws,
                     stream=None):
    rc = load().omni_router_topk(_ptr(x), _ptr(W_r), _ptr(W_c), L, d, N_r, N_c, K, _ptr(p_r),
                                 _ptr(p_c), _ptr(idx), _ptr(score), _ptr(gate), flags, _ptr(ws),
                                 ws.numel(), _stream(stream))
    _check("omni_router_topk", rc)


def omni_schedule(idx, gate, L, K, N, B, task_token, task_expert, task_gate, group_offsets,
                  group_counts, active_groups, num_active, num_distinct, ws, stream=None):
    rc = load().omni_schedule(_ptr(idx), _ptr(gate), L, K, N, B, _ptr(task_token),
                              _ptr(task_expert), _ptr(task_gate), _ptr(group_offsets),
                              _ptr(group_counts), _ptr(active_groups), _ptr(num_active),
                              _ptr(num_distinct), _ptr(ws), ws.numel(), _stream(stream))
    _check("omni_schedule", rc)


def omni_grouped_expert_fwd(x, W, V, L, d, K, N, B, task_token, task_expert, task_gate,
                            group_offsets, active_groups, num_active, y, flags, ws, stream=None):
    rc = load().omni_grouped_expert_fwd(_ptr(x), _ptr(W), _ptr(V), L, d, K, N, B,
                                        _ptr(task_token), _ptr(task_expert), _ptr(task_gate),
                                        _ptr(group_offsets), _ptr(active_groups),
                                        _ptr(num_active), _ptr(y), flags, _ptr(ws), ws.numel(),
                                        _stream(stream))
    _check("omni_grouped_expert_fwd", rc)


def omni_routed_fwd(x, W, V, W_r, W_c, L, d, N_r, N_c, K, B, y, idx_out, gate_out, flags, ws,
                    stream=None):
    rc = load().omni_routed_fwd(_ptr(x), _ptr(W), _ptr(V), _ptr(W_r), _ptr(W_c), L, d, N_r, N_c,
                                K, B, _ptr(y), _ptr(idx_out), _ptr(gate_out), flags, _ptr(ws),
                                ws.numel(), _stream(stream))
    _check("omni_routed_fwd", rc)


def omni_routed_bwd_workspace_size(L, d, N_r, N_c, K) -> int:
    return load().omni_routed_bwd_workspace_size(L, d, N_r, N_c, K)


def omni_routed_bwd(x, W, V, W_r, W_c, L, d, N_r, N_c, K, idx, gate, dy, dx, dW, dV, dW_r, dW_c,
                    flags, ws, stream=None):
    rc = load().omni_routed_bwd(_ptr(x), _ptr(W), _ptr(V), _ptr(W_r), _ptr(W_c), L, d, N_r, N_c,
                                K, _ptr(idx), _ptr(gate), _ptr(dy), _ptr(dx), _ptr(dW), _ptr(dV),
                                _ptr(dW_r), _ptr(dW_c), flags, _ptr(ws), ws.numel(),
                                _stream(stream))
    _check("omni_routed_bwd", rc)


def omni_shared_mlp_workspace_size(L, d, F) -> int:
    return int(load().omni_shared_mlp_workspace_size(L, d, F))


def shared_mlp_workspace(L, d, F, device="cuda") -> torch.Tensor:
    return _alloc(omni_shared_mlp_workspace_size(L, d, F), device)


def omni_shared_mlp_fwd(x, W_g, W_u, W_d, L, d, F, y, flags, ws, stream=None):
    rc = load().omni_shared_mlp_fwd(_ptr(x), _ptr(W_g), _ptr(W_u), _ptr(W_d), L, d, F, _ptr(y),
                                    flags, _ptr(ws), ws.numel(), _stream(stream))
    _check("omni_shared_mlp_fwd", rc)


def omni_get_device_status(ws, stream=None) -> int:
    out = ctypes.c_int(0)
    rc = load().omni_get_device_status(_ptr(ws), ws.numel(), _stream(stream), ctypes.byref(out))
    if rc not in (0, -5):
        raise OmniError("omni_get_device_status", rc)
    return int(out.value)


def omni_selftest_wait_timeout(ws, limit_ms: int, stream=None) -> None:
    rc = load().omni_selftest_wait_timeout(_ptr(ws), ws.numel(), limit_ms, _stream(stream))
    _check("omni_selftest_wait_timeout", rc)


def omni_grouped_expert_fwd_noalloc(x, W, V, L, d, K, N, B, task_token, task_expert, task_gate,
                                    group_offsets, active_groups, num_active, y, flags,
                                    stream=None):
    """The grouped expert call without a workspace (scratch inside the library)."""
    rc = load().omni_grouped_expert_fwd_noalloc(
        _ptr(x), _ptr(W), _ptr(V), L, d, K, N, B, _ptr(task_token), _ptr(task_expert),
        _ptr(task_gate), _ptr(group_offsets), _ptr(active_groups), _ptr(num_active), _ptr(y),
        flags, _stream(stream))
    _check("omni_grouped_expert_fwd_noalloc", rc)


def omni_noalloc_get_device_status(stream=None) -> int:
    """Status word of the no-workspace call's array on the current device
    (synchronises the stream, then clears the word)."""
    out = ctypes.c_int(0)
    rc = load().omni_noalloc_get_device_status(_stream(stream), ctypes.byref(out))
    if rc not in (0, -5):
        raise OmniError("omni_noalloc_get_device_status", rc)
    return int(out.value)
