"""The C-ABI library on the host: it loads, exports what include/omni.h
declares, sizes workspaces and rejects bad arguments before touching a GPU."""
import ctypes
import os
import re

import pytest

import atomic_expert_layer_b200 as omni
from atomic_expert_layer_b200 import _lib, build, configs

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "omni.h")


@pytest.fixture(scope="module")
def lib():
    build.build()
    return _lib.load()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(omni_[a-z_]+)\s*\(", src)))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for n in ("omni_router_topk", "omni_schedule", "omni_grouped_expert_fwd", "omni_routed_fwd",
              "omni_workspace_size", "omni_get_device_status"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
        assert name in _lib.SIGNATURES, f"binding lacks {name}"


def test_version_and_strings(lib):
    assert lib.omni_version() == 1
    assert lib.omni_status_string(-3) == b"OMNI_ERR_WORKSPACE"
    assert lib.omni_device_status_string(2) == b"OMNI_DEV_WAIT_TIMEOUT"


def test_workspace_sizes(lib):
    h = configs.HEADLINE
    full = omni.omni_workspace_size(h.L, h.d, h.N_r, h.N_c, h.K, h.B)
    assert full > 0 and full % 256 == 0
    r = omni.omni_router_workspace_size(h.L, h.N_r, h.N_c, h.K)
    s = omni.omni_schedule_workspace_size(h.L, h.K, h.N, h.B)
    e = omni.omni_expert_workspace_size(h.L, h.d, h.K, h.N, h.B)
    assert 0 < r < full and 0 < s < full and 0 < e < full
    # the scores s_r, s_c dominate the router part
    assert r >= 4 * h.L * (h.N_r + h.N_c)
    assert omni.omni_workspace_size(0, 8, 4, 4, 1, 1) == 0
    assert omni.omni_workspace_size(4, 8, 4, 4, 17, 1) == 0         # K > N
    assert omni.omni_workspace_size(4, 8, 4, 4, 4, 2048) == 0       # B above the limit
    assert omni.omni_workspace_size(4, 8, 9000, 4, 4, 4) == 0       # axis above the limit
    # flags: token order needs no schedule; the tensor-core expert path adds
    # its buffers (gate matrix G fp32 and P bf16 [L, cap], W_D and V_D^T
    # [cap, d] bf16, the compacted task list) when it is forced, and by
    # default only for large stages (L * K * d >= 2^31)
    DENSE, SPARSE, TOKEN = omni.OMNI_EXPERT_DENSE, omni.OMNI_EXPERT_SPARSE, omni.OMNI_TOKEN_ORDER
    fl = lambda c, f: omni.omni_workspace_size_flags(c.L, c.d, c.N_r, c.N_c, c.K, c.B, f)
    assert fl(h, 0) == full
    assert fl(h, SPARSE) == full
    assert fl(h, TOKEN) < full
    thr = max(32, -(-h.L // 96))
    cap = min(4096, -(-(h.M // thr) // 256) * 256)
    assert fl(h, DENSE) >= full + 6 * h.L * cap + 4 * cap * h.d
    z = configs.SKEW
    assert z.M * z.d >= 2 ** 31
    assert fl(z, 0) == fl(z, DENSE) > fl(z, SPARSE)
    assert (omni.omni_expert_workspace_size_flags(h.L, h.d, h.K, h.N, h.B, DENSE) >
            omni.omni_expert_workspace_size(h.L, h.d, h.K, h.N, h.B))
    # shared MLP: the status header plus h [L, F] bf16
    F = configs.mlp_hidden(h.d)
    assert omni.omni_shared_mlp_workspace_size(h.L, h.d, F) == 256 + 2 * h.L * F
    assert omni.omni_shared_mlp_workspace_size(0, h.d, F) == 0
    # backward: the status header, two bitmaps over the N experts, a counter
    # and 256 (token, ds) slots per router row
    words = -(-h.N // 32)
    rows = h.N_r + h.N_c
    assert omni.omni_routed_bwd_workspace_size(h.L, h.d, h.N_r, h.N_c, h.K) == \
        256 + 2 * (-(-4 * words // 256) * 256) + (-(-4 * rows // 256) * 256) + 8 * rows * 256
    assert omni.omni_routed_bwd_workspace_size(h.L, h.d, h.N_r, h.N_c, 0) == 0


def _p(v):
    return ctypes.c_void_p(v)


def test_bad_arguments_rejected_on_host(lib):
    """Every check below returns before any CUDA call (no GPU here)."""
    fake = _p(1 << 20)                      # 16-byte aligned, never dereferenced
    ws_small = 256
    L, d, Nr, Nc, K, B = 4, 256, 4, 4, 2, 2
    # null pointer
    assert lib.omni_routed_fwd(None, fake, fake, fake, fake, L, d, Nr, Nc, K, B, fake, None, None,
                               0, fake, 1 << 30, None) == -1
    # K > N
    assert lib.omni_routed_fwd(fake, fake, fake, fake, fake, L, d, Nr, Nc, 17, B, fake, None,
                               None, 0, fake, 1 << 30, None) == -1
    # d not a multiple of 256 for the expert stage
    assert lib.omni_routed_fwd(fake, fake, fake, fake, fake, L, 264, Nr, Nc, K, B, fake, None,
                               None, 0, fake, 1 << 30, None) == -2
    # workspace too small
    assert lib.omni_routed_fwd(fake, fake, fake, fake, fake, L, d, Nr, Nc, K, B, fake, None, None,
                               0, fake, ws_small, None) == -3
    # misaligned bf16 pointer
    assert lib.omni_routed_fwd(_p((1 << 20) + 2), fake, fake, fake, fake, L, d, Nr, Nc, K, B,
                               fake, None, None, 0, fake, 1 << 30, None) == -1
    # misaligned workspace
    assert lib.omni_schedule(fake, fake, L, K, 16, B, fake, fake, fake, fake, fake, fake, fake,
                             fake, _p((1 << 20) + 64), 1 << 30, None) == -1
    # N <= 0
    assert lib.omni_grouped_expert_fwd(fake, fake, fake, L, d, K, 0, B, fake, fake, fake, fake,
                                       fake, fake, fake, 0, fake, 1 << 30, None) == -1
    # router: d must be a multiple of 8
    assert lib.omni_router_topk(fake, fake, fake, L, 12, Nr, Nc, K, fake, fake, fake, fake, fake,
                                0, fake, 1 << 30, None) == -2
    # blockwise selection: only on caller log-probabilities, and K <= (N_r + N_c) / 4
    lp_bw = 1 | 8                           # OMNI_ROUTER_LOGPROBS_IN | OMNI_TOPK_BLOCKWISE
    assert lib.omni_router_topk(fake, fake, fake, L, d, Nr, Nc, K, fake, fake, fake, fake, fake,
                                8, fake, 1 << 30, None) == -2
    assert lib.omni_router_topk(None, None, None, L, 0, 8, 8, 16, fake, fake, fake, fake, fake,
                                lp_bw, fake, 1 << 30, None) == -2
    # ... and not through the whole forward
    assert lib.omni_routed_fwd(fake, fake, fake, fake, fake, L, d, Nr, Nc, K, B, fake, None,
                               None, 8, fake, 1 << 30, None) == -2
    # backward: null gradient buffer, unknown flag, d off the 256 grid, tiny workspace
    assert lib.omni_routed_bwd(fake, fake, fake, fake, fake, L, d, Nr, Nc, K, fake, fake, fake,
                               fake, None, fake, fake, fake, 0, fake, 256, None) == -1
    assert lib.omni_routed_bwd(fake, fake, fake, fake, fake, L, d, Nr, Nc, K, fake, fake, fake,
                               fake, fake, fake, fake, fake, 1, fake, 256, None) == -1
    assert lib.omni_routed_bwd(fake, fake, fake, fake, fake, L, 264, Nr, Nc, K, fake, fake, fake,
                               fake, fake, fake, fake, fake, 0, fake, 256, None) == -2
    assert lib.omni_routed_bwd(fake, fake, fake, fake, fake, L, d, Nr, Nc, K, fake, fake, fake,
                               fake, fake, fake, fake, fake, 0, fake, 64, None) == -3
    # shared MLP: null weight, unknown flag, d or F off the 64 grid, misaligned y, small workspace
    mlp_ws = omni.omni_shared_mlp_workspace_size(L, d, 128)
    assert lib.omni_shared_mlp_fwd(fake, None, fake, fake, L, d, 128, fake, 0, fake, mlp_ws,
                                   None) == -1
    assert lib.omni_shared_mlp_fwd(fake, fake, fake, fake, L, d, 128, fake, 4, fake, mlp_ws,
                                   None) == -1
    assert lib.omni_shared_mlp_fwd(fake, fake, fake, fake, L, 96, 128, fake, 0, fake, mlp_ws,
                                   None) == -2
    assert lib.omni_shared_mlp_fwd(fake, fake, fake, fake, L, d, 96, fake, 0, fake, mlp_ws,
                                   None) == -2
    assert lib.omni_shared_mlp_fwd(fake, fake, fake, fake, L, d, 128, _p((1 << 20) + 4), 0, fake,
                                   mlp_ws, None) == -1
    assert lib.omni_shared_mlp_fwd(fake, fake, fake, fake, L, d, 128, fake, 2, fake, mlp_ws - 1,
                                   None) == -3
    # status query needs a workspace
    out = ctypes.c_int(7)
    assert lib.omni_get_device_status(None, 0, None, ctypes.byref(out)) == -1


def test_binding_refuses_cpu_tensors(lib):
    import torch
    x = torch.zeros(4, 256, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        _lib._ptr(x)
