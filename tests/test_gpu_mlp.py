"""GPU parity of the shared dense MLP (omni_shared_mlp_fwd) and of the whole
layer y = routed(x) + MLP(x), through the C ABI, against the CPU oracle.

Tolerance: the GPU holds h = SiLU(x W_g^T) * (x W_u^T) in bf16 (the operand
type of the second product), a relative rounding of at most 2^-9 per hidden
unit; with fp32 accumulation elsewhere that gives a rel-L2 error near
2^-9 / sqrt(3) ~ 1.1e-3 on y, inside the y bar shared with the routed branch
(max-abs 2e-2, rel-L2 5e-3) at these inits (|y| ~ 0.5).
"""
import numpy as np
import pytest
import torch

import oracle
import atomic_expert_layer_b200 as omni
from atomic_expert_layer_b200 import configs, inputs

from _parity import check_y, host

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    omni.load()


def _x(L, d, seed):
    cfg = configs.LayerConfig("mlp", L, d, 1, 1, 1, 1)
    return inputs.make_inputs(cfg, DEV, seed=seed, with_experts=False)["x"]


def _rows(L, n):
    """n sampled token rows, always including the first and the last."""
    if L <= n:
        return np.arange(L, dtype=np.int32)
    rng = np.random.default_rng(L)
    mid = rng.choice(np.arange(1, L - 1), size=n - 2, replace=False)
    return np.sort(np.concatenate([[0, L - 1], mid])).astype(np.int32)


@pytest.mark.parametrize("L,d,F,rows", [
    (256, 256, configs.mlp_hidden(256), None),      # tiny layer width, half-filled last hidden tile
    (300, 768, configs.mlp_hidden(768), None),      # ragged token tile, three output tiles
    (77, 320, 192, None),                           # one token tile; second output box past d
    (1, 64, 64, None),                              # smallest shape
    (4096, 1024, configs.mlp_hidden(1024), 64),     # headline width, sampled rows
    (1000, 2048, configs.mlp_hidden(2048), 24),     # widest layer, sampled rows
])
def test_shared_mlp_against_oracle(L, d, F, rows):
    x = _x(L, d, seed=L + d)
    w = inputs.make_mlp_weights(d, F, DEV, seed=d + F)
    ws = omni.shared_mlp_workspace(L, d, F)
    y = omni.shared_mlp_fwd(x, w["W_g"], w["W_u"], w["W_d"], ws=ws)
    assert omni.omni_get_device_status(ws) == 0
    tok = _rows(L, rows) if rows else None
    ref = oracle.shared_mlp(host(x), host(w["W_g"]), host(w["W_u"]), host(w["W_d"]), tokens=tok)
    got = host(y) if tok is None else host(y)[tok]
    assert np.abs(ref).max() > 0.1                  # not vacuous
    check_y(got, ref, "mlp")


def test_shared_mlp_accumulates_and_is_deterministic():
    L, d, F = 200, 512, 384
    x = _x(L, d, seed=5)
    w = inputs.make_mlp_weights(d, F, DEV, seed=6)
    y = omni.shared_mlp_fwd(x, w["W_g"], w["W_u"], w["W_d"])
    again = omni.shared_mlp_fwd(x, w["W_g"], w["W_u"], w["W_d"])
    assert torch.equal(y, again)                     # one tile per element, fixed order
    base = torch.randn(L, d, device=DEV)
    acc = base.clone()
    omni.shared_mlp_fwd(x, w["W_g"], w["W_u"], w["W_d"], y=acc, accumulate=True)
    assert torch.equal(acc, base + y)                # one fp32 add per element


def test_layer_fwd_is_routed_plus_mlp():
    cfg = configs.TINY
    t = inputs.make_inputs(cfg, DEV, seed=2)
    F = configs.mlp_hidden(cfg.d)
    w = inputs.make_mlp_weights(cfg.d, F, DEV, seed=2)
    _, idx, gate = omni.routed_fwd(t["x"], t["W"], t["V"], t["W_r"], t["W_c"], cfg.K, cfg.B,
                                   want_routing=True)
    y = omni.layer_fwd(t["x"], t["W"], t["V"], t["W_r"], t["W_c"], w["W_g"], w["W_u"], w["W_d"],
                       cfg.K, cfg.B)
    u = {k: host(v) for k, v in t.items()}
    ref = (oracle.expert_fwd_token_centric(u["x"], u["W"], u["V"], host(idx), host(gate))
           + oracle.shared_mlp(u["x"], host(w["W_g"]), host(w["W_u"]), host(w["W_d"])))
    check_y(host(y), ref, "layer")
