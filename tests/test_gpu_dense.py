"""GPU parity of the expert stage's tensor-core path (dense experts).

The grouped GEMM of the pages, O_q = (G_q . SiLU(X_q W_q^T)) V_q, runs on the
tensor cores for the experts that at least thr = max(32, ceil(L / 96)) tasks
use, and task by task on the CUDA cores for the rest.  These tests feed
skewed routings (an additive Zipf log-bias on the router, so that a few
experts carry most tasks and hot groups hold thousands of tokens) and check
y element by element against the fp64 oracle on the same routing, with the
tensor-core path forced on ("dense"), forced off ("sparse") and by the
default size rule.  They also check the schedule checks the path performs.
"""
import numpy as np
import pytest
import torch

import oracle
import atomic_expert_layer_b200 as omni
from atomic_expert_layer_b200 import configs, inputs

from _parity import check_routing_near_ties, check_y, host

pytestmark = pytest.mark.gpu

DEV = "cuda"

# hot groups of ~4096 tokens: L = 4096, 128 x 128 grid, K = 32, B = 64
SKEW_4K = configs.LayerConfig("skew_L4096_d512_N16384_K32_B64_zipf", 4096, 512, 128, 128, 32,
                              64, zipf=True)
# ragged token count (not a multiple of the 128-row tile), narrow width
SKEW_RAGGED = configs.LayerConfig("skew_L1000_d256_N4096_K16_B32_zipf", 1000, 256, 64, 64, 16, 32,
                                  zipf=True)
# more dense experts than the column cap (4096): the rest stay task by task
OVER_CAP = configs.LayerConfig("dense_L16384_d256_N10000_K128_B100", 16384, 256, 100, 100, 128,
                               100)


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    omni.load()


def _routing_and_schedule(cfg, seed):
    """Inputs on the GPU, the oracle's routing and schedule on the host."""
    t = inputs.make_inputs(cfg, DEV, seed=seed)
    u = {k: host(v) for k, v in t.items()}
    p_r, p_c = oracle.router_logprobs(u["x"], u["W_r"], u["W_c"])
    idx, _, gate = oracle.topk_from_logprobs(p_r, p_c, cfg.K)
    sched = oracle.schedule(idx, gate, cfg.N, cfg.B)
    s_dev = {k: torch.as_tensor(np.atleast_1d(v).astype(np.float32 if k == "task_gate"
                                                        else np.int32)).to(DEV)
             for k, v in sched.items()}
    return t, u, idx, gate, sched, s_dev


def _dense_stats(idx, L, N):
    """(threshold, number of dense experts, share of tasks on them)."""
    thr = max(32, -(-L // 96))
    use = np.bincount(idx.ravel().astype(np.int64), minlength=N)
    hot = use >= thr
    return thr, int(hot.sum()), float(use[hot].sum() / idx.size)


@pytest.mark.parametrize("cfg", [SKEW_4K, SKEW_RAGGED, OVER_CAP], ids=lambda c: c.name)
def test_dense_expert_stage_on_oracle_schedule(cfg):
    torch.cuda.empty_cache()
    t, u, idx, gate, sched, s_dev = _routing_and_schedule(cfg, seed=3)
    thr, n_dense, share = _dense_stats(idx, cfg.L, cfg.N)
    assert n_dense > 0 and share > 0.3, (thr, n_dense, share)     # the case exercises the tiles
    if cfg is SKEW_4K:
        # the hottest group's tokens are (nearly) all 4096 tokens of the batch
        q = sched["task_expert"] // cfg.B
        hottest = int(np.argmax(np.bincount(q)))
        assert len(np.unique(sched["task_token"][q == hottest])) >= 0.9 * cfg.L
    if cfg is OVER_CAP:
        assert n_dense > 4096                                     # more than the column cap
    y_ref = oracle.expert_fwd_token_centric(u["x"], u["W"], u["V"], idx, gate)
    y_dense = omni.grouped_expert_fwd(t["x"], t["W"], t["V"], s_dev, cfg.K, cfg.B,
                                      expert_mode="dense")
    torch.cuda.synchronize()
    check_y(host(y_dense), y_ref, "dense path")
    y_sparse = omni.grouped_expert_fwd(t["x"], t["W"], t["V"], s_dev, cfg.K, cfg.B,
                                       expert_mode="sparse")
    check_y(host(y_sparse), y_ref, "task-by-task path")
    # accumulate mode adds both paths' parts to what is there
    y0 = torch.full_like(y_dense, 0.25)
    omni.grouped_expert_fwd(t["x"], t["W"], t["V"], s_dev, cfg.K, cfg.B, y=y0, accumulate=True,
                            expert_mode="dense")
    check_y(host(y0), y_ref + 0.25, "dense path, accumulate")
    del t, s_dev
    torch.cuda.empty_cache()


def test_dense_path_without_dense_experts():
    """Forced on a uniform tiny layer no expert reaches the threshold: the
    tiles do no work and every task runs on the CUDA cores."""
    cfg = configs.TINY
    t, u, idx, gate, sched, s_dev = _routing_and_schedule(cfg, seed=1)
    assert _dense_stats(idx, cfg.L, cfg.N)[1] == 0
    ws = omni.expert_workspace(cfg.L, cfg.d, cfg.K, cfg.N, cfg.B, DEV, omni.OMNI_EXPERT_DENSE)
    y = omni.grouped_expert_fwd(t["x"], t["W"], t["V"], s_dev, cfg.K, cfg.B, ws=ws,
                                expert_mode="dense")
    assert omni.omni_get_device_status(ws) == 0
    check_y(host(y), oracle.expert_fwd_token_centric(u["x"], u["W"], u["V"], idx, gate))


def test_routed_fwd_dense_end_to_end():
    """The whole routed branch with the tensor-core path forced: routing under
    the near-tie rule, y on every token against the oracle on the GPU's
    routing, and the same y as the task-by-task path."""
    cfg = SKEW_4K
    t = inputs.make_inputs(cfg, DEV, seed=0)
    u = {k: host(v) for k, v in t.items()}
    ws = omni.workspace(cfg.L, cfg.d, cfg.N_r, cfg.N_c, cfg.K, cfg.B, DEV, omni.OMNI_EXPERT_DENSE)
    y, idx, gate = omni.routed_fwd(t["x"], t["W"], t["V"], t["W_r"], t["W_c"], cfg.K, cfg.B,
                                   ws=ws, want_routing=True, expert_mode="dense")
    assert omni.omni_get_device_status(ws) == 0
    p_r, p_c = oracle.router_logprobs(u["x"], u["W_r"], u["W_c"])
    idx_ref, score_ref, _ = oracle.topk_from_logprobs(p_r, p_c, cfg.K)
    check_routing_near_ties(host(idx), idx_ref, score_ref, p_r, p_c, cfg.N_c)
    y_ref = oracle.expert_fwd_token_centric(u["x"], u["W"], u["V"], host(idx), host(gate))
    check_y(host(y), y_ref, "routed, dense")
    y_sp = omni.routed_fwd(t["x"], t["W"], t["V"], t["W_r"], t["W_c"], cfg.K, cfg.B, ws=ws,
                           expert_mode="sparse")
    check_y(host(y_sp), y_ref, "routed, task by task")


def _status_after(cfg, s_dev, t, mode):
    ws = omni.expert_workspace(cfg.L, cfg.d, cfg.K, cfg.N, cfg.B, DEV,
                               omni.OMNI_EXPERT_DENSE if mode == "dense" else 0)
    omni.grouped_expert_fwd(t["x"], t["W"], t["V"], s_dev, cfg.K, cfg.B, ws=ws, expert_mode=mode)
    return omni.omni_get_device_status(ws)


@pytest.mark.parametrize("mode", ["dense", "sparse"])
def test_expert_stage_checks_group_arrays(mode):
    """A wrong schedule is reported as OMNI_DEV_BAD_SCHEDULE (3), with every
    access kept in bounds: offsets shifted by one task (both paths); on the
    tensor-core path also num_active out of range or one too small (a group
    left out, so the active groups no longer cover every task)."""
    cfg = SKEW_RAGGED
    t, u, idx, gate, sched, s_dev = _routing_and_schedule(cfg, seed=5)
    assert _status_after(cfg, s_dev, t, mode) == 0
    bad = dict(s_dev)
    off = s_dev["group_offsets"].clone()
    q = int(sched["active_groups"][1])
    off[q] += 1                                        # the group's first task moves to q - 1
    bad["group_offsets"] = off
    assert _status_after(cfg, bad, t, mode) == 3
    if mode == "dense":
        G = (cfg.N + cfg.B - 1) // cfg.B
        for na in (G + 1, int(sched["num_active"]) - 1, -1):
            bad = dict(s_dev)
            bad["num_active"] = torch.tensor([na], dtype=torch.int32, device=DEV)
            assert _status_after(cfg, bad, t, mode) == 3, na
    assert _status_after(cfg, s_dev, t, mode) == 0
