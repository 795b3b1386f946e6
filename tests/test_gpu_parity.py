"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle.

Bar (see include/omni.h for the semantics):
  - integer / index work bit-exact: top-K indices (and scores, which are one
    fp32 addition) from identical fp32 log-probabilities, the sorted task
    order, group offsets / counts / active list, distinct-expert count;
  - gates within a few fp32 ulps (the oracle rounds an fp64 softmax once);
  - y within max-abs 2e-2 and rel-L2 5e-3 of the fp64 oracle;
  - end to end, the GPU's own log-probabilities differ from the oracle's in
    the last bits, so index sets may differ only in cells whose score is
    within 1e-5 of the K-th score, and y is then checked against the oracle
    run on the GPU's routing.
"""
import numpy as np
import pytest
import torch

import oracle
import atomic_expert_layer_b200 as omni
from atomic_expert_layer_b200 import configs, inputs

from _parity import (check_routing_near_ties, check_y, distinct_random_idx, host,
                     oracle_y_rows)

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    omni.load()


# ---------------------------------------------------- router top-K, exact
@pytest.mark.parametrize("L,N_r,N_c,K,quantum,seed", [
    (256, 64, 64, 16, None, 0),       # tiny grid
    (300, 512, 512, 64, None, 1),     # small grid
    (97, 1304, 1304, 64, None, 2),    # headline grid, ragged token count
    (64, 1024, 1024, 128, None, 3),   # skewed-config grid, K = 128
    (50, 8, 64, 16, None, 4),         # K > N_r
    (50, 1, 300, 40, None, 5),        # single row
    (40, 300, 1, 40, None, 6),        # single column
    (30, 8, 8, 64, None, 7),          # K = N
    (200, 40, 24, 20, 0.25, 8),       # forced exact ties
    (120, 64, 64, 64, 2.0 ** -4, 9),  # forced ties, K = 64
    (33, 12, 12, 1, None, 10),        # K = 1
    (17, 2000, 3000, 512, None, 11),  # K at the limit
])
def test_router_topk_from_logprobs_bitexact(L, N_r, N_c, K, quantum, seed):
    p_r = inputs.random_logprobs(L, N_r, seed, quantum)
    p_c = inputs.random_logprobs(L, N_c, seed + 1000, quantum)
    idx, score, gate = oracle.topk_from_logprobs(p_r, p_c, K)
    out = omni.router_topk(None, None, None, K, p_r=torch.from_numpy(p_r).to(DEV),
                           p_c=torch.from_numpy(p_c).to(DEV), logprobs_in=True)
    np.testing.assert_array_equal(host(out["idx"]), idx)
    np.testing.assert_array_equal(host(out["score"]), score)
    np.testing.assert_allclose(host(out["gate"]), gate, rtol=4e-6, atol=1e-12)


@pytest.mark.parametrize("L,N_r,N_c,K,quantum,seed", [
    (300, 512, 512, 64, None, 21),        # small grid, 4 bands
    (97, 1304, 1304, 64, None, 22),       # headline grid, 10 bands
    (64, 1024, 1024, 128, None, 23),      # skewed-config grid, K = 128
    (50, 8, 64, 16, None, 24),            # K > N_r, one band
    (50, 1, 300, 40, None, 25),           # single row
    (40, 300, 1, 40, None, 26),           # single column
    (33, 12, 12, 1, None, 27),            # K = 1, more bands than needed rows
    (17, 2000, 3000, 512, None, 28),      # K at the limit
    (64, 256, 256, 32, 2.0 ** -3, 29),    # forced exact ties across bands
    (100, 96, 160, 16, 0.25, 30),         # forced ties, coarse quantum
])
def test_router_topk_blockwise_bitexact(L, N_r, N_c, K, quantum, seed):
    """The pages' blockwise grid top-K gives the oracle's selection exactly."""
    p_r = inputs.random_logprobs(L, N_r, seed, quantum)
    p_c = inputs.random_logprobs(L, N_c, seed + 1000, quantum)
    idx, score, gate = oracle.topk_from_logprobs(p_r, p_c, K)
    out = omni.router_topk(None, None, None, K, p_r=torch.from_numpy(p_r).to(DEV),
                           p_c=torch.from_numpy(p_c).to(DEV), logprobs_in=True, blockwise=True)
    np.testing.assert_array_equal(host(out["idx"]), idx)
    np.testing.assert_array_equal(host(out["score"]), score)
    np.testing.assert_allclose(host(out["gate"]), gate, rtol=4e-6, atol=1e-12)


def test_router_topk_blockwise_limits():
    """K above (N_r + N_c) / 4 is refused on the host, before any launch."""
    p_r = torch.zeros((4, 8), device=DEV)
    p_c = torch.zeros((4, 8), device=DEV)
    with pytest.raises(omni.OmniError):
        omni.router_topk(None, None, None, 8, p_r=p_r, p_c=p_c, logprobs_in=True, blockwise=True)


def test_router_full_tiny_against_oracle():
    cfg = configs.TINY
    t = inputs.make_inputs(cfg, DEV, seed=0, with_experts=False)
    u = {k: host(v) for k, v in t.items()}
    p_r, p_c = oracle.router_logprobs(u["x"], u["W_r"], u["W_c"])
    out = omni.router_topk(t["x"], t["W_r"], t["W_c"], cfg.K)
    # fp32 tensor-core logits + fp32 LogSoftmax vs fp64
    np.testing.assert_allclose(host(out["p_r"]), p_r, rtol=0, atol=2e-5)
    np.testing.assert_allclose(host(out["p_c"]), p_c, rtol=0, atol=2e-5)
    # selection on the GPU's own p is exact
    idx2, score2, _ = oracle.topk_from_logprobs(host(out["p_r"]), host(out["p_c"]), cfg.K)
    np.testing.assert_array_equal(host(out["idx"]), idx2)
    np.testing.assert_array_equal(host(out["score"]), score2)
    # against the oracle's p only near-ties may differ
    idx, score, _ = oracle.topk_from_logprobs(p_r, p_c, cfg.K)
    check_routing_near_ties(host(out["idx"]), idx, score, p_r, p_c, cfg.N_c)


@pytest.mark.parametrize("L,d,N_r,N_c", [(1, 256, 64, 64), (130, 768, 100, 37),
                                          (257, 2048, 1304, 1304), (64, 200, 16, 300),
                                          (16, 2048, 1304, 1304), (7, 200, 100, 37),
                                          (3, 512, 8, 2000), (17, 1024, 1304, 1304)])
def test_router_gemm_logprobs_shapes(L, d, N_r, N_c):
    """Ragged L, N_r, N_c and d (d = 200 is not a multiple of the 64-wide K step);
    L <= 4 takes the streamed projection with LogSoftmax in the axis kernels,
    larger L the tensor-core GEMM with fused partials."""
    cfg = configs.LayerConfig("t", L, d, N_r, N_c, 4, 4)
    t = inputs.make_inputs(cfg, DEV, seed=5, with_experts=False)
    u = {k: host(v) for k, v in t.items()}
    p_r, p_c = oracle.router_logprobs(u["x"], u["W_r"], u["W_c"])
    out = omni.router_topk(t["x"], t["W_r"], t["W_c"], min(4, N_r * N_c))
    np.testing.assert_allclose(host(out["p_r"]), p_r, rtol=0, atol=3e-5)
    np.testing.assert_allclose(host(out["p_c"]), p_c, rtol=0, atol=3e-5)


# ---------------------------------------------------------- schedule, exact
def _compare_schedule(got, ref):
    for k in ("task_token", "task_expert", "task_gate", "group_offsets", "group_counts"):
        np.testing.assert_array_equal(host(got[k]), ref[k], err_msg=k)
    na = int(host(got["num_active"])[0])
    assert na == ref["num_active"]
    np.testing.assert_array_equal(host(got["active_groups"])[:na], ref["active_groups"][:na])
    assert int(host(got["num_distinct"])[0]) == ref["num_distinct"]


@pytest.mark.parametrize("L,K,N,B,seed", [
    (256, 16, 4096, 32, 0),          # tiny: 128 groups, one radix pass
    (1000, 64, 262144, 64, 1),       # small grid: 4096 groups
    (3000, 64, 1700416, 128, 2),     # headline grid: 13,285 groups, two passes
    (70, 5, 1000, 1, 3),             # B = 1
    (64, 4, 64, 64, 4),              # a single group: no radix pass
    (700, 32, 1 << 21, 1, 5),        # 2M groups: three passes
    (1, 7, 50, 3, 6),                # one token
    (4097, 3, 97, 5, 7),             # ragged tiles
])
def test_schedule_bitexact(L, K, N, B, seed):
    idx = distinct_random_idx(L, K, N, seed)
    gate = np.random.default_rng(seed).random((L, K)).astype(np.float32)
    ref = oracle.schedule(idx, gate, N, B)
    got = omni.schedule(torch.from_numpy(idx).to(DEV), torch.from_numpy(gate).to(DEV), N, B)
    _compare_schedule(got, ref)


def test_schedule_reports_bad_expert():
    idx = np.array([[0, 5], [7, 99]], np.int32)        # 99 >= N
    gate = np.ones((2, 2), np.float32)
    ws = omni.schedule_workspace(2, 2, 10, 2)
    omni.schedule(torch.from_numpy(idx).to(DEV), torch.from_numpy(gate).to(DEV), 10, 2, ws=ws)
    assert omni.omni_get_device_status(ws) == 1        # OMNI_DEV_BAD_EXPERT
    assert omni.omni_get_device_status(ws) == 0        # cleared by the read


def test_bounded_wait_ends_with_status():
    ws = torch.zeros(4096, dtype=torch.uint8, device=DEV)
    omni.omni_selftest_wait_timeout(ws, 50)
    assert omni.omni_get_device_status(ws) == 2        # OMNI_DEV_WAIT_TIMEOUT
    # the context is still usable
    assert torch.ones(4, device=DEV).sum().item() == 4


# ------------------------------------------------------- grouped expert stage
def _oracle_routing(cfg, u):
    p_r, p_c = oracle.router_logprobs(u["x"], u["W_r"], u["W_c"])
    return oracle.topk_from_logprobs(p_r, p_c, cfg.K)


@pytest.mark.parametrize("cfg", [configs.TINY,
                                 configs.LayerConfig("d512_B7", 300, 512, 32, 40, 24, 7),
                                 configs.LayerConfig("d1024_B1000", 200, 1024, 64, 64, 32, 1000)],
                         ids=lambda c: c.name)
def test_grouped_expert_on_oracle_schedule(cfg):
    t = inputs.make_inputs(cfg, DEV, seed=1)
    u = {k: host(v) for k, v in t.items()}
    idx, score, gate = _oracle_routing(cfg, u)
    sched = oracle.schedule(idx, gate, cfg.N, cfg.B)
    y_ref = oracle.expert_fwd_expert_centric(u["x"], u["W"], u["V"], sched, cfg.B)
    s_dev = {k: torch.as_tensor(np.atleast_1d(v).astype(np.float32 if k == "task_gate"
                                                        else np.int32)).to(DEV)
             for k, v in sched.items()}
    y = omni.grouped_expert_fwd(t["x"], t["W"], t["V"], s_dev, cfg.K, cfg.B)
    check_y(host(y), y_ref)
    # accumulate mode adds to what is there
    y0 = torch.full_like(y, 0.25)
    omni.grouped_expert_fwd(t["x"], t["W"], t["V"], s_dev, cfg.K, cfg.B, y=y0, accumulate=True)
    check_y(host(y0), y_ref + 0.25)


def test_grouped_expert_big_group_and_single_token():
    """One token choosing K = 512 experts of one group of B = 1024: a group
    spans several work items and several expert chunks."""
    cfg = configs.LayerConfig("one_group", 3, 256, 32, 32, 512, 1024)
    t = inputs.make_inputs(cfg, DEV, seed=2)
    u = {k: host(v) for k, v in t.items()}
    idx = distinct_random_idx(cfg.L, cfg.K, cfg.N, 3)
    gate = np.random.default_rng(3).random((cfg.L, cfg.K)).astype(np.float32)
    sched = oracle.schedule(idx, gate, cfg.N, cfg.B)
    y_ref = oracle.expert_fwd_token_centric(u["x"], u["W"], u["V"], idx, gate)
    got = omni.schedule(torch.from_numpy(idx).to(DEV), torch.from_numpy(gate).to(DEV), cfg.N,
                        cfg.B)
    _compare_schedule(got, sched)
    y = omni.grouped_expert_fwd(t["x"], t["W"], t["V"], got, cfg.K, cfg.B)
    check_y(host(y), y_ref)


# ------------------------------------------------------------- end to end
def test_routed_fwd_tiny_full():
    cfg = configs.TINY
    t = inputs.make_inputs(cfg, DEV, seed=0)
    u = {k: host(v) for k, v in t.items()}
    p_r, p_c = oracle.router_logprobs(u["x"], u["W_r"], u["W_c"])
    idx_ref, score_ref, gate_ref = oracle.topk_from_logprobs(p_r, p_c, cfg.K)
    ws = omni.workspace(cfg.L, cfg.d, cfg.N_r, cfg.N_c, cfg.K, cfg.B)
    y, idx, gate = omni.routed_fwd(t["x"], t["W"], t["V"], t["W_r"], t["W_c"], cfg.K, cfg.B,
                                   ws=ws, want_routing=True)
    assert omni.omni_get_device_status(ws) == 0
    check_routing_near_ties(host(idx), idx_ref, score_ref, p_r, p_c, cfg.N_c)
    y_pinned = oracle.expert_fwd_token_centric(u["x"], u["W"], u["V"], host(idx), host(gate))
    check_y(host(y), y_pinned)
    if np.array_equal(host(idx), idx_ref):
        check_y(host(y), oracle.expert_fwd_token_centric(u["x"], u["W"], u["V"], idx_ref, gate_ref))
    # repeated calls give the same routing and (up to fp32 add order) the same y
    y2 = omni.routed_fwd(t["x"], t["W"], t["V"], t["W_r"], t["W_c"], cfg.K, cfg.B, ws=ws)
    np.testing.assert_allclose(host(y2), host(y), rtol=0, atol=1e-6)


@pytest.mark.parametrize("cfg", [configs.TINY, configs.SMALL], ids=lambda c: c.name)
def test_routed_fwd_token_order(cfg):
    """OMNI_TOKEN_ORDER: the expert stage in token order without the schedule
    (the path every call with L <= 16 takes) gives the same y, checked on
    sampled rows against the oracle on the GPU's routing, and agrees with
    the scheduled path up to fp32 summation order."""
    torch.cuda.empty_cache()
    t = inputs.make_inputs(cfg, DEV, seed=0)
    ws = omni.workspace(cfg.L, cfg.d, cfg.N_r, cfg.N_c, cfg.K, cfg.B)
    y_tok, idx, gate = omni.routed_fwd(t["x"], t["W"], t["V"], t["W_r"], t["W_c"], cfg.K,
                                       cfg.B, ws=ws, want_routing=True, token_order=True)
    assert omni.omni_get_device_status(ws) == 0
    rng = np.random.default_rng(2)
    tokens = np.unique(np.concatenate([[0, cfg.L - 1],
                                       rng.choice(cfg.L, min(cfg.L, 48), replace=False)]))
    y_ref = oracle_y_rows(t["x"], t["W"], t["V"], idx, gate, tokens)
    check_y(host(y_tok)[tokens], y_ref)
    y_sched, idx2, _ = omni.routed_fwd(t["x"], t["W"], t["V"], t["W_r"], t["W_c"], cfg.K,
                                       cfg.B, ws=ws, want_routing=True)
    assert np.array_equal(host(idx2), host(idx))
    np.testing.assert_allclose(host(y_tok), host(y_sched), rtol=0, atol=1e-5)
    del t, ws
    torch.cuda.empty_cache()


FULL = [configs.SMALL, configs.HEADLINE, configs.SKEW] + [configs.sweep(L) for L in configs.SWEEP_L]


@pytest.mark.parametrize("cfg", FULL, ids=lambda c: c.name)
def test_routed_fwd_full_size_sampled(cfg):
    """Full-size configurations, in the launch configuration the bench times:
    routing on sampled tokens (near-tie rule), the whole schedule bit-exact,
    y on sampled rows against the oracle on the GPU's routing."""
    torch.cuda.empty_cache()
    t = inputs.make_inputs(cfg, DEV, seed=0)
    ws = omni.workspace(cfg.L, cfg.d, cfg.N_r, cfg.N_c, cfg.K, cfg.B)
    y, idx, gate = omni.routed_fwd(t["x"], t["W"], t["V"], t["W_r"], t["W_c"], cfg.K, cfg.B,
                                   ws=ws, want_routing=True)
    assert omni.omni_get_device_status(ws) == 0
    rng = np.random.default_rng(1)
    ns = min(cfg.L, 48)
    tokens = np.unique(np.concatenate([[0, cfg.L - 1], rng.choice(cfg.L, ns, replace=False)]))
    # routing of the sampled tokens
    xs = host(t["x"][torch.as_tensor(tokens, device=DEV)])
    p_r, p_c = oracle.router_logprobs(xs, host(t["W_r"]), host(t["W_c"]))
    idx_ref, score_ref, _ = oracle.topk_from_logprobs(p_r, p_c, cfg.K)
    idx_h = host(idx)
    check_routing_near_ties(idx_h[tokens], idx_ref, score_ref, p_r, p_c, cfg.N_c)
    # every token's experts are distinct and in range
    assert idx_h.min() >= 0 and idx_h.max() < cfg.N
    srt = np.sort(idx_h, axis=1)
    assert np.all(srt[:, 1:] != srt[:, :-1])
    g = host(gate)
    np.testing.assert_allclose(g.astype(np.float64).sum(1), 1.0, atol=2e-5)
    # the schedule of the GPU's routing, whole, bit-exact
    sched_ref = oracle.schedule(idx_h, g, cfg.N, cfg.B)
    _compare_schedule(omni.schedule(idx, gate, cfg.N, cfg.B), sched_ref)
    # y rows
    y_ref = oracle_y_rows(t["x"], t["W"], t["V"], idx, gate, tokens)
    check_y(host(y)[tokens], y_ref)
    del t, ws, y
    torch.cuda.empty_cache()


@pytest.mark.parametrize("L,d,N_r,N_c,K,B", [
    (17, 256, 40, 24, 20, 7),      # just above the fused decode size; ragged groups
    (33, 512, 1, 300, 40, 300),    # a single group: no radix pass, tasks copied in token order
    (50, 256, 300, 1, 40, 1),      # one expert per group (G = N)
    (64, 256, 8, 8, 32, 4),        # crowded groups (M >= 64 G): the CTA-gathered scatter
    (300, 256, 64, 48, 64, 16),    # crowded, several CTAs of tasks
])
def test_routed_fwd_schedule_variants(L, d, N_r, N_c, K, B):
    """The routed forward on shapes that reach each way it builds its
    schedule (grouping by one atomic scatter, by CTA-gathered atomics for
    crowded groups, or no grouping with a single group), and the first size
    past the fused decode step: every token's routing under the near-tie rule
    and every y row against the oracle on the GPU's routing."""
    cfg = configs.LayerConfig("variant", L, d, N_r, N_c, K, B)
    t = inputs.make_inputs(cfg, DEV, seed=4)
    u = {k: host(v) for k, v in t.items()}
    ws = omni.workspace(L, d, N_r, N_c, K, B)
    ws.fill_(0xff)
    y, idx, gate = omni.routed_fwd(t["x"], t["W"], t["V"], t["W_r"], t["W_c"], K, B, ws=ws,
                                   want_routing=True)
    assert omni.omni_get_device_status(ws) == 0
    p_r, p_c = oracle.router_logprobs(u["x"], u["W_r"], u["W_c"])
    idx_ref, score_ref, _ = oracle.topk_from_logprobs(p_r, p_c, K)
    check_routing_near_ties(host(idx), idx_ref, score_ref, p_r, p_c, N_c)
    check_y(host(y), oracle.expert_fwd_token_centric(u["x"], u["W"], u["V"], host(idx),
                                                     host(gate)))


def test_routed_fwd_skips_mlp_and_accumulates():
    cfg = configs.LayerConfig("acc", 40, 256, 16, 16, 8, 16)
    t = inputs.make_inputs(cfg, DEV, seed=4)
    y = omni.routed_fwd(t["x"], t["W"], t["V"], t["W_r"], t["W_c"], cfg.K, cfg.B)
    base = torch.randn_like(y)
    y2 = base.clone()
    omni.routed_fwd(t["x"], t["W"], t["V"], t["W_r"], t["W_c"], cfg.K, cfg.B, y=y2,
                    accumulate=True)
    np.testing.assert_allclose(host(y2), host(base + y), rtol=0, atol=1e-5)


# ------------------------------------------------------------------ backward
def _check_grad(got, ref, name, tol=2e-4):
    """fp32 reductions vs the fp64 oracle: max-abs within tol of the largest
    reference magnitude, and rel-L2 within tol."""
    scale = float(np.abs(ref).max())
    assert scale > 0, name
    err = np.abs(got - ref)
    assert float(err.max()) <= tol * scale, (name, float(err.max()), scale)
    rel = float(np.linalg.norm(got - ref) / np.linalg.norm(ref))
    assert rel <= tol, (name, rel)


def _bwd_case(cfg, L_sub, seed, marks="full"):
    """marks: "full", a workspace with the expert bitmaps (rows used once get a
    plain read-add-write) and the router-row lists; "bitmaps", room for the
    bitmaps only (router rows reduced); "min", the 256-byte minimum (every
    row reduced)."""
    t = inputs.make_inputs(cfg, DEV, seed=0)
    x = t["x"][:L_sub].contiguous()
    rt = omni.router_topk(x, t["W_r"], t["W_c"], cfg.K)
    g = torch.Generator(device=DEV)
    g.manual_seed(seed)
    dy = torch.randn((L_sub, cfg.d), generator=g, device=DEV, dtype=torch.float32)
    n_ws = {"full": omni.omni_routed_bwd_workspace_size(L_sub, cfg.d, cfg.N_r, cfg.N_c, cfg.K),
            "bitmaps": 256 + 2 * (-(-4 * (-(-cfg.N // 32)) // 256) * 256),
            "min": 256}[marks]
    ws = torch.full((n_ws,), 0xff, dtype=torch.uint8, device=DEV)   # the call clears what it uses
    out = omni.routed_bwd(x, t["W"], t["V"], t["W_r"], t["W_c"], rt["idx"], rt["gate"], dy, ws=ws)
    assert omni.omni_get_device_status(ws) == 0
    # oracle on the GPU's routing; expert rows compacted to the ones used
    idx = rt["idx"].long()
    uniq, inv = torch.unique(idx, return_inverse=True)
    ref = oracle.expert_bwd(host(x), host(t["W"][uniq]), host(t["V"][uniq]),
                            inv.to(torch.int32).cpu().numpy(), host(rt["gate"]), host(dy))
    # the router part needs the real expert ids n = i * N_c + j
    ref.update(oracle.router_bwd(host(x), host(t["W_r"]), host(t["W_c"]), host(rt["p_r"]),
                                 host(rt["p_c"]), host(rt["idx"]), host(rt["gate"]),
                                 ref["dgate"], dx=ref["dx"]))
    _check_grad(host(out["dx"]), ref["dx"], "dx")
    _check_grad(host(out["dW"][uniq]), ref["dW"], "dW")
    _check_grad(host(out["dV"][uniq]), ref["dV"], "dV")
    _check_grad(host(out["dW_r"]), ref["dW_r"], "dW_r")
    _check_grad(host(out["dW_c"]), ref["dW_c"], "dW_c")
    # rows of experts no token used stay untouched (zero)
    used = torch.zeros(cfg.N, dtype=torch.bool, device=DEV)
    used[uniq] = True
    if not bool(used.all()):
        assert float(out["dW"][~used].abs().max()) == 0.0
    return t, x, rt, dy, out


# 1024 tokens on a 4 x 64 grid: each grid row is met by hundreds of tokens,
# more than a router-row list holds, so its extra pairs take the reductions
BWD_CROWDED_ROWS = configs.LayerConfig("bwd_rows_L1024_d256_N256_K16_B16", 1024, 256, 4, 64, 16, 16)


@pytest.mark.parametrize("marks", ["full", "bitmaps", "min"])
@pytest.mark.parametrize("cfg,L_sub", [(configs.TINY, configs.TINY.L),
                                       (configs.HEADLINE, 48),
                                       (configs.sweep(16), 16),
                                       (BWD_CROWDED_ROWS, BWD_CROWDED_ROWS.L)],
                         ids=lambda v: getattr(v, "name", str(v)))
def test_routed_bwd_against_oracle(cfg, L_sub, marks):
    """Backward through the C ABI against the fp64 oracle backward on the
    GPU's own routing: every token of the tiny layer (experts shared by many
    tasks), a token batch at the full headline and d = 2048 shapes (N = 1.7M
    experts, almost all used once), and a layer whose grid rows overflow
    their lists; with the full workspace (expert bitmaps and router-row
    lists), the bitmaps only, and the 256-byte minimum."""
    torch.cuda.empty_cache()
    t, x, rt, dy, out = _bwd_case(cfg, L_sub, seed=5, marks=marks)
    if cfg is configs.TINY:
        counts = torch.bincount(rt["idx"].long().flatten(), minlength=cfg.N)
        assert int((counts == 1).sum()) > 0 and int((counts > 1).sum()) > 0   # both kinds of row
    if cfg is BWD_CROWDED_ROWS:
        rows_per_token = [len(set((host(rt["idx"])[i] // cfg.N_c).tolist())) for i in range(cfg.L)]
        assert max(np.bincount(np.concatenate([np.unique(host(rt["idx"])[i] // cfg.N_c)
                                               for i in range(cfg.L)]))) > 256, rows_per_token[:4]
    torch.cuda.empty_cache()


def test_routed_bwd_accumulates():
    """Weight gradients are accumulated (+=): a second call doubles them and
    leaves dx (overwritten) the same."""
    cfg = configs.TINY
    t, x, rt, dy, out = _bwd_case(cfg, cfg.L, seed=6)
    out2 = omni.routed_bwd(x, t["W"], t["V"], t["W_r"], t["W_c"], rt["idx"], rt["gate"], dy,
                           dW=out["dW"].clone(), dV=out["dV"].clone(),
                           dW_r=out["dW_r"].clone(), dW_c=out["dW_c"].clone())
    np.testing.assert_allclose(host(out2["dx"]), host(out["dx"]), rtol=0, atol=1e-6)
    for k in ("dW", "dV", "dW_r", "dW_c"):
        # fp32 reductions land in a run-dependent order: compare at fp32 scale
        ref = 2 * host(out[k])
        np.testing.assert_allclose(host(out2[k]), ref, rtol=0,
                                   atol=1e-5 * float(np.abs(ref).max()))


# ------------------------------------------------------- fused decode step
@pytest.mark.parametrize("L,d,N_r,N_c,K", [
    (1, 2048, 1304, 1304, 64),     # the decode sweep's grid and width
    (16, 2048, 1304, 1304, 64),
    (3, 256, 100, 37, 16),         # ragged axes (37: rows not a multiple of 4)
    (5, 512, 64, 64, 128),         # K = 128 on a small grid (K > N_r)
    (16, 1024, 512, 512, 128),
    (2, 512, 200, 300, 32),        # two tokens (CUDA-core projection), unequal axes
    (4, 256, 2400, 2400, 32),      # more than 16 router rows per CTA (two row tiles)
])
def test_decode_step_against_oracle(L, d, N_r, N_c, K):
    """L <= 16 runs the whole routed step (projection, selection, gates,
    token-order expert work) in one cooperative launch: routing against the
    oracle under the near-tie rule, y on every token against the oracle on
    the GPU's routing, idx_out / gate_out, and OMNI_Y_ACCUMULATE.  The
    workspace starts filled with 0xff bytes: the step needs no cleared state
    (its barrier word is tagged per call), and a second call on the same
    workspace (the accumulating one) still synchronises."""
    torch.cuda.empty_cache()
    cfg = configs.LayerConfig("decode", L, d, N_r, N_c, K, 64)
    t = inputs.make_inputs(cfg, DEV, seed=9)
    u = {k: host(v) for k, v in t.items() if k in ("x", "W_r", "W_c")}
    ws = omni.workspace(L, d, N_r, N_c, K, cfg.B)
    ws.fill_(0xff)           # the step clears its own status and barrier state
    y, idx, gate = omni.routed_fwd(t["x"], t["W"], t["V"], t["W_r"], t["W_c"], K, cfg.B, ws=ws,
                                   want_routing=True)
    assert omni.omni_get_device_status(ws) == 0
    p_r, p_c = oracle.router_logprobs(u["x"], u["W_r"], u["W_c"])
    idx_ref, score_ref, _ = oracle.topk_from_logprobs(p_r, p_c, K)
    check_routing_near_ties(host(idx), idx_ref, score_ref, p_r, p_c, N_c)
    g = host(gate)
    np.testing.assert_allclose(g.astype(np.float64).sum(1), 1.0, atol=2e-5)
    y_ref = oracle_y_rows(t["x"], t["W"], t["V"], idx, gate, np.arange(L))
    check_y(host(y), y_ref, "decode step")
    # accumulate adds to what is there
    base = torch.randn_like(y)
    y2 = base.clone()
    omni.routed_fwd(t["x"], t["W"], t["V"], t["W_r"], t["W_c"], K, cfg.B, y=y2, ws=ws,
                    accumulate=True)
    check_y(host(y2), host(base).astype(np.float64) + y_ref, "decode step, accumulate")
    del t, ws
    torch.cuda.empty_cache()
