"""Pins of the CPU oracle against things other than itself (CPU only).

Each test ties one oracle function to an independent fact: a case worked by
hand (tests/golden), brute force over the materialised score grid, a closed
form, an invariant, or a library routine.  A dropped term, a wrong sign or
index, or a transposed operand anywhere in the oracle fails one of them.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from atomic_expert_layer_b200 import configs, inputs

GOLDEN = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "hand_examples.json")))


def bf16_u16(a) -> np.ndarray:
    """Exact small values -> bf16 bit patterns."""
    return inputs.to_u16(torch.tensor(np.asarray(a, np.float32)).to(torch.bfloat16))


def brute_force_topk(p_r, p_c, K):
    """Materialise all N = N_r * N_c scores and sort them by the full key."""
    L, N_r = p_r.shape
    N_c = p_c.shape[1]
    idx = np.empty((L, K), np.int64)
    sc = np.empty((L, K), np.float32)
    n = np.arange(N_r * N_c)
    for t in range(L):
        S = (p_r[t][:, None] + p_c[t][None, :]).astype(np.float32).ravel()   # fp32 adds
        pr = np.repeat(p_r[t], N_c)
        pc = np.tile(p_c[t], N_r)
        order = np.lexsort((n, -pc, -pr, -S))        # last key is the primary one
        idx[t] = order[:K]
        sc[t] = S[order[:K]]
    return idx, sc


# ---------------------------------------------------------------- hand cases
@pytest.mark.parametrize("case", GOLDEN["router"], ids=lambda c: c["name"])
def test_topk_hand_examples(case):
    p_r = np.array([case["p_r"]], np.float32)
    p_c = np.array([case["p_c"]], np.float32)
    idx, score, gate = oracle.topk_from_logprobs(p_r, p_c, case["K"])
    assert idx[0].tolist() == case["idx"]
    np.testing.assert_allclose(gate[0], case["gate"], rtol=2e-6)
    assert np.all(score[0] == (p_r[0][np.array(case["idx"]) // p_c.shape[1]]
                               + p_c[0][np.array(case["idx"]) % p_c.shape[1]]))


@pytest.mark.parametrize("case", GOLDEN["schedule"], ids=lambda c: c["name"])
def test_schedule_hand_examples(case):
    s = oracle.schedule(np.array(case["idx"], np.int32), np.array(case["gate"], np.float32),
                        case["N"], case["B"])
    for key in ("task_token", "task_expert", "group_counts", "group_offsets"):
        assert s[key].tolist() == case[key], key
    np.testing.assert_array_equal(s["task_gate"], np.array(case["task_gate"], np.float32))
    assert s["num_active"] == case["num_active"]
    assert s["active_groups"][: s["num_active"]].tolist() == case["active_groups"]
    assert s["num_distinct"] == case["num_distinct"]


@pytest.mark.parametrize("case", GOLDEN["expert"], ids=lambda c: c["name"])
def test_expert_hand_examples(case):
    x, W, V = bf16_u16(case["x"]), bf16_u16(case["W"]), bf16_u16(case["V"])
    idx = np.array(case["idx"], np.int32)
    gate = np.array(case["gate"], np.float32)
    y = oracle.expert_fwd_token_centric(x, W, V, idx, gate)
    np.testing.assert_allclose(y, np.array(case["y"]), rtol=1e-14, atol=1e-15)
    sched = oracle.schedule(idx, gate, W.shape[0], 2)
    y2 = oracle.expert_fwd_expert_centric(x, W, V, sched, 2)
    np.testing.assert_allclose(y2, np.array(case["y"]), rtol=1e-14, atol=1e-15)


# ------------------------------------------------------- router, step A1/A2
def test_router_matches_library_log_softmax():
    cfg = configs.TINY
    t = inputs.make_inputs(cfg, "cpu", seed=3, with_experts=False)
    x, Wr, Wc = (inputs.to_u16(t[k]) for k in ("x", "W_r", "W_c"))
    p_r, p_c = oracle.router_logprobs(x, Wr, Wc)
    xf = t["x"].double()
    ref_r = torch.log_softmax(xf @ t["W_r"].double().T, dim=1).float().numpy()
    ref_c = torch.log_softmax(xf @ t["W_c"].double().T, dim=1).float().numpy()
    np.testing.assert_allclose(p_r, ref_r, rtol=0, atol=2e-6)
    np.testing.assert_allclose(p_c, ref_c, rtol=0, atol=2e-6)
    # log-probabilities: each row sums to one in probability space
    np.testing.assert_allclose(np.log(np.exp(p_r.astype(np.float64)).sum(1)), 0, atol=1e-6)
    np.testing.assert_allclose(np.log(np.exp(p_c.astype(np.float64)).sum(1)), 0, atol=1e-6)
    # the row projection uses W_r and the column one W_c (not swapped)
    assert not np.allclose(p_r, p_c)


# ------------------------------------------------------- top-K, step A3/A4
@pytest.mark.parametrize("N_r,N_c,K,quantum,seed", [
    (64, 64, 16, None, 0), (8, 64, 16, None, 1), (64, 8, 33, None, 2), (1, 50, 7, None, 3),
    (50, 1, 7, None, 4), (5, 7, 35, None, 5), (16, 16, 64, 2.0 ** -4, 6), (40, 24, 20, 0.25, 7),
    (12, 12, 1, None, 8), (3, 3, 9, 1.0, 9),
    # both axes at least K, at the K of the full-size layers (64 and 128), so
    # the pruned (a+1)(b+1) <= K block is the whole argument, as on the GPU
    (160, 160, 64, None, 10), (200, 150, 128, None, 11), (130, 130, 128, 2.0 ** -4, 12),
    (128, 256, 64, 0.25, 13), (300, 260, 128, 2.0 ** -3, 14),
])
def test_topk_matches_bruteforce(N_r, N_c, K, quantum, seed):
    L = 24
    p_r = inputs.random_logprobs(L, N_r, seed, quantum)
    p_c = inputs.random_logprobs(L, N_c, seed + 100, quantum)
    idx, score, gate = oracle.topk_from_logprobs(p_r, p_c, K)
    bidx, bsc = brute_force_topk(p_r, p_c, K)
    np.testing.assert_array_equal(idx, bidx)
    np.testing.assert_array_equal(score, bsc)


@pytest.mark.parametrize("K,quantum", [(64, None), (128, 2.0 ** -4)])
def test_topk_matches_bruteforce_headline_grid(K, quantum):
    # the 1304 x 1304 grid of the headline layer (1.7M cells per token),
    # brute force over every cell for a few tokens
    L, n = 3, 1304
    p_r = inputs.random_logprobs(L, n, 21 + K, quantum)
    p_c = inputs.random_logprobs(L, n, 22 + K, quantum)
    idx, score, _ = oracle.topk_from_logprobs(p_r, p_c, K)
    bidx, bsc = brute_force_topk(p_r, p_c, K)
    np.testing.assert_array_equal(idx, bidx)
    np.testing.assert_array_equal(score, bsc)


def test_topk_tiny_config_from_router():
    cfg = configs.TINY
    t = inputs.make_inputs(cfg, "cpu", seed=0, with_experts=False)
    p_r, p_c = oracle.router_logprobs(*(inputs.to_u16(t[k]) for k in ("x", "W_r", "W_c")))
    idx, score, gate = oracle.topk_from_logprobs(p_r, p_c, cfg.K)
    bidx, bsc = brute_force_topk(p_r, p_c, cfg.K)
    np.testing.assert_array_equal(idx, bidx)
    np.testing.assert_array_equal(score, bsc)
    # block invariant: every selected cell has row rank a, column rank b, (a+1)(b+1) <= K
    rr = np.argsort(np.argsort(-p_r, axis=1, kind="stable"), axis=1, kind="stable")
    cr = np.argsort(np.argsort(-p_c, axis=1, kind="stable"), axis=1, kind="stable")
    a = np.take_along_axis(rr, idx // cfg.N_c, 1)
    b = np.take_along_axis(cr, idx % cfg.N_c, 1)
    assert np.all((a + 1) * (b + 1) <= cfg.K)
    assert np.all(a < cfg.K) and np.all(b < cfg.K)
    # gates: positive, sum to one, ordered like the scores
    assert np.all(gate > 0)
    np.testing.assert_allclose(gate.astype(np.float64).sum(1), 1.0, atol=1e-6)
    assert np.all(np.diff(gate, axis=1) <= 0)
    assert np.all(np.diff(score, axis=1) <= 0)


def test_topk_single_row_is_stable_argsort():
    p_c = inputs.random_logprobs(10, 300, 11, 0.125)
    p_r = np.full((10, 1), -0.5, np.float32)
    idx, _, _ = oracle.topk_from_logprobs(p_r, p_c, 40)
    # S = p_r + p_c is monotone in p_c; equal S keep index order
    S = (p_r + p_c).astype(np.float32)
    ref = np.argsort(-S, axis=1, kind="stable")[:, :40]
    np.testing.assert_array_equal(idx, ref)


def test_gates_closed_form_when_K_equals_N():
    """K = N selects every cell; softmax over all S of true log-probabilities is
    the product of the two axis distributions."""
    rng = np.random.default_rng(5)
    lr, lc = rng.normal(0, 1, (6, 8)), rng.normal(0, 1, (6, 8))
    p_r = torch.log_softmax(torch.tensor(lr), 1).float().numpy()
    p_c = torch.log_softmax(torch.tensor(lc), 1).float().numpy()
    idx, score, gate = oracle.topk_from_logprobs(p_r, p_c, 64)
    pr, pc = np.exp(p_r.astype(np.float64)), np.exp(p_c.astype(np.float64))
    pr /= pr.sum(1, keepdims=True)
    pc /= pc.sum(1, keepdims=True)
    joint = np.take_along_axis((pr[:, :, None] * pc[:, None, :]).reshape(6, 64), idx, 1)
    np.testing.assert_allclose(gate, joint, rtol=3e-6)
    assert sorted(idx[0].tolist()) == list(range(64))


def test_topk_rejects_nonfinite():
    p = np.zeros((1, 4), np.float32)
    p[0, 2] = np.nan
    with pytest.raises(ValueError):
        oracle.topk_from_logprobs(p, np.zeros((1, 4), np.float32), 2)


# ------------------------------------------------------ schedule, A6/A7
@pytest.mark.parametrize("L,K,N,B,seed", [(256, 16, 4096, 32, 0), (100, 7, 1000, 7, 1),
                                          (33, 5, 64, 64, 2), (50, 12, 997, 1, 3)])
def test_schedule_matches_lexsort(L, K, N, B, seed):
    rng = np.random.default_rng(seed)
    idx = np.stack([rng.choice(N, K, replace=False) for _ in range(L)]).astype(np.int32)
    gate = rng.random((L, K)).astype(np.float32)
    s = oracle.schedule(idx, gate, N, B)
    t = np.repeat(np.arange(L), K)
    e = idx.ravel().astype(np.int64)
    order = np.lexsort((e, t, e // B))
    np.testing.assert_array_equal(s["task_token"], t[order])
    np.testing.assert_array_equal(s["task_expert"], e[order])
    np.testing.assert_array_equal(s["task_gate"], gate.ravel()[order])
    G = (N + B - 1) // B
    counts = np.bincount(e // B, minlength=G)
    np.testing.assert_array_equal(s["group_counts"], counts)
    np.testing.assert_array_equal(s["group_offsets"], np.concatenate([[0], np.cumsum(counts)]))
    act = np.nonzero(counts)[0]
    assert s["num_active"] == len(act)
    np.testing.assert_array_equal(s["active_groups"][: len(act)], act)
    assert s["num_distinct"] == len(np.unique(e))


# ---------------------------------------------------- expert stage, A8/A9
def _tiny_routing(seed=0, K=None):
    cfg = configs.TINY
    t = inputs.make_inputs(cfg, "cpu", seed=seed)
    u = {k: inputs.to_u16(v) for k, v in t.items()}
    p_r, p_c = oracle.router_logprobs(u["x"], u["W_r"], u["W_c"])
    idx, score, gate = oracle.topk_from_logprobs(p_r, p_c, K or cfg.K)
    return cfg, t, u, idx, gate


def test_token_centric_equals_expert_centric():
    cfg, t, u, idx, gate = _tiny_routing()
    y1 = oracle.expert_fwd_token_centric(u["x"], u["W"], u["V"], idx, gate)
    s = oracle.schedule(idx, gate, cfg.N, cfg.B)
    y2 = oracle.expert_fwd_expert_centric(u["x"], u["W"], u["V"], s, cfg.B)
    np.testing.assert_allclose(y1, y2, rtol=1e-12, atol=1e-14)


def test_expert_k1_reduces_to_one_expert():
    cfg, t, u, idx, gate = _tiny_routing(K=1)
    y = oracle.expert_fwd_token_centric(u["x"], u["W"], u["V"], idx, gate)
    x = t["x"].double().numpy()
    e = idx[:, 0]
    h = np.einsum("td,td->t", x, t["W"].double().numpy()[e])
    ref = (gate[:, 0] * h / (1 + np.exp(-h)))[:, None] * t["V"].double().numpy()[e]
    np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-15)
    np.testing.assert_array_equal(gate, 1.0)


def test_expert_closed_form_all_experts():
    """K = N: y = ((G) . SiLU(x W^T)) V with a dense gate matrix, by matmul."""
    rng = np.random.default_rng(9)
    L, d, N = 5, 16, 12
    x = bf16_u16(rng.normal(0, 1, (L, d)))
    W = bf16_u16(rng.normal(0, 0.3, (N, d)))
    V = bf16_u16(rng.normal(0, 0.3, (N, d)))
    idx = np.stack([rng.permutation(N) for _ in range(L)]).astype(np.int32)
    gate = rng.random((L, N)).astype(np.float32)
    y = oracle.expert_fwd_token_centric(x, W, V, idx, gate)
    f = lambda a: torch.tensor(a.view(np.int16)).view(torch.bfloat16).double().numpy()
    Gd = np.zeros((L, N))
    np.put_along_axis(Gd, idx.astype(np.int64), gate.astype(np.float64), 1)
    H = f(x) @ f(W).T
    ref = (Gd * (H / (1 + np.exp(-H)))) @ f(V)
    np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-14)


def test_expert_linear_in_V_and_zero():
    cfg, t, u, idx, gate = _tiny_routing(seed=1)
    zero = np.zeros_like(u["V"])
    y0 = oracle.expert_fwd_token_centric(u["x"], u["W"], zero, idx, gate)
    assert np.all(y0 == 0)
    y1 = oracle.expert_fwd_token_centric(u["x"], u["W"], u["V"], idx, gate)
    V2 = inputs.to_u16(t["V"] * 2)                     # exact in bf16
    y2 = oracle.expert_fwd_token_centric(u["x"], u["W"], V2, idx, gate)
    np.testing.assert_allclose(y2, 2 * y1, rtol=1e-13, atol=1e-16)
    # gates scale the output linearly too
    y3 = oracle.expert_fwd_token_centric(u["x"], u["W"], u["V"], idx, gate * 0.5)
    np.testing.assert_allclose(y3, 0.5 * y1, rtol=1e-13, atol=1e-16)


def test_routed_fwd_token_subset_matches_full():
    cfg, t, u, idx, gate = _tiny_routing()
    full = oracle.routed_fwd(u["x"], u["W"], u["V"], u["W_r"], u["W_c"], cfg.K, cfg.B)
    toks = np.array([3, 200, 17], np.int32)
    part = oracle.routed_fwd(u["x"], u["W"], u["V"], u["W_r"], u["W_c"], cfg.K, cfg.B, tokens=toks)
    np.testing.assert_array_equal(part["idx"], full["idx"][toks])
    np.testing.assert_array_equal(part["y"], full["y"][toks])
    np.testing.assert_array_equal(full["idx"], idx)


# ------------------------------------------------------------------ backward
def _bf16_values(rng, shape, scale):
    """Random values that are exact in bf16: (bit patterns, float64 values)."""
    t = torch.tensor(rng.normal(0.0, scale, size=shape).astype(np.float32)).to(torch.bfloat16)
    return inputs.to_u16(t), t.to(torch.float64).numpy()


def _np_forward(x, W, V, W_r, W_c, idx, N_c):
    """The routed branch in numpy fp64 with the expert selection idx fixed:
    an implementation independent of the oracle's C code, used only to take
    finite differences."""
    def log_softmax(s):
        m = s.max(axis=1, keepdims=True)
        return s - (m + np.log(np.exp(s - m).sum(axis=1, keepdims=True)))
    p_r, p_c = log_softmax(x @ W_r.T), log_softmax(x @ W_c.T)
    rows = np.arange(x.shape[0])[:, None]
    S = p_r[rows, idx // N_c] + p_c[rows, idx % N_c]
    g = np.exp(S - S.max(axis=1, keepdims=True))
    g /= g.sum(axis=1, keepdims=True)
    h = np.einsum("td,tkd->tk", x, W[idx])
    a = h / (1.0 + np.exp(-h))
    return np.einsum("tk,tkd->td", g * a, V[idx])


def test_backward_matches_finite_differences():
    """Every gradient of the oracle's backward (expert and router parts,
    through gates, LogSoftmax and both projections) against central finite
    differences of an independent fp64 forward, the selection held fixed."""
    rng = np.random.default_rng(7)
    L, d, N_r, N_c, K = 3, 8, 5, 4, 6
    xu, x = _bf16_values(rng, (L, d), 1.0)
    Wu, W = _bf16_values(rng, (N_r * N_c, d), 0.6)
    Vu, V = _bf16_values(rng, (N_r * N_c, d), 0.6)
    Wru, W_r = _bf16_values(rng, (N_r, d), 0.5)
    Wcu, W_c = _bf16_values(rng, (N_c, d), 0.5)
    dy = rng.normal(0.0, 1.0, size=(L, d)).astype(np.float32)
    p_r, p_c = oracle.router_logprobs(xu, Wru, Wcu)
    idx, _, gate = oracle.topk_from_logprobs(p_r, p_c, K)
    grads = oracle.routed_bwd(xu, Wu, Vu, Wru, Wcu, p_r, p_c, idx, gate, dy)
    params = dict(x=x, W=W, V=V, W_r=W_r, W_c=W_c)
    names = dict(x="dx", W="dW", V="dV", W_r="dW_r", W_c="dW_c")
    dy64 = dy.astype(np.float64)
    eps = 1e-6
    for pname, P in params.items():
        fd = np.zeros_like(P)
        for pos in np.ndindex(P.shape):
            keep = P[pos]
            P[pos] = keep + eps
            up = (_np_forward(**params, idx=idx, N_c=N_c) * dy64).sum()
            P[pos] = keep - eps
            dn = (_np_forward(**params, idx=idx, N_c=N_c) * dy64).sum()
            P[pos] = keep
            fd[pos] = (up - dn) / (2 * eps)
        got = grads[names[pname]]
        scale = np.abs(fd).max()
        assert scale > 1e-3, pname                      # the check is not vacuous
        # the oracle runs on fp32 gates and log-probabilities (as the GPU does)
        np.testing.assert_allclose(got, fd, rtol=0, atol=2e-5 * scale, err_msg=pname)


def test_backward_single_expert_has_no_router_gradient():
    """K = 1: the gate is softmax of one score, identically 1, so nothing
    reaches the router; the expert part reduces to one SiLU unit."""
    rng = np.random.default_rng(8)
    L, d, N_r, N_c = 4, 16, 6, 6
    xu, x = _bf16_values(rng, (L, d), 1.0)
    Wu, W = _bf16_values(rng, (N_r * N_c, d), 0.4)
    Vu, V = _bf16_values(rng, (N_r * N_c, d), 0.4)
    Wru, _ = _bf16_values(rng, (N_r, d), 0.5)
    Wcu, _ = _bf16_values(rng, (N_c, d), 0.5)
    dy = rng.normal(0.0, 1.0, size=(L, d)).astype(np.float32)
    p_r, p_c = oracle.router_logprobs(xu, Wru, Wcu)
    idx, _, gate = oracle.topk_from_logprobs(p_r, p_c, 1)
    assert np.all(gate == 1.0)
    g = oracle.routed_bwd(xu, Wu, Vu, Wru, Wcu, p_r, p_c, idx, gate, dy)
    assert np.abs(g["dW_r"]).max() < 1e-12 and np.abs(g["dW_c"]).max() < 1e-12
    for t in range(L):
        e = idx[t, 0]
        h = x[t] @ W[e]
        s = 1.0 / (1.0 + np.exp(-h))
        c = dy[t].astype(np.float64) @ V[e]
        np.testing.assert_allclose(g["dgate"][t, 0], h * s * c, rtol=1e-12)
        np.testing.assert_allclose(g["dx"][t], c * s * (1 + h * (1 - s)) * W[e], rtol=1e-10,
                                   atol=1e-14)


# ------------------------------------------------------ shared dense MLP
@pytest.mark.parametrize("case", GOLDEN["mlp"], ids=lambda c: c["name"])
def test_shared_mlp_hand_examples(case):
    out = oracle.shared_mlp(bf16_u16(case["x"]), bf16_u16(case["W_g"]), bf16_u16(case["W_u"]),
                            bf16_u16(case["W_d"]))
    np.testing.assert_allclose(out, np.array(case["y"]), rtol=1e-14, atol=1e-15)


def test_shared_mlp_one_hot_weights_reduce_to_library_silu():
    """One-hot rows turn every product into a lookup: with W_g[f] = 2 e_{pg(f)},
    W_u[f] = e_{pu(f)} and W_d[c] = e_{pd(c)}, MLP(x)[c] = silu(2 x[pg(pd(c))])
    * x[pu(pd(c))], with torch's silu.  The index maps reach every input
    feature and both ends of the hidden range, and d != F, so a transposed
    operand, swapped gate and up roles or a dropped term all change the result."""
    d, F, L = 16, 24, 5
    pg = (5 * np.arange(F) + 3) % d
    pu = (3 * np.arange(F) + 7) % d
    pd = (7 * np.arange(d) + 2) % F
    assert set(pg) == set(range(d)) and set(pu) == set(range(d)) and {0, F - 1} <= set(pd)
    W_g = np.zeros((F, d)); W_g[np.arange(F), pg] = 2.0
    W_u = np.zeros((F, d)); W_u[np.arange(F), pu] = 1.0
    W_d = np.zeros((d, F)); W_d[np.arange(d), pd] = 1.0
    rng = np.random.default_rng(11)
    xu, x = _bf16_values(rng, (L, d), 1.5)
    out = oracle.shared_mlp(xu, bf16_u16(W_g), bf16_u16(W_u), bf16_u16(W_d))
    xt = torch.tensor(x, dtype=torch.float64)
    want = torch.nn.functional.silu(2.0 * xt[:, pg[pd]]) * xt[:, pu[pd]]
    np.testing.assert_allclose(out, want.numpy(), rtol=1e-14, atol=0)


def test_shared_mlp_linear_in_down_projection_and_zero_gate():
    """MLP is linear in W_d (exact small bf16 values, so W_d1 + W_d2 is exact
    too), and a zero gate projection gives SiLU(0) = 0 everywhere."""
    rng = np.random.default_rng(12)
    d, F, L = 8, 12, 6
    xu, _ = _bf16_values(rng, (L, d), 1.0)
    W_g = bf16_u16(rng.integers(-4, 5, size=(F, d)) / 8.0)
    W_u = bf16_u16(rng.integers(-4, 5, size=(F, d)) / 8.0)
    D1 = rng.integers(-4, 5, size=(d, F)) / 8.0
    D2 = rng.integers(-4, 5, size=(d, F)) / 8.0
    o1 = oracle.shared_mlp(xu, W_g, W_u, bf16_u16(D1))
    o2 = oracle.shared_mlp(xu, W_g, W_u, bf16_u16(D2))
    o12 = oracle.shared_mlp(xu, W_g, W_u, bf16_u16(D1 + D2))
    assert np.abs(o1).max() > 0.1 and np.abs(o2).max() > 0.1
    np.testing.assert_allclose(o12, o1 + o2, rtol=1e-13, atol=1e-13)
    zero = oracle.shared_mlp(xu, bf16_u16(np.zeros((F, d))), W_u, bf16_u16(D1))
    assert np.all(zero == 0.0)


def test_shared_mlp_token_subset_matches_full():
    w = inputs.make_mlp_weights(64, 128, seed=3)
    x = inputs.make_inputs(configs.TINY, with_experts=False)["x"][:40, :64].contiguous()
    args = [inputs.to_u16(t) for t in (x, w["W_g"], w["W_u"], w["W_d"])]
    full = oracle.shared_mlp(*args)
    tok = np.array([39, 0, 17, 17, 5], np.int32)
    np.testing.assert_array_equal(oracle.shared_mlp(*args, tokens=tok), full[tok])
