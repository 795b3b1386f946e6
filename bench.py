#!/usr/bin/env python3
"""Benchmark of the routed-branch forward of an OmniMoE layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--impl omni|reference]

One step = one pass of the whole routed branch (router GEMM, LogSoftmax,
row/column top-K, grid merge + gates, expert-centric schedule, grouped
expert stage) over one batch of L synthetic tokens, through the C ABI
(omni_routed_fwd).  Inputs are resident in HBM when timing starts; L2 is
flushed (256 MB write) between timed steps, outside the timed events.

With N > 1 (launched by torchrun) every rank holds a replica of the weights
and routes its own L tokens: the layer shards by token batch with no
data-path collective (weak scaling); only the timing is reduced (max).

Prints ONE JSON line on rank 0.  ``--impl reference`` times the CPU oracle
(the plain C implementation under oracle/) on a bounded sample instead.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from atomic_expert_layer_b200 import configs, inputs  # noqa: E402

METRIC = "routed-layer tokens/s at L=4096, N≈1.7M (1×B200); % of HBM/tensor roofline"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
L2_FLUSH_BYTES = 256 << 20
E2E_BATCHES = 4
GRAPH_MAX_L = 256          # batches this small are also timed as one CUDA graph replay


# ------------------------------------------------------------------ helpers
def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def reduce_max(value: float, world: int, device) -> float:
    """Max over ranks (timing only)."""
    if world == 1:
        return value
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_seed(rank: int) -> int:
    """Seed of a replica's own token batch (rank 0 of a 1-GPU run keeps seed 0)."""
    return 0 if rank == 0 else 1000 + rank


def job_throughput(world: int, tokens_per_rank: int, ms_max: float) -> float:
    """Whole-job tokens/s: every rank's tokens over the slowest rank's time."""
    return world * tokens_per_rank / (ms_max * 1e-3)


def med_ms(pairs) -> float:
    """Median duration (ms) of (start, end) CUDA event pairs."""
    return float(np.median([a.elapsed_time(b) for a, b in pairs]))


def config_of(cfg, world: int) -> dict:
    """The workload's `config` object (the same keys on both arms)."""
    return {"workload": cfg.name, "L": cfg.L, "d": cfg.d, "N_r": cfg.N_r, "N_c": cfg.N_c,
            "N": cfg.N, "K": cfg.K, "B": cfg.B, "tokens_per_gpu": cfg.L,
            "parallelism": f"replicas x{world} (token batches)",
            "l2": "flushed between timed steps (256 MB write)"}


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def peaks_hbm() -> float:
    return measured_peaks()["hbm_gbs"]


def measured_peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return dict(hbm_gbs=float(d["hbm_gbs"]), bf16_tflops=float(d["bf16_tflops"]),
                    bf16_tflops_sustained=float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                    source="measured")
    return dict(hbm_gbs=FALLBACK_HBM_GBS, bf16_tflops=FALLBACK_BF16_TFLOPS,
                bf16_tflops_sustained=1400.0, source="fallback")


def radix_passes(G: int) -> int:
    bits = 0
    while bits < 31 and (1 << bits) < G:
        bits += 1
    return (bits + 7) // 8


def launches_per_step(cfg) -> int:
    """Library kernels one omni_routed_fwd launches (memsets not counted)."""
    nmax = max(cfg.N_r, cfg.N_c)
    kmax = min(cfg.K, nmax)
    cap = ((kmax + 64 + 31) // 32) * 32 if kmax <= 1024 else 0
    reg = cfg.N_r % 4 == 0 and cfg.N_c % 4 == 0 and nmax <= 2048 and 0 < cap <= 320
    router = 1 + (2 if reg else 1) + 1            # GEMM, axis top-K (+ flagged redo), merge
    p = radix_passes(cfg.G)
    sched = 1 + (p + max(p - 1, 0))               # scan, scatters, histogram scans (the
    if cfg.L <= 16 and cfg.K <= 128 and cfg.d % 256 == 0 and cfg.d <= 2048:
        return 1                                  # the fused decode step: one launch
    # the tensor-core expert path (default for L * K * d >= 2^31): expert use,
    # dense marks, column scan, column list, gather, split, two tile GEMMs
    dense = 8 if cfg.L > 16 and cfg.M * cfg.d >= 2 ** 31 else 0
    return router + sched + 2 + dense             # group pass, token pass


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled during the timed region."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100", "-i", str(self.gpu)],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            time.sleep(0.15)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self) -> dict:
        rows = []
        try:
            for line in open(self.path):
                f = [c.strip() for c in line.split(",")]
                if len(f) >= 9 and f[1].replace(".", "").isdigit():
                    rows.append(f)
        finally:
            if self.path and os.path.exists(self.path):
                os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0}
        sm = [float(r[1]) for r in rows]
        smax = max(float(r[2]) for r in rows)
        power = [float(r[3]) for r in rows if r[3].replace(".", "").isdigit()]
        # samples under load: power well above idle
        load_idx = [i for i, r in enumerate(rows) if power and float(r[3]) > 0.5 * max(power)]
        sm_load = [sm[i] for i in load_idx] or sm
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            for n, v in zip(names, r[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": float(np.median(sm_load)), "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(rows),
                "samples_under_load": len(load_idx)}


def traffic_from_profile(kernel_src: str) -> float | None:
    """DRAM bytes (read + write) of one grouped expert stage call (both
    kernels) from the committed ncu summary, if it was taken on the current
    kernel source."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p)).get("grouped_expert_stage")
    if not d:
        return None
    sha = hashlib.sha256(open(kernel_src, "rb").read()).hexdigest()
    if d.get("source_sha256") != sha:
        return None
    return float(d["dram_bytes_per_launch_full_size"])


# ------------------------------------------------------------ omni arm
def run_omni(args, cfg, world, rank, local):
    import atomic_expert_layer_b200 as omni
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    omni.load()
    t = inputs.make_inputs(cfg, dev, seed=0)
    if world > 1:                                   # each rank routes its own tokens
        t["x"] = inputs.make_inputs(cfg, dev, seed=replica_seed(rank), with_experts=False)["x"]
    L, d = cfg.L, cfg.d
    ws = omni.workspace(L, d, cfg.N_r, cfg.N_c, cfg.K, cfg.B, dev)
    y = torch.empty((L, d), dtype=torch.float32, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def step():
        omni.omni_routed_fwd(t["x"], t["W"], t["V"], t["W_r"], t["W_c"], L, d, cfg.N_r, cfg.N_c,
                             cfg.K, cfg.B, y, None, None, 0, ws)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if omni.omni_get_device_status(ws) != 0:
        raise RuntimeError("device status set during warm-up")

    # ---- timed region: K steps of omni_routed_fwd
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    with ClockSampler(local) as clk:
        barrier(world)
        torch.cuda.synchronize()
        for i in range(args.steps):
            flush.zero_()                            # L2 flush, outside the events
            ev[i][0].record(stream)
            step()
            ev[i][1].record(stream)
        torch.cuda.synchronize()
        barrier(world)
    clocks = clk.summary()
    ms = med_ms(ev)
    ms_mean = float(np.mean([a.elapsed_time(b) for a, b in ev]))
    ms_max = reduce_max(ms, world, dev)

    # ---- ablation: the same layer with the expert stage in token order and
    # no expert-centric schedule (OMNI_TOKEN_ORDER; the path L <= 16 always takes)
    def step_token_order():
        omni.omni_routed_fwd(t["x"], t["W"], t["V"], t["W_r"], t["W_c"], L, d, cfg.N_r, cfg.N_c,
                             cfg.K, cfg.B, y, None, None, omni.OMNI_TOKEN_ORDER, ws)

    for _ in range(3):
        step_token_order()
    aev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    barrier(world)
    torch.cuda.synchronize()
    for i in range(args.steps):
        flush.zero_()
        aev[i][0].record(stream)
        step_token_order()
        aev[i][1].record(stream)
    torch.cuda.synchronize()
    barrier(world)
    tok_ms = reduce_max(med_ms(aev), world, dev)
    # device memory of each path beyond the shared inputs (x, W, V, W_r, W_c)
    # and the output y: the library allocates nothing, so it is the workspace
    # each path needs; and what an implementation that materialises every
    # token's gathered expert rows (W[idx], V[idx] as [L, K, d] bf16) would
    # allocate for them
    ws_ec = omni.omni_workspace_size_flags(L, d, cfg.N_r, cfg.N_c, cfg.K, cfg.B, 0)
    ws_to = omni.omni_workspace_size_flags(L, d, cfg.N_r, cfg.N_c, cfg.K, cfg.B,
                                           omni.OMNI_TOKEN_ORDER)
    gathered = 2 * 2 * L * cfg.K * d
    ablation = {"token_order_ms_per_step": tok_ms, "expert_centric_ms_per_step": ms_max,
                "token_order_over_expert_centric": tok_ms / ms_max,
                "workspace_bytes_expert_centric": ws_ec,
                "workspace_bytes_token_order": ws_to,
                "materialised_gather_bytes": gathered,
                "materialised_gather_over_expert_centric_workspace": gathered / ws_ec}

    # ---- small batches are launch-bound: the same step as one CUDA graph
    graph = None
    if L <= GRAPH_MAX_L:
        try:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                step()
            for _ in range(3):
                g.replay()
            gev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                   for _ in range(args.steps)]
            barrier(world)
            torch.cuda.synchronize()
            for i in range(args.steps):
                flush.zero_()
                gev[i][0].record(stream)
                g.replay()
                gev[i][1].record(stream)
            torch.cuda.synchronize()
            barrier(world)
            gms = reduce_max(med_ms(gev), world, dev)
            graph = {"value": job_throughput(world, L, gms), "unit": "tokens/s", "ms_per_step": gms}
            del g
        except RuntimeError as exc:                   # a step that cannot be captured
            graph = {"unavailable": str(exc).splitlines()[0]}
            torch.cuda.synchronize()

    # ---- staged loop: the same kernels through the three stage calls, for
    # per-stage times and the grouped-expert kernel's duration
    rt = omni.router_topk(t["x"], t["W_r"], t["W_c"], cfg.K)
    sc = omni.schedule(rt["idx"], rt["gate"], cfg.N, cfg.B)
    U = int(sc["num_distinct"].item())
    ws_r = omni.router_workspace(L, cfg.N_r, cfg.N_c, cfg.K, dev)
    ws_s = omni.schedule_workspace(L, cfg.K, cfg.N, cfg.B, dev)
    ws_e = omni.expert_workspace(L, d, cfg.K, cfg.N, cfg.B, dev)
    y2 = torch.zeros_like(y)

    def staged(evs=None):
        if evs:
            evs[0].record(stream)
        omni.omni_router_topk(t["x"], t["W_r"], t["W_c"], L, d, cfg.N_r, cfg.N_c, cfg.K,
                              rt["p_r"], rt["p_c"], rt["idx"], rt["score"], rt["gate"], 0, ws_r)
        if evs:
            evs[1].record(stream)
        omni.omni_schedule(rt["idx"], rt["gate"], L, cfg.K, cfg.N, cfg.B, sc["task_token"],
                           sc["task_expert"], sc["task_gate"], sc["group_offsets"],
                           sc["group_counts"], sc["active_groups"], sc["num_active"],
                           sc["num_distinct"], ws_s)
        if evs:
            evs[2].record(stream)
        omni.omni_grouped_expert_fwd(t["x"], t["W"], t["V"], L, d, cfg.K, cfg.N, cfg.B,
                                     sc["task_token"], sc["task_expert"], sc["task_gate"],
                                     sc["group_offsets"], sc["active_groups"], sc["num_active"],
                                     y2, omni.OMNI_Y_ACCUMULATE, ws_e)
        if evs:
            evs[3].record(stream)

    for _ in range(max(3, args.warmup)):
        staged()
    sev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    barrier(world)
    torch.cuda.synchronize()
    for i in range(args.steps):
        flush.zero_()
        staged(sev[i])
    torch.cuda.synchronize()
    barrier(world)
    st_router = med_ms([(e[0], e[1]) for e in sev])
    st_sched = med_ms([(e[1], e[2]) for e in sev])
    st_expert = med_ms([(e[2], e[3]) for e in sev])

    # ---- the selection (row / column top-K + merge, on the same p) against the
    # pages' blockwise grid scan; a few steps, the scan scores all N cells
    topk_cmp = None
    if 4 * cfg.K <= cfg.N_r + cfg.N_c:
        ws_r2 = omni.router_workspace(L, cfg.N_r, cfg.N_c, cfg.K, dev)
        o = {k: torch.empty_like(rt[k]) for k in ("idx", "score", "gate")}
        res = {}
        for name, fl in (("pruned", omni.OMNI_ROUTER_LOGPROBS_IN),
                         ("blockwise", omni.OMNI_ROUTER_LOGPROBS_IN | omni.OMNI_TOPK_BLOCKWISE)):
            def sel(fl=fl):
                omni.omni_router_topk(None, None, None, L, 0, cfg.N_r, cfg.N_c, cfg.K,
                                      rt["p_r"], rt["p_c"], o["idx"], o["score"], o["gate"],
                                      fl, ws_r2)
            sel()
            reps = 5
            cev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                   for _ in range(reps)]
            torch.cuda.synchronize()
            for i in range(reps):
                flush.zero_()
                cev[i][0].record(stream)
                sel()
                cev[i][1].record(stream)
            torch.cuda.synchronize()
            res[name] = med_ms(cev)
        topk_cmp = {"pruned_ms": res["pruned"], "blockwise_ms": res["blockwise"],
                    "blockwise_over_pruned": res["blockwise"] / res["pruned"]}
        del ws_r2, o


    # ---- backward of the routed branch (routing of the forward fixed): dx,
    # and fp32 weight gradients accumulated into resident buffers
    bwd = None
    free_b, _ = torch.cuda.mem_get_info(dev)
    need = 8 * cfg.N * d + 16 * L * d + (64 << 20)
    if free_b > need + (4 << 30):
        f32 = dict(dtype=torch.float32, device=dev)
        g_dW, g_dV = torch.zeros((cfg.N, d), **f32), torch.zeros((cfg.N, d), **f32)
        g_dWr, g_dWc = torch.zeros((cfg.N_r, d), **f32), torch.zeros((cfg.N_c, d), **f32)
        g_dx = torch.empty((L, d), **f32)
        gen = torch.Generator(device=dev)
        gen.manual_seed(11)
        g_dy = torch.randn((L, d), generator=gen, **f32)
        ws_b = torch.empty(omni.omni_routed_bwd_workspace_size(L, d, cfg.N_r, cfg.N_c, cfg.K),
                           dtype=torch.uint8, device=dev)        # with the expert bitmaps

        def bstep():
            omni.omni_routed_bwd(t["x"], t["W"], t["V"], t["W_r"], t["W_c"], L, d, cfg.N_r,
                                 cfg.N_c, cfg.K, rt["idx"], rt["gate"], g_dy, g_dx, g_dW, g_dV,
                                 g_dWr, g_dWc, 0, ws_b)

        for _ in range(3):
            bstep()
        nb = max(3, min(args.steps, 20))
        bev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(nb)]
        torch.cuda.synchronize()
        for i in range(nb):
            flush.zero_()
            bev[i][0].record(stream)
            bstep()
            bev[i][1].record(stream)
        torch.cuda.synchronize()
        if omni.omni_get_device_status(ws_b) != 0:
            raise RuntimeError("device status set in the backward")
        bms = med_ms(bev)
        # read x, dy and the U distinct W, V rows; read-modify-write their fp32
        # dW, dV rows; write dx
        bbytes = 4.0 * d * U + 16.0 * d * U + 2.0 * L * d + 4.0 * L * d + 4.0 * L * d
        bwd = {"ms_per_step": bms, "value": L / (bms * 1e-3), "unit": "tokens/s",
               "steps": nb, "algorithmic_bytes": bbytes,
               "hbm_frac": bbytes / (bms * 1e-3) / (peaks_hbm() * 1e9)}
        del g_dW, g_dV, g_dWr, g_dWc, g_dx, g_dy, ws_b
        torch.cuda.empty_cache()

    # ---- the shared dense MLP beside the routed branch (gated form, hidden
    # width F = mlp_hidden(d)) alone, and the whole layer y = routed(x) + MLP(x)
    F = configs.mlp_hidden(d)
    mw = inputs.make_mlp_weights(d, F, dev, seed=0)
    ws_m = omni.shared_mlp_workspace(L, d, F, dev)

    def mstep():
        omni.omni_shared_mlp_fwd(t["x"], mw["W_g"], mw["W_u"], mw["W_d"], L, d, F, y,
                                 omni.OMNI_Y_ACCUMULATE, ws_m)

    def lstep():
        step()
        mstep()

    res = {}
    for name, fn in (("mlp", mstep), ("layer", lstep)):
        for _ in range(3):
            fn()
        mev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(args.steps)]
        barrier(world)
        torch.cuda.synchronize()
        for i in range(args.steps):
            flush.zero_()
            mev[i][0].record(stream)
            fn()
            mev[i][1].record(stream)
        torch.cuda.synchronize()
        barrier(world)
        res[name] = reduce_max(med_ms(mev), world, dev)
    if omni.omni_get_device_status(ws_m) != 0:
        raise RuntimeError("device status set in the shared MLP")
    mlp_flops = 6.0 * L * d * F                      # x W_g^T, x W_u^T, h W_d^T
    mlp_tflops = mlp_flops / (res["mlp"] * 1e-3) / 1e12
    mlp = {"F": F, "ms_per_step": res["mlp"], "value": job_throughput(world, L, res["mlp"]),
           "unit": "tokens/s", "flops": mlp_flops, "achieved_tflops": mlp_tflops,
           "peak_tflops": measured_peaks()["bf16_tflops"],
           "frac": mlp_tflops / measured_peaks()["bf16_tflops"],
           "layer_ms_per_step": res["layer"],
           "layer_value": job_throughput(world, L, res["layer"])}
    del mw, ws_m

    # ---- end to end: host buffers, copies inside the timed region.  Every
    # step copies its token batch in from pinned host memory and its y out to
    # pinned host memory.  Steps are pipelined over three streams (copy-in of
    # step i+1 and copy-out of step i-1 overlap the layer of step i), with
    # two device buffers each for x and y.  The batches cycle through
    # E2E_BATCHES distinct token draws, so every step routes a new batch and
    # gathers about 1 GB of expert rows (more than L2); no L2 flush.
    x_host = [inputs.make_inputs(cfg, dev, seed=5000 + 64 * rank + b,
                                 with_experts=False)["x"].cpu().pin_memory()
              for b in range(E2E_BATCHES)]
    y_host = [torch.empty((L, d), dtype=torch.float32).pin_memory() for _ in range(2)]
    x_dev = [torch.empty_like(t["x"]) for _ in range(2)]
    y_dev = [torch.empty((L, d), dtype=torch.float32, device=dev) for _ in range(2)]
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    in_done = [torch.cuda.Event() for _ in range(2)]
    cmp_done = [torch.cuda.Event() for _ in range(2)]
    out_done = [torch.cuda.Event() for _ in range(2)]

    def e2e_run(n):
        for i in range(n):
            b = i % 2
            with torch.cuda.stream(s_in):
                if i >= 2:
                    s_in.wait_event(cmp_done[b])      # step i-2 has finished reading x_dev[b]
                x_dev[b].copy_(x_host[i % E2E_BATCHES], non_blocking=True)
                in_done[b].record(s_in)
            stream.wait_event(in_done[b])
            if i >= 2:
                stream.wait_event(out_done[b])        # y_dev[b] of step i-2 is on the host
            omni.omni_routed_fwd(x_dev[b], t["W"], t["V"], t["W_r"], t["W_c"], L, d, cfg.N_r,
                                 cfg.N_c, cfg.K, cfg.B, y_dev[b], None, None, 0, ws)
            cmp_done[b].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(cmp_done[b])
                y_host[b].copy_(y_dev[b], non_blocking=True)
                out_done[b].record(s_out)
        for b in range(min(n, 2)):
            stream.wait_event(out_done[b])

    e2e_run(max(3, args.warmup))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    e0.record(stream)
    s_in.wait_event(e0)
    s_out.wait_event(e0)
    e2e_run(args.steps)
    e1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    e2e_ms = reduce_max(e0.elapsed_time(e1) / args.steps, world, dev)
    if omni.omni_get_device_status(ws) != 0:
        raise RuntimeError("device status set during timing")

    peaks = measured_peaks()
    # algorithmic bytes: the U distinct W and V rows, x read once, y written once
    exp_bytes = 4.0 * d * U + 2.0 * L * d + 4.0 * L * d
    layer_bytes = exp_bytes + 2.0 * d * (cfg.N_r + cfg.N_c)
    layer_flops = 2.0 * L * d * (cfg.N_r + cfg.N_c) + 4.0 * cfg.M * d
    achieved = exp_bytes / (st_expert * 1e-3) / 1e9
    t_roof = max(layer_bytes / (peaks["hbm_gbs"] * 1e9),
                 layer_flops / (peaks["bf16_tflops_sustained"] * 1e12))
    out = {
        "metric": METRIC,
        "value": job_throughput(world, L, ms_max),
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms_max,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded Gaussian inputs and random-init weights of the layer's shapes)",
        "config": config_of(cfg, world),
        "timing": "median of the timed steps' CUDA-event durations (mean in ms_per_step_mean)",
        "ms_per_step_mean": ms_mean,
        "stages_ms": {"router_topk": st_router, "schedule": st_sched,
                      "grouped_expert": st_expert},
        "distinct_experts": U,
        "roofline": {"bound": "hbm", "kernel": "grouped_expert (omni_grouped_expert_fwd)",
                     "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": achieved / peaks["hbm_gbs"],
                     "peak_source": peaks["source"],
                     "traffic": traffic_from_profile(
                         os.path.join(ROOT, "atomic_expert_layer_b200", "csrc", "expert.cu")),
                     "algorithmic_bytes_per_launch": exp_bytes},
        "layer_roofline": {"t_roof_ms": t_roof * 1e3, "t_meas_ms": ms_max,
                           "frac": t_roof * 1e3 / ms_max, "bytes": layer_bytes,
                           "flops": layer_flops},
        "e2e": {"value": job_throughput(world, L, e2e_ms), "unit": "tokens/s",
                "h2d_bytes_per_step": 2 * L * d, "d2h_bytes_per_step": 4 * L * d,
                "ms_per_step": e2e_ms,
                "method": f"omni_routed_fwd on pinned host x/y, copies pipelined over 3 streams, "
                          f"{E2E_BATCHES} distinct token batches cycled, no L2 flush"},
        "gpu_launches": launches_per_step(cfg) * args.steps,
        "graph": graph,
        "ablation": ablation,
        "topk_compare": topk_cmp,
        "backward": bwd,
        "shared_mlp": mlp,
        "clocks": clocks,
    }
    del t, ws, flush
    torch.cuda.empty_cache()
    return out


def profile_stage(args, cfg):
    """Run one stage (or the whole layer) W + K times, synchronising at the end."""
    import atomic_expert_layer_b200 as omni
    dev = torch.device("cuda", 0)
    omni.load()
    t = inputs.make_inputs(cfg, dev, seed=0,
                           with_experts=args.profile_stage in ("expert", "all", "backward"))
    L, d = cfg.L, cfg.d
    rt = omni.router_topk(t["x"], t["W_r"], t["W_c"], cfg.K)
    sc = omni.schedule(rt["idx"], rt["gate"], cfg.N, cfg.B)
    ws = omni.workspace(L, d, cfg.N_r, cfg.N_c, cfg.K, cfg.B, dev)
    y = torch.zeros((L, d), dtype=torch.float32, device=dev)
    if args.profile_stage == "mlp":
        F = configs.mlp_hidden(d)
        mw = inputs.make_mlp_weights(d, F, dev, seed=0)
        ws_m = omni.shared_mlp_workspace(L, d, F, dev)
    if args.profile_stage == "backward":
        f32 = dict(dtype=torch.float32, device=dev)
        g = dict(dx=torch.empty((L, d), **f32), dW=torch.zeros((cfg.N, d), **f32),
                 dV=torch.zeros((cfg.N, d), **f32), dW_r=torch.zeros((cfg.N_r, d), **f32),
                 dW_c=torch.zeros((cfg.N_c, d), **f32))
        dy = torch.ones((L, d), **f32)
        ws = torch.empty(omni.omni_routed_bwd_workspace_size(L, d, cfg.N_r, cfg.N_c, cfg.K),
                         dtype=torch.uint8, device=dev)
    for _ in range(args.warmup + args.steps):
        if args.profile_stage == "backward":
            omni.omni_routed_bwd(t["x"], t["W"], t["V"], t["W_r"], t["W_c"], L, d, cfg.N_r,
                                 cfg.N_c, cfg.K, rt["idx"], rt["gate"], dy, g["dx"], g["dW"],
                                 g["dV"], g["dW_r"], g["dW_c"], 0, ws)
        elif args.profile_stage == "mlp":
            omni.omni_shared_mlp_fwd(t["x"], mw["W_g"], mw["W_u"], mw["W_d"], L, d, F, y,
                                     omni.OMNI_Y_ACCUMULATE, ws_m)
        elif args.profile_stage == "router":
            omni.omni_router_topk(t["x"], t["W_r"], t["W_c"], L, d, cfg.N_r, cfg.N_c, cfg.K,
                                  rt["p_r"], rt["p_c"], rt["idx"], rt["score"], rt["gate"], 0, ws)
        elif args.profile_stage == "schedule":
            omni.omni_schedule(rt["idx"], rt["gate"], L, cfg.K, cfg.N, cfg.B, sc["task_token"],
                               sc["task_expert"], sc["task_gate"], sc["group_offsets"],
                               sc["group_counts"], sc["active_groups"], sc["num_active"],
                               sc["num_distinct"], ws)
        elif args.profile_stage == "expert":
            omni.omni_grouped_expert_fwd(t["x"], t["W"], t["V"], L, d, cfg.K, cfg.N, cfg.B,
                                         sc["task_token"], sc["task_expert"], sc["task_gate"],
                                         sc["group_offsets"], sc["active_groups"],
                                         sc["num_active"], y, omni.OMNI_Y_ACCUMULATE, ws)
        else:
            omni.omni_routed_fwd(t["x"], t["W"], t["V"], t["W_r"], t["W_c"], L, d, cfg.N_r,
                                 cfg.N_c, cfg.K, cfg.B, y, None, None, 0, ws)
    torch.cuda.synchronize()
    status = omni.omni_get_device_status(ws)
    if status != 0:
        raise RuntimeError(f"device status {status}")
    print(f"profile-stage {args.profile_stage} {cfg.name}: {args.warmup + args.steps} runs ok")


def timeline(args, cfg):
    """In-stream kernel timeline of omni_routed_fwd (CUPTI through
    torch.profiler): start and end of every library launch of the last step,
    relative to the step's first kernel.  With programmatic dependent launch a
    kernel's CTAs start before its predecessor ends, so a kernel's cost is the
    gap between consecutive end times ("end delta")."""
    import atomic_expert_layer_b200 as omni
    from torch.profiler import profile, ProfilerActivity
    dev = torch.device("cuda", 0)
    omni.load()
    t = inputs.make_inputs(cfg, dev, seed=0)
    L, d = cfg.L, cfg.d
    ws = omni.workspace(L, d, cfg.N_r, cfg.N_c, cfg.K, cfg.B, dev)
    y = torch.empty((L, d), dtype=torch.float32, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)

    def step():
        omni.omni_routed_fwd(t["x"], t["W"], t["V"], t["W_r"], t["W_c"], L, d, cfg.N_r, cfg.N_c,
                             cfg.K, cfg.B, y, None, None, 0, ws)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    with profile(activities=[ProfilerActivity.CUDA]) as prof:
        for _ in range(args.steps):
            flush.zero_()
            step()
        torch.cuda.synchronize()
    rows = sorted((e.time_range.start, e.time_range.end, e.name) for e in prof.events()
                  if e.device_type == torch.autograd.DeviceType.CUDA)
    steps, cur = [], None
    for a, b, n in rows:
        if "router_gemm" in n or "router_small" in n or "decode_fused" in n:   # a step's first kernel
            cur = []
            steps.append(cur)
        if cur is not None and "omni::" in n:
            cur.append((a, b, n))
    spans = [st[-1][1] - st[0][0] for st in steps]
    last = steps[-1]
    t0, prev_end = last[0][0], last[0][0]
    print(f"{'kernel':44s} {'start us':>9s} {'end us':>9s} {'end delta':>10s}")
    for a, b, n in last:
        m = re.search(r"(\w+(?:<[\d, ]+>)?)\((?!anonymous)", n)    # the kernel's own name
        short = (m.group(1) if m else n)[:44]
        print(f"{short:44s} {a - t0:9.2f} {b - t0:9.2f} {b - prev_end:10.2f}")
        prev_end = max(prev_end, b)
    print(f"first kernel start to last kernel end, per step (us): "
          f"{', '.join(f'{x:.1f}' for x in spans)}")


# ------------------------------------------------------- oracle (CPU) arm
def time_oracle(cfg, n_tokens: int, seed: int = 0, repeats: int = 1) -> dict:
    """Time the CPU oracle on the first n_tokens of the workload (router,
    top-K, gates, schedule, expert stage), `repeats` times over the same
    host arrays; inputs are made on the GPU if one is present, else on the
    CPU, and only the expert rows the sample uses are copied to the host
    (copying is not timed)."""
    import oracle
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    t = inputs.make_inputs(cfg, dev, seed=seed)
    x = inputs.to_u16(t["x"][:n_tokens])
    Wr, Wc = inputs.to_u16(t["W_r"]), inputs.to_u16(t["W_c"])
    secs = 0.0
    Wu = Vu = idx_local = None
    for _ in range(repeats):
        t0 = time.perf_counter()
        p_r, p_c = oracle.router_logprobs(x, Wr, Wc)
        idx, score, gate = oracle.topk_from_logprobs(p_r, p_c, cfg.K)
        t1 = time.perf_counter()
        if Wu is None:
            tok = torch.as_tensor(idx.astype(np.int64), device=dev)
            uniq, inv = torch.unique(tok, return_inverse=True)
            Wu, Vu = inputs.to_u16(t["W"][uniq]), inputs.to_u16(t["V"][uniq])
            idx_local = inv.to(torch.int32).cpu().numpy()
        t2 = time.perf_counter()
        oracle.schedule(idx, gate, cfg.N, cfg.B)
        oracle.expert_fwd_token_centric(x, Wu, Vu, idx_local, gate)
        t3 = time.perf_counter()
        secs += (t1 - t0) + (t3 - t2)
    del t
    return {"seconds": secs, "tokens": n_tokens * repeats, "value": n_tokens * repeats / secs,
            "cores": oracle.max_threads()}


def cpu_baseline(cfg, budget_s: float = 25.0) -> dict:
    """The oracle on a bounded sample: the first n tokens (n sized to about
    budget_s of CPU work), or all L tokens repeated until about budget_s."""
    probe = min(cfg.L, 64)
    r = time_oracle(cfg, probe)
    per_tok = r["seconds"] / probe
    n = int(max(probe, min(cfg.L, budget_s / max(per_tok, 1e-9))))
    reps = 1
    if n == cfg.L:
        reps = int(max(1, min(20, budget_s // max(per_tok * cfg.L, 1e-9))))
    if n > probe or reps > 1:
        r = time_oracle(cfg, n, repeats=reps)
    what = (f"first {n} of {cfg.L} tokens" if n < cfg.L else f"all {cfg.L} tokens x {reps} runs")
    return {"value": r["value"], "unit": "tokens/s", "cores": r["cores"], "kind": "oracle",
            "sample": f"{what} of {cfg.name}, whole routed branch in the C oracle (fp64), "
                      f"{r['seconds']:.1f} s"}


def run_reference(args, cfg, world, rank):
    if rank != 0:
        return None
    n = min(cfg.L, 512)
    for _ in range(args.warmup):
        time_oracle(cfg, min(n, 16))
    secs, toks, cores = 0.0, 0, 1
    for _ in range(args.steps):
        r = time_oracle(cfg, n)
        secs += r["seconds"]
        toks += r["tokens"]
        cores = r["cores"]
    value = toks / secs
    sample = (f"first {n} of {cfg.L} tokens of {cfg.name} per step, whole routed branch in "
              f"the C oracle (fp64)")
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * cfg.L / value, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_of(cfg, world),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


# -------------------------------------------------------------------- main
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", default=configs.HEADLINE.name,
                    help="workload name: " + ", ".join(c.name for c in configs.ALL))
    ap.add_argument("--impl", choices=["omni", "reference"], default="omni")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--profile-stage", choices=["router", "schedule", "expert", "all", "backward", "mlp"],
                    help="run only this stage W + K times (for profiler captures; no JSON)")
    ap.add_argument("--timeline", action="store_true",
                    help="print the in-stream kernel timeline of the last of K steps (no JSON)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    cfg = configs.BY_NAME[args.config]
    world, rank, local = dist_env()
    if world > 1 and args.impl == "omni":
        import torch.distributed as dist
        from datetime import timedelta
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=timedelta(seconds=120))
    try:
        if args.profile_stage:
            profile_stage(args, cfg)
            return
        if args.timeline:
            timeline(args, cfg)
            return
        if args.impl == "reference":
            out = run_reference(args, cfg, world, rank)
        else:
            out = run_omni(args, cfg, world, rank, local)
            if rank == 0 and world == 1 and not args.no_cpu_baseline:
                out["cpu_baseline"] = cpu_baseline(cfg)
        if rank == 0 and out is not None:
            print(json.dumps(out), flush=True)
    finally:
        if world > 1 and args.impl == "omni":
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
