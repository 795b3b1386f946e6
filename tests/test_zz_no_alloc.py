"""The grouped expert call that needs no workspace.

Callers that cannot allocate device memory when they run the layer use
omni_grouped_expert_fwd_noalloc, whose scratch is a fixed array inside the
library.  It must give the same y as the workspace call, call after call
(the array is shared and keeps the previous call's contents), and refuse
sizes beyond its array.  This file is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import atomic_expert_layer_b200 as omni
from atomic_expert_layer_b200 import _lib, configs, inputs

from _parity import check_y, host


def test_noalloc_rejects_sizes_beyond_its_array():
    lib = _lib.load()
    fake = ctypes.c_void_p(1 << 20)
    # 16385 tokens: above the array's token limit (host check, nothing enqueued)
    assert lib.omni_grouped_expert_fwd_noalloc(fake, fake, fake, 16385, 256, 4, 4096, 32, fake,
                                               fake, fake, fake, fake, fake, fake, 0, None) == -2
    # 4096 tokens x 128 experts = 524288 tasks: above the task limit
    assert lib.omni_grouped_expert_fwd_noalloc(fake, fake, fake, 4096, 256, 128, 4096, 32, fake,
                                               fake, fake, fake, fake, fake, fake, 0, None) == -2
    assert lib.omni_grouped_expert_fwd_noalloc(None, fake, fake, 16, 256, 4, 4096, 32, fake,
                                               fake, fake, fake, fake, fake, fake, 0, None) == -1


@pytest.mark.gpu
@pytest.mark.parametrize("cfg", [configs.TINY,
                                 configs.LayerConfig("d1024", 2048, 1024, 256, 256, 64, 128)],
                         ids=lambda c: c.name)
def test_noalloc_matches_workspace_call_twice(cfg):
    dev = "cuda"
    t = inputs.make_inputs(cfg, dev, seed=7)
    rt = omni.router_topk(t["x"], t["W_r"], t["W_c"], cfg.K)
    sched = omni.schedule(rt["idx"], rt["gate"], cfg.N, cfg.B)
    y_ws = omni.grouped_expert_fwd(t["x"], t["W"], t["V"], sched, cfg.K, cfg.B)
    for _ in range(2):                      # the shared array is reused as is
        y = torch.full((cfg.L, cfg.d), float("nan"), dtype=torch.float32, device=dev)
        omni.omni_grouped_expert_fwd_noalloc(
            t["x"], t["W"], t["V"], cfg.L, cfg.d, cfg.K, cfg.N, cfg.B, sched["task_token"],
            sched["task_expert"], sched["task_gate"], sched["group_offsets"],
            sched["active_groups"], sched["num_active"], y, 0)
        torch.cuda.synchronize()
        check_y(host(y), host(y_ws).astype(np.float64), "noalloc vs workspace call")
    # and both agree with the CPU oracle on the same routing (sampled rows)
    toks = np.arange(0, cfg.L, max(1, cfg.L // 16))
    u = {k: host(v) for k, v in t.items()}
    y_ref = oracle.expert_fwd_token_centric(u["x"], u["W"], u["V"], host(rt["idx"]),
                                            host(rt["gate"]), tokens=toks)
    check_y(host(y)[toks], y_ref)


@pytest.mark.gpu
def test_noalloc_reports_bad_schedule_through_its_own_status_word():
    # a task whose expert id is out of range: the call clamps it (every access
    # stays in bounds) and records OMNI_DEV_BAD_SCHEDULE in the array's status
    # word, which only omni_noalloc_get_device_status can read
    cfg = configs.TINY
    dev = "cuda"
    t = inputs.make_inputs(cfg, dev, seed=7)
    rt = omni.router_topk(t["x"], t["W_r"], t["W_c"], cfg.K)
    sched = omni.schedule(rt["idx"], rt["gate"], cfg.N, cfg.B)
    y = torch.zeros((cfg.L, cfg.d), dtype=torch.float32, device=dev)

    def call(task_expert):
        omni.omni_grouped_expert_fwd_noalloc(
            t["x"], t["W"], t["V"], cfg.L, cfg.d, cfg.K, cfg.N, cfg.B, sched["task_token"],
            task_expert, sched["task_gate"], sched["group_offsets"], sched["active_groups"],
            sched["num_active"], y, 0)

    omni.omni_noalloc_get_device_status()           # clear whatever an earlier call left
    bad = sched["task_expert"].clone()
    bad[5] = cfg.N                                  # one past the last expert
    call(bad)
    assert omni.omni_noalloc_get_device_status() == 3    # OMNI_DEV_BAD_SCHEDULE
    assert omni.omni_noalloc_get_device_status() == 0    # the read cleared it
    call(sched["task_expert"])                      # a clean call leaves it clear
    assert omni.omni_noalloc_get_device_status() == 0
