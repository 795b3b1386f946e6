"""Host logic of the N > 1 benchmark path, run as two gloo ranks on the CPU.

The layer shards by token batch with no data-path collective, so what the
multi-rank path adds is the barrier around the timed region, the max over
ranks of the measured time, the whole-job throughput and each replica's own
token seed.  These run here exactly as they do under torchrun with NCCL.
"""
import json
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    sys.path.insert(0, ROOT)
    import bench
    from atomic_expert_layer_b200 import configs
    from datetime import timedelta

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        w, r, _ = bench.dist_env()
        bench.barrier(world)
        ms = 1.0 + 0.25 * rank                       # per-rank "measured" time
        ms_max = bench.reduce_max(ms, world, torch.device("cpu"))
        bench.barrier(world)
        ref = bench.run_reference(None, configs.TINY, world, rank) if rank != 0 else "rank0"
        res = {"env": [w, r], "ms_max": ms_max,
               "value": bench.job_throughput(world, 4096, ms_max),
               "seed": bench.replica_seed(rank), "ref": ref}
    finally:
        dist.destroy_process_group()
    with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
        json.dump(res, f)


def test_two_replicas_barrier_and_max_timing(tmp_path):
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       join=True, start_method="spawn")
    res = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(world)]
    for r, d in enumerate(res):
        assert d["env"] == [world, r]
        assert d["ms_max"] == pytest.approx(1.25)               # the slowest rank's time
        assert d["value"] == pytest.approx(2 * 4096 / 1.25e-3)  # all ranks' tokens / that time
    assert res[0]["seed"] != res[1]["seed"]                      # each replica routes its own batch
    assert res[1]["ref"] is None                                 # the oracle arm runs on rank 0 only
