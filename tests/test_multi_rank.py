"""Host side of the multi-GPU benchmark mode on CPU (gloo, world size 2):
replicas get distinct seeded sequences of the same workload shape, and the job
time is the maximum over ranks.  No data-path collective exists: the layer
prefill of one sequence runs on one GPU."""
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from sparse_attention_long_block_b200.inputs import generate


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        wl = bench.replica_workload("tiny_fp32_1k", rank)
        x = generate(wl)
        ms = 10.0 + rank * 5.0  # stand-in device times
        job = bench.max_over_ranks(ms, torch.device("cpu"))
        out[rank] = (wl.seed, float(x["q"][5, 1, 3]), job, wl.n)
    finally:
        dist.destroy_process_group()


def test_replicas_are_distinct_and_time_is_max_over_ranks():
    world = 2
    port = _free_port()
    # the manager process is spawned too: this process may already run
    # threads (the oracle's OpenMP pool), and forking it could deadlock
    manager = mp.get_context("spawn").Manager()
    out = manager.dict()
    mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
    seeds = {out[r][0] for r in range(world)}
    assert len(seeds) == world                        # distinct sequences
    assert out[0][1] != out[1][1]
    assert out[0][2] == out[1][2] == 15.0             # slowest rank defines the time
    assert out[0][3] == out[1][3]                     # same per-rank work (weak scaling)
