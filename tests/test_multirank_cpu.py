"""Multi-rank host logic of bench.py on CPU with gloo, world size 2.

The attention path shards by (batch, head) with no exchange step, so the
only cross-rank operations are the barrier and the max-over-ranks timing
reduction; both are exercised here without a GPU.
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from seeded_inputs import make_qkv, workload


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        local_ms = 10.0 + 5.0 * rank
        job_ms = bench.max_over_ranks(local_ms, dist, torch.device("cpu"))
        w = workload(0)
        q, _, _ = make_qkv(1, 1, 8, 8, 64, "fp16", bench.rank_seed(w, rank))
        dist.barrier()
        out[rank] = (job_ms, float(q.float().sum()))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_rank_slices():
    world = 2
    port = _free_port()
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
    assert out[0][0] == out[1][0] == 15.0          # slowest rank sets the job time
    assert out[0][1] != out[1][1]                   # each rank draws its own slice


def test_job_throughput_is_whole_job():
    w = workload(1)
    one = bench.job_tflops(1, w.flops, 10, 1.0)
    two = bench.job_tflops(2, w.flops, 10, 1.0)
    assert two == pytest.approx(2 * one)
    assert bench.max_over_ranks(3.5, None, None) == 3.5
