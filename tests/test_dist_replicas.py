"""Multi-rank host logic of the benchmark, on CPU with the gloo backend (world size 2).

The path shards into independent replicas (one sequence stack per rank, no data-path
collective). What has to be right across ranks is the bookkeeping: every rank draws its own
seeded inputs, the job time is the slowest rank's, and the whole-job throughput counts every
rank's tokens over that time.
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from sliding_window_attention_chunked_b200 import workloads as wl


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        ms_local = 100.0 + 37.5 * rank               # rank 1 is the slow one
        ms = bench.max_over_ranks(ms_local)
        value = bench.job_throughput(131072, 5, world, ms)
        q = wl.stack_layer_inputs(0, 1, 2, 64, 16, 16, seed_base=bench.replica_seed_base(rank))[0]
        gathered = [torch.zeros_like(q.float()) for _ in range(world)]
        dist.all_gather(gathered, q.float())
        out[rank] = (ms, value, bool(torch.equal(gathered[0], gathered[1])))
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_two_gloo_ranks_agree_on_max_time_and_throughput():
    world = 2
    manager = mp.Manager()
    out = manager.dict()
    mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    slow = 100.0 + 37.5
    for rank in range(world):
        ms, value, same_inputs = out[rank]
        assert ms == slow                                 # both ranks report the slowest rank
        assert value == pytest.approx(131072 * 5 * world / (slow / 1e3))
        assert not same_inputs                            # replicas draw different inputs


def test_single_process_helpers_without_a_process_group():
    assert bench.max_over_ranks(12.5) == 12.5
    assert bench.job_throughput(1000, 4, 1, 2000.0) == pytest.approx(2000.0)
    assert bench.replica_seed_base(0) != bench.replica_seed_base(1)
