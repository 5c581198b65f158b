"""Host logic of the multi-GPU bench path (independent replicas, one per rank),
run as two gloo ranks on the CPU: the timed region's duration is the max over
ranks and the reported value aggregates every rank's tokens."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = bench.max_over_ranks(10.0 + 5.0 * rank, dist, torch.device("cpu"))
        ws, r, local = bench.dist_info()
        out[rank] = (ms, ws, r, local, bench.job_throughput(ws, 1000, ms))
    finally:
        dist.destroy_process_group()


def test_two_rank_timing_is_max_over_ranks():
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(2, port, out), nprocs=2, join=True)
        res = dict(out)
    for rank in (0, 1):
        ms, ws, r, local, tput = res[rank]
        assert ms == 15.0 and ws == 2 and r == rank and local == rank
        assert tput == pytest.approx(2 * 1000 / 15e-3)


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks(3.5, None, None) == 3.5
    assert bench.job_throughput(1, 100, 2.0) == pytest.approx(50000.0)
