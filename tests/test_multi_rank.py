"""The benchmark's multi-rank plumbing on CPU: two gloo ranks, each an independent replica, the reported time
is the maximum over ranks, and every rank takes the same collective steps."""
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import bench
    ws, r, local = bench.dist_setup()
    assert (ws, r) == (world, rank)
    bench.barrier(ws)
    t = bench.max_over_ranks(10.0 + 5.0 * rank, ws)      # each replica's own elapsed time
    # throughput over all ranks divides the units of every rank by the slowest rank's time
    value = ws * 1000 / (t / 1e3)
    results[rank] = (t, value)
    import torch.distributed as dist
    dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_two_gloo_ranks_report_the_slowest_rank():
    world, port = 2, _free_port()
    results = mp.Manager().dict()
    mp.spawn(_worker, args=(world, port, results), nprocs=world, join=True)
    assert results[0] == results[1]
    t, value = results[0]
    assert t == 15.0
    assert value == pytest.approx(2 * 1000 / 0.015)


def test_single_rank_needs_no_process_group():
    import bench
    assert bench.max_over_ranks(3.5, 1) == 3.5
    bench.barrier(1)
    assert not torch.distributed.is_initialized()
