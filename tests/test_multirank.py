"""The benchmark's multi-rank plumbing on CPU: two gloo ranks, max-over-ranks timing and the
whole-job throughput that rank 0 reports (the same helpers the GPU run calls over NCCL)."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank: int, world: int, port: int, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        own = [0.5, 2.0][rank]                       # rank 1 is the slow one
        dist.barrier()
        slowest = bench.max_over_ranks(own, world, torch.device("cpu"))
        e2e = bench.max_over_ranks([3.0, 1.0][rank], world, torch.device("cpu"))
        out.put((rank, slowest, e2e, bench.job_tokens_per_s(world, 131072, 5, slowest)))
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_two_gloo_ranks_take_the_slowest_time():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=90) for _ in range(world))
    for p in procs:
        p.join(timeout=30)
        assert p.exitcode == 0
    for rank, slowest, e2e, value in res:
        assert slowest == 2.0 and e2e == 3.0
        assert value == pytest.approx(2 * 131072 * 5 / 2.0)


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks(1.5, 1, torch.device("cpu")) == 1.5
    assert bench.job_tokens_per_s(1, 4096, 2, 0.5) == 4096 * 2 / 0.5
