"""The multi-GPU path is replicas only: ranks share no data, and the bench reports the slowest
rank's time. These world-size-2 checks run the same reduction on CPU ranks over gloo."""
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


def _rank(rank: int, world: int, port: int, q) -> None:
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # each replica times a different step length; all must agree on the max
        ms = [120.0, 180.5][rank]
        got = bench.max_over_ranks(ms, world, torch.device("cpu"))
        value = bench.replica_throughput(world, 10, 126.6e12, got)
        q.put((rank, got, value))
    finally:
        dist.destroy_process_group()


def test_two_replicas_report_the_slowest_rank():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[1] for r in res] == [180.5, 180.5]
    expected = 2 * 10 * 126.6e12 / 0.1805 / 1e12
    assert all(abs(r[2] - expected) < 1e-9 * expected for r in res)


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks(3.5, 1, None) == 3.5
    assert bench.replica_throughput(1, 4, 1e12, 1000.0) == pytest.approx(4.0)
