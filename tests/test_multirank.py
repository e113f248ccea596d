"""The N>1 bench path on CPU: two gloo ranks, each a replica with its own
time; the job time is the maximum over ranks and the throughput sums the
replicas' work over that time (no data-path collective)."""

import os
import socket

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank: int, world: int, port: int, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        my_time = [0.40, 0.55][rank]          # seconds for this replica's steps
        t = bench.reduce_max(my_time, world, torch.device("cpu"))
        value = bench.aggregate(1000.0, t, world)
        q.put((rank, t, value))
    finally:
        dist.destroy_process_group()


def test_two_rank_aggregation():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    for rank, t, value in res:
        assert t == 0.55                      # every rank sees the slowest rank's time
        assert abs(value - 2 * 1000.0 / 0.55) < 1e-9


def test_single_rank_is_identity():
    assert bench.reduce_max(0.3, 1, None) == 0.3
    assert bench.aggregate(10.0, 2.0, 1) == 5.0
