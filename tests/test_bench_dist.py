"""The benchmark's multi-rank host logic on CPU: two gloo ranks agree on the max
time and on the whole-job throughput (no GPU needed)."""
from __future__ import annotations

import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    local_ms = [12.5, 20.0][rank]
    ms = bench.reduce_max(dist, local_ms, torch.device("cpu"))
    value = bench.tokens_per_second(world, 64, 100, ms)
    q.put((rank, ms, value))
    dist.barrier()
    dist.destroy_process_group()


def test_two_gloo_ranks_max_time_and_throughput():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[1] for r in res] == [20.0, 20.0]                 # max over ranks
    assert res[0][2] == res[1][2] == pytest.approx(2 * 64 * 100 / 0.020)


def test_single_process_helpers():
    import bench
    assert bench.reduce_max(None, 3.0, None) == 3.0
    assert bench.tokens_per_second(1, 64, 1000, 250.0) == pytest.approx(256000.0)
