"""Multi-process host logic of the benchmark on CPU: two gloo ranks.

The attention call does not shard (replicas only); what spans processes is
bench.py's aggregation: the slowest rank's time and the whole-job throughput
of all ranks. Two ranks with different local times must agree on both.
"""

from __future__ import annotations

import os
import socket
import sys
from pathlib import Path

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = Path(__file__).resolve().parent.parent


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank: int, world: int, port: int, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, str(ROOT))
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_ms = [200.0, 250.0][rank]
        ms, value = bench.replica_throughput(local_ms, 1.0e14, world)
        bench.barrier(world)
        results[rank] = (ms, value)
    finally:
        dist.destroy_process_group()


def test_two_replicas_agree_on_slowest_rank():
    ctx = mp.get_context("spawn")
    manager = ctx.Manager()
    results = manager.dict()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, results)) for r in range(2)]
    for pr in procs:
        pr.start()
    for pr in procs:
        pr.join(timeout=120)
        assert pr.exitcode == 0
    assert results[0] == results[1]
    ms, value = results[0]
    assert ms == 250.0
    assert value == pytest.approx(2 * 1.0e14 / 0.25 / 1e12)


def test_single_process_needs_no_group():
    sys.path.insert(0, str(ROOT))
    import bench
    assert bench.replica_throughput(100.0, 2.0e12, 1) == (100.0, pytest.approx(20.0))
