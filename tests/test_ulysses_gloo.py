"""Ulysses sequence parallelism ("HunyuanVideo 模型结构与数学原理" §9.2) on CPU:
world_size 2 and 3 ``gloo`` ranks run the exchange logic of
``joint_full_attention_b200/ulysses.py`` around the float64 oracle (standing in
for the GPU kernel, which these CPU tests cannot run) and must reproduce the
single-process oracle output exactly: the exchange only moves data, and the
oracle computes every head independently."""

from __future__ import annotations

import os
import socket
import sys
from pathlib import Path

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = Path(__file__).resolve().parent.parent


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _problem(grid, text_len, valid, heads, seed):
    n = grid[0] * grid[1] * grid[2]
    rng = np.random.default_rng(seed)
    q, k, v = (rng.standard_normal((len(valid), n + text_len, heads, 128)) for _ in range(3))
    return q, k, v


def _oracle_attn(q, k, v, grid, text_len, text_valid):
    from oracle import hv_oracle as O
    return torch.from_numpy(O.joint_attention(q.numpy(), k.numpy(), v.numpy(), grid, text_len, text_valid))


def _rank(rank, world, port, grid, text_len, valid, heads, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, str(ROOT))
    from joint_full_attention_b200 import ulysses as U
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        q, k, v = (torch.from_numpy(x) for x in _problem(grid, text_len, valid, heads, seed=7))
        layout = U.ulysses_layout(grid, heads, world)
        n = layout.n_video
        shard = [U.shard_video(x[:, :n], layout, rank) for x in (q, k, v)]
        text = [x[:, n:].contiguous() for x in (q, k, v)]
        vid_out, txt_out = U.ulysses_attention(*shard, *text, grid, valid, attn=_oracle_attn)
        results[rank] = (vid_out.numpy(), txt_out.numpy(), layout.shard_positions(rank).numpy(), layout.axis)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,grid,text_len,valid,heads", [
    (2, (2, 6, 4), 5, [3, 5], 4),      # slabs of H'/2 rows
    (3, (2, 6, 4), 5, [0, 2], 6),
    (2, (2, 5, 6), 7, [7], 4),         # H'/2 = 5 odd: slabs of W'/2 columns
    (2, (1, 4, 2), 0, [0], 2),         # no text
])
def test_ulysses_matches_single_process(world, grid, text_len, valid, heads):
    from oracle import hv_oracle as O
    ctx = mp.get_context("spawn")
    manager = ctx.Manager()
    results = manager.dict()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, world, port, grid, text_len, valid, heads, results))
             for r in range(world)]
    for pr in procs:
        pr.start()
    for pr in procs:
        pr.join(timeout=300)
        assert pr.exitcode == 0
    q, k, v = _problem(grid, text_len, valid, heads, seed=7)
    ref = O.joint_attention(q, k, v, grid, text_len, valid)
    n = grid[0] * grid[1] * grid[2]
    for r in range(world):
        vid_out, txt_out, pos, axis = results[r]
        assert axis == (1 if grid[1] % world == 0 else 2)
        np.testing.assert_array_equal(vid_out, ref[:, pos])
        np.testing.assert_array_equal(txt_out, ref[:, n:])


def test_ulysses_layout_rules():
    sys.path.insert(0, str(ROOT))
    from joint_full_attention_b200 import ulysses as U
    # the pages' example: 7 ranks divide neither 45 nor 80 of the 720p grid
    with pytest.raises(ValueError):
        U.ulysses_layout((33, 45, 80), 24, 7)
    with pytest.raises(ValueError):
        U.ulysses_layout((5, 34, 60), 24, 7)
    # the Ulysses degree must divide the 24 heads
    with pytest.raises(ValueError):
        U.ulysses_layout((33, 45, 80), 24, 16)
    lay = U.ulysses_layout((33, 45, 80), 24, 8)      # 45 % 8 != 0, 80 % 8 == 0
    assert lay.axis == 2 and lay.shard_tokens == 118800 // 8 and lay.heads_per_rank == 3
    lay = U.ulysses_layout((33, 45, 80), 24, 3)
    assert lay.axis == 1
    # the shards tile the video tokens exactly once
    lay = U.ulysses_layout((3, 4, 6), 6, 2)
    allpos = torch.cat([lay.shard_positions(r) for r in range(2)])
    assert torch.equal(torch.sort(allpos).values, torch.arange(72))
    order = lay.gather_order()
    assert torch.equal(allpos[order], torch.arange(72))
