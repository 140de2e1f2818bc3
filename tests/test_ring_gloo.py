"""Ring attention ("HunyuanVideo 模型结构与数学原理" §9.2) on CPU: world_size 2
and 3 ``gloo`` ranks run the ring of ``joint_full_attention_b200/ring.py`` with
the float64 oracle's block attention and merge standing in for the GPU
kernels, and must reproduce the single-process oracle output (the merges
reorder float64 sums only)."""

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


def _problem(grid, text_len, batch, heads, seed):
    n = grid[0] * grid[1] * grid[2]
    rng = np.random.default_rng(seed)
    return tuple(rng.standard_normal((batch, n + text_len, heads, 128)) for _ in range(3))


def _block_oracle(q, k, v, grid, q_video, q_pos0, k_video, k_pos0, kv_len):
    from oracle import hv_oracle as O
    b_sz, sq, heads, d = q.shape
    o = np.empty((b_sz, sq, heads, d))
    lse = np.empty((b_sz, sq, heads))
    for b in range(b_sz):
        for h in range(heads):
            o[b, :, h], lse[b, :, h] = O.joint_attention_block(q[b, :, h].numpy(), k[b, :, h].numpy(),
                                                               v[b, :, h].numpy(), grid, q_video, q_pos0, k_video,
                                                               k_pos0, int(kv_len[b]))
    return torch.from_numpy(o), torch.from_numpy(lse)


def _merge_oracle(acc_o, acc_lse, o, lse, out=None):
    from oracle import hv_oracle as O
    d = acc_o.shape[-1]
    merged, m_lse = O.merge_blocks([acc_o.reshape(-1, d).numpy(), o.reshape(-1, d).numpy()],
                                   [acc_lse.reshape(-1).numpy(), lse.reshape(-1).numpy()])
    acc_o.copy_(torch.from_numpy(merged).view(acc_o.shape))
    acc_lse.copy_(torch.from_numpy(m_lse).view(acc_lse.shape))
    if out is not None:
        out.copy_(acc_o)


def _rank(rank, world, port, grid, text_len, valid, heads, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, str(ROOT))
    from joint_full_attention_b200 import ring as R
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        q, k, v = (torch.from_numpy(x) for x in _problem(grid, text_len, len(valid), heads, seed=9))
        n = grid[0] * grid[1] * grid[2]
        start, cnt = R.ring_chunks(n, world)[rank]
        run = [x[:, start:start + cnt].contiguous() for x in (q, k, v)]
        text = [x[:, n:].contiguous() for x in (q, k, v)]
        vid, txt = R.ring_attention(*run, *text, grid, valid, block=_block_oracle, merge=_merge_oracle)
        results[rank] = (vid.numpy(), txt.numpy(), start, cnt)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,grid,text_len,valid,heads", [
    (2, (2, 3, 5), 6, [4, 0], 2),      # a sample with no valid text key
    (3, (1, 1, 31), 6, [6], 2),        # runs of 10, 10 and 11 tokens
    (2, (1, 4, 2), 0, [0], 1),         # no text
])
def test_ring_matches_single_process(world, grid, text_len, valid, heads):
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
    q, k, v = _problem(grid, text_len, len(valid), heads, seed=9)
    ref = O.joint_attention(q, k, v, grid, text_len, valid)
    n = grid[0] * grid[1] * grid[2]
    for r in range(world):
        vid, txt, start, cnt = results[r]
        np.testing.assert_allclose(vid, ref[:, start:start + cnt], rtol=0, atol=1e-12)
        np.testing.assert_allclose(txt, ref[:, n:], rtol=0, atol=1e-12)


def test_ring_chunks():
    sys.path.insert(0, str(ROOT))
    from joint_full_attention_b200 import ring as R
    assert R.ring_chunks(31, 3) == [(0, 10), (10, 10), (20, 11)]
    assert R.ring_chunks(118800, 7)[-1] == (101828, 16972)     # any world size works, e.g. 7
    with pytest.raises(ValueError):
        R.ring_chunks(2, 3)
