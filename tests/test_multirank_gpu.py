"""Ulysses and ring attention ("HunyuanVideo 模型结构与数学原理" §9.2) with the
real kernels on several ranks: world_size 2 and 3 ``gloo`` processes, all on
cuda:0. The exchanges (all-to-all, all-gather, ring send/recv) run on CPU
tensors through gloo; every attention step of every rank runs in the library
through the C ABI (``hv_attn_forward`` for Ulysses, ``hv_attn_forward_block``
and ``hv_attn_merge`` for ring attention). No kernel waits on another rank.
The gathered output is compared element by element with the float64 oracle's
joint attention of the whole problem: max |Δ| <= 2e-2, mean |Δ| <= 2e-3.

Values cross the exchanges as float32 holding exact bf16 numbers, so the
exchange itself changes nothing."""

from __future__ import annotations

import os
import socket
import sys
from pathlib import Path

import numpy as np
import pytest
import torch

ROOT = Path(__file__).resolve().parent.parent
MAX_ABS = 2e-2
MEAN_ABS = 2e-3

pytestmark = pytest.mark.gpu


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _problem(grid, text_len, valid, heads, seed):
    sys.path.insert(0, str(ROOT))
    from joint_full_attention_b200 import workloads as W
    wl = W.Workload("multirank", "multirank", len(valid), heads, tuple(grid), text_len, valid=tuple(valid))
    inp = W.make_inputs(wl, seed=seed)
    return tuple(W.bf16_bits_to_f32(inp[n]) for n in ("q", "k", "v"))


def _gpu_attn(q, k, v, grid, text_len, text_valid):
    from joint_full_attention_b200 import hvattn as H
    dev = torch.device("cuda", 0)
    qd, kd, vd = (x.to(dev, torch.bfloat16).contiguous() for x in (q, k, v))
    o = H.attn_forward(qd, kd, vd, grid, text_len, text_valid)
    torch.cuda.synchronize(dev)
    assert H.last_device_error() == 0
    return o.float().cpu()


def _gpu_block(q, k, v, grid, q_video, q_pos0, k_video, k_pos0, kv_len):
    from joint_full_attention_b200 import hvattn as H
    dev = torch.device("cuda", 0)
    qd, kd, vd = (x.to(dev, torch.bfloat16).contiguous() for x in (q, k, v))
    o, lse = H.attn_forward_block(qd, kd, vd, grid, q_video, q_pos0, k_video, k_pos0, kv_len)
    torch.cuda.synchronize(dev)
    assert H.last_device_error() == 0
    return o.cpu(), lse.cpu()


def _gpu_merge(acc_o, acc_lse, o, lse, out=None):
    from joint_full_attention_b200 import hvattn as H
    dev = torch.device("cuda", 0)
    ao = acc_o.to(dev, torch.float32).contiguous()
    al = acc_lse.to(dev, torch.float32).contiguous()
    od = o.to(dev).contiguous()
    ld = lse.to(dev, torch.float32).contiguous()
    outd = None if out is None else torch.empty(out.shape, dtype=torch.bfloat16, device=dev)
    H.attn_merge(ao, al, od, ld, out=outd)
    torch.cuda.synchronize(dev)
    acc_o.copy_(ao.cpu().to(acc_o.dtype))
    acc_lse.copy_(al.cpu().to(acc_lse.dtype))
    if out is not None:
        out.copy_(outd.cpu().to(out.dtype))


def _ulysses_rank(rank, world, port, grid, text_len, valid, heads, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, str(ROOT))
    import torch.distributed as dist

    from joint_full_attention_b200 import ulysses as U
    torch.cuda.set_device(0)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        q, k, v = (torch.from_numpy(x) for x in _problem(grid, text_len, valid, heads, seed=21))
        layout = U.ulysses_layout(grid, heads, world)
        n = layout.n_video
        shard = [U.shard_video(x[:, :n], layout, rank) for x in (q, k, v)]
        text = [x[:, n:].contiguous() for x in (q, k, v)]
        vid, txt = U.ulysses_attention(*shard, *text, grid, valid, attn=_gpu_attn)
        results[rank] = (vid.numpy(), txt.numpy(), layout.shard_positions(rank).numpy())
    finally:
        dist.destroy_process_group()


def _ring_rank(rank, world, port, grid, text_len, valid, heads, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, str(ROOT))
    import torch.distributed as dist

    from joint_full_attention_b200 import ring as R
    torch.cuda.set_device(0)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        q, k, v = (torch.from_numpy(x) for x in _problem(grid, text_len, valid, heads, seed=22))
        n = grid[0] * grid[1] * grid[2]
        start, cnt = R.ring_chunks(n, world)[rank]
        run = [x[:, start:start + cnt].contiguous() for x in (q, k, v)]
        text = [x[:, n:].contiguous() for x in (q, k, v)]
        vid, txt = R.ring_attention(*run, *text, grid, valid, block=_gpu_block, merge=_gpu_merge)
        results[rank] = (vid.float().numpy(), txt.float().numpy(), start, cnt)
    finally:
        dist.destroy_process_group()


def _spawn(target, world, *args):
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    manager = ctx.Manager()
    results = manager.dict()
    port = _free_port()
    procs = [ctx.Process(target=target, args=(r, world, port, *args, results)) for r in range(world)]
    for pr in procs:
        pr.start()
    for pr in procs:
        pr.join(timeout=600)
        assert pr.exitcode == 0, f"rank exited with {pr.exitcode}"
    return dict(results)


def _check(got, ref, what):
    err = np.abs(got.astype(np.float64) - ref)
    print(f"[parity] {what}: max abs err {err.max():.3e}, mean {err.mean():.3e}")
    assert np.all(np.isfinite(got)), what
    assert err.max() <= MAX_ABS and err.mean() <= MEAN_ABS, what


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    sys.path.insert(0, str(ROOT))
    from joint_full_attention_b200 import build as B
    B.build()


@pytest.mark.parametrize("world,grid,text_len,valid,heads", [
    (2, (2, 6, 4), 5, [3, 0], 4),        # slabs of H'/2 rows; a sample with no valid text
    (3, (2, 6, 4), 5, [0, 2], 6),
    (2, (2, 5, 6), 7, [7], 4),           # H'/2 = 5 odd: slabs of W'/2 columns
    (2, (3, 8, 20), 40, [25], 4),        # 520 rows: several tiles and a ragged tail
    (3, (2, 9, 30), 19, [11], 3),        # 559 rows, three ranks of one head each
])
def test_ulysses_ranks_run_the_kernel(world, grid, text_len, valid, heads):
    from oracle import hv_oracle as O
    res = _spawn(_ulysses_rank, world, grid, text_len, valid, heads)
    q, k, v = (x.astype(np.float64) for x in _problem(grid, text_len, valid, heads, seed=21))
    ref = O.joint_attention(q, k, v, grid, text_len, valid)
    n = grid[0] * grid[1] * grid[2]
    for r in range(world):
        vid, txt, pos = res[r]
        _check(vid, ref[:, pos], f"ulysses world {world} rank {r} video")
        _check(txt, ref[:, n:], f"ulysses world {world} rank {r} text")


@pytest.mark.parametrize("world,grid,text_len,valid,heads", [
    (2, (3, 8, 20), 40, [25, 0], 3),     # a sample with no valid text key
    (3, (1, 1, 301), 16, [16], 2),       # uneven runs of 100, 100 and 101 tokens
    (3, (2, 7, 23), 0, [0], 2),          # no text at all
])
def test_ring_ranks_run_the_kernels(world, grid, text_len, valid, heads):
    from oracle import hv_oracle as O
    res = _spawn(_ring_rank, world, grid, text_len, valid, heads)
    q, k, v = (x.astype(np.float64) for x in _problem(grid, text_len, valid, heads, seed=22))
    ref = O.joint_attention(q, k, v, grid, text_len, valid)
    n = grid[0] * grid[1] * grid[2]
    for r in range(world):
        vid, txt, start, cnt = res[r]
        _check(vid, ref[:, start:start + cnt], f"ring world {world} rank {r} video")
        if text_len:
            _check(txt, ref[:, n:], f"ring world {world} rank {r} text")
