"""The Ulysses wrapper on one GPU: a one-rank NCCL group, the library's kernel
as the attention step. With one rank the exchanges move nothing, so the
result must equal a direct hv_attn_forward call bit for bit. (More ranks need
more GPUs than a test here gets; the multi-rank exchange is covered by the
gloo tests on CPU.)"""

from __future__ import annotations

import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist

from joint_full_attention_b200 import build as B
from joint_full_attention_b200 import hvattn as H
from joint_full_attention_b200 import ulysses as U
from joint_full_attention_b200 import workloads as W

pytestmark = pytest.mark.gpu


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_one_rank_nccl_equals_direct_call():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    B.build()
    torch.cuda.set_device(0)
    store = dist.TCPStore("127.0.0.1", _free_port(), 1, True)
    dist.init_process_group("nccl", store=store, rank=0, world_size=1, device_id=torch.device("cuda", 0))
    try:
        wl = W.WORKLOADS["img256"]
        inp = W.make_inputs(wl, seed=31)
        q, k, v = (torch.from_numpy(inp[n].view(np.int16)).view(torch.bfloat16).cuda() for n in ("q", "k", "v"))
        n = wl.n_video
        ref = H.attn_forward(q, k, v, wl.grid, wl.text_len, inp["text_valid"])
        lay = U.ulysses_layout(wl.grid, wl.heads, 1)
        shard = [U.shard_video(x[:, :n], lay, 0) for x in (q, k, v)]
        text = [x[:, n:].contiguous() for x in (q, k, v)]
        vid, txt = U.ulysses_attention(*shard, *text, wl.grid, inp["text_valid"])
        torch.cuda.synchronize()
        assert H.last_device_error() == 0
        assert torch.equal(vid, ref[:, :n]) and torch.equal(txt, ref[:, n:])
    finally:
        dist.destroy_process_group()
