"""The Ulysses wrapper on one GPU with NCCL: a one-rank group, the library's
kernel as the attention step, compared with the float64 oracle (max |Δ| <=
2e-2, mean |Δ| <= 2e-3). With one rank the exchanges move nothing, so the
result also equals a direct hv_attn_forward call bit for bit. Several ranks
running the kernel are covered by tests/test_multirank_gpu.py (gloo ranks on
one GPU); NCCL across GPUs needs more GPUs than a test here gets."""

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
from oracle import hv_oracle as O

pytestmark = pytest.mark.gpu


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_one_rank_nccl_matches_oracle():
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
        x = {nm: W.bf16_bits_to_f64(inp[nm]) for nm in ("q", "k", "v")}
        want = O.joint_attention(x["q"], x["k"], x["v"], wl.grid, wl.text_len, inp["text_valid"])
        got = torch.cat([vid, txt], dim=1).float().cpu().numpy().astype(np.float64)
        err = np.abs(got - want)
        print(f"[parity] one-rank ulysses: max abs err {err.max():.3e}, mean {err.mean():.3e}")
        assert np.all(np.isfinite(got)) and err.max() <= 2e-2 and err.mean() <= 2e-3
        assert torch.equal(vid, ref[:, :n]) and torch.equal(txt, ref[:, n:])
    finally:
        dist.destroy_process_group()
