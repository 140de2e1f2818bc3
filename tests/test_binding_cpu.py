"""Python binding checks that need no GPU: argument validation happens
before any device work, and the host-side helpers (head groups, layouts)
behave as documented."""

from __future__ import annotations

import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist

from joint_full_attention_b200 import build as B
from joint_full_attention_b200 import hvattn as H


@pytest.fixture(scope="module", autouse=True)
def _lib():
    B.build()
    H.lib()


def test_device_calls_reject_host_and_malformed_tensors():
    cpu = torch.zeros(1, 40, 2, 128, dtype=torch.bfloat16)
    with pytest.raises(TypeError):
        H.attn_forward(cpu, cpu, cpu, (2, 4, 4), 8, [5])
    with pytest.raises(TypeError):
        H.attn_forward_ws(cpu, cpu, cpu, (2, 4, 4), 8, [5])
    with pytest.raises(TypeError):
        H.attn_forward_block(cpu, cpu, cpu, (2, 4, 4), 32, 0, 32, 0, [40])


def test_host_call_rejects_bad_host_tensors():
    good = torch.zeros(1, 40, 2, 128, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        H.attn_forward_host(good.float(), good, good, (2, 4, 4), 8, [5])
    with pytest.raises(ValueError):
        H.attn_forward_host(good, good[:, :39], good, (2, 4, 4), 8, [5])
    with pytest.raises(ValueError):
        H.attn_forward_host(good.transpose(1, 2), good, good, (2, 4, 4), 8, [5])
    with pytest.raises(ValueError):
        H.attn_forward_host(good, good, good, (2, 4, 4), 8, [5, 6])


def test_default_head_groups():
    assert H.default_head_groups(24) == 8
    assert H.default_head_groups(18) == 6
    assert H.default_head_groups(4) == 4
    assert H.default_head_groups(9) == 3
    assert H.default_head_groups(7) == 1


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_wrappers_check_their_slabs_on_one_rank():
    from joint_full_attention_b200 import ring as R
    from joint_full_attention_b200 import ulysses as U
    store = dist.TCPStore("127.0.0.1", _free_port(), 1, True)
    dist.init_process_group("gloo", store=store, rank=0, world_size=1)
    try:
        x = torch.zeros(1, 31, 2, 128, dtype=torch.float64)
        t = torch.zeros(1, 4, 2, 128, dtype=torch.float64)
        with pytest.raises(ValueError):          # 31 tokens, the one-rank slab of a 32-token grid has 32
            U.ulysses_attention(x, x, x, t, t, t, (2, 4, 4), [4], attn=lambda *a, **k: None)
        with pytest.raises(ValueError):
            R.ring_attention(x, x, x, t, t, t, (2, 4, 4), [4], block=lambda *a, **k: None,
                             merge=lambda *a, **k: None)
    finally:
        dist.destroy_process_group()
