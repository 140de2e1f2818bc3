"""The no-allocation entry point, hv_attn_forward_noalloc.

It exists for callers that cannot allocate device memory when they run
attention (their allocator owns the GPU, or they cannot afford cudaMalloc's
implicit synchronisation) and have no buffer to lend as workspace: the
rotated keys go to a 64 MiB scratch array built into the library instead.

This file is named so that pytest collects it last. It calls the entry point
through the C ABI twice in a row, on different inputs, and compares each
result with hv_attn_forward's within the parity tolerance (they are in fact
bit-identical, and that is checked too), then checks that a problem larger
than the built-in scratch is refused before any launch.
"""

from __future__ import annotations

import ctypes

import numpy as np
import pytest
import torch

from joint_full_attention_b200 import build as B
from joint_full_attention_b200 import hvattn as H
from joint_full_attention_b200 import workloads as W

MAX_ABS = 2e-2
MEAN_ABS = 2e-3
NOALLOC_MAX_BYTES = 64 << 20

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    B.build()
    return H.lib()


def _dev(bits):
    return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).cuda()


def _noalloc(lib, q, k, v, out, grid, text_len, text_valid):
    b_sz, _, heads, _ = q.shape
    valid = (ctypes.c_int * b_sz)(*[int(x) for x in text_valid])
    return lib.hv_attn_forward_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), b_sz, heads,
                                       grid[0], grid[1], grid[2], text_len, valid, 256.0, 1.0 / np.sqrt(128),
                                       ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def test_noalloc_matches_forward_on_two_calls(lib):
    cases = [(W.WORKLOADS["img256"], 11), (W.Workload("e", "edge", 2, 3, (5, 3, 11), 100, valid=(1, 77)), 12)]
    for wl, seed in cases:     # two calls in a row; the second sees the first call's scratch contents
        inp = W.make_inputs(wl, seed=seed)
        q, k, v = (_dev(inp[n]) for n in ("q", "k", "v"))
        assert wl.batch * wl.seq_len * wl.heads * 256 <= NOALLOC_MAX_BYTES
        ref = H.attn_forward(q, k, v, wl.grid, wl.text_len, inp["text_valid"])
        out = torch.full_like(q, float("nan"))
        st = _noalloc(lib, q, k, v, out, wl.grid, wl.text_len, inp["text_valid"])
        assert st == 0, H.status_string(st)
        torch.cuda.synchronize()
        assert H.last_device_error() == 0
        err = (out.float() - ref.float()).abs()
        assert torch.isfinite(out.float()).all()
        assert err.max().item() <= MAX_ABS and err.mean().item() <= MEAN_ABS
        assert torch.equal(out, ref)


def test_noalloc_refuses_problems_beyond_its_scratch(lib):
    wl = W.WORKLOADS["v544x960x129"]          # rotated keys: 415 MB > 64 MiB
    shape = (wl.batch, wl.seq_len, wl.heads, 128)
    q = torch.zeros(shape, dtype=torch.bfloat16, device="cuda")
    out = torch.empty_like(q)
    st = _noalloc(lib, q, q, q, out, wl.grid, wl.text_len, [wl.text_len])
    assert st == 12 and "HV_NOALLOC_MAX_BYTES" in H.status_string(st)
    assert H.last_device_error() == 0
