"""GPU parity of the ring-attention step ("HunyuanVideo 模型结构与数学原理"
§9.2) through the C ABI: hv_attn_forward_block (outputs and log-sum-exp)
against the oracle's block attention, hv_attn_merge against the merge rule,
and a one-rank ring (NCCL) against the oracle's joint attention. Tolerance as
for the plain call: max |Δ| <= 2e-2, mean |Δ| <= 2e-3 (outputs and lse)."""

from __future__ import annotations

import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist

from joint_full_attention_b200 import build as B
from joint_full_attention_b200 import hvattn as H
from joint_full_attention_b200 import ring as R
from joint_full_attention_b200 import workloads as W
from oracle import hv_oracle as O

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    B.build()
    H.lib()
    assert H.last_device_error() == 0


def _bits(shape, seed):
    rng = np.random.default_rng(seed)
    return W.round_to_bf16_bits(rng.standard_normal(shape).astype(np.float32))


def _dev(bits):
    return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).cuda()


def check(got, ref, what):
    fin = np.isfinite(ref)
    err = np.abs(got[fin] - ref[fin])
    print(f"[parity] ring {what}: max abs err {err.max():.3e}, mean {err.mean():.3e}")
    assert np.all(np.isfinite(got[fin])), what
    assert err.max() <= 2e-2 and err.mean() <= 2e-3, what


@pytest.mark.parametrize("sq,q_video,q_pos0,sk,k_video,k_pos0,kv", [
    (240, 200, 100, 200, 200, 50, [200]),     # video rows of both at offsets, text queries after
    (240, 200, 100, 40, 0, 0, [25]),          # the text key block, padding masked
    (77, 77, 403, 130, 130, 350, [130]),      # ragged tiles, a run at the end of the grid
    (300, 0, 0, 300, 100, 0, [170]),          # queries all text, keys past the valid ones masked
])
def test_block_matches_oracle(sq, q_video, q_pos0, sk, k_video, k_pos0, kv):
    grid = (3, 8, 20)                                   # 480 video tokens
    heads = 3
    qb, kb, vb = _bits((1, sq, heads, 128), 1), _bits((1, sk, heads, 128), 2), _bits((1, sk, heads, 128), 3)
    o, lse = H.attn_forward_block(_dev(qb), _dev(kb), _dev(vb), grid, q_video, q_pos0, k_video, k_pos0, kv)
    torch.cuda.synchronize()
    assert H.last_device_error() == 0
    q, k, v = (W.bf16_bits_to_f64(x) for x in (qb, kb, vb))
    ref_o = np.empty((sq, heads, 128))
    ref_l = np.empty((sq, heads))
    for h in range(heads):
        ref_o[:, h], ref_l[:, h] = O.joint_attention_block(q[0, :, h], k[0, :, h], v[0, :, h], grid, q_video, q_pos0,
                                                           k_video, k_pos0, kv[0])
    check(o[0].float().cpu().numpy().astype(np.float64), ref_o, f"block out Sq={sq} Sk={sk}")
    check(lse[0].cpu().numpy().astype(np.float64), ref_l, f"block lse Sq={sq} Sk={sk}")


def test_whole_sequence_block_is_the_plain_call():
    wl = W.WORKLOADS["img256"]
    inp = W.make_inputs(wl, seed=8)
    q, k, v = (_dev(inp[n]) for n in ("q", "k", "v"))
    ref = H.attn_forward(q, k, v, wl.grid, wl.text_len, inp["text_valid"])
    n = wl.n_video
    kv = [n + int(x) for x in inp["text_valid"]]
    o, _ = H.attn_forward_block(q, k, v, wl.grid, n, 0, n, 0, kv, out_dtype=torch.bfloat16)
    o32, _ = H.attn_forward_block(q, k, v, wl.grid, n, 0, n, 0, kv)
    torch.cuda.synchronize()
    assert torch.equal(o, ref)
    # the fp32 partial is the same result before its rounding to bf16
    assert o32.dtype == torch.float32 and torch.equal(o32.to(torch.bfloat16), ref)


def test_block_on_grid_without_table():
    """A grid whose rotation table would not fit in shared memory (8*T' + 28*(H'/2 + W'/2) = 3928
    entries against 3840): the block kernel's per-pair sincospif form, against the oracle at run
    offsets, and over the whole sequence equal to the plain call (which takes the same form)."""
    grid = (1, 100, 40)                                 # 4000 video tokens
    heads = 2
    sq, q_video, q_pos0, sk, k_video, k_pos0, kv = 240, 200, 3700, 300, 300, 100, [300]
    qb, kb, vb = _bits((1, sq, heads, 128), 11), _bits((1, sk, heads, 128), 12), _bits((1, sk, heads, 128), 13)
    o, lse = H.attn_forward_block(_dev(qb), _dev(kb), _dev(vb), grid, q_video, q_pos0, k_video, k_pos0, kv)
    torch.cuda.synchronize()
    assert H.last_device_error() == 0
    q, k, v = (W.bf16_bits_to_f64(x) for x in (qb, kb, vb))
    ref_o = np.empty((sq, heads, 128))
    ref_l = np.empty((sq, heads))
    for h in range(heads):
        ref_o[:, h], ref_l[:, h] = O.joint_attention_block(q[0, :, h], k[0, :, h], v[0, :, h], grid, q_video, q_pos0,
                                                           k_video, k_pos0, kv[0])
    check(o[0].float().cpu().numpy().astype(np.float64), ref_o, "block out, no table")
    check(lse[0].cpu().numpy().astype(np.float64), ref_l, "block lse, no table")
    text_len, valid = 30, [12]
    n = grid[0] * grid[1] * grid[2]
    qw, kw, vw = (_dev(_bits((1, n + text_len, heads, 128), s)) for s in (14, 15, 16))
    ref = H.attn_forward(qw, kw, vw, grid, text_len, valid)
    whole, _ = H.attn_forward_block(qw, kw, vw, grid, n, 0, n, 0, [n + valid[0]], out_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    assert torch.equal(whole, ref)


def test_merge_kernel_matches_rule():
    rows = 1000
    rng = np.random.default_rng(4)
    acc_o = rng.standard_normal((rows, 128)).astype(np.float32)
    acc_l = (rng.standard_normal(rows) * 4).astype(np.float32)
    acc_l[:10] = -np.inf
    acc_o[:10] = 0
    part_b = W.round_to_bf16_bits(rng.standard_normal((rows, 128)).astype(np.float32))
    part_l = (rng.standard_normal(rows) * 4).astype(np.float32)
    part_l[5:15] = -np.inf                            # rows 5..9: both empty
    ao, al = torch.from_numpy(acc_o).cuda(), torch.from_numpy(acc_l).cuda()
    out = torch.empty((rows, 128), dtype=torch.bfloat16, device="cuda")
    H.attn_merge(ao, al, _dev(part_b), torch.from_numpy(part_l).cuda(), out=out)
    torch.cuda.synchronize()
    ref_o, ref_l = O.merge_blocks([acc_o.astype(np.float64), W.bf16_bits_to_f64(part_b)],
                                  [acc_l.astype(np.float64), part_l.astype(np.float64)])
    got_o = ao.cpu().numpy().astype(np.float64)
    np.testing.assert_allclose(got_o, ref_o, rtol=1e-5, atol=1e-5)
    got_l = al.cpu().numpy().astype(np.float64)
    assert np.array_equal(np.isinf(got_l), np.isinf(ref_l))
    np.testing.assert_allclose(got_l[np.isfinite(ref_l)], ref_l[np.isfinite(ref_l)], rtol=1e-5, atol=1e-5)
    np.testing.assert_allclose(out.float().cpu().numpy(), got_o, rtol=2 ** -8, atol=1e-6)
    # fp32 partials (what the ring passes): merged without a bf16 rounding of the part
    part_f = rng.standard_normal((rows, 128)).astype(np.float32)
    ao2, al2 = torch.from_numpy(acc_o).cuda(), torch.from_numpy(acc_l).cuda()
    H.attn_merge(ao2, al2, torch.from_numpy(part_f).cuda(), torch.from_numpy(part_l).cuda())
    torch.cuda.synchronize()
    ref_o2, _ = O.merge_blocks([acc_o.astype(np.float64), part_f.astype(np.float64)],
                               [acc_l.astype(np.float64), part_l.astype(np.float64)])
    np.testing.assert_allclose(ao2.cpu().numpy().astype(np.float64), ref_o2, rtol=1e-5, atol=1e-5)


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_one_rank_ring_nccl_matches_oracle():
    torch.cuda.set_device(0)
    store = dist.TCPStore("127.0.0.1", _free_port(), 1, True)
    dist.init_process_group("nccl", store=store, rank=0, world_size=1, device_id=torch.device("cuda", 0))
    try:
        wl = W.Workload("ring", "ring", 2, 3, (3, 8, 20), 40, valid=(25, 0))
        inp = W.make_inputs(wl, seed=12)
        q, k, v = (_dev(inp[n]) for n in ("q", "k", "v"))
        n = wl.n_video
        vid, txt = R.ring_attention(q[:, :n].contiguous(), k[:, :n].contiguous(), v[:, :n].contiguous(),
                                    q[:, n:].contiguous(), k[:, n:].contiguous(), v[:, n:].contiguous(),
                                    wl.grid, inp["text_valid"])
        torch.cuda.synchronize()
        assert H.last_device_error() == 0
        x = {nm: W.bf16_bits_to_f64(inp[nm]) for nm in ("q", "k", "v")}
        ref = O.joint_attention(x["q"], x["k"], x["v"], wl.grid, wl.text_len, inp["text_valid"])
        got = torch.cat([vid, txt], dim=1).float().cpu().numpy().astype(np.float64)
        check(got, ref, "one-rank ring")
    finally:
        dist.destroy_process_group()
