"""Ring attention around the joint attention call.

"HunyuanVideo 模型结构与数学原理" §9.2 (xDiT/USP): with ring attention each
rank keeps a segment of the queries and the K/V blocks travel around a ring
of ranks; the partial results of the blocks are combined through their
log-sum-exp. Unlike Ulysses it needs no divisibility of the grid or of the
heads.

Layout (one process per GPU, ``torch.distributed``):

* the N video tokens are cut into `world` contiguous runs of the (t, h, w)
  sequence (``ring_chunks``); rank r holds run r of Q, K and V, and the whole
  text segment (replicated);
* step s: rank r attends its queries [run r ; text] to the K/V run of rank
  r - s (``hv_attn_forward_block``, RoPE at the run's global token indices,
  the block's result kept in fp32) while it passes that run on to rank r + 1
  and receives the next one; ``hv_attn_merge`` folds each block into an fp32
  accumulator, so no step of the ring rounds to bf16 before the last;
* a last block attends to the text keys (padding masked per sample) and
  writes the bf16 output.

Every rank computes the text query rows against all keys, so each returns
the full text output (equal across ranks up to the order of the merges).
"""

from __future__ import annotations

import torch
import torch.distributed as dist


def ring_chunks(n_video: int, world: int) -> list[tuple[int, int]]:
    """(first global token index, token count) of each rank's run of video tokens."""
    if world < 1 or n_video < world:
        raise ValueError(f"cannot cut {n_video} video tokens into {world} non-empty runs")
    bounds = [r * n_video // world for r in range(world + 1)]
    return [(bounds[r], bounds[r + 1] - bounds[r]) for r in range(world)]


def ring_attention(q_video: torch.Tensor, k_video: torch.Tensor, v_video: torch.Tensor,
                   q_text: torch.Tensor, k_text: torch.Tensor, v_text: torch.Tensor, grid, text_valid,
                   group=None, block=None, merge=None, **block_kwargs):
    """Joint attention of a sequence-sharded problem by ring attention.

    q_video, k_video, v_video: this rank's run of video tokens [B, n_r, H, D]
    (runs as ``ring_chunks``); q_text, k_text, v_text: the whole text segment
    [B, L, H, D] on every rank. ``block`` and ``merge`` default to the
    library's ``hvattn.attn_forward_block`` and ``hvattn.attn_merge``.

    Returns (video output run [B, n_r, H, D], text output [B, L, H, D]).
    """
    if block is None or merge is None:
        from . import hvattn
        block = block or hvattn.attn_forward_block
        merge = merge or hvattn.attn_merge
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    t_lat, hp, wp = (int(x) for x in grid)
    chunks = ring_chunks(t_lat * hp * wp, world)
    start, n_r = chunks[rank]
    b_sz, n_loc, heads, d = q_video.shape
    if n_loc != n_r:
        raise ValueError(f"rank {rank} holds {n_loc} video tokens, its run has {n_r}")
    text_len = q_text.shape[1]
    q = torch.cat([q_video, q_text], dim=1).contiguous()
    acc_dtype = torch.float32 if q.is_cuda else torch.float64
    acc_o = torch.zeros((b_sz, n_r + text_len, heads, d), dtype=acc_dtype, device=q.device)
    acc_lse = torch.full((b_sz, n_r + text_len, heads), float("-inf"), dtype=acc_dtype, device=q.device)
    out = torch.empty_like(q)
    nxt_rank, prv_rank = (rank + 1) % world, (rank - 1) % world
    cur_k, cur_v = k_video.contiguous(), v_video.contiguous()
    for step in range(world):
        src = (rank - step) % world
        reqs = []
        if step + 1 < world:
            # post the hand-over first so that it overlaps this block's attention
            n_in = chunks[(src - 1) % world][1]
            in_k = torch.empty((b_sz, n_in, heads, d), dtype=cur_k.dtype, device=cur_k.device)
            in_v = torch.empty_like(in_k)
            ops = [dist.P2POp(dist.isend, cur_k, nxt_rank, group), dist.P2POp(dist.isend, cur_v, nxt_rank, group),
                   dist.P2POp(dist.irecv, in_k, prv_rank, group), dist.P2POp(dist.irecv, in_v, prv_rank, group)]
            reqs = dist.batch_isend_irecv(ops)
        k0, nk = chunks[src]
        o, lse = block(q, cur_k, cur_v, grid, n_r, start, nk, k0, [nk] * b_sz, **block_kwargs)
        last = step + 1 == world and text_len == 0
        merge(acc_o, acc_lse, o, lse, out=out if last else None)
        for r in reqs:
            r.wait()
        if step + 1 < world:
            cur_k, cur_v = in_k, in_v
    if text_len > 0:
        # the text keys, the same on every rank; a sample with no valid text key
        # contributes nothing (its block result is dropped through lse = -inf)
        valid = [int(x) for x in text_valid]
        o, lse = block(q, k_text.contiguous(), v_text.contiguous(), grid, n_r, start, 0, 0,
                       [max(1, x) for x in valid], **block_kwargs)
        for b, x in enumerate(valid):
            if x == 0:
                lse[b].fill_(float("-inf"))
        merge(acc_o, acc_lse, o, lse, out=out)
    return out[:, :n_r].contiguous(), out[:, n_r:].contiguous()
