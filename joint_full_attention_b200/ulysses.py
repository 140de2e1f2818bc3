"""Ulysses sequence parallelism around the joint attention call.

"HunyuanVideo 模型结构与数学原理" §9.2 (xDiT/USP): Ulysses re-lays the
activations between a sequence-sharded and a head-sharded layout with
all-to-all, so that every rank runs full attention over the whole joint
sequence for a slice of the heads. The fork requires one patched spatial axis
(H' or W') to be divisible by the world size, and the Ulysses degree has to
divide the head count.

Layout here (one process per GPU, ``torch.distributed``):

* input on rank r: the video tokens of its slab of the token grid (the rows
  h of block r of H'/2, or, when H'/2 is not divisible, the columns w of
  block r of W'/2), in (t, h, w) order, as [B, N/P, heads, 128]; the text
  tokens, replicated on every rank, as [B, L, heads, 128].
* all-to-all #1 sends head block j of the local video rows to rank j; rank r
  then holds every video token for heads [r H/P, (r+1) H/P), puts them back
  in the global (t, h, w) order and appends its head block of the text.
* the attention call (``hv_attn_forward`` by default) runs on [B, S, H/P, 128].
* all-to-all #2 returns each rank's video rows for every head block;
  an all-gather over head blocks gives every rank the full text output.

The exchange steps are plain ``torch.distributed`` collectives (NCCL on the
GPUs); the attention itself is the library's kernel. This file holds layout
and exchange logic only.
"""

from __future__ import annotations

from dataclasses import dataclass

import torch
import torch.distributed as dist


@dataclass(frozen=True)
class UlyssesLayout:
    world: int
    grid: tuple[int, int, int]   # (T', H'/2, W'/2)
    heads: int
    axis: int                    # 1: slabs of H'/2 rows, 2: slabs of W'/2 columns

    @property
    def n_video(self) -> int:
        t, hp, wp = self.grid
        return t * hp * wp

    @property
    def shard_tokens(self) -> int:
        return self.n_video // self.world

    @property
    def heads_per_rank(self) -> int:
        return self.heads // self.world

    def shard_positions(self, rank: int) -> torch.Tensor:
        """Global sequence indices of rank ``rank``'s video tokens, in the order it holds them."""
        t_lat, hp, wp = self.grid
        t = torch.arange(t_lat).view(-1, 1, 1)
        if self.axis == 1:
            blk = hp // self.world
            h = torch.arange(rank * blk, (rank + 1) * blk).view(1, -1, 1)
            w = torch.arange(wp).view(1, 1, -1)
        else:
            blk = wp // self.world
            h = torch.arange(hp).view(1, -1, 1)
            w = torch.arange(rank * blk, (rank + 1) * blk).view(1, 1, -1)
        return (t * (hp * wp) + h * wp + w).reshape(-1)

    def gather_order(self) -> torch.Tensor:
        """For global video token n, its row in the concatenation of all shards (rank-major)."""
        cat = torch.cat([self.shard_positions(r) for r in range(self.world)])
        order = torch.empty_like(cat)
        order[cat] = torch.arange(cat.numel())
        return order


def ulysses_layout(grid, heads: int, world: int) -> UlyssesLayout:
    """The slab layout for ``world`` ranks, or ValueError where the pages' rule forbids it."""
    t_lat, hp, wp = (int(x) for x in grid)
    if world < 1:
        raise ValueError("world size must be >= 1")
    if heads % world:
        raise ValueError(f"{heads} heads cannot be split over {world} ranks (Ulysses degree must divide the heads)")
    if hp % world == 0:
        axis = 1
    elif wp % world == 0:
        axis = 2
    else:
        raise ValueError(f"neither H'/2 = {hp} nor W'/2 = {wp} is divisible by the world size {world}")
    return UlyssesLayout(world, (t_lat, hp, wp), heads, axis)


def shard_video(x: torch.Tensor, layout: UlyssesLayout, rank: int) -> torch.Tensor:
    """Rank ``rank``'s video slab of a full [B, S, heads, D] tensor (for building inputs)."""
    return x[:, layout.shard_positions(rank).to(x.device)].contiguous()


def _all_to_all_heads(x: torch.Tensor, layout: UlyssesLayout, group) -> torch.Tensor:
    """[B, n, H, D] sharded by tokens -> [P, B, n, H/P, D]: block j comes from rank j,
    holding its n tokens for this rank's heads."""
    b_sz, n, heads, d = x.shape
    p = layout.world
    send = x.view(b_sz, n, p, heads // p, d).permute(2, 0, 1, 3, 4).contiguous()
    recv = torch.empty_like(send)
    dist.all_to_all_single(recv, send, group=group)
    return recv


def ulysses_attention(q_video: torch.Tensor, k_video: torch.Tensor, v_video: torch.Tensor,
                      q_text: torch.Tensor, k_text: torch.Tensor, v_text: torch.Tensor, grid, text_valid,
                      attn=None, group=None, **attn_kwargs):
    """Joint attention of a sequence-sharded problem with Ulysses all-to-all.

    q_video, k_video, v_video: this rank's video slab [B, N/P, heads, D];
    q_text, k_text, v_text: the whole text segment [B, L, heads, D] (the same on
    every rank). ``attn(q, k, v, grid, text_len, text_valid, **attn_kwargs)``
    computes joint attention of [B, S, heads/P, D] tensors; by default the
    library's ``hv_attn_forward`` through ``hvattn.attn_forward``.

    Returns (video output slab [B, N/P, heads, D], text output [B, L, heads, D]).
    """
    if attn is None:
        from . import hvattn
        attn = hvattn.attn_forward
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    b_sz, n_loc, heads, d = q_video.shape
    layout = ulysses_layout(grid, heads, world)
    if n_loc != layout.shard_tokens:
        raise ValueError(f"video slab has {n_loc} tokens, layout needs {layout.shard_tokens}")
    text_len = q_text.shape[1]
    hl = layout.heads_per_rank
    order = layout.gather_order().to(q_video.device)
    my_heads = slice(rank * hl, (rank + 1) * hl)

    def to_heads(xv: torch.Tensor, xt: torch.Tensor) -> torch.Tensor:
        blocks = _all_to_all_heads(xv, layout, group)                      # [P, B, n_loc, hl, D]
        video = blocks.permute(1, 0, 2, 3, 4).reshape(b_sz, world * n_loc, hl, d)
        video = video.index_select(1, order)                               # global (t, h, w) order
        return torch.cat([video, xt[:, :, my_heads]], dim=1).contiguous()

    q, k, v = to_heads(q_video, q_text), to_heads(k_video, k_text), to_heads(v_video, v_text)
    out = attn(q, k, v, grid, text_len, text_valid, **attn_kwargs)        # [B, S, hl, D]

    # video rows back to their slabs: block s holds rank s's tokens for my heads
    out_video = out[:, :layout.n_video]
    back = torch.stack([out_video.index_select(1, layout.shard_positions(s).to(out.device))
                        for s in range(world)])                            # [P, B, n_loc, hl, D]
    recv = torch.empty_like(back)
    dist.all_to_all_single(recv, back.contiguous(), group=group)
    video_out = recv.permute(1, 2, 0, 3, 4).reshape(b_sz, n_loc, heads, d)

    # text rows: every rank computed its head block; gather all blocks
    if text_len == 0:
        return video_out.contiguous(), q_text.new_empty((b_sz, 0, heads, d))
    text_blocks = [torch.empty_like(out[:, layout.n_video:]) for _ in range(world)]
    dist.all_gather(text_blocks, out[:, layout.n_video:].contiguous(), group=group)
    text_out = torch.cat(text_blocks, dim=2)
    return video_out.contiguous(), text_out.contiguous()
