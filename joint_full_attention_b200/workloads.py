"""Seeded synthetic workloads for the joint 3D-RoPE attention call.

This module only *generates inputs*: shapes, seeded random tensors rounded to
bfloat16, per-sample text valid lengths and sampled output rows. It holds none
of the attention or RoPE arithmetic, so that the CUDA path and the float64
oracle can both be fed from it without sharing any of the computation.

Shapes follow the pages' workloads ("HunyuanVideo 模型结构与数学原理" §4 and
§5.6; the README mirror's supported-size table): video-token grids of
(T', H'/2, W'/2), up to 256 text tokens, 24 heads of 128 channels, tensors in
the [B, S, heads, 128] layout with S = video tokens + text_len. They stand in
for real DiT activations, which the pages do not provide.

Recipe: PCG64(seed) -> independent child streams for Q, K, V and the
metadata; Q, K, V ~ N(0, 1) drawn as float32, then rounded to bfloat16
(round-to-nearest-even). Valid text lengths are uniform integers in
[20, 256] (or fixed for the tiny case). The 720x1280x129 workload also
multiplies K per head by U[0.5, 2] (in float32, before rounding) to vary the
softmax sharpness.
"""

from __future__ import annotations

from dataclasses import dataclass

import numpy as np

HEAD_DIM = 128


@dataclass(frozen=True)
class Workload:
    name: str
    label: str                 # what the clip is: "FxHxW" or a description
    batch: int
    heads: int
    grid: tuple[int, int, int]  # (T', H'/2, W'/2) video-token grid
    text_len: int
    valid: tuple[int, ...] | None = None   # fixed valid lengths, else U[20, 256]
    k_head_scale: bool = False
    full_check: bool = True    # full-output oracle check (else sampled rows)

    @property
    def n_video(self) -> int:
        t, hp, wp = self.grid
        return t * hp * wp

    @property
    def seq_len(self) -> int:
        return self.n_video + self.text_len


WORKLOADS: dict[str, Workload] = {
    "tiny": Workload("tiny", "B1 2 heads grid 2x4x4 + 8 text (5 valid)", 1, 2, (2, 4, 4), 8, valid=(5,)),
    "img256": Workload("img256", "256x256 single image (F=1)", 2, 24, (1, 16, 16), 256),
    "v544x960x17": Workload("v544x960x17", "544x960x17 short video", 1, 24, (5, 34, 60), 256),
    "v544x960x129": Workload("v544x960x129", "544x960x129 video", 1, 24, (33, 34, 60), 256, full_check=False),
    "v720x1280x129": Workload("v720x1280x129", "720x1280x129 video", 1, 24, (33, 45, 80), 256,
                              k_head_scale=True, full_check=False),
    # other supported sizes of the README's table (same ~118k-token scale, other aspect ratios)
    "v960x960x129": Workload("v960x960x129", "960x960x129 video", 1, 24, (33, 60, 60), 256, full_check=False),
    "v1104x832x129": Workload("v1104x832x129", "1104x832x129 video", 1, 24, (33, 69, 52), 256,
                              full_check=False),
    # two-branch classifier-free guidance: conditional and unconditional prompts
    # batched together, each with its own valid text length
    "cfg544x960x129": Workload("cfg544x960x129", "544x960x129 video, B=2 (CFG pair)", 2, 24, (33, 34, 60), 256,
                               full_check=False),
}

BENCH_WORKLOAD = "v720x1280x129"


def round_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """float32 -> bfloat16 bit patterns (uint16), round to nearest even."""
    bits = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    rounded = bits + np.uint32(0x7FFF) + ((bits >> np.uint32(16)) & np.uint32(1))
    return (rounded >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """bfloat16 bit patterns (uint16) -> float64 (exact widening)."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def _normal_bf16(rng: np.random.Generator, shape, head_scale: np.ndarray | None = None,
                 chunk_rows: int = 1 << 14) -> np.ndarray:
    """N(0,1) float32 draws rounded to bf16 bits, generated in row chunks."""
    b_sz, s_len, heads, d = shape
    out = np.empty(shape, dtype=np.uint16)
    for b in range(b_sz):
        for s0 in range(0, s_len, chunk_rows):
            s1 = min(s_len, s0 + chunk_rows)
            x = rng.standard_normal((s1 - s0, heads, d), dtype=np.float32)
            if head_scale is not None:
                x *= head_scale[None, :, None].astype(np.float32)
            out[b, s0:s1] = round_to_bf16_bits(x)
    return out


def _streams(wl: Workload, seed: int):
    root = np.random.SeedSequence([seed, sum(map(ord, wl.name))])
    return root.spawn(4)


def _meta(wl: Workload, s_meta) -> tuple[np.ndarray, np.ndarray | None]:
    meta = np.random.Generator(np.random.PCG64(s_meta))
    if wl.valid is not None:
        text_valid = np.asarray(wl.valid, dtype=np.int32)
    else:
        text_valid = meta.integers(20, 257, size=wl.batch).astype(np.int32)
    text_valid = np.minimum(text_valid, wl.text_len).astype(np.int32)
    k_scale = meta.uniform(0.5, 2.0, size=wl.heads).astype(np.float32) if wl.k_head_scale else None
    return text_valid, k_scale


def text_valid_of(wl: Workload, seed: int = 0) -> np.ndarray:
    """The valid text lengths ``make_inputs(wl, seed)`` draws, without drawing the tensors."""
    return _meta(wl, _streams(wl, seed)[0])[0]


def make_device_inputs(wl: Workload, seed: int, device) -> dict:
    """Inputs of the workload's shape and distribution drawn on the GPU (torch's seeded
    Philox generator): for timing runs, where drawing 100+ million values on the host
    would dominate. Same recipe as ``make_inputs`` (N(0, 1) in float32, K scaled per
    head when the workload asks for it, rounded to bf16); not the same values.
    """
    import torch

    text_valid, k_scale = _meta(wl, _streams(wl, seed)[0])
    gen = torch.Generator(device=device)
    gen.manual_seed(int(seed) * 1000003 + sum(map(ord, wl.name)))
    shape = (wl.batch, wl.seq_len, wl.heads, HEAD_DIM)
    out = {}
    for name in ("q", "k", "v"):
        x = torch.randn(shape, generator=gen, device=device, dtype=torch.float32)
        if name == "k" and k_scale is not None:
            x *= torch.from_numpy(k_scale).to(device).view(1, 1, -1, 1)
        out[name] = x.to(torch.bfloat16)
        del x
    out["text_valid"] = text_valid
    return out


def make_inputs(wl: Workload, seed: int = 0) -> dict:
    """Seeded inputs of a workload.

    Returns dict with q, k, v as uint16 bf16 bit arrays [B, S, heads, 128],
    text_valid (int32 [B]) and k_scale (float32 [heads] or None).
    """
    s_meta, s_q, s_k, s_v = _streams(wl, seed)
    text_valid, k_scale = _meta(wl, s_meta)
    shape = (wl.batch, wl.seq_len, wl.heads, HEAD_DIM)
    q = _normal_bf16(np.random.Generator(np.random.PCG64(s_q)), shape)
    k = _normal_bf16(np.random.Generator(np.random.PCG64(s_k)), shape, head_scale=k_scale)
    v = _normal_bf16(np.random.Generator(np.random.PCG64(s_v)), shape)
    return {"q": q, "k": k, "v": v, "text_valid": text_valid, "k_scale": k_scale}


def sample_triples(batch: int, heads: int, n_video: int, text_len: int, text_valid, count: int,
                   seed: int = 0, tile: int = 128) -> np.ndarray:
    """Seeded (b, head, row) triples, with forced coverage of the edge rows.

    About a quarter are forced: rows 0 and S-1, either side of the video/text
    boundary, valid and padded text rows, the last (partial) 128-row tile,
    and rows on both sides of tile boundaries; the rest are uniform.
    """
    s_len = n_video + text_len
    rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, 7919])))
    forced_rows: list[int] = [0, s_len - 1, n_video - 1]
    if text_len > 0:
        forced_rows += [n_video, s_len - 1]
    for b in range(batch):
        vb = int(text_valid[b])
        if vb > 0:
            forced_rows += [n_video + vb - 1]
        if vb < text_len:
            forced_rows += [n_video + vb]
    last_tile = (s_len - 1) // tile * tile
    forced_rows += list(range(last_tile, s_len, max(1, (s_len - last_tile) // 8)))
    for t0 in (tile, 2 * tile, (s_len // tile) * tile, ((s_len // tile) - 1) * tile):
        for r in (t0 - 1, t0):
            if 0 <= r < s_len:
                forced_rows.append(r)
    forced_rows = sorted(set(r for r in forced_rows if 0 <= r < s_len))
    triples = []
    n_forced = max(len(forced_rows), count // 4)
    for i in range(min(count, n_forced)):
        r = forced_rows[i % len(forced_rows)]
        triples.append((int(rng.integers(batch)), int(rng.integers(heads)), r))
    while len(triples) < count:
        triples.append((int(rng.integers(batch)), int(rng.integers(heads)), int(rng.integers(s_len))))
    return np.asarray(triples[:count], dtype=np.int64)
