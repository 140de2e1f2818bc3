"""Float64 CPU oracle for joint full attention with 3D RoPE.

TEST INFRASTRUCTURE ONLY. This module is the correctness reference for the
CUDA path and is not part of the product: only ``tests/``,
``__graft_entry__.smoke()`` and ``bench.py`` (its CPU-baseline and reference
arms) may import it. It shares no code with ``joint_full_attention_b200``;
it imports nothing from that package and that package imports nothing from
here. It takes plain numpy arrays; the seeded input generators that feed both
sides live in ``joint_full_attention_b200/workloads.py`` and hold none of the
arithmetic below.

Sources (pages on HunyuanVideo; cited by page title and section):

* [P1] "HunyuanVideo 模型结构与数学原理" (note.shouss.top, research/video_generation/
  hunyuan_video):
  - §4 "Causal 3D VAE": latent grid T' = floor((F-1)/4)+1, H' = H/8, W' = W/8,
    and the 1x2x2 patch embedding giving N = T'·(H'/2)·(W'/2) video tokens;
    worked example 544x960x17 -> T'=5, H'=68, W'=120, N=10200; 720x1280x129
    -> 33x45x80 = 118800.
  - §5.2 "双流块": Q=[Q_v;Q_t] (same for K, V), Attn = softmax(QK^T/sqrt(128))V,
    joint length S = N + L with L the valid text length.
  - §5.4 "归一化、条件调制和残差门": RMSNorm on the Q and K of every
    attention head, RMSNorm(x) = gamma * x / sqrt((1/d) sum_j x_j^2 + eps).
  - §5.5 "3D RoPE": q'_p = R(p) q_p, k'_p = R(p) k_p; head dim 128 split
    (d_t, d_h, d_w) = (16, 56, 56); R_3D = R_t (+) R_h (+) R_w; theta = 256;
    applied to the video Q, K only, text tokens are not rotated.
  - §5.6 (shape chain): QKV last three dims [S, 24, 128]; joint length about
    10456 for the 17-frame example; 10456^2 ~ 1.09e8 score elements per head.
  - §9.1 "FlashAttention": exact attention, the kernel never materialises the
    N x N matrix but the result is that of the definition above.
* [P2] "HunyuanVideo" summary (zhao9797.github.io, ai-research/omni/2024/
  hunyuan-video), "Diffusion backbone (13B DiT)": 3D RoPE splits the channels
  into (dt, dh, dw) segments, each rotated by the time/height/width coordinate
  frequency, then concatenated; Table 2: 24 heads, head dim 128,
  (dt, dh, dw) = (16, 56, 56).
* [P4] README mirror (gittoolsai.com, Tencent-Hunyuan--HunyuanVideo),
  "单 GPU 推理": the supported height/width/frame settings.

Readings where the pages are silent:

  R1 pairing: adjacent channel pairs (2i, 2i+1) inside each axis segment (the
     RoFormer rotation the pages cite in [P1] §5.5).
  R2 axis order inside the head: t -> channels [0,16), h -> [16,72),
     w -> [72,128), the order (d_t, d_h, d_w) is listed in.
  R3 frequency law: pair i of an axis with d_a channels turns by
     pos · theta^(-2i/d_a), i = 0 .. d_a/2-1 (RoFormer form, per-axis d_a).
  R4 positions: integer, 0-based t in [0,T'), h in [0,H'/2), w in [0,W'/2).
  R5 rotation sign: (x0, x1) -> (x0 cos - x1 sin, x0 sin + x1 cos).
  R6 token order: video first, flattened t-major then h then w; text after.
  R7 text padding sits at the end of the text segment; keys at or past
     N + valid are masked out; padded text *query* rows are computed like any
     other row (they attend to the valid keys).
  R8 scale is a parameter, default 1/sqrt(128).
  R13 QK RMSNorm ([P1] §5.4, optional prologue): over the head dim d = 128 of
     each (token, head) row, y = gamma * x / sqrt(mean_j x_j^2 + eps), with one
     gamma of 128 channels shared by all heads (the formula has no head index).
  R14 video rows take the video stream's gamma, text rows the text stream's
     ([P1] §5.2: the double-stream blocks keep separate parameters per
     modality); a single-stream block passes the same gamma twice.
  R16 ring-attention blocks ([P1] §9.2): a query or key block is a run of
     consecutive joint-sequence rows given by its count of leading video rows
     and the global token index of the first; results of disjoint key blocks
     combine through their per-row log-sum-exp (the softmax over the union).
  R15 order: RMSNorm first, then the 3D rotation of the video rows (the norm
     acts on Q, K as projected, §5.4; RoPE rotates the Q, K that attention
     uses, §5.5). eps is a parameter (the pages give none).

Parity status: every function here is pinned by ``tests/test_oracle_pins.py``
(closed forms, invariants, a second independent formulation, a library SDPA
special case, and the pages' worked numbers in ``tests/golden/``). Parity
against real HunyuanVideo activations is unpinned: the pages carry no weights
and no printed attention outputs.
"""

from __future__ import annotations

import math

import numpy as np

HEAD_DIM = 128
# [P1] §5.5, [P2] Table 2: (d_t, d_h, d_w), summing to the head dim.
ROPE_AXIS_DIMS = (16, 56, 56)
DEFAULT_THETA = 256.0


def latent_grid(frames: int, height: int, width: int) -> tuple[int, int, int]:
    """Video-token grid (T', H'/2, W'/2) of an F x H x W clip.

    [P1] §4: the causal VAE keeps the first frame on its own, so
    T' = floor((F-1)/4) + 1 for F = 4k+1; space is compressed 8x
    (H' = H/8, W' = W/8); the DiT patch is 1x2x2, halving H' and W' again.
    Raises ValueError where the pages' formula does not give an integer grid.
    """
    if frames < 1 or (frames - 1) % 4 != 0:
        raise ValueError(f"frame count {frames} is not of the form 4k+1")
    if height % 16 or width % 16 or height <= 0 or width <= 0:
        raise ValueError(f"{height}x{width} is not a multiple of 16 (VAE 8x, patch 2x)")
    t_lat = (frames - 1) // 4 + 1
    h_lat = height // 8
    w_lat = width // 8
    return t_lat, h_lat // 2, w_lat // 2


def video_token_count(frames: int, height: int, width: int) -> int:
    """N = T' · (H'/2) · (W'/2)  ([P1] §4)."""
    t, hp, wp = latent_grid(frames, height, width)
    return t * hp * wp


def token_positions(t_lat: int, hp: int, wp: int) -> np.ndarray:
    """(N, 3) integer (t, h, w) of each video token, in sequence order.

    Reading R6/R4: the patch grid is flattened t-major, then h, then w, and
    coordinates are 0-based integers.
    """
    n = t_lat * hp * wp
    pos = np.empty((n, 3), dtype=np.int64)
    idx = 0
    for t in range(t_lat):
        for h in range(hp):
            for w in range(wp):
                pos[idx] = (t, h, w)
                idx += 1
    return pos


def axis_frequencies(theta: float = DEFAULT_THETA) -> list[np.ndarray]:
    """Per-axis rotation frequencies, reading R3: theta^(-2i/d_a)."""
    out = []
    for d_a in ROPE_AXIS_DIMS:
        i = np.arange(d_a // 2, dtype=np.float64)
        out.append(np.power(float(theta), -2.0 * i / d_a))
    return out


def rope3d_rotate(x: np.ndarray, pos: np.ndarray, theta: float = DEFAULT_THETA) -> np.ndarray:
    """Apply R_3D(pos) = R_t (+) R_h (+) R_w to each row of ``x``.

    [P1] §5.5 / [P2]: the 128 channels are cut into the t, h and w segments
    (16, 56, 56) (reading R2); inside a segment adjacent channels (2i, 2i+1)
    form a pair (R1) turned by the angle pos_axis · theta^(-2i/d_a) (R3) as
    (x0, x1) -> (x0 cos - x1 sin, x0 sin + x1 cos) (R5).

    x: (n, 128) float64; pos: (n, 3) integer (t, h, w). Returns a new array.
    """
    x = np.asarray(x, dtype=np.float64)
    pos = np.asarray(pos)
    assert x.ndim == 2 and x.shape[1] == HEAD_DIM and pos.shape == (x.shape[0], 3)
    out = x.copy()
    freqs = axis_frequencies(theta)
    offset = 0
    for axis, d_a in enumerate(ROPE_AXIS_DIMS):
        p = pos[:, axis].astype(np.float64)
        for i in range(d_a // 2):
            c0 = offset + 2 * i
            angle = p * freqs[axis][i]
            cos = np.cos(angle)
            sin = np.sin(angle)
            x0 = x[:, c0]
            x1 = x[:, c0 + 1]
            out[:, c0] = x0 * cos - x1 * sin
            out[:, c0 + 1] = x0 * sin + x1 * cos
        offset += d_a
    return out


def rotate_sequence(x: np.ndarray, grid: tuple[int, int, int], theta: float = DEFAULT_THETA) -> np.ndarray:
    """Rotate the video rows of one head's joint sequence; text rows unchanged.

    x: (S, 128) for one (batch, head) in token order (video first, R6).
    [P1] §5.5: RoPE acts on the visual Q, K only.
    """
    t_lat, hp, wp = grid
    n = t_lat * hp * wp
    out = np.asarray(x, dtype=np.float64).copy()
    out[:n] = rope3d_rotate(out[:n], token_positions(t_lat, hp, wp), theta)
    return out


def rms_norm(x: np.ndarray, gamma: np.ndarray, eps: float) -> np.ndarray:
    """RMSNorm over the last axis ([P1] §5.4): gamma * x / sqrt(mean(x^2) + eps).

    x: (..., d) float64; gamma: (d,). Returns a new float64 array.
    """
    x = np.asarray(x, dtype=np.float64)
    gamma = np.asarray(gamma, dtype=np.float64)
    assert gamma.shape == (x.shape[-1],)
    mean_sq = np.mean(x * x, axis=-1, keepdims=True)
    return gamma * (x / np.sqrt(mean_sq + eps))


def qk_norm_rows(x: np.ndarray, is_video: np.ndarray, gamma_video: np.ndarray, gamma_text: np.ndarray,
                 eps: float) -> np.ndarray:
    """Per-head QK RMSNorm of rows of one head (R13-R14): video rows with the
    video stream's gamma, text rows with the text stream's gamma."""
    x = np.asarray(x, dtype=np.float64)
    out = np.empty_like(x)
    vid = np.asarray(is_video, dtype=bool)
    out[vid] = rms_norm(x[vid], gamma_video, eps)
    out[~vid] = rms_norm(x[~vid], gamma_text, eps)
    return out


def joint_attention_head(q: np.ndarray, k: np.ndarray, v: np.ndarray, grid: tuple[int, int, int],
                         valid: int, theta: float = DEFAULT_THETA, scale: float | None = None,
                         rows: np.ndarray | None = None, qk_norm: dict | None = None) -> np.ndarray:
    """Joint full attention of one (batch, head), float64.

    [P1] §5.2: over the concatenation [video ; text] compute
    softmax(Q'K'^T · scale) V with Q', K' the 3D-RoPE-rotated queries and keys
    (§5.5, video rows only). Keys are the N video tokens and the first
    ``valid`` text tokens (joint length N + L, L the valid text length);
    padded keys take no part (R7). ``rows`` selects query rows (default: all
    S rows, padded text rows included). ``qk_norm``, if given, is a dict with
    gamma_q_video, gamma_k_video, gamma_q_text, gamma_k_text (128 each) and
    eps: the RMSNorm prologue (R13-R15), applied before the rotation.

    q, k, v: (S, 128). Returns (len(rows), 128) float64.
    """
    if scale is None:
        scale = 1.0 / math.sqrt(HEAD_DIM)
    t_lat, hp, wp = grid
    n = t_lat * hp * wp
    s_len = q.shape[0]
    assert k.shape[0] == s_len and v.shape[0] == s_len
    assert 0 <= valid <= s_len - n
    if rows is None:
        rows = np.arange(s_len)
    rows = np.asarray(rows, dtype=np.int64)
    kv_len = n + valid

    qr = np.asarray(q, dtype=np.float64)[rows].copy()
    kr = np.asarray(k, dtype=np.float64)[:kv_len].copy()
    vid = rows < n
    if qk_norm is not None:
        eps = float(qk_norm["eps"])
        qr = qk_norm_rows(qr, vid, qk_norm["gamma_q_video"], qk_norm["gamma_q_text"], eps)
        kr = qk_norm_rows(kr, np.arange(kv_len) < n, qk_norm["gamma_k_video"], qk_norm["gamma_k_text"], eps)
    if vid.any():
        qr[vid] = rope3d_rotate(qr[vid], token_positions(t_lat, hp, wp)[rows[vid]], theta)
    kr = rotate_sequence(kr, grid, theta)
    vv = np.asarray(v, dtype=np.float64)[:kv_len]

    scores = (qr @ kr.T) * scale                     # (rows, N + valid)
    scores -= scores.max(axis=1, keepdims=True)      # max-subtracted softmax
    p = np.exp(scores)
    p /= p.sum(axis=1, keepdims=True)
    return p @ vv


def joint_attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, grid: tuple[int, int, int],
                    text_len: int, text_valid, theta: float = DEFAULT_THETA,
                    scale: float | None = None, qk_norm: dict | None = None) -> np.ndarray:
    """Full output [B, S, heads, 128] float64 of the joint attention call.

    Inputs in the boundary layout [B, S, heads, 128] with S = N + text_len
    ([P1] §5.6: QKV reshaped to [S, 24, 128] per sample).
    """
    b_sz, s_len, heads, d = q.shape
    t_lat, hp, wp = grid
    assert d == HEAD_DIM and s_len == t_lat * hp * wp + text_len
    out = np.empty((b_sz, s_len, heads, d), dtype=np.float64)
    for b in range(b_sz):
        for h in range(heads):
            out[b, :, h, :] = joint_attention_head(q[b, :, h], k[b, :, h], v[b, :, h], grid,
                                                   int(text_valid[b]), theta, scale, qk_norm=qk_norm)
    return out


def joint_attention_samples(q: np.ndarray, k: np.ndarray, v: np.ndarray, grid: tuple[int, int, int],
                            text_len: int, text_valid, samples: np.ndarray, theta: float = DEFAULT_THETA,
                            scale: float | None = None, qk_norm: dict | None = None) -> np.ndarray:
    """Outputs of selected (b, head, row) triples, float64, shape (n_samples, 128).

    Same definition as ``joint_attention``; heads are grouped so that each
    (b, head) rotates its keys once.
    """
    samples = np.asarray(samples, dtype=np.int64)
    out = np.empty((samples.shape[0], HEAD_DIM), dtype=np.float64)
    keys = samples[:, 0] * q.shape[2] + samples[:, 1]
    for key in np.unique(keys):
        sel = np.nonzero(keys == key)[0]
        b, h = int(samples[sel[0], 0]), int(samples[sel[0], 1])
        out[sel] = joint_attention_head(q[b, :, h], k[b, :, h], v[b, :, h], grid,
                                        int(text_valid[b]), theta, scale, rows=samples[sel, 2], qk_norm=qk_norm)
    return out


def joint_attention_block(q: np.ndarray, k: np.ndarray, v: np.ndarray, grid: tuple[int, int, int],
                          q_video: int, q_pos0: int, k_video: int, k_pos0: int, kv_len: int,
                          theta: float = DEFAULT_THETA, scale: float | None = None,
                          qk_norm: dict | None = None) -> tuple[np.ndarray, np.ndarray]:
    """Attention of a block of query rows against a block of key rows, with
    the log-sum-exp of each row: the step of ring attention ([P1] §9.2: each
    rank keeps a segment of queries while K/V blocks pass around the ring).

    Reading R16: a block holds a run of consecutive joint-sequence rows; its
    first ``*_video`` rows are video tokens whose global token indices start at
    ``*_pos0`` (rotated by the 3D RoPE of those tokens, R4/R6), the rest are
    text rows (not rotated). Only the first ``kv_len`` key rows take part.
    Returns O = softmax(scores) V over those keys and
    lse = log(sum_j exp(score_j)) (natural log of the scaled scores), per row;
    a block with kv_len = 0 gives O = 0 and lse = -inf (it contributes
    nothing when merged).

    q: (Sq, 128), k, v: (Sk, 128) for one (batch, head).
    """
    if scale is None:
        scale = 1.0 / math.sqrt(HEAD_DIM)
    t_lat, hp, wp = grid
    pos = token_positions(t_lat, hp, wp)
    qr = np.asarray(q, dtype=np.float64).copy()
    kr = np.asarray(k, dtype=np.float64)[:kv_len].copy()
    vv = np.asarray(v, dtype=np.float64)[:kv_len]
    if qk_norm is not None:
        eps = float(qk_norm["eps"])
        qr = qk_norm_rows(qr, np.arange(qr.shape[0]) < q_video, qk_norm["gamma_q_video"],
                          qk_norm["gamma_q_text"], eps)
        kr = qk_norm_rows(kr, np.arange(kv_len) < k_video, qk_norm["gamma_k_video"], qk_norm["gamma_k_text"], eps)
    if q_video > 0:
        qr[:q_video] = rope3d_rotate(qr[:q_video], pos[q_pos0:q_pos0 + q_video], theta)
    kv_vid = min(k_video, kv_len)
    if kv_vid > 0:
        kr[:kv_vid] = rope3d_rotate(kr[:kv_vid], pos[k_pos0:k_pos0 + kv_vid], theta)
    if kv_len == 0:
        return np.zeros_like(qr), np.full(qr.shape[0], -np.inf)
    scores = (qr @ kr.T) * scale
    mx = scores.max(axis=1, keepdims=True)
    p = np.exp(scores - mx)
    tot = p.sum(axis=1, keepdims=True)
    return (p / tot) @ vv, (mx + np.log(tot))[:, 0]


def merge_blocks(outs, lses) -> tuple[np.ndarray, np.ndarray]:
    """Combine the results of disjoint key blocks of the same query rows:
    O = sum_i exp(lse_i - lse) O_i with lse = log(sum_i exp(lse_i))
    (the softmax over the union of the blocks' keys)."""
    lses = np.stack([np.asarray(x, dtype=np.float64) for x in lses])       # (blocks, rows)
    top = lses.max(axis=0)
    safe = np.where(np.isfinite(top), top, 0.0)
    w = np.exp(lses - safe)                                                # (blocks, rows)
    tot = w.sum(axis=0)
    out = sum(w[i][:, None] * np.asarray(o, dtype=np.float64) for i, o in enumerate(outs))
    with np.errstate(invalid="ignore", divide="ignore"):
        out = np.where(tot[:, None] > 0, out / np.where(tot > 0, tot, 1.0)[:, None], 0.0)
        lse = np.where(tot > 0, safe + np.log(np.where(tot > 0, tot, 1.0)), -np.inf)
    return out, lse


def attention_flops(batch: int, heads: int, grid: tuple[int, int, int], text_len: int, text_valid) -> float:
    """Algorithmic FLOPs of one call: 2 GEMMs of S x (N+valid) x 128 per (b, head).

    Masked padding keys are not counted.
    """
    n = grid[0] * grid[1] * grid[2]
    s_len = n + text_len
    total = 0.0
    for b in range(batch):
        total += 4.0 * heads * s_len * (n + int(text_valid[b])) * HEAD_DIM
    return total
