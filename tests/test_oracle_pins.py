"""Pins for the float64 oracle: what the pages and the mathematics fix.

Each test checks the oracle against something other than itself: the pages'
worked numbers (tests/golden/), closed forms, invariants, a second and
independent formulation of the rotation, brute force on tiny inputs, and a
library attention routine in a special case. ``test_planted_mistakes`` plants
plausible errors in a copy of the oracle (on the CPU) and checks that a pin
fails for each.
"""

from __future__ import annotations

import math
from pathlib import Path

import numpy as np
import pytest
import scipy.linalg
import torch

from oracle import hv_oracle as O

GOLDEN = Path(__file__).parent / "golden"


def _rows(name):
    out = []
    for line in (GOLDEN / name).read_text().splitlines():
        line = line.split("#", 1)[0].strip()
        if line:
            out.append(line.split())
    return out


# ---------------------------------------------------------------- token grid

def test_token_grid_worked_examples():
    rows = _rows("token_grids.txt")
    assert len(rows) == 2
    for f, h, w, t, hp, wp, n in (map(int, r) for r in rows):
        assert O.latent_grid(f, h, w) == (t, hp, wp)
        assert O.video_token_count(f, h, w) == n


def test_supported_sizes_give_integer_grids():
    for h, w, f in (map(int, r) for r in _rows("supported_sizes.txt")):
        t, hp, wp = O.latent_grid(f, h, w)
        assert t == 33                       # 129 frames -> 33 latent frames
        assert hp * 16 == h and wp * 16 == w


def test_image_is_single_latent_frame():
    assert O.latent_grid(1, 256, 256) == (1, 16, 16)
    assert O.video_token_count(1, 256, 256) == 256
    assert O.video_token_count(129, 544, 960) == 33 * 34 * 60 == 67320


def test_token_grid_rejects_non_grid_sizes():
    for f, h, w in [(16, 544, 960), (17, 540, 960), (17, 544, 968), (0, 544, 960)]:
        with pytest.raises(ValueError):
            O.latent_grid(f, h, w)


def test_shape_chain():
    g = {r[0]: r[1:] for r in _rows("shape_chain.txt")}
    n = int(g["video_tokens"][0])
    s = n + int(g["text_tokens"][0])
    assert s == int(g["joint_len"][0])
    assert abs(s * s - float(g["score_elems_per_head_approx"][0])) / 1.09e8 < 0.005
    _, c, t, h_lat, w_lat = map(int, g["latent_shape"])
    assert c * 1 * 2 * 2 == 64                     # 16 latent channels x 1x2x2 patch
    assert (t, h_lat // 2, w_lat // 2) == O.latent_grid(17, 544, 960)
    assert sum(map(int, g["rope_split"])) == int(g["head_dim"][0]) == O.HEAD_DIM
    assert tuple(map(int, g["rope_split"])) == O.ROPE_AXIS_DIMS


def test_token_order_is_row_major_over_grid():
    grid = (3, 4, 5)
    pos = O.token_positions(*grid)
    t, h, w = np.unravel_index(np.arange(np.prod(grid)), grid)
    assert np.array_equal(pos, np.stack([t, h, w], axis=1))


# ------------------------------------------------------------------ 3D RoPE

def _rand(shape, seed=0):
    return np.random.default_rng(seed).standard_normal(shape)


def _rand_pos(n, seed=1, hi=(33, 45, 80)):
    rng = np.random.default_rng(seed)
    return np.stack([rng.integers(0, hi[a], n) for a in range(3)], axis=1)


def test_rope_preserves_norm_per_row_and_per_pair():
    x = _rand((64, 128))
    pos = _rand_pos(64)
    y = O.rope3d_rotate(x, pos)
    np.testing.assert_allclose(np.linalg.norm(y, axis=1), np.linalg.norm(x, axis=1), rtol=1e-12)
    pair_x = x[:, 0::2] ** 2 + x[:, 1::2] ** 2
    pair_y = y[:, 0::2] ** 2 + y[:, 1::2] ** 2
    np.testing.assert_allclose(pair_y, pair_x, rtol=1e-12, atol=1e-14)


def test_rope_identity_at_origin():
    x = _rand((8, 128))
    y = O.rope3d_rotate(x, np.zeros((8, 3), dtype=np.int64))
    assert np.array_equal(x, y)


def test_rope_relative_position_property():
    """(R_m q) . (R_n k) depends only on m - n per axis (RoFormer, cited in §5.5)."""
    rng = np.random.default_rng(3)
    q = _rand((32, 128), 4)
    k = _rand((32, 128), 5)
    m = _rand_pos(32, 6, hi=(10, 20, 30))
    n = _rand_pos(32, 7, hi=(10, 20, 30))
    delta = np.stack([rng.integers(0, 20, 32), rng.integers(0, 20, 32), rng.integers(0, 40, 32)], axis=1)
    d0 = np.sum(O.rope3d_rotate(q, m) * O.rope3d_rotate(k, n), axis=1)
    d1 = np.sum(O.rope3d_rotate(q, m + delta) * O.rope3d_rotate(k, n + delta), axis=1)
    np.testing.assert_allclose(d1, d0, rtol=1e-12, atol=1e-11)
    # and it does depend on the offset: moving only one side changes it
    d2 = np.sum(O.rope3d_rotate(q, m + delta) * O.rope3d_rotate(k, n), axis=1)
    assert np.max(np.abs(d2 - d0)) > 1e-3


def _complex_route(x, pos, theta):
    """Second formulation: each adjacent pair as a complex number times e^{i phi}."""
    z = x[:, 0::2] + 1j * x[:, 1::2]                      # 64 pairs
    angles = np.empty((x.shape[0], 64))
    col = 0
    for axis, d_a in enumerate((16, 56, 56)):
        for i in range(d_a // 2):
            angles[:, col] = pos[:, axis] * theta ** (-(2.0 * i) / d_a)
            col += 1
    zr = z * np.exp(1j * angles)
    out = np.empty_like(x)
    out[:, 0::2] = zr.real
    out[:, 1::2] = zr.imag
    return out


def test_rope_matches_complex_formulation():
    x = _rand((48, 128), 8)
    pos = _rand_pos(48, 9)
    for theta in (256.0, 10000.0):
        np.testing.assert_allclose(O.rope3d_rotate(x, pos, theta), _complex_route(x, pos, theta),
                                   rtol=0, atol=1e-12)


def test_rope_matches_matrix_exponential_of_generator():
    """Third formulation: R = expm(G), G block-diagonal with [[0,-phi],[phi,0]] blocks."""
    x = _rand((6, 128), 10)
    pos = _rand_pos(6, 11, hi=(5, 7, 9))
    for r in range(6):
        gen = np.zeros((128, 128))
        col = 0
        for axis, d_a in enumerate((16, 56, 56)):
            for i in range(d_a // 2):
                phi = pos[r, axis] * 256.0 ** (-(2.0 * i) / d_a)
                c = col + 2 * i
                gen[c + 1, c] = phi
                gen[c, c + 1] = -phi
            col += d_a
        rot = scipy.linalg.expm(gen)
        np.testing.assert_allclose(O.rope3d_rotate(x[r:r + 1], pos[r:r + 1])[0], rot @ x[r], atol=1e-10)


def test_rope_axis_segments_are_isolated():
    """Channels of one axis only see that axis' coordinate (R_t (+) R_h (+) R_w)."""
    x = _rand((4, 128), 12)
    segs = {0: slice(0, 16), 1: slice(16, 72), 2: slice(72, 128)}
    for axis, sl in segs.items():
        only = np.zeros_like(x)
        only[:, sl] = x[:, sl]
        pos = _rand_pos(4, 13)
        pos_other = pos.copy()
        pos_other[:, [a for a in range(3) if a != axis]] = 0
        y = O.rope3d_rotate(only, pos)
        assert np.array_equal(y, O.rope3d_rotate(only, pos_other))
        outside = np.ones(128, dtype=bool)
        outside[sl] = False
        assert np.all(y[:, outside] == 0)


def test_rope_first_pair_of_each_axis_turns_by_position():
    """theta^0 = 1: pair 0 of every axis turns by exactly pos radians, any theta."""
    for axis, c0 in enumerate((0, 16, 72)):
        e = np.zeros((1, 128))
        e[0, c0] = 1.0
        pos = np.zeros((1, 3), dtype=np.int64)
        pos[0, axis] = 7
        for theta in (256.0, 3.0):
            y = O.rope3d_rotate(e, pos, theta)
            assert math.isclose(math.atan2(y[0, c0 + 1], y[0, c0]), 7 - 2 * math.pi, abs_tol=1e-12)


def test_rope_theta_one_turns_every_pair_alike():
    x = _rand((3, 128), 14)
    pos = np.array([[2, 2, 2], [5, 5, 5], [1, 1, 1]])
    y = O.rope3d_rotate(x, pos, theta=1.0)
    for r in range(3):
        ang = pos[r, 0]
        c, s = math.cos(ang), math.sin(ang)
        np.testing.assert_allclose(y[r, 0::2], x[r, 0::2] * c - x[r, 1::2] * s, atol=1e-12)
        np.testing.assert_allclose(y[r, 1::2], x[r, 0::2] * s + x[r, 1::2] * c, atol=1e-12)


def test_rope_frequencies_decrease_geometrically():
    """Angle per unit position, read back off a rotated basis vector."""
    for axis, (c0, d_a) in enumerate(((0, 16), (16, 56), (72, 56))):
        angles = []
        for i in range(d_a // 2):
            e = np.zeros((1, 128))
            e[0, c0 + 2 * i] = 1.0
            pos = np.zeros((1, 3), dtype=np.int64)
            pos[0, axis] = 1
            y = O.rope3d_rotate(e, pos)
            angles.append(math.atan2(y[0, c0 + 2 * i + 1], y[0, c0 + 2 * i]))
        a = np.array(angles)
        assert a[0] == pytest.approx(1.0, abs=1e-14)
        assert np.all(np.diff(a) < 0)
        ratios = a[1:] / a[:-1]
        np.testing.assert_allclose(ratios, ratios[0], rtol=1e-12)
        # the geometric ladder spans theta^0 .. theta^-(d-2)/d
        assert a[-1] == pytest.approx(a[0] * ratios[0] ** (d_a // 2 - 1), rel=1e-12)


def test_text_rows_untouched_by_rotation():
    grid = (2, 3, 4)
    x = _rand((24 + 10, 128), 15)
    y = O.rotate_sequence(x, grid)
    assert np.array_equal(y[24:], x[24:])
    assert not np.array_equal(y[1:24], x[1:24])
    assert np.array_equal(y[0], x[0])                    # token 0 sits at (0,0,0)


# ---------------------------------------------------------------- attention

def _brute_force_attention(q, k, v, grid, text_len, valid, scale):
    """Explicit S x S score matrix, additive -inf mask, python loops for softmax."""
    n = grid[0] * grid[1] * grid[2]
    s_len = q.shape[0]
    pos = np.zeros((s_len, 3), dtype=np.int64)
    pos[:n] = O.token_positions(*grid)
    qr, kr = q.copy(), k.copy()
    qr[:n] = _complex_route(q[:n], pos[:n], 256.0)
    kr[:n] = _complex_route(k[:n], pos[:n], 256.0)
    mask = np.zeros((s_len, s_len))
    mask[:, n + valid:] = -np.inf
    scores = qr @ kr.T * scale + mask
    out = np.zeros_like(q)
    for i in range(s_len):
        mx = max(scores[i])
        w = [math.exp(s - mx) if s != -np.inf else 0.0 for s in scores[i]]
        tot = math.fsum(w)
        for j in range(s_len):
            if w[j]:
                out[i] += (w[j] / tot) * v[j]
    return out


@pytest.mark.parametrize("valid", [5, 0, 8])
def test_attention_matches_brute_force_on_tiny(valid):
    grid, text_len = (2, 4, 4), 8
    s_len = 32 + text_len
    q, k, v = (_rand((s_len, 128), s) for s in (20, 21, 22))
    ref = _brute_force_attention(q, k, v, grid, text_len, valid, 1 / math.sqrt(128))
    got = O.joint_attention_head(q, k, v, grid, valid)
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)


def test_attention_batched_layout_matches_per_head():
    grid, text_len = (1, 2, 3), 4
    s_len = 6 + text_len
    q, k, v = (_rand((2, s_len, 3, 128), s) for s in (30, 31, 32))
    valid = [4, 1]
    full = O.joint_attention(q, k, v, grid, text_len, valid)
    for b in range(2):
        for h in range(3):
            np.testing.assert_array_equal(full[b, :, h], O.joint_attention_head(q[b, :, h], k[b, :, h],
                                                                                v[b, :, h], grid, valid[b]))
    samples = np.array([[0, 2, 9], [1, 0, 0], [1, 1, 5], [0, 2, 1]])
    np.testing.assert_allclose(O.joint_attention_samples(q, k, v, grid, text_len, valid, samples),
                               full[samples[:, 0], samples[:, 2], samples[:, 1]], atol=1e-14)


def test_attention_single_video_token_equals_library_sdpa():
    """T'=H'/2=W'/2=1: the one video token sits at the origin, RoPE is the identity."""
    grid, text_len = (1, 1, 1), 40
    s_len = 1 + text_len
    q, k, v = (_rand((s_len, 128), s) for s in (40, 41, 42))
    for valid in (40, 17, 0):
        got = O.joint_attention_head(q, k, v, grid, valid)
        keep = torch.zeros(s_len, dtype=torch.bool)
        keep[:1 + valid] = True
        ref = torch.nn.functional.scaled_dot_product_attention(
            torch.from_numpy(q)[None, None], torch.from_numpy(k)[None, None], torch.from_numpy(v)[None, None],
            attn_mask=keep[None, None, None, :])[0, 0].numpy()
        np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)


def test_attention_composition_equals_library_sdpa_on_rotated_inputs():
    """RoPE is pinned above; this pins the attention around it against SDPA."""
    grid, text_len, valid = (2, 5, 6), 20, 13
    n = 60
    s_len = n + text_len
    q, k, v = (_rand((s_len, 128), s) for s in (50, 51, 52))
    pos = O.token_positions(*grid)
    qr, kr = q.copy(), k.copy()
    qr[:n] = _complex_route(q[:n], pos, 256.0)
    kr[:n] = _complex_route(k[:n], pos, 256.0)
    keep = torch.zeros(s_len, dtype=torch.bool)
    keep[:n + valid] = True
    for scale in (None, 0.05):
        ref = torch.nn.functional.scaled_dot_product_attention(
            torch.from_numpy(qr)[None, None], torch.from_numpy(kr)[None, None], torch.from_numpy(v)[None, None],
            attn_mask=keep[None, None, None, :], scale=scale)[0, 0].numpy()
        np.testing.assert_allclose(O.joint_attention_head(q, k, v, grid, valid, scale=scale), ref,
                                   rtol=0, atol=1e-12)


def test_softmax_rows_sum_to_one():
    grid, text_len = (2, 3, 3), 6
    s_len = 18 + text_len
    q, k = _rand((s_len, 128), 60) * 3, _rand((s_len, 128), 61) * 3
    out = O.joint_attention_head(q, k, np.ones((s_len, 128)), grid, 4)
    np.testing.assert_allclose(out, 1.0, rtol=0, atol=1e-12)


def test_zero_query_gives_mean_of_valid_values():
    grid, text_len, valid = (2, 3, 3), 6, 4
    s_len = 18 + text_len
    k, v = _rand((s_len, 128), 62), _rand((s_len, 128), 63)
    out = O.joint_attention_head(np.zeros((s_len, 128)), k, v, grid, valid)
    np.testing.assert_allclose(out, np.broadcast_to(v[:18 + valid].mean(axis=0), out.shape), atol=1e-12)


def test_padding_invariance():
    grid, text_len, valid = (2, 3, 3), 6, 2
    s_len = 18 + text_len
    q, k, v = (_rand((s_len, 128), s) for s in (64, 65, 66))
    base = O.joint_attention_head(q, k, v, grid, valid)
    k2, v2 = k.copy(), v.copy()
    k2[18 + valid:] = 1e3
    v2[18 + valid:] = -7.0
    np.testing.assert_array_equal(O.joint_attention_head(q, k2, v2, grid, valid), base)


def test_attention_flops_worked_sizes():
    # 4 * heads * S * (N + valid) * 128, masked padding not counted
    f = O.attention_flops(1, 24, (33, 45, 80), 256, [138])
    assert f == pytest.approx(174.0e12, rel=0.002)
    assert O.attention_flops(1, 24, (5, 34, 60), 256, [138]) == pytest.approx(1.33e12, rel=0.01)


# ------------------------------------------------ planted mistakes are caught

def _pins_fail(monkeypatch, patch):
    """Apply ``patch`` to the oracle module, run the pins, report whether one fails."""
    patch(monkeypatch)
    checks = [test_rope_matches_complex_formulation, test_rope_relative_position_property,
              test_rope_axis_segments_are_isolated, test_rope_first_pair_of_each_axis_turns_by_position,
              test_rope_frequencies_decrease_geometrically,
              lambda: test_attention_matches_brute_force_on_tiny(5),
              test_attention_composition_equals_library_sdpa_on_rotated_inputs,
              test_token_order_is_row_major_over_grid, test_token_grid_worked_examples]
    for check in checks:
        try:
            check()
        except AssertionError:
            return True
    return False


def test_planted_mistakes(monkeypatch):
    orig_rotate = O.rope3d_rotate
    orig_freqs = O.axis_frequencies
    orig_positions = O.token_positions

    def wrong_sign(mp):
        mp.setattr(O, "rope3d_rotate", lambda x, pos, theta=256.0: orig_rotate(x, -np.asarray(pos), theta))

    def wrong_freq(mp):
        mp.setattr(O, "axis_frequencies", lambda theta=256.0: [np.power(float(theta), -np.arange(d // 2) / d)
                                                               for d in O.ROPE_AXIS_DIMS])

    def swapped_axes(mp):
        mp.setattr(O, "ROPE_AXIS_DIMS", (56, 16, 56))

    def wrong_order(mp):
        def f(t, hp, wp):
            p = orig_positions(t, hp, wp)
            return p[:, [0, 2, 1]] if hp == wp else p[np.lexsort((p[:, 1], p[:, 2], p[:, 0]))]
        mp.setattr(O, "token_positions", f)

    def wrong_grid(mp):
        mp.setattr(O, "latent_grid", lambda f, h, w: (f // 4, h // 16, w // 16))

    for patch in (wrong_sign, wrong_freq, swapped_axes, wrong_order, wrong_grid):
        with monkeypatch.context() as mp:
            assert _pins_fail(mp, patch), patch.__name__
    assert O.rope3d_rotate is orig_rotate and O.axis_frequencies is orig_freqs
