"""Pins for the oracle's QK-RMSNorm prologue ("HunyuanVideo 模型结构与数学原理"
§5.4: RMSNorm on the Q and K of every attention head).

Closed forms and invariants of RMSNorm, a library RMSNorm (torch's, in
float64) as the independent formulation, and the composition with the rest
of the oracle: norm per modality first, then the 3D rotation. Plausible
mistakes are planted in a copy of the oracle's source (on the CPU) and a pin
must fail for each.
"""

from __future__ import annotations

import math
import types
from pathlib import Path

import numpy as np
import pytest
import torch

from oracle import hv_oracle as O

ORACLE_SRC = Path(O.__file__).read_text()


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def _lib_rms(x, gamma, eps):
    t = torch.from_numpy(np.ascontiguousarray(x))
    return torch.nn.functional.rms_norm(t, (x.shape[-1],), torch.from_numpy(np.asarray(gamma, np.float64)),
                                        eps).numpy()


def _norm_params(seed, eps=1e-6):
    rng = np.random.default_rng(seed)
    g = lambda: rng.uniform(0.25, 2.0, 128)
    return {"gamma_q_video": g(), "gamma_k_video": g(), "gamma_q_text": g(), "gamma_k_text": g(), "eps": eps}


# ------------------------------------------------------------- RMSNorm alone

def check_worked_vector(M=O):
    # x = (3, 4, 0, ..., 0) over d = 128: mean of squares 25/128, so
    # y = x * sqrt(128) / 5 with gamma = 1 and eps = 0.
    x = np.zeros(128)
    x[0], x[1] = 3.0, 4.0
    y = M.rms_norm(x, np.ones(128), 0.0)
    assert y[0] == pytest.approx(3 * math.sqrt(128) / 5, rel=1e-15)
    assert y[1] == pytest.approx(4 * math.sqrt(128) / 5, rel=1e-15)
    assert np.all(y[2:] == 0)


def check_matches_library(M=O):
    x = _rand((7, 3, 128), 1) * 3.0
    gamma = np.random.default_rng(2).uniform(-2, 2, 128)
    for eps in (0.0, 1e-6, 0.5):
        np.testing.assert_allclose(M.rms_norm(x, gamma, eps), _lib_rms(x, gamma, eps), rtol=1e-13, atol=1e-14)


def test_rms_norm_worked_vector():
    check_worked_vector()


def test_rms_norm_matches_library():
    check_matches_library()


def test_rms_norm_unit_rms_and_scale_invariance():
    x = _rand((50, 128), 3)
    y = O.rms_norm(x, np.ones(128), 0.0)
    np.testing.assert_allclose(np.sqrt(np.mean(y * y, axis=-1)), 1.0, rtol=1e-14)
    np.testing.assert_allclose(O.rms_norm(7.5 * x, np.ones(128), 0.0), y, rtol=1e-14, atol=1e-15)


def test_rms_norm_gamma_is_channelwise():
    x = _rand((9, 128), 4)
    gamma = np.random.default_rng(5).uniform(-3, 3, 128)
    np.testing.assert_allclose(O.rms_norm(x, gamma, 1e-3), gamma * O.rms_norm(x, np.ones(128), 1e-3), rtol=1e-15)


def test_rms_norm_eps_limits():
    assert np.all(O.rms_norm(np.zeros((2, 128)), np.ones(128), 1e-6) == 0)
    x = _rand((3, 128), 6) * 1e-6        # mean square ~1e-12, far below eps
    np.testing.assert_allclose(O.rms_norm(x, np.ones(128), 1e-2), x / math.sqrt(1e-2), rtol=1e-9)


def test_rms_norm_rows_are_independent():
    x = _rand((6, 128), 7)
    y = O.rms_norm(x, np.ones(128), 1e-6)
    x2 = x.copy()
    x2[3] *= 100.0
    x2[4] = 0.0
    y2 = O.rms_norm(x2, np.ones(128), 1e-6)
    np.testing.assert_array_equal(np.delete(y2, [3, 4], axis=0), np.delete(y, [3, 4], axis=0))


# ------------------------------------------------- prologue inside attention

def check_attention_equals_prenormalised(M=O):
    """norm per modality (library RMSNorm), then the oracle without the prologue."""
    grid, text_len, valid = (2, 3, 5), 12, 7
    n = 30
    s_len = n + text_len
    q, k, v = (_rand((s_len, 128), s) * 2.0 for s in (10, 11, 12))
    prm = _norm_params(13, eps=1e-3)
    qn, kn = q.copy(), k.copy()
    qn[:n] = _lib_rms(q[:n], prm["gamma_q_video"], prm["eps"])
    qn[n:] = _lib_rms(q[n:], prm["gamma_q_text"], prm["eps"])
    kn[:n] = _lib_rms(k[:n], prm["gamma_k_video"], prm["eps"])
    kn[n:] = _lib_rms(k[n:], prm["gamma_k_text"], prm["eps"])
    ref = O.joint_attention_head(qn, kn, v, grid, valid)
    got = M.joint_attention_head(q, k, v, grid, valid, qk_norm=prm)
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)
    rows = np.array([0, 29, 30, 41, 5])
    np.testing.assert_allclose(M.joint_attention_head(q, k, v, grid, valid, rows=rows, qk_norm=prm), ref[rows],
                               rtol=0, atol=1e-12)


def test_attention_with_prologue_equals_prenormalised_inputs():
    check_attention_equals_prenormalised()


def test_prologue_batched_and_sampled_forms_agree():
    grid, text_len = (1, 2, 3), 4
    s_len = 6 + text_len
    q, k, v = (_rand((2, s_len, 3, 128), s) for s in (20, 21, 22))
    valid = [4, 1]
    prm = _norm_params(23)
    full = O.joint_attention(q, k, v, grid, text_len, valid, qk_norm=prm)
    for b in range(2):
        for h in range(3):
            np.testing.assert_array_equal(full[b, :, h], O.joint_attention_head(q[b, :, h], k[b, :, h], v[b, :, h],
                                                                                grid, valid[b], qk_norm=prm))
    samples = np.array([[0, 2, 9], [1, 0, 0], [1, 1, 5], [0, 2, 1]])
    np.testing.assert_allclose(O.joint_attention_samples(q, k, v, grid, text_len, valid, samples, qk_norm=prm),
                               full[samples[:, 0], samples[:, 2], samples[:, 1]], atol=1e-14)


def test_unit_gamma_zero_eps_removes_input_scale():
    """With gamma = 1 and eps = 0 the prologue makes attention blind to the
    per-row scale of Q and K."""
    grid, text_len, valid = (1, 3, 4), 6, 6
    s_len = 12 + text_len
    q, k, v = (_rand((s_len, 128), s) for s in (30, 31, 32))
    prm = {n: np.ones(128) for n in ("gamma_q_video", "gamma_k_video", "gamma_q_text", "gamma_k_text")}
    prm["eps"] = 0.0
    row_scale = np.random.default_rng(33).uniform(0.1, 10.0, (s_len, 1))
    a = O.joint_attention_head(q, k, v, grid, valid, qk_norm=prm)
    b = O.joint_attention_head(q * row_scale, k * row_scale[::-1], v, grid, valid, qk_norm=prm)
    np.testing.assert_allclose(a, b, rtol=0, atol=1e-12)


# ----------------------------------------------------------- planted mistakes

def _planted(old: str, new: str) -> types.ModuleType:
    assert ORACLE_SRC.count(old) == 1, old
    mod = types.ModuleType("planted_oracle")
    exec(compile(ORACLE_SRC.replace(old, new), "planted_oracle", "exec"), mod.__dict__)
    return mod


_NORM = '    if qk_norm is not None:\n        eps = float(qk_norm["eps"])\n        qr = qk_norm_rows(qr, vid, qk_norm["gamma_q_video"], qk_norm["gamma_q_text"], eps)\n        kr = qk_norm_rows(kr, np.arange(kv_len) < n, qk_norm["gamma_k_video"], qk_norm["gamma_k_text"], eps)\n'
_ROT = '    if vid.any():\n        qr[vid] = rope3d_rotate(qr[vid], token_positions(t_lat, hp, wp)[rows[vid]], theta)\n    kr = rotate_sequence(kr, grid, theta)\n'

PLANTS = {
    "sum instead of mean": ("np.mean(x * x, axis=-1, keepdims=True)", "np.sum(x * x, axis=-1, keepdims=True)"),
    "eps outside the root": ("np.sqrt(mean_sq + eps)", "(np.sqrt(mean_sq) + eps)"),
    "norm over tokens": ("np.mean(x * x, axis=-1, keepdims=True)", "np.mean(x * x, axis=0, keepdims=True)"),
    "text gamma on video rows": ('qr = qk_norm_rows(qr, vid, qk_norm["gamma_q_video"], qk_norm["gamma_q_text"], eps)',
                                 'qr = qk_norm_rows(qr, vid, qk_norm["gamma_q_text"], qk_norm["gamma_q_video"], eps)'),
    "q gamma on keys": ('kr = qk_norm_rows(kr, np.arange(kv_len) < n, qk_norm["gamma_k_video"], '
                        'qk_norm["gamma_k_text"], eps)',
                        'kr = qk_norm_rows(kr, np.arange(kv_len) < n, qk_norm["gamma_q_video"], '
                        'qk_norm["gamma_k_text"], eps)'),
    "rotate before norm": (_NORM + _ROT, _ROT + _NORM),
}


@pytest.mark.parametrize("name", sorted(PLANTS))
def test_planted_prologue_mistakes_are_caught(name):
    mod = _planted(*PLANTS[name])
    failed = False
    for check in (check_worked_vector, check_matches_library, check_attention_equals_prenormalised):
        try:
            check(mod)
        except AssertionError:
            failed = True
            break
    assert failed, name
