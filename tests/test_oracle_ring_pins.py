"""Pins for the oracle's ring-attention step ("HunyuanVideo 模型结构与数学原理"
§9.2): block attention with per-row log-sum-exp, and the merge of blocks.
The already pinned joint attention is the reference: any partition of the
keys into blocks must merge back to it, and the log-sum-exp is checked by
brute force."""

from __future__ import annotations

import math

import numpy as np
import pytest

from oracle import hv_oracle as O


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def _full_lse(q, k, grid, valid):
    """log of the softmax denominator, by plain loops over the rotated rows."""
    n = grid[0] * grid[1] * grid[2]
    qr = O.rotate_sequence(q, grid)
    kr = O.rotate_sequence(k[:n + valid], grid)
    out = np.empty(q.shape[0])
    for i in range(q.shape[0]):
        s = [float(np.dot(qr[i], kr[j])) / math.sqrt(128) for j in range(n + valid)]
        m = max(s)
        out[i] = m + math.log(math.fsum(math.exp(x - m) for x in s))
    return out


@pytest.mark.parametrize("cuts", [[0, 40], [0, 13, 27, 40], [0, 1, 2, 40]])
def test_key_blocks_merge_to_joint_attention(cuts):
    grid, text_len, valid = (2, 4, 5), 9, 6
    n = 40
    s_len = n + text_len
    q, k, v = (_rand((s_len, 128), s) for s in (1, 2, 3))
    ref = O.joint_attention_head(q, k, v, grid, valid)
    outs, lses = [], []
    for a, b in zip(cuts[:-1], cuts[1:]):          # video key blocks [a, b)
        o, l = O.joint_attention_block(q, k[a:b], v[a:b], grid, n, 0, b - a, a, b - a)
        outs.append(o)
        lses.append(l)
    o, l = O.joint_attention_block(q, k[n:], v[n:], grid, n, 0, 0, n, valid)   # the text block
    outs.append(o)
    lses.append(l)
    got, lse = O.merge_blocks(outs, lses)
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, _full_lse(q, k, grid, valid), rtol=0, atol=1e-10)


def test_query_blocks_with_offsets_match_rows_of_the_full_call():
    grid, text_len, valid = (3, 3, 4), 7, 5
    n = 36
    s_len = n + text_len
    q, k, v = (_rand((s_len, 128), s) for s in (4, 5, 6))
    ref = O.joint_attention_head(q, k, v, grid, valid)
    # query block = video rows [10, 30) followed by all text rows
    qb = np.concatenate([q[10:30], q[n:]])
    o, _ = O.joint_attention_block(qb, k, v, grid, 20, 10, n, 0, n + valid)
    np.testing.assert_allclose(o[:20], ref[10:30], rtol=0, atol=1e-12)
    np.testing.assert_allclose(o[20:], ref[n:], rtol=0, atol=1e-12)


def test_empty_block_contributes_nothing():
    grid = (1, 2, 2)
    q, k, v = (_rand((6, 128), s) for s in (7, 8, 9))
    o0, l0 = O.joint_attention_block(q, k[4:], v[4:], grid, 4, 0, 0, 4, 0)
    assert np.all(o0 == 0) and np.all(l0 == -np.inf)
    o1, l1 = O.joint_attention_block(q, k, v, grid, 4, 0, 4, 0, 6)
    got, lse = O.merge_blocks([o1, o0], [l1, l0])
    np.testing.assert_array_equal(got, o1)
    np.testing.assert_array_equal(lse, l1)


def test_merge_is_order_free_and_weights_by_lse():
    rng = np.random.default_rng(10)
    o = [rng.standard_normal((5, 128)) for _ in range(3)]
    l = [rng.standard_normal(5) * 3 for _ in range(3)]
    a, la = O.merge_blocks(o, l)
    b, lb = O.merge_blocks(o[::-1], l[::-1])
    np.testing.assert_allclose(a, b, atol=1e-14)
    np.testing.assert_allclose(la, lb, atol=1e-14)
    # two blocks with equal lse: plain average
    c, lc = O.merge_blocks(o[:2], [np.zeros(5), np.zeros(5)])
    np.testing.assert_allclose(c, (o[0] + o[1]) / 2, atol=1e-15)
    np.testing.assert_allclose(lc, math.log(2), atol=1e-15)


def test_block_with_prologue_merges_to_prologue_call():
    grid, text_len, valid = (2, 3, 3), 5, 3
    n = 18
    q, k, v = (_rand((n + text_len, 128), s) for s in (11, 12, 13))
    rng = np.random.default_rng(14)
    prm = {nm: rng.uniform(0.5, 1.5, 128) for nm in ("gamma_q_video", "gamma_k_video", "gamma_q_text",
                                                     "gamma_k_text")}
    prm["eps"] = 1e-6
    ref = O.joint_attention_head(q, k, v, grid, valid, qk_norm=prm)
    o1, l1 = O.joint_attention_block(q, k[:7], v[:7], grid, n, 0, 7, 0, 7, qk_norm=prm)
    o2, l2 = O.joint_attention_block(q, k[7:n], v[7:n], grid, n, 0, n - 7, 7, n - 7, qk_norm=prm)
    o3, l3 = O.joint_attention_block(q, k[n:], v[n:], grid, n, 0, 0, n, valid, qk_norm=prm)
    got, _ = O.merge_blocks([o1, o2, o3], [l1, l2, l3])
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)


# ----------------------------------------------------------- planted mistakes

import types
from pathlib import Path

ORACLE_SRC = Path(O.__file__).read_text()

PLANTS = {
    "key offset ignored": ("pos[k_pos0:k_pos0 + kv_vid]", "pos[0:kv_vid]"),
    "query offset ignored": ("pos[q_pos0:q_pos0 + q_video]", "pos[0:q_video]"),
    "lse in log2": ("(mx + np.log(tot))[:, 0]", "(mx + np.log2(tot))[:, 0]"),
    "merge without weights": ("out = sum(w[i][:, None] * np.asarray(o, dtype=np.float64) for i, o in enumerate(outs))",
                              "out = sum(np.asarray(o, dtype=np.float64) for o in outs) * tot[:, None] / len(outs)"),
}


@pytest.mark.parametrize("name", sorted(PLANTS))
def test_planted_ring_mistakes_are_caught(name, monkeypatch):
    old, new = PLANTS[name]
    assert ORACLE_SRC.count(old) == 1, old
    mod = types.ModuleType("planted_oracle")
    exec(compile(ORACLE_SRC.replace(old, new), "planted_oracle", "exec"), mod.__dict__)
    monkeypatch.setattr(O, "joint_attention_block", mod.joint_attention_block)
    monkeypatch.setattr(O, "merge_blocks", mod.merge_blocks)
    failed = False
    for check in (lambda: test_key_blocks_merge_to_joint_attention([0, 13, 27, 40]),
                  test_query_blocks_with_offsets_match_rows_of_the_full_call):
        try:
            check()
        except AssertionError:
            failed = True
            break
    assert failed, name
