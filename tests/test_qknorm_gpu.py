"""GPU parity of the QK-RMSNorm prologue ("HunyuanVideo 模型结构与数学原理"
§5.4) through the C ABI: hv_attn_forward_qknorm and its two-stage variant
against the float64 oracle, with the same tolerance as the plain call
(max |gpu - oracle| <= 2e-2, mean <= 2e-3)."""

from __future__ import annotations

import numpy as np
import pytest
import torch

from joint_full_attention_b200 import build as B
from joint_full_attention_b200 import hvattn as H
from joint_full_attention_b200 import workloads as W
from oracle import hv_oracle as O

MAX_ABS = 2e-2
MEAN_ABS = 2e-3
EPS = 1e-6

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    B.build()
    H.lib()
    assert H.last_device_error() == 0


def gammas(seed, same_streams=False):
    rng = np.random.default_rng(seed)
    g = rng.uniform(0.5, 1.5, (4, 128)).astype(np.float32)
    if same_streams:
        g[2], g[3] = g[0], g[1]
    prm = {"gamma_q_video": g[0].astype(np.float64), "gamma_k_video": g[1].astype(np.float64),
           "gamma_q_text": g[2].astype(np.float64), "gamma_k_text": g[3].astype(np.float64), "eps": EPS}
    return torch.from_numpy(g).cuda(), prm


def to_dev(bits):
    return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).cuda()


def f64(inp):
    return {n: W.bf16_bits_to_f64(inp[n]) for n in ("q", "k", "v")}


def check(got, ref, what):
    err = np.abs(got - ref)
    print(f"[parity] qknorm {what}: max abs err {err.max():.3e}, mean {err.mean():.3e}")
    assert np.all(np.isfinite(got)), what
    assert err.max() <= MAX_ABS, f"{what}: max abs err {err.max():.3e}"
    assert err.mean() <= MEAN_ABS, f"{what}: mean abs err {err.mean():.3e}"


def run_both(inp, grid, text_len, g, theta=256.0):
    q, k, v = (to_dev(inp[n]) for n in ("q", "k", "v"))
    one = H.attn_forward_qknorm(q, k, v, grid, text_len, inp["text_valid"], g, EPS, rope_theta=theta)
    ws = torch.empty(H.workspace_bytes(q.shape[0], q.shape[2], grid, text_len) // 2, dtype=torch.bfloat16,
                     device="cuda")
    two = H.attn_forward_qknorm(q, k, v, grid, text_len, inp["text_valid"], g, EPS, rope_theta=theta, workspace=ws)
    torch.cuda.synchronize()
    assert H.last_device_error() == 0
    return one, two, ws


def _small(grid, text_len, valid, heads=3, seed=5, row_scale=False):
    wl = W.Workload("edge", "edge case", len(valid), heads, grid, text_len, valid=tuple(valid))
    inp = W.make_inputs(wl, seed=seed)
    if row_scale:
        # rows of very different size: the prologue removes the scale
        rng = np.random.default_rng(seed + 100)
        for n in ("q", "k"):
            x = W.bf16_bits_to_f32(inp[n])
            x *= np.exp(rng.uniform(-5, 5, x.shape[:3] + (1,))).astype(np.float32)
            inp[n] = W.round_to_bf16_bits(x)
    return inp


@pytest.mark.parametrize("name", ["tiny", "img256", "v544x960x17"])
def test_qknorm_full_parity_and_two_stage_identical(name):
    wl = W.WORKLOADS[name]
    inp = W.make_inputs(wl, seed=21)
    g, prm = gammas(22)
    one, two, _ = run_both(inp, wl.grid, wl.text_len, g)
    assert torch.equal(one, two), "two-stage output differs"
    x = f64(inp)
    ref = O.joint_attention(x["q"], x["k"], x["v"], wl.grid, wl.text_len, inp["text_valid"], qk_norm=prm)
    check(one.float().cpu().numpy().astype(np.float64), ref, name)


def test_qknorm_sampled_parity_720p():
    wl = W.WORKLOADS["v720x1280x129"]
    inp = W.make_inputs(wl, seed=23)
    g, prm = gammas(24)
    one, two, _ = run_both(inp, wl.grid, wl.text_len, g)
    assert torch.equal(one, two), "two-stage output differs"
    samples = W.sample_triples(wl.batch, wl.heads, wl.n_video, wl.text_len, inp["text_valid"], 4096, seed=25)
    got = one[samples[:, 0], samples[:, 2], samples[:, 1]].float().cpu().numpy().astype(np.float64)
    x = f64(inp)
    ref = O.joint_attention_samples(x["q"], x["k"], x["v"], wl.grid, wl.text_len, inp["text_valid"], samples,
                                    qk_norm=prm)
    check(got, ref, "v720x1280x129")


@pytest.mark.parametrize("grid,text_len,valid,same", [
    ((1, 1, 1), 0, [0], False),
    ((1, 1, 1), 256, [0], False),
    ((3, 5, 7), 37, [0], False),
    ((5, 3, 11), 100, [1], True),
    ((4, 8, 9), 19, [19, 3, 0], False),
    ((4, 8, 8), 0, [0], False),          # S = 256: the key statistics need no padding entries
    ((1, 100, 40), 30, [12], False),     # table too large: (cos, sin) per pair
])
def test_qknorm_edge_shapes(grid, text_len, valid, same):
    inp = _small(grid, text_len, valid, heads=2, row_scale=True)
    g, prm = gammas(26, same_streams=same)
    one, two, _ = run_both(inp, grid, text_len, g, theta=1000.0)
    assert torch.equal(one, two)
    x = f64(inp)
    ref = O.joint_attention(x["q"], x["k"], x["v"], grid, text_len, inp["text_valid"], theta=1000.0, qk_norm=prm)
    check(one.float().cpu().numpy().astype(np.float64), ref, f"grid {grid} text {text_len}")


def test_plain_call_on_grid_without_table():
    grid, text_len = (1, 100, 40), 30
    inp = _small(grid, text_len, [12], heads=2)
    q, k, v = (to_dev(inp[n]) for n in ("q", "k", "v"))
    o = H.attn_forward(q, k, v, grid, text_len, inp["text_valid"])
    ws = H.attn_forward_ws(q, k, v, grid, text_len, inp["text_valid"])
    torch.cuda.synchronize()
    assert torch.equal(o, ws)
    x = f64(inp)
    ref = O.joint_attention(x["q"], x["k"], x["v"], grid, text_len, inp["text_valid"])
    check(o.float().cpu().numpy().astype(np.float64), ref, "plain, no table")


def test_workspace_holds_normalised_rotated_keys():
    grid, text_len = (3, 5, 7), 24
    n = 105
    inp = _small(grid, text_len, [9], heads=2, row_scale=True)
    g, prm = gammas(27)
    _, _, ws = run_both(inp, grid, text_len, g)
    got = ws.view(1, n + text_len, 2, 128).float().cpu().numpy().astype(np.float64)
    k = W.bf16_bits_to_f64(inp["k"])
    for h in range(2):
        normed = O.qk_norm_rows(k[0, :, h], np.arange(n + text_len) < n, prm["gamma_k_video"],
                                prm["gamma_k_text"], EPS)
        exact = normed.copy()
        exact[:n] = O.rope3d_rotate(normed[:n], O.token_positions(*grid))
        # one bf16 step of the result plus fp32 rounding of the norm and rotation
        step = np.abs(exact) * 2.0 ** -7 + 1e-4
        assert np.all(np.abs(got[0, :, h] - exact) <= step)


def test_qknorm_errors_on_device():
    q = torch.zeros(1, 40, 2, 128, dtype=torch.bfloat16, device="cuda")
    g = torch.ones(4, 128, dtype=torch.float32, device="cuda")
    with pytest.raises(H.HVError) as e:
        H.attn_forward_qknorm(q, q, q, (2, 4, 4), 8, [5], g, -1.0)
    assert e.value.status == 7
    small = torch.empty(100, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(H.HVError) as e:
        H.attn_forward_qknorm(q, q, q, (2, 4, 4), 8, [5], g, workspace=small)
    assert e.value.status == 11
    # out overlapping gamma: out is a view whose storage starts inside gamma's
    buf = torch.zeros(4 * 128 * 2 + 40 * 2 * 128, dtype=torch.bfloat16, device="cuda")
    g_in = buf[:1024].view(torch.float32).view(4, 128)
    out = buf[512:512 + 40 * 2 * 128].view(1, 40, 2, 128)
    with pytest.raises(H.HVError) as e:
        H.attn_forward_qknorm(q, q, q, (2, 4, 4), 8, [5], g_in, out=out)
    assert e.value.status == 6
    assert H.last_device_error() == 0
