"""GPU parity: the sm_100a kernel (called through the C ABI) against the
float64 oracle on the same seeded bf16 inputs.

Tolerance (bf16 I/O, unit-variance inputs): max |gpu - oracle| <= 2e-2 and
mean |gpu - oracle| <= 2e-3, on the full output for the small workloads and
on 4096 seeded (batch, head, row) samples for the two 129-frame workloads.
"""

from __future__ import annotations

import ctypes
import math

import numpy as np
import pytest
import torch

from joint_full_attention_b200 import build as B
from joint_full_attention_b200 import hvattn as H
from joint_full_attention_b200 import workloads as W
from oracle import hv_oracle as O

MAX_ABS = 2e-2
MEAN_ABS = 2e-3

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    B.build()
    H.lib()
    assert H.last_device_error() == 0


def to_dev(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).cuda()


def out_f64(t: torch.Tensor) -> np.ndarray:
    return t.float().cpu().numpy().astype(np.float64)


def run_gpu(inp, grid, text_len, theta=256.0, scale=None, out=None):
    q, k, v = (to_dev(inp[n]) for n in ("q", "k", "v"))
    o = H.attn_forward(q, k, v, grid, text_len, inp["text_valid"], theta, scale, out=out)
    torch.cuda.synchronize()
    assert H.last_device_error() == 0
    return o


def f64(inp):
    return {n: W.bf16_bits_to_f64(inp[n]) for n in ("q", "k", "v")}


def check(got, ref, what):
    err = np.abs(got - ref)
    print(f"[parity] {what}: max abs err {err.max():.3e}, mean {err.mean():.3e}")
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    assert err.max() <= MAX_ABS, f"{what}: max abs err {err.max():.3e}"
    assert err.mean() <= MEAN_ABS, f"{what}: mean abs err {err.mean():.3e}"
    return err.max(), err.mean()


def full_check(inp, grid, text_len, theta=256.0, scale=None):
    o = run_gpu(inp, grid, text_len, theta, scale)
    x = f64(inp)
    ref = O.joint_attention(x["q"], x["k"], x["v"], grid, text_len, inp["text_valid"], theta, scale)
    return check(out_f64(o), ref, f"grid {grid} text {text_len}")


@pytest.mark.parametrize("name", ["tiny", "img256", "v544x960x17"])
def test_full_output_parity(name):
    wl = W.WORKLOADS[name]
    inp = W.make_inputs(wl, seed=1)
    full_check(inp, wl.grid, wl.text_len)


@pytest.mark.parametrize("name", ["v544x960x129", "v720x1280x129", "v960x960x129", "v1104x832x129",
                                  "cfg544x960x129"])
def test_sampled_parity_large(name):
    wl = W.WORKLOADS[name]
    inp = W.make_inputs(wl, seed=2)
    o = run_gpu(inp, wl.grid, wl.text_len)
    samples = W.sample_triples(wl.batch, wl.heads, wl.n_video, wl.text_len, inp["text_valid"], 4096, seed=3)
    got = o[samples[:, 0], samples[:, 2], samples[:, 1]].float().cpu().numpy().astype(np.float64)
    x = f64(inp)
    ref = O.joint_attention_samples(x["q"], x["k"], x["v"], wl.grid, wl.text_len, inp["text_valid"], samples)
    check(got, ref, name)


def _small(grid, text_len, valid, batch=1, heads=3, seed=5, k_scale=1.0):
    wl = W.Workload("edge", "edge case", batch, heads, grid, text_len, valid=tuple(valid))
    inp = W.make_inputs(wl, seed=seed)
    if k_scale != 1.0:
        inp["k"] = W.round_to_bf16_bits(W.bf16_bits_to_f32(inp["k"]) * np.float32(k_scale))
    return inp


@pytest.mark.parametrize("grid,text_len,valid", [
    ((1, 1, 1), 0, [0]),            # one video token, no text
    ((1, 1, 1), 256, [0]),          # all text padded
    ((2, 4, 4), 8, [8]),            # no padding
    ((3, 5, 7), 37, [0]),           # ragged, text present but none valid
    ((1, 9, 15), 256, [256]),       # full text
    ((5, 3, 11), 100, [1]),         # 265 rows: ragged Q unit and K tile
    ((2, 16, 16), 0, [0]),          # exactly 512 rows, no text
    ((4, 8, 9), 19, [19, 3, 0]),    # batch of 3 with different valid lengths
])
def test_edge_shapes(grid, text_len, valid):
    inp = _small(grid, text_len, valid, batch=len(valid))
    full_check(inp, grid, text_len)


def test_theta_and_scale_parameters():
    grid, text_len = (3, 6, 10), 30
    inp = _small(grid, text_len, [17])
    full_check(inp, grid, text_len, theta=10000.0)
    full_check(inp, grid, text_len, scale=0.05)
    full_check(inp, grid, text_len, theta=2.0, scale=1.0 / math.sqrt(64))


def test_sharp_softmax_rescaling():
    """Sharper softmax: K scaled by 2, the top of the per-head K scale range of
    the 720x1280x129 workload; exercises the running-max rescale of O."""
    grid, text_len = (4, 10, 10), 64
    inp = _small(grid, text_len, [50], k_scale=2.0)
    full_check(inp, grid, text_len)


def test_sharp_softmax_error_curve():
    """Error against the oracle as K is scaled by 1, 2, 3 and 4 (sharper and
    sharper softmax). The tolerance holds up to x2, the top of the
    720x1280x129 workload's per-head K scale; x3 and x4 are measured and
    printed, not bounded. Beside each, the error against the oracle's
    attention on bf16-rounded rotated operands (R(q), R(k) rounded to bf16, as
    the tensor core receives them) shows how much of it that rounding explains:
    it grows with |score|, since a relative operand error of 2^-9 becomes an
    absolute score error of about |score| * 2^-8."""
    grid, text_len, valid = (4, 10, 10), 64, 50
    n = grid[0] * grid[1] * grid[2]
    curve = {}
    for ks in (1.0, 2.0, 3.0, 4.0):
        inp = _small(grid, text_len, [valid], k_scale=ks)
        got = out_f64(run_gpu(inp, grid, text_len))[0]
        x = f64(inp)
        ref = O.joint_attention(x["q"], x["k"], x["v"], grid, text_len, [valid])[0]
        ref_rounded = np.empty_like(ref)
        for h in range(x["q"].shape[2]):
            rq = O.rotate_sequence(x["q"][0, :, h], grid)
            rk = O.rotate_sequence(x["k"][0, :, h], grid)
            rq, rk = (W.bf16_bits_to_f64(W.round_to_bf16_bits(a.astype(np.float32))) for a in (rq, rk))
            ref_rounded[:, h], _ = O.joint_attention_block(rq, rk, x["v"][0, :, h], grid, 0, 0, 0, 0, n + valid)
        e, e2 = np.abs(got - ref), np.abs(got - ref_rounded)
        curve[ks] = (e.max(), e.mean(), e2.max(), e2.mean())
        print(f"[sharp] K x {ks:g}: vs oracle max {e.max():.3e} mean {e.mean():.3e}; "
              f"vs bf16-rounded R(q), R(k) max {e2.max():.3e} mean {e2.mean():.3e}")
    for ks in (1.0, 2.0):
        assert curve[ks][0] <= MAX_ABS and curve[ks][1] <= MEAN_ABS, f"K x {ks}"


def test_padding_invariance_and_determinism():
    grid, text_len = (2, 8, 8), 64
    inp = _small(grid, text_len, [10])
    o1 = run_gpu(inp, grid, text_len).clone()
    o2 = run_gpu(inp, grid, text_len)
    assert torch.equal(o1, o2), "two runs differ"
    n = 128
    inp2 = dict(inp)
    for name in ("k", "v"):
        arr = inp[name].copy()
        arr[:, n + 10:] = W.round_to_bf16_bits(np.full(arr[:, n + 10:].shape, 3.5, dtype=np.float32))
        inp2[name] = arr
    o3 = run_gpu(inp2, grid, text_len)
    assert torch.equal(o1, o3), "padded keys changed the output"


def test_output_canary_untouched():
    grid, text_len = (3, 7, 5), 21
    inp = _small(grid, text_len, [11])
    s_len = 105 + text_len
    buf = torch.full((1, s_len + 64, 3, 128), 7.0, dtype=torch.bfloat16, device="cuda")
    out = buf[:, :s_len]
    assert out.is_contiguous()
    run_gpu(inp, grid, text_len, out=out)
    assert torch.all(buf[:, s_len:] == 7.0), "kernel wrote past the output"


def test_errors_on_device():
    q = torch.zeros(1, 40, 2, 128, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(H.HVError) as e:
        H.attn_forward(q, q, q, (2, 4, 4), 8, [9])
    assert e.value.status == 4
    with pytest.raises(H.HVError) as e:
        H.attn_forward(q, q, q, (2, 4, 4), 8, [5], out=q)
    assert e.value.status == 6
    flat = torch.zeros(1 * 40 * 2 * 128 + 8, dtype=torch.bfloat16, device="cuda")
    mis = flat[1:1 + 40 * 2 * 128].view(1, 40, 2, 128)
    with pytest.raises(H.HVError) as e:
        H.attn_forward(mis, q, q, (2, 4, 4), 8, [5], out=torch.empty_like(q))
    assert e.value.status == 2
    assert H.last_device_error() == 0


def test_bounded_wait_times_out_cleanly():
    word = H.selftest_timeout(20000)
    assert word & 1 and (word >> 8) & 0xFF == 5
    assert H.last_device_error() == 0
    # the context is still usable
    inp = _small((2, 4, 4), 8, [5])
    full_check(inp, (2, 4, 4), 8)


def test_attention_kernel_abort_path():
    """The attention kernel's own abort path (hv_attn_selftest_abort): with one K
    tile load of CTA 0 withheld and 20 ms wait limits, a wait in that CTA runs
    out (the RoPE warps' for those keys, or the producer's for the stage they
    hold); that CTA's roles stop, drain their copies and MMAs, free TMEM and
    return, while the other CTAs finish. The timeout is then visible without
    synchronising: the next call returns HV_ERR_DEVICE_TIMEOUT without
    launching, until hv_attn_last_device_error reads the word (timeout bit,
    role) and clears it. A normal call afterwards matches the oracle."""
    grid, text_len = (2, 8, 20), 64            # 384 rows: two work units per head
    inp = _small(grid, text_len, [40], heads=4)
    q, k, v = (to_dev(inp[n]) for n in ("q", "k", "v"))
    assert H.last_device_error() == 0
    assert H.selftest_abort(q, k, v, grid, text_len, [40], withhold_k=1, timeout_us=20000) == 0
    # every entry point that launches work refuses while the status word is set
    gam = torch.ones((4, 128), dtype=torch.float32, device="cuda")
    n = grid[0] * grid[1] * grid[2]
    acc_o = torch.zeros((1, n + text_len, 4, 128), dtype=torch.float32, device="cuda")
    acc_l = torch.full((1, n + text_len, 4), float("-inf"), dtype=torch.float32, device="cuda")
    refused = [
        lambda: H.attn_forward(q, k, v, grid, text_len, [40]),
        lambda: H.attn_forward_ws(q, k, v, grid, text_len, [40]),
        lambda: H.attn_forward_qknorm(q, k, v, grid, text_len, [40], gam),
        lambda: H.attn_forward_qknorm(q, k, v, grid, text_len, [40], gam, use_workspace=True),
        lambda: H.attn_forward_block(q, k, v, grid, n, 0, n, 0, [n + 40]),
        lambda: H.attn_merge(acc_o, acc_l, acc_o.clone(), acc_l.clone()),
    ]
    for call in refused:
        with pytest.raises(H.HVError) as e:
            call()
        assert e.value.status == 10
    b_sz, _, heads, _ = q.shape
    valid = (ctypes.c_int * 1)(40)
    st = H.lib().hv_attn_forward_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), torch.empty_like(q).data_ptr(),
                                         b_sz, heads, *grid, text_len, valid, 256.0, 1.0 / math.sqrt(128),
                                         ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 10
    word = H.last_device_error()
    # bit 0: a wait ran out; bits 8..15: the role(s) that recorded it. The RoPE
    # warps (waiting for the withheld tile) and the producer (waiting for the
    # stage behind it to free) both wait on it, and which of them times out
    # first is a race between their polling windows, so any waiting role counts.
    assert word & 1 and (word >> 8) & 0xFF, hex(word)
    assert ((word >> 8) & 0xFF) & ~0x7 == 0, hex(word)
    assert H.last_device_error() == 0
    full_check(inp, grid, text_len)


# ------------------------------------------------ workspace (pre-rotated K) path

def _run_both(inp, grid, text_len, theta=256.0):
    q, k, v = (to_dev(inp[n]) for n in ("q", "k", "v"))
    fused = H.attn_forward(q, k, v, grid, text_len, inp["text_valid"], theta)
    ws = torch.empty(H.workspace_bytes(q.shape[0], q.shape[2], grid, text_len) // 2, dtype=torch.bfloat16,
                     device="cuda")
    two = H.attn_forward_ws(q, k, v, grid, text_len, inp["text_valid"], theta, workspace=ws)
    torch.cuda.synchronize()
    assert H.last_device_error() == 0
    return fused, two, ws


@pytest.mark.parametrize("name", ["tiny", "img256", "v544x960x17", "v720x1280x129", "v1104x832x129",
                                  "cfg544x960x129"])
def test_workspace_path_bit_identical(name):
    wl = W.WORKLOADS[name]
    inp = W.make_inputs(wl, seed=4)
    fused, two, _ = _run_both(inp, wl.grid, wl.text_len)
    assert torch.equal(fused, two)


@pytest.mark.parametrize("grid,text_len,valid", [((1, 1, 1), 0, [0]), ((5, 3, 11), 100, [1]),
                                                 ((4, 8, 9), 19, [19, 3, 0])])
def test_workspace_path_edge_shapes(grid, text_len, valid):
    inp = _small(grid, text_len, valid, batch=len(valid))
    fused, two, _ = _run_both(inp, grid, text_len, theta=1000.0)
    assert torch.equal(fused, two)


def test_workspace_holds_rotated_keys():
    """The first stage writes R(K): video rows rotated (bf16 of the exact
    rotation, within one bf16 step), text rows copied bit for bit."""
    grid, text_len = (3, 5, 7), 24
    inp = _small(grid, text_len, [9], heads=2)
    _, _, ws = _run_both(inp, grid, text_len)
    n = 105
    got = ws.view(1, n + text_len, 2, 128).float().cpu().numpy().astype(np.float64)
    k = W.bf16_bits_to_f64(inp["k"])
    for h in range(2):
        exact = O.rope3d_rotate(k[0, :n, h], O.token_positions(*grid))
        # one bf16 step of the result, plus fp32 rounding of the rotation itself
        step = np.abs(exact) * 2.0 ** -7 + 1e-5
        assert np.all(np.abs(got[0, :n, h] - exact) <= step)
        assert np.array_equal(got[0, n:, h], k[0, n:, h])


def test_workspace_errors():
    q = torch.zeros(1, 40, 2, 128, dtype=torch.bfloat16, device="cuda")
    small = torch.empty(100, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(H.HVError) as e:
        H.attn_forward_ws(q, q, q, (2, 4, 4), 8, [5], workspace=small)
    assert e.value.status == 11
    with pytest.raises(H.HVError) as e:
        H.attn_forward_ws(q, q, q, (2, 4, 4), 8, [5], out=torch.empty_like(q), workspace=q.view(-1))
    assert e.value.status == 11
    assert H.last_device_error() == 0


# ------------------------------------------------------- host-buffer pipeline

@pytest.mark.parametrize("name,groups,pinned", [("img256", 1, True), ("img256", 4, True), ("img256", 24, False),
                                                ("v544x960x17", 3, True), ("v544x960x17", 8, False)])
def test_host_pipeline_bit_identical(name, groups, pinned):
    """hv_attn_forward_host (per-head-group copies overlapping the kernels)
    returns exactly what hv_attn_forward computes on device buffers."""
    wl = W.WORKLOADS[name]
    inp = W.make_inputs(wl, seed=6)
    q, k, v = (to_dev(inp[n]) for n in ("q", "k", "v"))
    ref = H.attn_forward(q, k, v, wl.grid, wl.text_len, inp["text_valid"]).cpu()
    host = []
    for n in ("q", "k", "v"):
        t = torch.from_numpy(inp[n].view(np.int16)).view(torch.bfloat16)
        host.append(t.pin_memory() if pinned else t.clone())
    work = {}
    for _ in range(2):      # the second call reuses the workspace and the copy streams
        out = H.attn_forward_host(*host, wl.grid, wl.text_len, inp["text_valid"], work=work, head_groups=groups)
        assert torch.equal(out, ref)
    assert H.last_device_error() == 0


@pytest.mark.parametrize("heads,groups", [(1, 1), (2, 1), (3, 1), (2, 2), (4, 2), (6, 3)])
def test_host_pipeline_pieces(heads, groups):
    """The pipeline's pieces: the first and the last head group are cut into one
    head and the rest (a single group of 2 or 3 heads becomes 1 + 1 or 1 + 2;
    groups of one head are not cut), alternating slots and kernel streams.
    Every split returns what hv_attn_forward computes, bit for bit, on a
    batch of two samples with different valid text lengths."""
    wl = W.Workload("pieces", "pieces", 2, heads, (2, 6, 5), 7, valid=(7, 3))
    inp = W.make_inputs(wl, seed=8)
    q, k, v = (to_dev(inp[n]) for n in ("q", "k", "v"))
    ref = H.attn_forward(q, k, v, wl.grid, wl.text_len, inp["text_valid"]).cpu()
    host = [torch.from_numpy(inp[n].view(np.int16)).view(torch.bfloat16).pin_memory() for n in ("q", "k", "v")]
    work = {}
    for _ in range(2):
        out = H.attn_forward_host(*host, wl.grid, wl.text_len, inp["text_valid"], work=work, head_groups=groups)
        assert torch.equal(out, ref)
    assert H.last_device_error() == 0
