"""C-ABI checks that need no GPU: the library builds, loads, exports every
symbol declared in include/hv_attn.h, computes token counts, and rejects bad
arguments with status codes before touching a device."""

from __future__ import annotations

import ctypes
import re
from pathlib import Path

import pytest

from joint_full_attention_b200 import build as B
from joint_full_attention_b200 import hvattn as H

ROOT = Path(__file__).resolve().parent.parent
HEADER = ROOT / "include" / "hv_attn.h"
GOLDEN = Path(__file__).parent / "golden"


@pytest.fixture(scope="module")
def lib():
    B.build()
    return H.lib()


def declared_functions():
    text = re.sub(r"/\*.*?\*/", "", HEADER.read_text(), flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[\w\s\*]+?\b(hv_\w+)\s*\(", text, flags=re.M)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for must in ("hv_attn_forward", "hv_video_tokens", "hv_attn_last_device_error"):
        assert must in names
    assert set(names) <= set(H.EXPORTED) | {n for n in names}


def test_library_exports_every_declared_symbol(lib):
    names = declared_functions()
    assert names, "no declarations parsed"
    for name in names:
        assert hasattr(lib, name), name
        assert ctypes.cast(getattr(lib, name), ctypes.c_void_p).value


def test_video_tokens_worked_examples(lib):
    for line in (GOLDEN / "token_grids.txt").read_text().splitlines():
        line = line.split("#", 1)[0].split()
        if line:
            f, h, w, *_, n = map(int, line)
            assert H.video_tokens(f, h, w) == n
    assert H.video_tokens(1, 256, 256) == 256
    assert H.video_tokens(129, 544, 960) == 67320
    for bad in [(16, 544, 960), (0, 544, 960), (17, 540, 960), (17, 544, 0), (-3, 16, 16)]:
        assert H.video_tokens(*bad) == -1


def test_status_strings(lib):
    for code, name in H.STATUS_NAMES.items():
        assert H.status_string(code)
    assert "unknown" in H.status_string(999)


def _call(lib, q=0x10000, k=0x20000, v=0x30000, out=0x40000, B_=1, heads=2, T=2, Hp=4, Wp=4, text_len=8,
          valid=(5,), theta=256.0, scale=0.088, stream=None):
    arr = None if valid is None else (ctypes.c_int * max(1, len(valid)))(*valid)
    return lib.hv_attn_forward(q, k, v, out, B_, heads, T, Hp, Wp, text_len, arr, theta, scale, stream)


def test_argument_validation_codes(lib):
    big = 1 << 40
    assert _call(lib, q=None) == 1
    assert _call(lib, valid=None) == 1
    assert _call(lib, k=0x20008) == 2
    assert _call(lib, B_=0) == 3
    assert _call(lib, heads=0) == 3
    assert _call(lib, Wp=0) == 3
    assert _call(lib, B_=513, valid=(5,) * 513) == 3
    assert _call(lib, text_len=257, valid=(5,)) == 4
    assert _call(lib, text_len=-1, valid=(0,)) == 4
    assert _call(lib, valid=(9,)) == 4
    assert _call(lib, valid=(-1,)) == 4
    assert _call(lib, theta=0.0) == 7
    assert _call(lib, theta=float("nan")) == 7
    assert _call(lib, scale=float("inf")) == 7
    assert _call(lib, T=40000, Hp=400, Wp=400) == 5
    # out overlapping an input
    assert _call(lib, q=big, k=big * 2, v=big * 3, out=big + 4096) == 6


def test_workspace_entry_points(lib):
    assert lib.hv_attn_workspace_bytes(1, 24, 33, 45, 80, 256) == 119056 * 24 * 256
    assert lib.hv_attn_workspace_bytes(2, 2, 2, 4, 4, 8) == 2 * 40 * 2 * 256
    assert lib.hv_attn_workspace_bytes(0, 2, 2, 4, 4, 8) == -1
    assert lib.hv_attn_workspace_bytes(1, 2, 2, 4, 4, 300) == -1
    valid = (ctypes.c_int * 1)(5)
    f = lib.hv_attn_forward_ws
    # argument errors come first, before the workspace is looked at
    assert f(None, 0x20000, 0x30000, 0x40000, 1, 2, 2, 4, 4, 8, valid, 256.0, 0.088, 0x90000, 1 << 20, None) == 1
    assert f(0x10000, 0x20000, 0x30000, 0x40000, 0, 2, 2, 4, 4, 8, valid, 256.0, 0.088, 0x90000, 1 << 20, None) == 3


def test_qknorm_entry_points_validate_arguments(lib):
    valid = (ctypes.c_int * 1)(5)
    f, fw = lib.hv_attn_forward_qknorm, lib.hv_attn_forward_qknorm_ws
    base = (0x10000, 0x20000, 0x30000, 0x40000, 1, 2, 2, 4, 4, 8, valid, 256.0, 0.088)
    g = 0x900000
    assert f(*base, None, 1e-6, None) == 1                      # gamma missing
    assert f(*base, g + 4, 1e-6, None) == 2                     # gamma misaligned
    assert f(*base, g, -1e-6, None) == 7                        # eps < 0
    assert f(*base, g, float("nan"), None) == 7
    assert f(*base, 0x40000 + 64, 1e-6, None) == 6              # gamma inside out
    assert f(*base, 0x40000 - 1024, 1e-6, None) == 6            # gamma running into out
    # shape and text errors come first, as in hv_attn_forward
    assert f(0x10000, 0x20000, 0x30000, 0x40000, 0, 2, 2, 4, 4, 8, valid, 256.0, 0.088, g, 1e-6, None) == 3
    # the workspace variant checks the same arguments first (its workspace is
    # looked at after the device check, in the GPU tests)
    assert fw(*base, None, 1e-6, 0x800000, 1 << 20, None) == 1
    assert fw(*base, g, float("inf"), 0x800000, 1 << 20, None) == 7


def test_host_entry_point_validates_arguments(lib):
    assert lib.hv_attn_host_workspace_bytes(1, 24, 33, 45, 80, 256, 4) == 8 * 119056 * 6 * 256
    assert lib.hv_attn_host_workspace_bytes(1, 24, 33, 45, 80, 256, 5) == -1     # 5 does not divide 24
    assert lib.hv_attn_host_workspace_bytes(1, 24, 33, 45, 80, 256, 0) == -1
    valid = (ctypes.c_int * 1)(5)
    f = lib.hv_attn_forward_host
    hq, hk, hv, ho = 1 << 30, 2 << 30, 3 << 30, 4 << 30
    args = (1, 2, 2, 4, 4, 8, valid, 256.0, 0.088)
    assert f(None, hk, hv, ho, *args, 2, 0x900000, 1 << 20, None) == 1
    assert f(hq, hk, hv, ho, *args, 2, None, 1 << 20, None) == 1
    assert f(hq, hk, hv, ho, *args, 3, 0x900000, 1 << 20, None) == 3          # 3 does not divide 2 heads
    assert f(hq, hk, hv, hq + 64, *args, 1, 0x900000, 1 << 20, None) == 6     # out over q
    assert f(hq, hk, hv, ho, *args, 2, 0x900008, 1 << 20, None) == 11         # misaligned workspace
    assert f(hq, hk, hv, ho, *args, 2, 0x900000, 1000, None) == 11            # too small


def test_block_and_merge_entry_points_validate_arguments(lib):
    kv = (ctypes.c_int * 1)(10)
    f = lib.hv_attn_forward_block
    q, k, v, o, lse = 0x100000, 0x200000, 0x300000, 0x400000, 0x500000
    grid = (2, 4, 4)                                   # 32 video tokens
    ok = (1, 2, *grid, 40, 20, 0, 16, 16, 8, kv, 256.0, 0.088, 1, None)
    assert f(None, k, v, o, lse, *ok) == 1
    assert f(q, k, v, o, lse + 2, *ok) == 2                                       # lse misaligned
    assert f(q, k, v, o, lse, 1, 2, *grid, 40, 41, 0, 16, 16, 8, kv, 256.0, 0.088, 1, None) == 3   # q_video > Sq
    assert f(q, k, v, o, lse, 1, 2, *grid, 40, 20, 13, 16, 16, 8, kv, 256.0, 0.088, 1, None) == 3  # past the grid
    assert f(q, k, v, o, lse, 1, 2, *grid, 40, 20, 0, 16, 16, 17, kv, 256.0, 0.088, 1, None) == 3  # k past the grid
    assert f(q, k, v, o, lse, 1, 2, *grid, 40, 20, 0, 16, 16, 8, kv, 256.0, 0.088, 2, None) == 3   # out_fp32 not 0/1
    bad = (ctypes.c_int * 1)(17)
    assert f(q, k, v, o, lse, 1, 2, *grid, 40, 20, 0, 16, 16, 8, bad, 256.0, 0.088, 1, None) == 4  # kv_len > Sk
    zero = (ctypes.c_int * 1)(0)
    assert f(q, k, v, o, lse, 1, 2, *grid, 40, 20, 0, 16, 16, 8, zero, 256.0, 0.088, 1, None) == 4
    assert f(q, k, v, q + 64, lse, *ok) == 6                                      # out over q
    assert f(q, k, v, o, o + 16, *ok) == 6                                        # lse over out
    # an fp32 out is twice as long as a bf16 one: 1 x 40 x 2 x 128 x 4 bytes = 40960
    assert f(q, k, v, o, o + 30000, *ok) == 6                                     # lse inside the fp32 out
    bf16 = ok[:-2] + (0, None)
    assert f(q, k, v, o, o + 30000, *bf16) != 6                                   # past the bf16 out
    m = lib.hv_attn_merge
    assert m(None, 0x10, 0x20, 1, 0x30, None, 4, None) == 1
    assert m(0x1008, 0x10, 0x20, 1, 0x30, None, 4, None) == 2                     # o_acc not 16-byte aligned
    assert m(0x1000, 0x10, 0x28, 1, 0x30, None, 4, None) == 2                     # fp32 o_part not 16-byte aligned
    assert m(0x1000, 0x10, 0x28, 0, 0x30, None, 0, None) == 0                     # bf16 o_part: 8 bytes suffice
    assert m(0x1000, 0x10, 0x20, 1, 0x30, None, -1, None) == 3
    assert m(0x1000, 0x10, 0x20, 2, 0x30, None, 4, None) == 3                     # o_part_fp32 not 0/1
    assert m(0x1000, 0x10, 0x20, 1, 0x30, None, 0, None) == 0                     # nothing to merge


def test_valid_arguments_without_gpu_fail_cleanly(lib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present; covered by the gpu tests")
    st = _call(lib, q=1 << 32, k=2 << 32, v=3 << 32, out=4 << 32)
    assert st in (8, 9)
    valid = (ctypes.c_int * 1)(5)
    st = lib.hv_attn_selftest_abort(1 << 32, 2 << 32, 3 << 32, 4 << 32, 1, 2, 2, 4, 4, 8, valid, 1, 20000, None)
    assert st in (8, 9)
    assert lib.hv_attn_selftest_abort(1 << 32, 2 << 32, 3 << 32, 4 << 32, 1, 2, 2, 4, 4, 8, valid, -1, 20000,
                                      None) == 7
    st = lib.hv_attn_forward_qknorm(1 << 32, 2 << 32, 3 << 32, 4 << 32, 1, 2, 2, 4, 4, 8, valid, 256.0, 0.088,
                                    5 << 32, 1e-6, None)
    assert st in (8, 9)
