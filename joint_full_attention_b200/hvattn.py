"""Python binding of the C ABI in ``include/hv_attn.h`` (ctypes).

Argument marshalling only: tensors are checked and their device pointers and
the current CUDA stream are handed to ``libhvattn.so``; every step of the
attention runs in the library's sm_100a kernel. There is no fallback: if the
library is missing or the device is not an sm_100 part the calls raise.
"""

from __future__ import annotations

import ctypes
import math
from pathlib import Path

import torch

_LIB_PATH = Path(__file__).resolve().parent / "libhvattn.so"
_lib = None

HV_OK = 0
HV_ERR_BAD_SHAPE = 3
STATUS_NAMES = {
    0: "HV_OK", 1: "HV_ERR_NULL_POINTER", 2: "HV_ERR_MISALIGNED", 3: "HV_ERR_BAD_SHAPE",
    4: "HV_ERR_BAD_TEXT", 5: "HV_ERR_TOO_LARGE", 6: "HV_ERR_ALIAS", 7: "HV_ERR_BAD_SCALAR",
    8: "HV_ERR_NO_DEVICE", 9: "HV_ERR_LAUNCH", 10: "HV_ERR_DEVICE_TIMEOUT", 11: "HV_ERR_WORKSPACE",
    12: "HV_ERR_NOALLOC_LIMIT",
}
EXPORTED = ("hv_attn_forward", "hv_attn_forward_ws", "hv_attn_forward_noalloc", "hv_attn_forward_qknorm",
            "hv_attn_forward_qknorm_ws", "hv_attn_forward_host", "hv_attn_host_workspace_bytes",
            "hv_attn_workspace_bytes", "hv_attn_forward_block", "hv_attn_merge",
            "hv_video_tokens",
            "hv_attn_last_device_error", "hv_attn_selftest_timeout", "hv_attn_selftest_abort",
            "hv_attn_status_string")


class HVError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {STATUS_NAMES.get(status, status)} ({status_string(status)})")


def lib() -> ctypes.CDLL:
    """Load ``libhvattn.so`` (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not _LIB_PATH.exists():
            raise RuntimeError(f"{_LIB_PATH} is missing: run joint_full_attention_b200.build.build() first")
        L = ctypes.CDLL(str(_LIB_PATH))
        L.hv_attn_forward.restype = ctypes.c_int
        L.hv_attn_forward.argtypes = [ctypes.c_void_p] * 4 + [ctypes.c_int] * 6 + [
            ctypes.POINTER(ctypes.c_int), ctypes.c_float, ctypes.c_float, ctypes.c_void_p]
        L.hv_attn_forward_ws.restype = ctypes.c_int
        L.hv_attn_forward_ws.argtypes = [ctypes.c_void_p] * 4 + [ctypes.c_int] * 6 + [
            ctypes.POINTER(ctypes.c_int), ctypes.c_float, ctypes.c_float, ctypes.c_void_p, ctypes.c_size_t,
            ctypes.c_void_p]
        L.hv_attn_forward_noalloc.restype = ctypes.c_int
        L.hv_attn_forward_noalloc.argtypes = [ctypes.c_void_p] * 4 + [ctypes.c_int] * 6 + [
            ctypes.POINTER(ctypes.c_int), ctypes.c_float, ctypes.c_float, ctypes.c_void_p]
        L.hv_attn_forward_qknorm.restype = ctypes.c_int
        L.hv_attn_forward_qknorm.argtypes = [ctypes.c_void_p] * 4 + [ctypes.c_int] * 6 + [
            ctypes.POINTER(ctypes.c_int), ctypes.c_float, ctypes.c_float, ctypes.c_void_p, ctypes.c_float,
            ctypes.c_void_p]
        L.hv_attn_forward_qknorm_ws.restype = ctypes.c_int
        L.hv_attn_forward_qknorm_ws.argtypes = [ctypes.c_void_p] * 4 + [ctypes.c_int] * 6 + [
            ctypes.POINTER(ctypes.c_int), ctypes.c_float, ctypes.c_float, ctypes.c_void_p, ctypes.c_float,
            ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]
        L.hv_attn_forward_host.restype = ctypes.c_int
        L.hv_attn_forward_host.argtypes = [ctypes.c_void_p] * 4 + [ctypes.c_int] * 6 + [
            ctypes.POINTER(ctypes.c_int), ctypes.c_float, ctypes.c_float, ctypes.c_int, ctypes.c_void_p,
            ctypes.c_size_t, ctypes.c_void_p]
        L.hv_attn_host_workspace_bytes.restype = ctypes.c_longlong
        L.hv_attn_host_workspace_bytes.argtypes = [ctypes.c_int] * 7
        L.hv_attn_forward_block.restype = ctypes.c_int
        L.hv_attn_forward_block.argtypes = [ctypes.c_void_p] * 5 + [ctypes.c_int] * 11 + [
            ctypes.POINTER(ctypes.c_int), ctypes.c_float, ctypes.c_float, ctypes.c_int, ctypes.c_void_p]
        L.hv_attn_merge.restype = ctypes.c_int
        L.hv_attn_merge.argtypes = [ctypes.c_void_p] * 3 + [ctypes.c_int] + [ctypes.c_void_p] * 2 + [
            ctypes.c_longlong, ctypes.c_void_p]
        L.hv_attn_selftest_abort.restype = ctypes.c_int
        L.hv_attn_selftest_abort.argtypes = [ctypes.c_void_p] * 4 + [ctypes.c_int] * 6 + [
            ctypes.POINTER(ctypes.c_int), ctypes.c_int, ctypes.c_int, ctypes.c_void_p]
        L.hv_attn_workspace_bytes.restype = ctypes.c_longlong
        L.hv_attn_workspace_bytes.argtypes = [ctypes.c_int] * 6
        L.hv_video_tokens.restype = ctypes.c_longlong
        L.hv_video_tokens.argtypes = [ctypes.c_int] * 3
        L.hv_attn_last_device_error.restype = ctypes.c_int
        L.hv_attn_last_device_error.argtypes = []
        L.hv_attn_selftest_timeout.restype = ctypes.c_int
        L.hv_attn_selftest_timeout.argtypes = [ctypes.c_int]
        L.hv_attn_status_string.restype = ctypes.c_char_p
        L.hv_attn_status_string.argtypes = [ctypes.c_int]
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().hv_attn_status_string(int(status)).decode()


def video_tokens(frames: int, height: int, width: int) -> int:
    """N video tokens of an F x H x W clip, or -1 (pure host computation in the library)."""
    return int(lib().hv_video_tokens(int(frames), int(height), int(width)))


def last_device_error() -> int:
    """Device error word of the library's kernels since the last read (synchronises)."""
    return int(lib().hv_attn_last_device_error())


def selftest_timeout(timeout_us: int = 20000) -> int:
    return int(lib().hv_attn_selftest_timeout(int(timeout_us)))


def selftest_abort(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, grid, text_len: int, text_valid,
                   withhold_k: int = 1, timeout_us: int = 20000, out: torch.Tensor | None = None) -> int:
    """``hv_attn_selftest_abort``: the attention kernel with one K load withheld and short
    wait limits; returns the call's status (the timeout shows in the error words)."""
    _check(q, "q")
    _check(k, "k", q.shape)
    _check(v, "v", q.shape)
    if out is None:
        out = torch.empty_like(q)
    b_sz, _, heads, _ = q.shape
    t_lat, hp, wp = (int(x) for x in grid)
    valid = (ctypes.c_int * b_sz)(*[int(x) for x in text_valid])
    stream = torch.cuda.current_stream(q.device)
    with torch.cuda.device(q.device):
        return int(lib().hv_attn_selftest_abort(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), b_sz,
                                                heads, t_lat, hp, wp, int(text_len), valid, int(withhold_k),
                                                int(timeout_us), ctypes.c_void_p(stream.cuda_stream)))


def _check(t: torch.Tensor, name: str, shape=None):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != torch.bfloat16:
        raise TypeError(f"{name} must be bfloat16, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous [B, S, heads, 128]")
    if t.dim() != 4 or t.shape[-1] != 128:
        raise ValueError(f"{name} must be [B, S, heads, 128], got {tuple(t.shape)}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} shape {tuple(t.shape)} != {tuple(shape)}")


def attn_forward(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, grid, text_len: int, text_valid,
                 rope_theta: float = 256.0, scale: float | None = None, out: torch.Tensor | None = None,
                 stream: torch.cuda.Stream | None = None) -> torch.Tensor:
    """Joint 3D-RoPE attention on device tensors; enqueued on ``stream`` (default: current)."""
    _check(q, "q")
    _check(k, "k", q.shape)
    _check(v, "v", q.shape)
    if out is None:
        out = torch.empty_like(q)
    _check(out, "out", q.shape)
    b_sz, _, heads, _ = q.shape
    t_lat, hp, wp = (int(x) for x in grid)
    valid = (ctypes.c_int * b_sz)(*[int(x) for x in text_valid])
    if len(text_valid) != b_sz:
        raise ValueError("text_valid needs one entry per batch sample")
    if scale is None:
        scale = 1.0 / math.sqrt(128)
    if stream is None:
        stream = torch.cuda.current_stream(q.device)
    with torch.cuda.device(q.device):
        st = lib().hv_attn_forward(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), b_sz, heads,
                                   t_lat, hp, wp, int(text_len), valid, float(rope_theta), float(scale),
                                   ctypes.c_void_p(stream.cuda_stream))
    if st != HV_OK:
        raise HVError(st, "hv_attn_forward")
    return out


def workspace_bytes(batch: int, heads: int, grid, text_len: int) -> int:
    """Device bytes ``attn_forward_ws`` needs for its rotated-key workspace."""
    t_lat, hp, wp = (int(x) for x in grid)
    return int(lib().hv_attn_workspace_bytes(int(batch), int(heads), t_lat, hp, wp, int(text_len)))


def attn_forward_ws(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, grid, text_len: int, text_valid,
                    rope_theta: float = 256.0, scale: float | None = None, out: torch.Tensor | None = None,
                    workspace: torch.Tensor | None = None, stream: torch.cuda.Stream | None = None) -> torch.Tensor:
    """Same result as ``attn_forward``, keys pre-rotated once into ``workspace``.

    ``workspace`` is any CUDA tensor of at least ``workspace_bytes(...)``
    bytes (allocated here if None); on return it holds the rotated keys.
    """
    _check(q, "q")
    _check(k, "k", q.shape)
    _check(v, "v", q.shape)
    if out is None:
        out = torch.empty_like(q)
    _check(out, "out", q.shape)
    b_sz, _, heads, _ = q.shape
    t_lat, hp, wp = (int(x) for x in grid)
    if len(text_valid) != b_sz:
        raise ValueError("text_valid needs one entry per batch sample")
    need = workspace_bytes(b_sz, heads, grid, text_len)
    if workspace is None:
        workspace = torch.empty(max(need, 0) // 2, dtype=torch.bfloat16, device=q.device)
    if not workspace.is_cuda or not workspace.is_contiguous():
        raise ValueError("workspace must be a contiguous CUDA tensor")
    valid = (ctypes.c_int * b_sz)(*[int(x) for x in text_valid])
    if scale is None:
        scale = 1.0 / math.sqrt(128)
    if stream is None:
        stream = torch.cuda.current_stream(q.device)
    with torch.cuda.device(q.device):
        st = lib().hv_attn_forward_ws(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), b_sz, heads,
                                      t_lat, hp, wp, int(text_len), valid, float(rope_theta), float(scale),
                                      workspace.data_ptr(), workspace.numel() * workspace.element_size(),
                                      ctypes.c_void_p(stream.cuda_stream))
    if st != HV_OK:
        raise HVError(st, "hv_attn_forward_ws")
    return out


def _check_gamma(g: torch.Tensor, device) -> None:
    if not isinstance(g, torch.Tensor) or not g.is_cuda or g.device != device:
        raise TypeError("qk_gamma must be a CUDA tensor on the device of q")
    if g.dtype != torch.float32 or not g.is_contiguous() or tuple(g.shape) != (4, 128):
        raise ValueError("qk_gamma must be contiguous float32 [4, 128] (Q video, K video, Q text, K text)")


def attn_forward_qknorm(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, grid, text_len: int, text_valid,
                        qk_gamma: torch.Tensor, qk_eps: float = 1e-6, rope_theta: float = 256.0,
                        scale: float | None = None, out: torch.Tensor | None = None,
                        workspace: torch.Tensor | None = None, use_workspace: bool = False,
                        stream: torch.cuda.Stream | None = None) -> torch.Tensor:
    """Joint 3D-RoPE attention with the per-head QK RMSNorm prologue.

    ``qk_gamma``: float32 [4, 128] CUDA tensor (Q video, K video, Q text,
    K text). ``use_workspace`` (or a ``workspace`` tensor) selects the
    two-stage path; its output is bit-identical.
    """
    _check(q, "q")
    _check(k, "k", q.shape)
    _check(v, "v", q.shape)
    _check_gamma(qk_gamma, q.device)
    if out is None:
        out = torch.empty_like(q)
    _check(out, "out", q.shape)
    b_sz, _, heads, _ = q.shape
    t_lat, hp, wp = (int(x) for x in grid)
    if len(text_valid) != b_sz:
        raise ValueError("text_valid needs one entry per batch sample")
    valid = (ctypes.c_int * b_sz)(*[int(x) for x in text_valid])
    if scale is None:
        scale = 1.0 / math.sqrt(128)
    if stream is None:
        stream = torch.cuda.current_stream(q.device)
    two_stage = use_workspace or workspace is not None
    if two_stage and workspace is None:
        workspace = torch.empty(max(workspace_bytes(b_sz, heads, grid, text_len), 0) // 2, dtype=torch.bfloat16,
                                device=q.device)
    with torch.cuda.device(q.device):
        if two_stage:
            if not workspace.is_cuda or not workspace.is_contiguous():
                raise ValueError("workspace must be a contiguous CUDA tensor")
            st = lib().hv_attn_forward_qknorm_ws(
                q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), b_sz, heads, t_lat, hp, wp,
                int(text_len), valid, float(rope_theta), float(scale), qk_gamma.data_ptr(), float(qk_eps),
                workspace.data_ptr(), workspace.numel() * workspace.element_size(),
                ctypes.c_void_p(stream.cuda_stream))
        else:
            st = lib().hv_attn_forward_qknorm(
                q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), b_sz, heads, t_lat, hp, wp,
                int(text_len), valid, float(rope_theta), float(scale), qk_gamma.data_ptr(), float(qk_eps),
                ctypes.c_void_p(stream.cuda_stream))
    if st != HV_OK:
        raise HVError(st, "hv_attn_forward_qknorm_ws" if two_stage else "hv_attn_forward_qknorm")
    return out


def attn_forward_block(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, grid, q_video: int, q_pos0: int,
                       k_video: int, k_pos0: int, kv_len, rope_theta: float = 256.0, scale: float | None = None,
                       out: torch.Tensor | None = None, lse: torch.Tensor | None = None,
                       out_dtype: torch.dtype = torch.float32, stream: torch.cuda.Stream | None = None):
    """One ring-attention step (``hv_attn_forward_block``): q [B, Sq, H, 128]
    against k, v [B, Sk, H, 128]; returns (out [B, Sq, H, 128] of ``out_dtype``:
    fp32 (default, the partial result kept exact for merging) or bf16, lse fp32
    [B, Sq, H])."""
    _check(q, "q")
    _check(k, "k")
    _check(v, "v", k.shape)
    if k.shape[0] != q.shape[0] or k.shape[2] != q.shape[2]:
        raise ValueError("q and k/v must agree in batch and heads")
    if out is None:
        out = torch.empty(q.shape, dtype=out_dtype, device=q.device)
    if out.dtype not in (torch.float32, torch.bfloat16) or not out.is_cuda or not out.is_contiguous() \
            or tuple(out.shape) != tuple(q.shape):
        raise ValueError("out must be a contiguous fp32 or bf16 CUDA tensor shaped like q")
    b_sz, sq, heads, _ = q.shape
    sk = k.shape[1]
    if lse is None:
        lse = torch.empty((b_sz, sq, heads), dtype=torch.float32, device=q.device)
    if lse.dtype != torch.float32 or not lse.is_contiguous() or tuple(lse.shape) != (b_sz, sq, heads):
        raise ValueError("lse must be contiguous float32 [B, Sq, heads]")
    if len(kv_len) != b_sz:
        raise ValueError("kv_len needs one entry per batch sample")
    t_lat, hp, wp = (int(x) for x in grid)
    kvl = (ctypes.c_int * b_sz)(*[int(x) for x in kv_len])
    if scale is None:
        scale = 1.0 / math.sqrt(128)
    if stream is None:
        stream = torch.cuda.current_stream(q.device)
    with torch.cuda.device(q.device):
        st = lib().hv_attn_forward_block(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(),
                                         b_sz, heads, t_lat, hp, wp, sq, int(q_video), int(q_pos0), sk,
                                         int(k_video), int(k_pos0), kvl, float(rope_theta), float(scale),
                                         1 if out.dtype == torch.float32 else 0,
                                         ctypes.c_void_p(stream.cuda_stream))
    if st != HV_OK:
        raise HVError(st, "hv_attn_forward_block")
    return out, lse


def attn_merge(o_acc: torch.Tensor, lse_acc: torch.Tensor, o_part: torch.Tensor, lse_part: torch.Tensor,
               out: torch.Tensor | None = None, stream: torch.cuda.Stream | None = None) -> None:
    """``hv_attn_merge``: fold (o_part fp32 or bf16, lse_part fp32) into (o_acc fp32, lse_acc fp32) in
    place; optionally also write the merged rows to ``out`` (bf16)."""
    rows = lse_acc.numel()
    part_dt = o_part.dtype if o_part.dtype in (torch.float32, torch.bfloat16) else torch.float32
    for name, t, dt in (("o_acc", o_acc, torch.float32), ("lse_acc", lse_acc, torch.float32),
                        ("o_part", o_part, part_dt), ("lse_part", lse_part, torch.float32)):
        if not t.is_cuda or t.dtype != dt or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous CUDA {dt} tensor")
    if o_acc.numel() != rows * 128 or o_part.numel() != rows * 128 or lse_part.numel() != rows:
        raise ValueError("o_acc / o_part must hold 128 channels per row of lse_acc; lse_part one per row")
    if out is not None and (out.dtype != torch.bfloat16 or out.numel() != rows * 128 or not out.is_contiguous()):
        raise ValueError("out must be contiguous bf16 with 128 channels per row")
    if stream is None:
        stream = torch.cuda.current_stream(o_acc.device)
    with torch.cuda.device(o_acc.device):
        st = lib().hv_attn_merge(o_acc.data_ptr(), lse_acc.data_ptr(), o_part.data_ptr(),
                                 1 if o_part.dtype == torch.float32 else 0, lse_part.data_ptr(),
                                 None if out is None else out.data_ptr(), rows, ctypes.c_void_p(stream.cuda_stream))
    if st != HV_OK:
        raise HVError(st, "hv_attn_merge")


def default_head_groups(heads: int) -> int:
    """Head groups of the host-buffer pipeline: the largest of 8, 6, 4, 3, 2
    that divides the heads (at 720p 8 groups left 5 ms of copies exposed, 1
    group 48 ms)."""
    for g in (8, 6, 4, 3, 2):
        if heads % g == 0:
            return g
    return 1


def attn_forward_host(q_host: torch.Tensor, k_host: torch.Tensor, v_host: torch.Tensor, grid, text_len: int,
                      text_valid, rope_theta: float = 256.0, scale: float | None = None,
                      device: int | torch.device = 0, out_host: torch.Tensor | None = None,
                      work: dict | None = None, head_groups: int | None = None) -> torch.Tensor:
    """Host-to-host call (``hv_attn_forward_host``): pinned host inputs in, output back in host memory.

    The library pipelines per head group: copy in, attention, copy out, with
    the copies overlapping the kernels. ``work`` may hold the reusable device
    workspace (key "host_ws") so that repeated calls allocate nothing on the
    device. Returns after the output is in ``out_host``.
    """
    dev = torch.device("cuda", device) if isinstance(device, int) else device
    for name, t in (("q_host", q_host), ("k_host", k_host), ("v_host", v_host)):
        if t.is_cuda or t.dtype != torch.bfloat16 or not t.is_contiguous() or t.dim() != 4 or t.shape[-1] != 128:
            raise ValueError(f"{name} must be a contiguous bfloat16 host tensor [B, S, heads, 128]")
        if tuple(t.shape) != tuple(q_host.shape):
            raise ValueError(f"{name} shape {tuple(t.shape)} != {tuple(q_host.shape)}")
    b_sz, _, heads, _ = q_host.shape
    if len(text_valid) != b_sz:
        raise ValueError("text_valid needs one entry per batch sample")
    groups = default_head_groups(heads) if head_groups is None else int(head_groups)
    t_lat, hp, wp = (int(x) for x in grid)
    need = int(lib().hv_attn_host_workspace_bytes(b_sz, heads, t_lat, hp, wp, int(text_len), groups))
    if need < 0:
        raise HVError(HV_ERR_BAD_SHAPE, "hv_attn_host_workspace_bytes")
    work = {} if work is None else work
    ws = work.get("host_ws")
    if ws is None or ws.device != dev or ws.numel() * ws.element_size() < need:
        ws = work["host_ws"] = torch.empty(need, dtype=torch.uint8, device=dev)
    if out_host is None:
        out_host = torch.empty(q_host.shape, dtype=q_host.dtype, pin_memory=True)
    valid = (ctypes.c_int * b_sz)(*[int(x) for x in text_valid])
    if scale is None:
        scale = 1.0 / math.sqrt(128)
    stream = torch.cuda.current_stream(dev)
    with torch.cuda.device(dev):
        st = lib().hv_attn_forward_host(q_host.data_ptr(), k_host.data_ptr(), v_host.data_ptr(),
                                        out_host.data_ptr(), b_sz, heads, t_lat, hp, wp, int(text_len), valid,
                                        float(rope_theta), float(scale), groups, ws.data_ptr(),
                                        ws.numel() * ws.element_size(), ctypes.c_void_p(stream.cuda_stream))
    if st != HV_OK:
        raise HVError(st, "hv_attn_forward_host")
    stream.synchronize()
    return out_host
