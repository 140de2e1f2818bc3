#!/usr/bin/env python
"""Benchmark of the joint 3D-RoPE attention call on B200.

One step = one ``hv_attn_forward`` call over the whole workload (default:
720x1280x129 -> 118800 video + 256 text tokens, B=1, 24 heads x 128, bf16),
i.e. every step of the hot path: RoPE-on-load, QK^T, key mask, online
softmax, PV and the bf16 epilogue, all inside one kernel launch.

Prints ONE JSON line (rank 0). ``value`` is whole-job TFLOP/s of algorithmic
work (4 * heads * S * (N + valid) * 128 per sample; masked padding not
counted) with inputs resident in HBM; ``e2e`` is the same metric through the
host-buffer API (pinned host -> device copies, the call, device -> host copy
of the output, all inside the timed region). Multi-GPU runs are independent
replicas (the call does not shard): ``value`` = work of all ranks / the
slowest rank's time.

``--impl reference`` times the float64 CPU oracle on bounded samples of the
same workload instead (the only other use of ``oracle/`` here besides the
``cpu_baseline`` leg).
"""

from __future__ import annotations

import argparse
import csv
import hashlib
import io
import json
import math
import os
import re
import statistics
import subprocess
import sys
import tempfile
import time
from pathlib import Path

import numpy as np

ROOT = Path(__file__).resolve().parent
sys.path.insert(0, str(ROOT))

METRIC = "joint 3D-RoPE attention TFLOP/s & ms/call at 720×1280×129, % of B200 dense-BF16 peak"
UNIT = "TFLOP/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
DATASHEET_BF16_TFLOPS = 2250.0
KERNEL_NAME = "hv_attn_fwd_kernel"
TRAFFIC_SUMMARY = ROOT / "profiles" / "hv_attn_fwd_kernel.v720x1280x129.dram.md"


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="v720x1280x129")
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-clocks", action="store_true")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer leg (for profiling runs)")
    ap.add_argument("--no-ws", action="store_true", help="skip timing the workspace (pre-rotated K) path")
    ap.add_argument("--no-qknorm", action="store_true", help="skip timing the QK RMSNorm prologue paths")
    ap.add_argument("--no-workloads", action="store_true", help="skip timing the other workloads")
    return ap.parse_args()


def workload_flops(wl, text_valid) -> float:
    s_len = wl.seq_len
    return float(sum(4.0 * wl.heads * s_len * (wl.n_video + int(v)) * 128 for v in text_valid))


def l2_note(wl) -> str:
    gb = 4 * wl.batch * wl.seq_len * wl.heads * 256 / 1e9
    if gb * 1e3 > 126:
        return "inputs larger than L2 (q,k,v,out = %.2f GB vs 126 MB L2), no flush" % gb
    return "inputs fit in L2 (q,k,v,out = %.1f MB vs 126 MB L2), no flush" % (gb * 1e3)


def config_of(wl, text_valid) -> dict:
    return {
        "workload": f"{wl.label}: B={wl.batch}, {wl.heads} heads x 128, {wl.n_video} video + {wl.text_len} text tokens",
        "name": wl.name,
        "batch": wl.batch,
        "heads": wl.heads,
        "head_dim": 128,
        "grid": list(wl.grid),
        "seq_len": wl.seq_len,
        "text_len": wl.text_len,
        "text_valid": [int(v) for v in text_valid],
        "rope_theta": 256.0,
        "scale": 1.0 / math.sqrt(128),
        "l2": l2_note(wl),
        "parallelism": "replicas",
    }


def load_peaks():
    p = ROOT / "MEASURED_PEAKS.json"
    if p.exists():
        d = json.loads(p.read_text())
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


_CODE_TOKENS = re.compile(r'//[^\n]*|/\*.*?\*/|"(?:\\.|[^"\\\n])*"|\S+', re.S)


def source_digest() -> str:
    """Hash of the CUDA sources' code: comments and layout are left out, so that
    a comment edit does not retire the DRAM figures taken on unchanged code."""
    h = hashlib.sha256()
    for f in sorted((ROOT / "joint_full_attention_b200" / "csrc").glob("*")):
        for tok in _CODE_TOKENS.findall(f.read_text(encoding="utf-8")):
            if not tok.startswith(("//", "/*")):
                h.update(tok.encode("utf-8") + b"\0")
    return h.hexdigest()[:16]


def traffic_per_launch(workload: str):
    """DRAM bytes per launch from the committed ncu summary, if it covers this
    workload and matches this source."""
    if not TRAFFIC_SUMMARY.exists() or f".{workload}." not in TRAFFIC_SUMMARY.name:
        return None
    text = TRAFFIC_SUMMARY.read_text()
    m_src = re.search(r"source_digest:\s*([0-9a-f]+)", text)
    m_b = re.search(r"traffic_bytes_per_launch:\s*([0-9.eE+]+)", text)
    if not (m_src and m_b) or m_src.group(1) != source_digest():
        return None
    return float(m_b.group(1))


class Clocks:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int, enabled: bool = True):
        self.index = index
        self.proc = None
        self.path = None
        if enabled:
            try:
                fd, self.path = tempfile.mkstemp(suffix=".csv")
                os.close(fd)
                self.fh = open(self.path, "w")
                self.proc = subprocess.Popen(
                    ["nvidia-smi", "-i", str(index), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                     "-lms", "200"], stdout=self.fh, stderr=subprocess.DEVNULL)
            except OSError:
                self.proc = None

    def stop(self) -> dict | None:
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.fh.close()
        rows = list(csv.reader(io.StringIO(Path(self.path).read_text())))
        os.unlink(self.path)
        sm, smax, reasons, power = [], 0.0, set(), []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            r = [x.strip() for x in r]
            if len(r) < 9:
                continue
            try:
                sm.append(float(r[1]))
                smax = max(smax, float(r[2]))
                power.append(float(r[3]))
            except ValueError:
                continue
            for name, val in zip(names, r[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": smax, "reasons": sorted(reasons),
                "samples": len(sm), "power_w_max": max(power) if power else None}


def dist_init(n_gpus: int):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=600))
    return rank, world, local


def allreduce_max(x: float, world: int) -> float:
    """Max of x over all ranks (a CUDA tensor under NCCL, a CPU tensor under gloo)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_throughput(local_ms: float, flops_per_rank: float, world: int) -> tuple[float, float]:
    """Independent replicas: (slowest rank's ms per step, whole-job TFLOP/s).

    Every rank runs the same workload; the job's throughput is the work of all
    ranks divided by the time of the slowest one.
    """
    ms = allreduce_max(local_ms, world)
    return ms, world * flops_per_rank / (ms / 1e3) / 1e12


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def oracle_rows(wl) -> int:
    """Rows per oracle sample: about 4e10 FLOP of float64 work against all valid keys (64..4096)."""
    kv = wl.n_video + wl.text_len
    return int(max(64, min(4096, round(4e10 / (4.0 * kv * 128)))))


def oracle_estimate(wl, seed: int = 0, rows: int | None = None, threads: int | None = None) -> dict:
    """Time the float64 oracle on one (b, head) of the workload and extrapolate to the whole call.

    The oracle rotates a head's keys once and then computes each query row
    against all valid keys, so its time for r rows of one head is a + b*r. Two
    calls of ``joint_attention_head`` (32 rows, then 32 + ``rows`` rows) give a
    (key preparation) and b (per row); the whole call takes B*heads*(a + b*S).
    Inputs: one head's q, k, v of the workload's shape from the seeded
    generator (the oracle's time does not depend on the values).
    ``threads``: limit of the BLAS thread pools (None: all).
    """
    from threadpoolctl import threadpool_info, threadpool_limits

    from joint_full_attention_b200 import workloads as W
    from oracle import hv_oracle as O

    one = W.Workload(wl.name + "-head", wl.label, 1, 1, wl.grid, wl.text_len, valid=wl.valid,
                     k_head_scale=False)
    inp = W.make_inputs(one, seed=seed)
    valid = int(inp["text_valid"][0])
    q, k, v = (W.bf16_bits_to_f64(inp[n][0, :, 0]) for n in ("q", "k", "v"))
    rows = oracle_rows(wl) if rows is None else int(rows)
    rng = np.random.default_rng(seed)

    def run(r):
        sel = rng.integers(0, wl.seq_len, r)
        t0 = time.perf_counter()
        O.joint_attention_head(q, k, v, wl.grid, valid, rows=sel)
        return time.perf_counter() - t0

    with threadpool_limits(limits=threads):
        used = max((d.get("num_threads", 1) for d in threadpool_info()), default=1)
        t_all = time.perf_counter()
        run(1)                                  # warm-up: first-touch and allocation effects
        t1 = min(run(32), run(32))
        t2 = run(32 + rows)
        t_all = time.perf_counter() - t_all
    per_row = max((t2 - t1) / rows, 1e-9)
    fixed = max(t1 - 32 * per_row, 0.0)
    call_s = wl.batch * wl.heads * (fixed + per_row * wl.seq_len)
    return {"call_seconds": call_s, "per_row_s": per_row, "per_head_fixed_s": fixed, "rows": rows,
            "threads": used, "sample_seconds": t_all,
            "sample": f"float64 oracle (joint_attention_head) on one (b, head) of this workload, all valid "
                      f"keys: after a warm-up call, 32 seeded query rows (best of 2) and {32 + rows} rows; "
                      f"time = a + b*rows fitted (a: the head's key rotation, b: per row), extrapolated to "
                      f"B*heads*(a + b*S)"}


def cpu_baseline_of(wl, flops: float, seed: int = 0, one_core: bool = True) -> dict:
    """The oracle on all host threads (and on one core), extrapolated to the whole call."""
    full = oracle_estimate(wl, seed)
    res = {"value": flops / full["call_seconds"] / 1e12, "unit": UNIT, "cores": full["threads"],
           "kind": "oracle", "sample": full["sample"],
           "rows": full["rows"], "ms_per_call_extrapolated": full["call_seconds"] * 1e3,
           "cpu_seconds": full["sample_seconds"], "host_cpus": os.cpu_count()}
    if one_core:
        one = oracle_estimate(wl, seed, rows=max(16, full["rows"] // 4), threads=1)
        res["one_core"] = {"value": flops / one["call_seconds"] / 1e12, "cores": 1, "rows": one["rows"],
                           "ms_per_call_extrapolated": one["call_seconds"] * 1e3,
                           "cpu_seconds": one["sample_seconds"]}
    return res


def run_reference(args, wl, rank, world):
    if rank != 0:
        return
    from joint_full_attention_b200 import workloads as W
    text_valid = W.text_valid_of(wl, seed=0)
    cfg = config_of(wl, text_valid)
    flops = workload_flops(wl, text_valid)
    for w in range(args.warmup):
        oracle_estimate(wl, seed=100 + w, rows=32)
    calls = []
    t_all = time.perf_counter()
    for s in range(args.steps):
        calls.append(oracle_estimate(wl, seed=s + 1))
    wall = time.perf_counter() - t_all
    call_s = statistics.mean(c["call_seconds"] for c in calls)
    value = flops / call_s / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": call_s * 1e3,
        "ms_per_step_extrapolated": True, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "config": cfg,
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": calls[-1]["threads"], "kind": "oracle",
                         "rows": calls[-1]["rows"],
                         "sample": calls[-1]["sample"] + f"; each step is one such estimate, {args.steps} "
                                   f"steps in {wall:.1f} s; ms_per_step is the extrapolated whole call, "
                                   f"not a measured call"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def time_calls(call, stream, steps: int, warmup: int) -> list[float]:
    """CUDA-event device time (ms) of each of `steps` calls after `warmup` untimed ones."""
    import torch
    for _ in range(warmup):
        call()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for a, b in ev:
        a.record(stream)
        call()
        b.record(stream)
    torch.cuda.synchronize()
    return [a.elapsed_time(b) for a, b in ev]


def other_workloads(args, dev, stream, peaks):
    """Device time, TFLOP/s and roofline fraction of the fused call on every other workload."""
    import torch

    from joint_full_attention_b200 import hvattn as H
    from joint_full_attention_b200 import workloads as W

    peak = float(peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))
    peak_burst = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    res = []
    for name, wl in W.WORKLOADS.items():
        if name == args.workload:
            continue
        inp = W.make_device_inputs(wl, seed=0, device=dev)
        tv = [int(x) for x in inp["text_valid"]]
        out = torch.empty_like(inp["q"])
        flops = workload_flops(wl, tv)
        call = lambda: H.attn_forward(inp["q"], inp["k"], inp["v"], wl.grid, wl.text_len, tv, out=out,
                                      stream=stream)
        one = statistics.median(time_calls(call, stream, 3, 2))
        steps = int(max(5, min(200, 1500.0 / max(one, 1e-3))))
        ms = time_calls(call, stream, steps, 2)
        if H.last_device_error() != 0:
            raise RuntimeError(f"device error on workload {name}")
        mean = statistics.mean(ms)
        achieved = flops / (mean / 1e3) / 1e12
        entry = {"workload": name, "label": wl.label, "batch": wl.batch, "heads": wl.heads, "grid": list(wl.grid),
                 "seq_len": wl.seq_len, "text_valid": tv, "flop_per_call": flops, "steps": steps,
                 "ms_per_call": mean, "ms_min": min(ms), "value": achieved, "unit": UNIT,
                 "frac_of_sustained": achieved / peak, "frac_of_burst": achieved / peak_burst,
                 "units_256_rows": wl.batch * wl.heads * -(-wl.seq_len // 256), "sms": sms}
        if not args.no_cpu_baseline:
            entry["cpu_baseline"] = cpu_baseline_of(wl, flops, one_core=False)
        res.append(entry)
        del inp, out
        torch.cuda.empty_cache()
    return res


def run_ours(args, wl, inp, rank, world, local):
    import torch

    from joint_full_attention_b200 import hvattn as H

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    H.lib()
    text_valid = [int(x) for x in inp["text_valid"]]
    to_dev = lambda bits: torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(dev)
    q, k, v = (to_dev(inp[n]) for n in ("q", "k", "v"))
    out = torch.empty_like(q)
    flops = workload_flops(wl, text_valid)
    stream = torch.cuda.current_stream(dev)

    def step():
        H.attn_forward(q, k, v, wl.grid, wl.text_len, text_valid, out=out, stream=stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    if H.last_device_error() != 0:
        raise RuntimeError("device error during warm-up")

    barrier(world)
    torch.cuda.synchronize(dev)
    clocks = Clocks(local, enabled=not args.no_clocks)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    for s in range(args.steps):
        ev[s][0].record(stream)
        step()
        ev[s][1].record(stream)
    t_end.record(stream)
    torch.cuda.synchronize(dev)
    barrier(world)
    clk = clocks.stop()
    total_ms = t_start.elapsed_time(t_end)
    launch_ms = [a.elapsed_time(b) for a, b in ev]
    if H.last_device_error() != 0:
        raise RuntimeError("device error during the timed region")

    ms_per_step, value = replica_throughput(total_ms / args.steps, flops, world)

    # the workspace path: K rotated once by a memory-bound kernel, then attention
    ws_line = None
    if not args.no_ws:
        ws = torch.empty(H.workspace_bytes(wl.batch, wl.heads, wl.grid, wl.text_len) // 2, dtype=torch.bfloat16,
                         device=dev)
        for _ in range(max(1, args.warmup)):
            H.attn_forward_ws(q, k, v, wl.grid, wl.text_len, text_valid, out=out, workspace=ws, stream=stream)
        torch.cuda.synchronize(dev)
        barrier(world)
        w0, w1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        w0.record(stream)
        for _ in range(args.steps):
            H.attn_forward_ws(q, k, v, wl.grid, wl.text_len, text_valid, out=out, workspace=ws, stream=stream)
        w1.record(stream)
        torch.cuda.synchronize(dev)
        if H.last_device_error() != 0:
            raise RuntimeError("device error in the workspace path")
        ws_ms, ws_value = replica_throughput(w0.elapsed_time(w1) / args.steps, flops, world)
        ws_line = {"value": ws_value, "unit": UNIT, "ms_per_step": ws_ms,
                   "gpu_launches_per_step": 2, "workspace_bytes": ws.numel() * 2,
                   "what": "hv_attn_forward_ws: keys rotated once into a caller workspace by a memory-bound "
                           "kernel, then the attention kernel rotating Q on load; output bit-identical"}
        del ws

    # the QK RMSNorm prologue (seeded gammas), one-kernel and two-stage forms
    qk_line = None
    if not args.no_qknorm:
        gam = torch.from_numpy(np.random.default_rng(1234).uniform(0.5, 1.5, (4, 128)).astype(np.float32)).to(dev)
        ws = torch.empty(H.workspace_bytes(wl.batch, wl.heads, wl.grid, wl.text_len) // 2, dtype=torch.bfloat16,
                         device=dev)
        qk_line = {"unit": UNIT, "what": "hv_attn_forward_qknorm / _qknorm_ws: per-head RMSNorm of Q and K "
                                         "(video and text gammas, eps 1e-6) before the rotation"}
        for key, wsp in (("fused", None), ("workspace", ws)):
            call = lambda: H.attn_forward_qknorm(q, k, v, wl.grid, wl.text_len, text_valid, gam, 1e-6, out=out,
                                                 workspace=wsp, stream=stream)
            for _ in range(max(1, args.warmup)):
                call()
            torch.cuda.synchronize(dev)
            barrier(world)
            a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a0.record(stream)
            for _ in range(args.steps):
                call()
            a1.record(stream)
            torch.cuda.synchronize(dev)
            if H.last_device_error() != 0:
                raise RuntimeError("device error in the QK-norm path")
            q_ms, q_value = replica_throughput(a0.elapsed_time(a1) / args.steps, flops, world)
            qk_line[key] = {"value": q_value, "ms_per_step": q_ms}
        del ws

    # end to end through the host-buffer API: pinned host in, pinned host out
    e2e = None
    if not args.no_e2e:
        to_host = lambda bits: torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).pin_memory()
        qh, kh, vh = (to_host(inp[n]) for n in ("q", "k", "v"))
        oh = torch.empty(qh.shape, dtype=qh.dtype).pin_memory()
        work = {"q": q, "k": k, "v": v, "out": out}
        H.attn_forward_host(qh, kh, vh, wl.grid, wl.text_len, text_valid, device=dev, out_host=oh, work=work)
        barrier(world)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.e2e_steps):
            H.attn_forward_host(qh, kh, vh, wl.grid, wl.text_len, text_valid, device=dev, out_host=oh, work=work)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        e2e_ms, e2e_value = replica_throughput(e0.elapsed_time(e1) / args.e2e_steps, flops, world)
        e2e = {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": 3 * qh.numel() * 2,
               "d2h_bytes_per_step": oh.numel() * 2, "ms_per_step": e2e_ms, "steps": args.e2e_steps}
        del qh, kh, vh, oh, work

    peaks, peak_kind = load_peaks()
    others = None
    if not args.no_workloads:
        del q, k, v, out
        torch.cuda.empty_cache()
        others = other_workloads(args, dev, stream, peaks)

    if rank != 0:
        return
    mean_launch = statistics.mean(launch_ms)
    achieved = flops / (mean_launch / 1e3) / 1e12
    peak = float(peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))
    peak_burst = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    roofline = {
        "bound": "tensor", "achieved": achieved, "peak": peak, "unit": UNIT, "frac": achieved / peak,
        "traffic": traffic_per_launch(args.workload), "kernel": KERNEL_NAME,
        "peak_source": f"bf16_tflops_sustained of {peak_kind} (cuBLAS bf16 loop under the power cap); "
                       "the step is a seconds-long loop of one kernel",
        "frac_of_burst": achieved / peak_burst, "frac_of_datasheet_2250": achieved / DATASHEET_BF16_TFLOPS,
        "algorithmic_flops_per_launch": flops,
        "launch_ms": {"mean": mean_launch, "median": statistics.median(launch_ms), "min": min(launch_ms),
                      "max": max(launch_ms), "count": len(launch_ms)},
    }
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "config": config_of(wl, text_valid),
        "roofline": roofline,
        "e2e": e2e,
        "gpu_launches": args.steps,
        "clocks": clk,
        "workspace_path": ws_line,
        "qk_norm_path": qk_line,
        "workloads": others,
    }
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline_of(wl, flops)
    print(json.dumps(line), flush=True)


def main():
    args = parse_args()
    from joint_full_attention_b200 import workloads as W
    wl = W.WORKLOADS[args.workload]
    if args.impl == "reference":
        # the oracle runs on rank 0's host cores only; other ranks exit at once
        rank = int(os.environ.get("RANK", "0"))
        world = int(os.environ.get("WORLD_SIZE", "1"))
        if rank == 0:
            run_reference(args, wl, rank, world)
        return
    rank, world, local = dist_init(args.gpus)
    inp = W.make_inputs(wl, seed=0)
    run_ours(args, wl, inp, rank, world, local)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
