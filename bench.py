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
    ap.add_argument("--cpu-seconds", type=float, default=15.0, help="target CPU time of the oracle sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-clocks", action="store_true")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer leg (for profiling runs)")
    ap.add_argument("--no-ws", action="store_true", help="skip timing the workspace (pre-rotated K) path")
    ap.add_argument("--no-qknorm", action="store_true", help="skip timing the QK RMSNorm prologue paths")
    return ap.parse_args()


def workload_flops(wl, text_valid) -> float:
    s_len = wl.seq_len
    return float(sum(4.0 * wl.heads * s_len * (wl.n_video + int(v)) * 128 for v in text_valid))


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
        "l2": "inputs larger than L2 (q,k,v,out = %.2f GB vs 126 MB L2), no flush" % (
            4 * wl.batch * wl.seq_len * wl.heads * 256 / 1e9),
        "parallelism": "replicas",
    }


def load_peaks():
    p = ROOT / "MEASURED_PEAKS.json"
    if p.exists():
        d = json.loads(p.read_text())
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


def source_digest() -> str:
    h = hashlib.sha256()
    for f in sorted((ROOT / "joint_full_attention_b200" / "csrc").glob("*")):
        h.update(f.read_bytes())
    return h.hexdigest()[:16]


def traffic_per_launch():
    """DRAM bytes per launch from the committed ncu summary, if it matches this source."""
    if not TRAFFIC_SUMMARY.exists():
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


def oracle_sample(wl, inp, seconds: float, seed: int = 0):
    """Time the float64 oracle on sampled query rows of one (b, head): returns (tflops, info)."""
    from threadpoolctl import threadpool_info

    from joint_full_attention_b200 import workloads as W
    from oracle import hv_oracle as O

    b, h = 0, 0
    valid = int(inp["text_valid"][b])
    q = W.bf16_bits_to_f64(inp["q"][b:b + 1, :, h:h + 1])
    k = W.bf16_bits_to_f64(inp["k"][b:b + 1, :, h:h + 1])
    v = W.bf16_bits_to_f64(inp["v"][b:b + 1, :, h:h + 1])
    rng = np.random.default_rng(seed)
    kv = wl.n_video + valid

    def run(rows):
        samples = np.stack([np.zeros(rows, np.int64), np.zeros(rows, np.int64),
                            rng.integers(0, wl.seq_len, rows)], axis=1)
        t0 = time.perf_counter()
        O.joint_attention_samples(q, k, v, wl.grid, wl.text_len, [valid], samples)
        return time.perf_counter() - t0

    rows = 32
    dt = run(rows)
    rows = int(max(32, min(1 << 16, rows * seconds / max(dt, 1e-3) * 0.8)))
    dt = run(rows)
    flops = 4.0 * rows * kv * 128
    threads = max((d.get("num_threads", 1) for d in threadpool_info()), default=1)
    info = {"rows": rows, "seconds": dt, "threads": threads,
            "sample": f"{rows} query rows of (b=0, head=0) against all {kv} valid keys, "
                      f"float64 numpy oracle incl. the per-head key rotation; TFLOP/s of the sampled rows"}
    return flops / dt / 1e12, info


def run_reference(args, wl, inp, rank, world):
    if rank != 0:
        return
    cfg = config_of(wl, inp["text_valid"])
    per_step = max(1.0, args.cpu_seconds / max(1, args.steps))
    for _ in range(args.warmup):
        oracle_sample(wl, inp, min(per_step, 2.0))
    vals, infos = [], []
    t_all = time.perf_counter()
    for s in range(args.steps):
        v, info = oracle_sample(wl, inp, per_step, seed=s + 1)
        vals.append(v)
        infos.append(info)
    wall = time.perf_counter() - t_all
    value = statistics.mean(vals)
    flops = workload_flops(wl, inp["text_valid"])
    ms = flops / (value * 1e12) * 1e3
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "config": cfg,
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": infos[-1]["threads"], "kind": "oracle",
                         "sample": infos[-1]["sample"] + f"; {args.steps} steps in {wall:.1f} s, "
                                   f"ms_per_step extrapolated to the full call"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


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

    if rank != 0:
        return
    peaks, peak_kind = load_peaks()
    mean_launch = statistics.mean(launch_ms)
    achieved = flops / (mean_launch / 1e3) / 1e12
    peak = float(peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))
    peak_burst = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    roofline = {
        "bound": "tensor", "achieved": achieved, "peak": peak, "unit": UNIT, "frac": achieved / peak,
        "traffic": traffic_per_launch(), "kernel": KERNEL_NAME,
        "peak_source": f"bf16_tflops_sustained of {peak_kind} (cuBLAS bf16 loop under the power cap); "
                       "the step is a seconds-long loop of one kernel",
        "frac_of_burst": achieved / peak_burst, "frac_of_datasheet_2250": achieved / DATASHEET_BF16_TFLOPS,
        "algorithmic_flops_per_launch": flops,
        "launch_ms": {"mean": mean_launch, "min": min(launch_ms), "max": max(launch_ms)},
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
    }
    if world == 1 and not args.no_cpu_baseline:
        cpu_value, info = oracle_sample(wl, inp, args.cpu_seconds)
        line["cpu_baseline"] = {"value": cpu_value, "unit": UNIT, "cores": info["threads"], "kind": "oracle",
                                "sample": info["sample"]}
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
            run_reference(args, wl, W.make_inputs(wl, seed=0), rank, world)
        return
    rank, world, local = dist_init(args.gpus)
    inp = W.make_inputs(wl, seed=0)
    run_ours(args, wl, inp, rank, world, local)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
