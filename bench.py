#!/usr/bin/env python
"""Benchmark of the SageSLA attention path on B200.

python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload NAME|all]

One step = one sagesla_attn call over the whole workload (every kernel of the
path: statistics, quantisation, pooled top-k mask, linear branch, sparse
flash).  Default workload: Wan2.1-14B-720P-shaped self-attention, B=1, H=40,
N=75600, d=128, block 64, topk 0.1, seeded synthetic bf16 inputs (2.3 GB, far
larger than L2, so no flush is needed between steps).  Prints one JSON line.
Under torchrun every rank runs its own replica of the workload (independent
problems, no collective on the data path): weak scaling.  `--workload all`
(one GPU) prints one shorter line per benchmark configuration instead: the
five configurations (tiny, 1.3B-480P, 14B-480P, 14B-720P at topk 0.1 and
0.05) and the sparsity sweep at 720p (block 64 and 128, topk 0.05 / 0.1 /
0.15, dense with the linear branch off).
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "SageSLA attn ms/call & dense-equiv TFLOPS at H40xN75600xd128; % roofline"


def _env_int(name, default):
    try:
        return int(os.environ.get(name, default))
    except ValueError:
        return default


def workloads():
    from sparse_bit_attention_smoothing_b200 import inputs as I
    d = {w.name: w for w in [I.TINY, I.WAN13_480P, I.WAN14_480P, I.WAN14_720P, I.WAN14_720P_K05] + I.sweep()}
    return d


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            m = json.load(f)
        return dict(hbm=m["hbm_gbs"], bf16=m["bf16_tflops"], bf16_sus=m.get("bf16_tflops_sustained"), src="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sus=1400.0, src="fallback")


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, ValueError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        out, _ = self.proc.communicate(timeout=10)
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, val in zip(names, f[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def flash_traffic(w):
    """DRAM bytes of one flash launch from the committed ncu capture, scaled by
    elements; None when the kernel source changed since the capture."""
    import hashlib
    p = os.path.join(ROOT, "profiles", "flash_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        t = json.load(f)
    with open(os.path.join(ROOT, t["source"]), "rb") as f:
        if hashlib.sha256(f.read()).hexdigest() != t["source_sha256"]:
            return None
    if w.block != 64:
        return None
    return t["dram_bytes"] / t["elements"] * (w.B * w.H * w.N * w.d)


def flops(w) -> dict:
    """Dense-equivalent and computed-block FLOPs of one call, and algorithmic HBM bytes."""
    from sparse_bit_attention_smoothing_b200 import topk_count
    BH, N, d = w.B * w.H, w.N, w.d
    nb = (N + w.block - 1) // w.block
    kc = topk_count(nb, w.topk)
    dense = 4.0 * BH * N * N * d
    blocks = 4.0 * BH * nb * kc * w.block * w.block * d
    E = BH * N * d
    hbm = 2 * E * 2 + 3 * E * 2 + 3 * E + 3 * E + 2 * E
    return dict(dense=dense, computed=blocks, hbm_bytes=float(hbm), nb=nb, kc=kc)


def cpu_baseline(w, q, k, v, pw, heads: int = 8, qblocks: int = 4) -> dict:
    """The oracle, as it stands, on a bounded sample of the workload; extrapolated to one call."""
    import numpy as np
    from oracle import oracle as orc
    orc.lib()
    BH, N, d = w.B * w.H, w.N, w.d
    nb = (N + w.block - 1) // w.block
    hs = min(heads, BH)
    qf = q.reshape(BH, N, d)[:hs].contiguous()
    kf = k.reshape(BH, N, d)[:hs].contiguous()
    vf = v.reshape(BH, N, d)[:hs].contiguous()
    sel0 = np.zeros((hs, nb), np.uint8)
    t0 = time.perf_counter()
    orc.sagesla(qf, kf, vf, pw, w.block, w.topk, qsel=sel0)
    t_fixed = time.perf_counter() - t0
    sel = np.zeros((hs, nb), np.uint8)
    picks = np.unique(np.linspace(0, nb - 1, qblocks).round().astype(int))
    sel[:, picks] = 1
    t0 = time.perf_counter()
    orc.sagesla(qf, kf, vf, pw, w.block, w.topk, qsel=sel)
    t_sample = time.perf_counter() - t0
    cores = orc.threads()
    t_qb = max(0.0, (t_sample - t_fixed) / len(picks))
    waves = math.ceil(BH / min(cores, hs)) if hs < cores else math.ceil(BH / cores)
    full_s = waves * (t_fixed + nb * t_qb)
    f = flops(w)
    return dict(value=f["dense"] / full_s / 1e12, unit="TFLOPS", cores=cores, kind="oracle",
                ms_per_call=full_s * 1e3,
                sample=(f"{hs} heads x {len(picks)} query blocks of {w.name} (fp64 C oracle, OpenMP over heads); "
                        f"per-head fixed part {t_fixed:.2f}s, {t_qb * 1e3:.1f} ms per query block; "
                        f"extrapolated to {BH} heads x {nb} query blocks"),
                sample_seconds=t_fixed + t_sample)


def run_all(args):
    """One line per benchmark configuration (kernel-only timing, one GPU)."""
    import torch
    from sparse_bit_attention_smoothing_b200 import build as sbuild
    sbuild.build()
    import sparse_bit_attention_smoothing_b200 as sg
    from sparse_bit_attention_smoothing_b200.inputs import make_inputs
    st = torch.cuda.current_stream()
    pk = peaks()
    peak8 = 2.0 * pk["bf16"]
    cache = {}
    for w in workloads().values():
        key = (w.B, w.H, w.N, w.d, w.outliers)
        if key not in cache:
            cache.clear()
            q, k, v, pw = make_inputs(w.B, w.H, w.N, w.d, seed=0, outliers=w.outliers)
            cache[key] = (q.cuda(), k.cuda(), v.cuda(), pw.cuda())
        dq, dk, dv, dw = cache[key]
        dw = dw if w.linear else None
        out = torch.empty_like(dq)
        for _ in range(max(3, args.warmup)):
            sg.sagesla_attn(dq, dk, dv, dw, out=out, block=w.block, topk=w.topk, stream=st)
        torch.cuda.synchronize()
        sg.profile(True)
        sg.profile_read()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(st)
        for _ in range(args.steps):
            sg.sagesla_attn(dq, dk, dv, dw, out=out, block=w.block, topk=w.topk, stream=st)
        e1.record(st)
        torch.cuda.synchronize()
        prof = sg.profile_read()
        sg.profile(False)
        ms = e0.elapsed_time(e1) / args.steps
        f = flops(w)
        fl_ms, fl_n = prof.get("flash", (0.0, 0))
        flash_ms = fl_ms / max(1, fl_n)
        achieved = f["computed"] / (flash_ms * 1e-3) / 1e12 if flash_ms > 0 else None
        t_roof = max(f["computed"] / (peak8 * 1e12), f["hbm_bytes"] / (pk["hbm"] * 1e9))
        line = {"workload": w.name, "B": w.B, "H": w.H, "N": w.N, "block": w.block, "topk": w.topk,
                "linear": w.linear, "k_blocks": f["kc"], "ms_per_call": ms,
                "dense_equiv_tflops": f["dense"] / (ms * 1e-3) / 1e12,
                "flash_ms": flash_ms, "flash_tflops": achieved,
                "flash_frac_of_8bit_peak": (achieved / peak8) if achieved else None,
                "path_frac_of_roofline": t_roof * 1e3 / ms, "device_status": sg.sync_status(),
                "kernels_ms": {kname: round(t / max(1, n), 4) for kname, (t, n) in prof.items()}}
        print(json.dumps(line), flush=True)
        del out
    return 0


def run_reference(args):
    rank = _env_int("RANK", 0)
    if rank != 0:
        return 0
    from sparse_bit_attention_smoothing_b200.inputs import make_workload
    w = workloads()[args.workload]
    q, k, v, pw = make_workload(w)
    vals = []
    for s in range(args.warmup + args.steps):
        cb = cpu_baseline(w, q, k, v, pw, heads=4, qblocks=2)
        if s >= args.warmup:
            vals.append(cb)
    val = statistics.median([c["value"] for c in vals])
    ms = statistics.median([c["ms_per_call"] for c in vals])
    line = {"impl": "reference", "metric": METRIC, "value": val, "unit": "TFLOPS", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": w.name, "B": w.B, "H": w.H, "N": w.N, "d": w.d, "block": w.block,
                       "topk": w.topk, "linear": w.linear},
            "cpu_baseline": {"value": val, "unit": "TFLOPS", "cores": vals[0]["cores"], "kind": "oracle",
                             "sample": vals[0]["sample"]},
            "e2e": {"value": val, "unit": "TFLOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="wan2.1-14b-720p_h40_n75600")
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-linear", action="store_true", help="proj_w = NULL (linear branch off)")
    args = ap.parse_args()
    if args.impl == "reference":
        return run_reference(args)
    if args.workload == "all":
        return run_all(args)

    import torch
    import torch.distributed as dist

    from sparse_bit_attention_smoothing_b200.replicas import job_throughput, max_over_ranks, rank_env

    rank, world, local = rank_env()
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=torch.device("cuda", local))
    from sparse_bit_attention_smoothing_b200 import build as sbuild
    sbuild.build()
    import sparse_bit_attention_smoothing_b200 as sg
    from sparse_bit_attention_smoothing_b200.inputs import make_workload

    w = workloads()[args.workload]
    q, k, v, pw = make_workload(w)
    if args.no_linear:
        pw = None
    dq, dk, dv = q.cuda(), k.cuda(), v.cuda()
    dw = pw.cuda() if pw is not None else None
    out = torch.empty_like(dq)
    st = torch.cuda.current_stream()

    def step():
        sg.sagesla_attn(dq, dk, dv, dw, out=out, block=w.block, topk=w.topk, stream=st)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    sg.profile(True)
    sg.profile_read()
    clk = ClockSampler(local)
    clk.start()
    time.sleep(0.3)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(st)
    for _ in range(args.steps):
        step()
    e1.record(st)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clocks = clk.stop()
    prof = sg.profile_read()
    sg.profile(False)
    status = sg.sync_status()
    ms = max_over_ranks([e0.elapsed_time(e1) / args.steps], device="cuda")[0]

    f = flops(w)
    value = job_throughput(f["dense"], world, ms) / 1e12
    pk = peaks()
    peak8 = 2.0 * pk["bf16"]  # 8-bit dense = 2 x bf16 (nominal 4.5 / 2.25 PFLOP/s)
    fl_ms, fl_n = prof.get("flash", (0.0, 0))
    flash_ms = fl_ms / max(1, fl_n)
    achieved = f["computed"] / (flash_ms * 1e-3) / 1e12 if flash_ms > 0 else None
    # profiler scopes -> kernels: the top-k scope launches pool_means, z_total
    # (linear branch on) and pool_topk; every other scope one kernel
    per_scope = {"pool_topk": 3 if (w.linear and pw is not None) else 2}
    launches = sum(n * per_scope.get(kname, 1) for kname, (_, n) in prof.items())
    t_roof = max(f["computed"] / (peak8 * 1e12), f["hbm_bytes"] / (pk["hbm"] * 1e9))

    # end to end through the host-buffer entry point (pinned memory)
    hq, hk, hv = q.pin_memory(), k.pin_memory(), v.pin_memory()
    hw = pw.pin_memory() if pw is not None else None
    hout = torch.empty_like(hq).pin_memory()
    sg.sagesla_attn_host(hq, hk, hv, hw, out=hout, block=w.block, topk=w.topk, stream=st)
    if world > 1:
        dist.barrier()
    t0 = time.perf_counter()
    for _ in range(args.e2e_steps):
        sg.sagesla_attn_host(hq, hk, hv, hw, out=hout, block=w.block, topk=w.topk, stream=st)
    e2e_ms = max_over_ranks([(time.perf_counter() - t0) * 1e3 / args.e2e_steps], device="cuda")[0]
    E = q.numel() * 2
    h2d = 3 * E + (pw.numel() * 2 if pw is not None else 0)

    line = {"metric": METRIC, "value": value, "unit": "TFLOPS", "n_gpus": world, "steps": args.steps,
            "warmup": max(3, args.warmup), "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "i8/e4m3 (fp32 accumulate, bf16 io)", "data": "synthetic",
            "config": {"workload": w.name, "B": w.B, "H": w.H, "N": w.N, "d": w.d, "block": w.block,
                       "topk": w.topk, "k_blocks": f["kc"], "nb": f["nb"], "linear": w.linear and pw is not None,
                       "l2": "inputs 2.3 GB > 126 MB L2, no flush", "parallelism": f"replicas x{world}"},
            "gpu_launches": launches, "device_status": status,
            "kernels_ms": {kname: round(t / max(1, n), 4) for kname, (t, n) in prof.items()},
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak8, "unit": "TFLOP/s",
                         "frac": (achieved / peak8) if achieved else None, "traffic": flash_traffic(w),
                         "kernel": "flash", "peak_note": f"8-bit = 2 x {pk['src']} bf16 burst {pk['bf16']}",
                         "path_t_roof_ms": t_roof * 1e3, "path_frac": t_roof * 1e3 / ms},
            "clocks": clocks,
            "e2e": {"value": job_throughput(f["dense"], world, e2e_ms) / 1e12, "unit": "TFLOPS", "ms_per_step": e2e_ms,
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": E}}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cb = cpu_baseline(w, q, k, v, pw)
        line["cpu_baseline"] = {kk: cb[kk] for kk in ("value", "unit", "cores", "kind", "sample", "ms_per_call")}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
