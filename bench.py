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


NOMINAL_8BIT_TFLOPS = 4500.0  # B200 dense INT8 / FP8, nominal


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


def flops(w, kc: int) -> dict:
    """Dense-equivalent and computed-block FLOPs of one call, and algorithmic HBM bytes.

    kc = key blocks kept per query block (the caller's topk_count: the library's
    in the GPU arm, the oracle's in the reference arm)."""
    BH, N, d = w.B * w.H, w.N, w.d
    nb = (N + w.block - 1) // w.block
    dense = 4.0 * BH * N * N * d
    blocks = 4.0 * BH * nb * kc * w.block * w.block * d
    E = BH * N * d
    hbm = 2 * E * 2 + 3 * E * 2 + 3 * E + 3 * E + 2 * E
    return dict(dense=dense, computed=blocks, hbm_bytes=float(hbm), nb=nb, kc=kc)


def _oracle():
    from oracle import oracle as orc
    orc.lib()
    return orc


def cpu_sample_plan(w, cores: int, qblocks: int = 2):
    """The oracle's bounded sample of a workload: one head per host core (all
    heads if there are fewer) x `qblocks` evenly spaced query blocks per head."""
    import numpy as np
    BH = w.B * w.H
    nb = (w.N + w.block - 1) // w.block
    heads = min(BH, max(1, cores))
    picks = np.unique(np.linspace(0, nb - 1, qblocks).round().astype(int))
    return heads, picks, nb


def cpu_fixed_part(w, q, k, v, pw, heads: int) -> float:
    """Seconds of the oracle's per-head work outside the query blocks (smoothing,
    quantisation, mask, linear-branch blocks) for `heads` heads run together."""
    import numpy as np
    orc = _oracle()
    BH, N, d = w.B * w.H, w.N, w.d
    nb = (N + w.block - 1) // w.block
    qf, kf, vf = (t.reshape(BH, N, d)[:heads].contiguous() for t in (q, k, v))
    t0 = time.perf_counter()
    orc.sagesla(qf, kf, vf, pw, w.block, w.topk, qsel=np.zeros((heads, nb), np.uint8))
    return time.perf_counter() - t0


def cpu_sample(w, q, k, v, pw, heads: int, picks, t_fixed: float) -> dict:
    """The oracle, as it stands, on the sample (the fixed part plus the picked
    query blocks of `heads` heads, one per core), extrapolated to one call:
    along query blocks (x nb / picks) and along heads by whole waves of one
    head per core (x ceil(BH / heads)).  Returns the rate and the sampled rows."""
    import numpy as np
    orc = _oracle()
    BH, N, d = w.B * w.H, w.N, w.d
    nb = (N + w.block - 1) // w.block
    qf, kf, vf = (t.reshape(BH, N, d)[:heads].contiguous() for t in (q, k, v))
    sel = np.zeros((heads, nb), np.uint8)
    sel[:, picks] = 1
    t0 = time.perf_counter()
    out, idx = orc.sagesla(qf, kf, vf, pw, w.block, w.topk, qsel=sel)
    t_sample = time.perf_counter() - t0
    t_q = max(0.0, t_sample - t_fixed) / len(picks)
    waves = math.ceil(BH / heads)
    full_s = waves * (t_fixed + nb * t_q)
    f = flops(w, orc.topk_count(nb, w.topk))
    return dict(value=f["dense"] / full_s / 1e12, unit="TFLOPS", cores=orc.threads(), kind="oracle",
                ms_per_call=full_s * 1e3, extrapolated=True,
                sample=(f"{heads} heads (one per host core) x {len(picks)} query blocks of {w.name} (fp64 C oracle, "
                        f"OpenMP over heads): fixed part {t_fixed:.2f} s, {t_q * 1e3:.1f} ms per query block; "
                        f"extrapolated to {nb} query blocks and to {BH} heads in {waves} waves"),
                sample_seconds=t_fixed + t_sample, out=out, idx=idx, heads=heads, picks=picks)


def cpu_baseline(w, q, k, v, pw, qblocks: int = 2) -> dict:
    orc = _oracle()
    heads, picks, _ = cpu_sample_plan(w, orc.threads(), qblocks)
    t_fixed = cpu_fixed_part(w, q, k, v, pw, heads)
    return cpu_sample(w, q, k, v, pw, heads, picks, t_fixed)


def _bf16_half_ulp(x):
    import numpy as np
    x = np.abs(np.asarray(x, np.float64))
    e = np.floor(np.log2(np.maximum(x, 2.0 ** -126)))
    return np.ldexp(1.0, (e - 8).astype(np.int64))


def parity(w, q, k, gpu_out, gpu_idx, cb, near_tie: float = 1e-5) -> dict:
    """Parity figures of the timed call: the block mask of every head against
    the oracle's (equal rows, and rows that differ only in near-ties of the
    k-th pooled score within `near_tie`); the sampled output rows against the
    oracle's quantised emulation (max-abs error beyond half a bf16 ulp, and
    cosine), on rows whose mask the two sides share."""
    import numpy as np
    orc = _oracle()
    BH, N, d = w.B * w.H, w.N, w.d
    nb = (N + w.block - 1) // w.block
    qf, kf = q.reshape(BH, N, d), k.reshape(BH, N, d)
    om = orc.mask(qf, kf, w.block, w.topk)["idx"]
    gi = gpu_idx.reshape(BH, nb, -1)
    eq_rows = (gi == om).all(axis=2)
    near = other = 0
    for h in np.nonzero(~eq_rows.all(axis=1))[0]:
        s64 = orc.block_scores_f64(qf[h:h + 1].contiguous(), kf[h:h + 1].contiguous(), w.block)[0]
        for i in np.nonzero(~eq_rows[h])[0]:
            kth = np.sort(s64[i])[::-1][gi.shape[2] - 1]
            diff = set(gi[h, i].tolist()) ^ set(om[h, i].tolist())
            if all(abs(s64[i, j] - kth) <= near_tie for j in diff):
                near += 1
            else:
                other += 1
    got, ref = [], []
    go = gpu_out.reshape(BH, N, d)
    for h in range(cb["heads"]):
        for i in cb["picks"]:
            if eq_rows[h, i]:
                r0, r1 = i * w.block, min(N, (i + 1) * w.block)
                got.append(go[h, r0:r1])
                ref.append(cb["out"][h, r0:r1])
    got = np.concatenate(got).astype(np.float64) if got else np.zeros((0, d))
    ref = np.concatenate(ref) if ref else np.zeros((0, d))
    err = float(np.max(np.abs(got - ref) - _bf16_half_ulp(ref))) if got.size else None
    cos = float((got * ref).sum() / np.sqrt((got * got).sum() * (ref * ref).sum())) if got.size else None
    return {"mask_rows": int(BH * nb), "mask_rows_equal": int(eq_rows.sum()), "mask_rows_near_tie": near,
            "mask_rows_other": other, "out_rows_compared": int(got.shape[0]), "max_abs_excess": err,
            "cosine": cos, "tolerance": {"max_abs_excess": 1e-2, "cosine": 0.9999, "near_tie": near_tie}}


def measure_8bit_peaks(n: int = 8192, reps: int = 10) -> dict:
    """Dense 8-bit library GEMM throughput on this GPU: torch._int_mm (INT8 x
    INT8 -> INT32) and torch._scaled_mm (E4M3 x E4M3 -> bf16), n^3, best of
    `reps`, CUDA events; 2 n^3 FLOP each."""
    import torch
    dev = torch.device("cuda")
    out = {}
    a8 = torch.randint(-127, 128, (n, n), dtype=torch.int8, device=dev)
    b8 = torch.randint(-127, 128, (n, n), dtype=torch.int8, device=dev)
    af = torch.randn(n, n, device=dev).to(torch.float8_e4m3fn)
    bf = torch.randn(n, n, device=dev).to(torch.float8_e4m3fn).t()
    one = torch.ones((), device=dev)

    def best(fn):
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        ts = []
        for _ in range(reps):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            fn()
            e1.record()
            torch.cuda.synchronize()
            ts.append(e0.elapsed_time(e1))
        return min(ts)
    for name, fn in (("int8", lambda: torch._int_mm(a8, b8.t().contiguous().t())),
                     ("e4m3", lambda: torch._scaled_mm(af, bf, scale_a=one, scale_b=one, out_dtype=torch.bfloat16))):
        try:
            ms = best(fn)
            out[name] = {"ms": ms, "tflops": 2.0 * n ** 3 / (ms * 1e-3) / 1e12}
        except Exception as e:  # report what failed, keep the other
            out[name] = {"error": str(e).splitlines()[0][:200]}
    return out


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
        nb = (w.N + w.block - 1) // w.block
        f = flops(w, sg.topk_count(nb, w.topk))
        fl_ms, fl_n = prof.get("flash", (0.0, 0))
        flash_ms = fl_ms / max(1, fl_n)
        achieved = f["computed"] / (flash_ms * 1e-3) / 1e12 if flash_ms > 0 else None
        t_roof = max(f["computed"] / (peak8 * 1e12), f["hbm_bytes"] / (pk["hbm"] * 1e9))
        line = {"workload": w.name, "B": w.B, "H": w.H, "N": w.N, "block": w.block, "topk": w.topk,
                "linear": w.linear, "k_blocks": f["kc"], "ms_per_call": ms,
                "dense_equiv_tflops": f["dense"] / (ms * 1e-3) / 1e12,
                "flash_ms": flash_ms, "flash_tflops": achieved,
                "flash_frac_of_8bit_peak": (achieved / peak8) if achieved else None,
                "flash_frac_of_nominal_8bit": (achieved / NOMINAL_8BIT_TFLOPS) if achieved else None,
                "path_frac_of_roofline": t_roof * 1e3 / ms, "device_status": sg.sync_status(),
                "kernels_ms": {kname: round(t / max(1, n), 4) for kname, (t, n) in prof.items()}}
        print(json.dumps(line), flush=True)
        del out
    return 0


def run_reference(args):
    """The oracle, as it stands, timed on the host cores on the same bounded
    sample as the GPU arm's cpu_baseline (one head per core x 2 query blocks),
    one sample per step; rank 0 only.  Loads only the oracle's library."""
    rank = _env_int("RANK", 0)
    if rank != 0:
        return 0
    from sparse_bit_attention_smoothing_b200.inputs import make_workload
    orc = _oracle()
    w = workloads()[args.workload]
    q, k, v, pw = make_workload(w)
    heads, picks, nb = cpu_sample_plan(w, orc.threads())
    t_fixed = cpu_fixed_part(w, q, k, v, pw, heads)
    vals = []
    for s in range(args.warmup + args.steps):
        cb = cpu_sample(w, q, k, v, pw, heads, picks, t_fixed)
        if s >= args.warmup:
            vals.append(cb)
    val = statistics.median([c["value"] for c in vals])
    ms = statistics.median([c["ms_per_call"] for c in vals])
    f = flops(w, orc.topk_count(nb, w.topk))
    line = {"impl": "reference", "metric": METRIC, "value": val, "unit": "TFLOPS", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "ms_per_step_extrapolated": True,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": w.name, "B": w.B, "H": w.H, "N": w.N, "d": w.d, "block": w.block,
                       "topk": w.topk, "k_blocks": f["kc"], "nb": nb, "linear": w.linear},
            "cpu_baseline": {"value": val, "unit": "TFLOPS", "cores": vals[0]["cores"], "kind": "oracle",
                             "sample": vals[0]["sample"], "extrapolated": True},
            "e2e": {"value": val, "unit": "TFLOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


W8A8_SHAPES = {  # tokens x in -> out: the Wan2.1-14B hidden size (5120) at the 720p token count
    "w8a8_wan14b_720p_qkvo": (75600, 5120, 5120),
    "w8a8_wan14b_720p_ffn_up": (75600, 5120, 13824),
}


def run_w8a8(args):
    """The W8A8 linear layer (x [M, K] quantised every call, W [N, K] quantised once):
    dense-equivalent TFLOPS = 2 M N K / t of one sagesla_w8a8_linear call."""
    import torch

    from sparse_bit_attention_smoothing_b200 import build as sbuild
    from sparse_bit_attention_smoothing_b200.replicas import job_throughput, max_over_ranks, rank_env
    rank, world, local = rank_env()
    torch.cuda.set_device(local)
    sbuild.build()
    import sparse_bit_attention_smoothing_b200 as sg
    M, K, N = W8A8_SHAPES[args.workload]
    g = torch.Generator().manual_seed(0)
    x = torch.randn(M, K, generator=g).bfloat16().cuda()
    w = (torch.randn(N, K, generator=g) * K ** -0.5).bfloat16().cuda()
    wq, sw = sg.sagesla_w8a8_quant(w)
    y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    st = torch.cuda.current_stream()
    for _ in range(max(3, args.warmup)):
        sg.sagesla_w8a8_linear(x, wq, sw, N, y=y, stream=st)
    torch.cuda.synchronize()
    sg.profile(True)
    sg.profile_read()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(st)
    for _ in range(args.steps):
        sg.sagesla_w8a8_linear(x, wq, sw, N, y=y, stream=st)
    e1.record(st)
    torch.cuda.synchronize()
    prof = sg.profile_read()
    sg.profile(False)
    ms = max_over_ranks([e0.elapsed_time(e1) / args.steps], device="cuda")[0]
    flops = 2.0 * M * N * K
    pk = peaks()
    peak8 = 2.0 * pk["bf16"]
    g_ms = prof["w8a8_gemm"][0] / max(1, prof["w8a8_gemm"][1])
    achieved = flops / (g_ms * 1e-3) / 1e12
    line = {"metric": "W8A8 linear dense TFLOPS (2MNK / t)", "value": job_throughput(flops, world, ms) / 1e12,
            "unit": "TFLOPS", "n_gpus": world, "steps": args.steps, "warmup": max(3, args.warmup),
            "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "i8 (int32 per 128-block, fp32 promotion, bf16 io)", "data": "synthetic",
            "config": {"workload": args.workload, "M": M, "K": K, "N": N, "block": 128,
                       "l2": "x 774 MB > 126 MB L2, no flush"},
            "kernels_ms": {kname: round(t / max(1, n), 4) for kname, (t, n) in prof.items()},
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak8, "unit": "TFLOP/s",
                         "frac": achieved / peak8, "kernel": "w8a8_gemm",
                         "frac_of_nominal_8bit": achieved / NOMINAL_8BIT_TFLOPS,
                         "peak_note": f"8-bit = 2 x {pk['src']} bf16 burst {pk['bf16']}"},
            "device_status": sg.sync_status()}
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def run_head_parallel(args):
    """One sagesla_attn call of the workload split over the ranks by head: each rank holds its token shard
    [B, H, N/P, d] of q, k, v, two all-to-alls (NCCL) regroup by head and back.  value = the whole call's
    dense-equivalent TFLOPS over the slowest rank's time (strong scaling)."""
    import datetime

    import torch
    import torch.distributed as dist

    from sparse_bit_attention_smoothing_b200 import build as sbuild
    from sparse_bit_attention_smoothing_b200.replicas import max_over_ranks, rank_env
    rank, world, local = rank_env()
    torch.cuda.set_device(local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=torch.device("cuda", local))
    sbuild.build()
    import sparse_bit_attention_smoothing_b200 as sg
    from sparse_bit_attention_smoothing_b200.headpar import sagesla_attn_head_parallel
    from sparse_bit_attention_smoothing_b200.inputs import make_workload
    w = workloads()[args.workload]
    q, k, v, pw = make_workload(w)
    if w.N % world or w.H % world:
        raise SystemExit(f"head-parallel run needs N ({w.N}) and H ({w.H}) divisible by {world}")
    Nl = w.N // world
    sl = slice(rank * Nl, (rank + 1) * Nl)
    ql, kl, vl = (t[:, :, sl].contiguous().cuda() for t in (q, k, v))
    dw = pw.cuda() if (w.linear and not args.no_linear) else None
    st = torch.cuda.current_stream()
    for _ in range(max(3, args.warmup)):
        sagesla_attn_head_parallel(ql, kl, vl, dw, block=w.block, topk=w.topk, stream=st)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(st)
    for _ in range(args.steps):
        out = sagesla_attn_head_parallel(ql, kl, vl, dw, block=w.block, topk=w.topk, stream=st)
    e1.record(st)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    ms = max_over_ranks([e0.elapsed_time(e1) / args.steps], device="cuda")[0]
    f = flops(w, sg.topk_count((w.N + w.block - 1) // w.block, w.topk))
    line = {"metric": METRIC + " (one call split by head over the ranks)", "value": f["dense"] / (ms * 1e-3) / 1e12,
            "unit": "TFLOPS", "n_gpus": world, "steps": args.steps, "warmup": max(3, args.warmup),
            "ms_per_step": ms, "higher_is_better": True, "scaling": "strong", "vs_baseline": None,
            "dtype": "i8/e4m3 (fp32 accumulate, bf16 io)", "data": "synthetic",
            "config": {"workload": w.name, "B": w.B, "H": w.H, "N": w.N, "d": w.d, "block": w.block, "topk": w.topk,
                       "linear": dw is not None, "parallelism": f"heads x{world} (all-to-all, NCCL)"},
            "device_status": sg.sync_status(), "out_shape": list(out.shape)}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
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
    ap.add_argument("--peaks", action="store_true", help="measure the 8-bit library GEMM peaks and exit")
    ap.add_argument("--parallel", default="replicas", choices=["replicas", "heads"],
                    help="replicas: one independent call per rank (weak scaling); heads: one call split over the "
                         "ranks by head with two all-to-alls (strong scaling)")
    args = ap.parse_args()
    if args.peaks:
        print(json.dumps({"n": 8192, "peaks": measure_8bit_peaks()}), flush=True)
        return 0
    if args.impl == "reference":
        return run_reference(args)
    if args.workload == "all":
        return run_all(args)
    if args.workload.startswith("w8a8"):
        return run_w8a8(args)
    if args.parallel == "heads":
        return run_head_parallel(args)

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

    f = flops(w, sg.topk_count((w.N + w.block - 1) // w.block, w.topk))
    value = job_throughput(f["dense"], world, ms) / 1e12
    pk = peaks()
    # the roofline peak: 8-bit dense = 2 x the measured bf16 burst (the
    # 60 % target is judged on this measured figure); the fraction of the
    # chip's nominal 8-bit dense peak (4.5 PFLOP/s) is reported beside it
    peak8 = 2.0 * pk["bf16"]
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
                         "frac_of_nominal_8bit": (achieved / NOMINAL_8BIT_TFLOPS) if achieved else None,
                         "nominal_8bit_peak": NOMINAL_8BIT_TFLOPS,
                         "path_t_roof_ms": t_roof * 1e3, "path_frac": t_roof * 1e3 / ms},
            "clocks": clocks,
            "e2e": {"value": job_throughput(f["dense"], world, e2e_ms) / 1e12, "unit": "TFLOPS", "ms_per_step": e2e_ms,
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": E}}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cb = cpu_baseline(w, q, k, v, pw)
        line["cpu_baseline"] = {kk: cb[kk] for kk in ("value", "unit", "cores", "kind", "sample", "ms_per_call",
                                                       "extrapolated")}
        gidx = sg.sagesla_get_mask(dq, dk, block=w.block, topk=w.topk, stream=st)["idx"]
        torch.cuda.synchronize()
        line["parity"] = parity(w, q, k, out.float().cpu().numpy(), gidx.cpu().numpy(), cb)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
