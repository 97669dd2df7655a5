"""Seeded synthetic inputs shaped like the Wan2.1 video-DiT attention calls.

This module holds random-number generation only, none of the method's
arithmetic; both the CUDA path and the CPU oracle consume what it returns.

Recipe (one CPU torch.Generator seeded with `seed`, drawn in this order):
  1. Q, K, V ~ N(0, 1), each [B, H, N, d] in fp32;
  2. K bias ~ N(0, 2) (variance 2), one per (b, h, channel), added to every token;
  3. outlier channels (only when `outliers`): for each of Q, K, V and each
     (b, h), ceil(0.01 * d) channels picked by randperm are scaled x10
     (before the bias is added to K);
  4. proj_w ~ N(0, 1/d), [d, d];
then every tensor is rounded to bf16 (round to nearest even).
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    N: int
    d: int
    block: int
    topk: float
    outliers: bool
    linear: bool = True  # False: linear branch off (proj_w = NULL)


# Token counts are latent grids: 4x16x16 = 1024, 21x30x52 = 32760, 21x45x80 = 75600.
TINY = Workload("tiny_h2_n1024", 1, 2, 1024, 128, 64, 0.25, False)
WAN13_480P = Workload("wan2.1-1.3b-480p_h12_n32760", 1, 12, 32760, 128, 64, 0.1, True)
WAN14_480P = Workload("wan2.1-14b-480p_h40_n32760", 1, 40, 32760, 128, 64, 0.1, True)
WAN14_720P = Workload("wan2.1-14b-720p_h40_n75600", 1, 40, 75600, 128, 64, 0.1, True)
WAN14_720P_K05 = Workload("wan2.1-14b-720p_h40_n75600_topk0.05", 1, 40, 75600, 128, 64, 0.05, True)


def sweep():
    """The sparsity sweep at H=40, N=75600 (same tensors as the 720p workload)."""
    out = []
    for block in (64, 128):
        for topk in (0.05, 0.1, 0.15):
            out.append(Workload(f"sweep_b{block}_topk{topk}", 1, 40, 75600, 128, block, topk, True))
        out.append(Workload(f"sweep_b{block}_dense", 1, 40, 75600, 128, block, 1.0, True, False))
    return out


def make_inputs(B: int, H: int, N: int, d: int, seed: int = 0, outliers: bool = True):
    """Return (q, k, v, proj_w) as contiguous CPU bf16 tensors."""
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    shape = (B, H, N, d)
    q = torch.randn(shape, generator=g, dtype=torch.float32)
    k = torch.randn(shape, generator=g, dtype=torch.float32)
    v = torch.randn(shape, generator=g, dtype=torch.float32)
    kbias = torch.randn((B, H, 1, d), generator=g, dtype=torch.float32) * math.sqrt(2.0)
    if outliers:
        n_out = max(1, math.ceil(0.01 * d))
        for t in (q, k, v):
            for b in range(B):
                for h in range(H):
                    ch = torch.randperm(d, generator=g)[:n_out]
                    t[b, h, :, ch] *= 10.0
    k += kbias
    w = torch.randn((d, d), generator=g, dtype=torch.float32) / math.sqrt(d)
    return (q.to(torch.bfloat16).contiguous(), k.to(torch.bfloat16).contiguous(),
            v.to(torch.bfloat16).contiguous(), w.to(torch.bfloat16).contiguous())


def make_workload(w: Workload, seed: int = 0):
    q, k, v, pw = make_inputs(w.B, w.H, w.N, w.d, seed=seed, outliers=w.outliers)
    return q, k, v, (pw if w.linear else None)
