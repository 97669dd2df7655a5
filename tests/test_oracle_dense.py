"""Pins of the oracle's dense attention and of K-smoothing (CPU only).

Dense softmax attention is the textbook definition; it is pinned against a
brute-force Python loop and against torch's own scaled_dot_product_attention
in float64.  Smoothing (subtracting the per-channel mean of K) is pinned by
the invariance of softmax to a per-row constant shift of the scores
("异常值平滑", 量子位 news 技术解密 1).
"""
import math

import numpy as np
import torch


def brute_attention(q, k, v):
    BH, N, d = q.shape
    out = np.zeros_like(q)
    for b in range(BH):
        for r in range(N):
            s = [sum(q[b, r, c] * k[b, n, c] for c in range(d)) / math.sqrt(d) for n in range(N)]
            m = max(s)
            e = [math.exp(x - m) for x in s]
            tot = sum(e)
            for c in range(d):
                out[b, r, c] = sum(e[n] * v[b, n, c] for n in range(N)) / tot
    return out


def test_dense_vs_bruteforce(orc):
    rng = np.random.default_rng(1)
    q, k, v = (rng.standard_normal((2, 7, 5)) for _ in range(3))
    np.testing.assert_allclose(orc.dense_attn(q, k, v), brute_attention(q, k, v), rtol=0, atol=1e-13)


def test_dense_vs_torch_sdpa_fp64(orc):
    g = torch.Generator().manual_seed(2)
    q, k, v = (torch.randn(3, 100, 16, generator=g, dtype=torch.float64) * 2 for _ in range(3))
    ref = torch.nn.functional.scaled_dot_product_attention(q, k, v).numpy()
    np.testing.assert_allclose(orc.dense_attn(q.numpy(), k.numpy(), v.numpy()), ref, rtol=0, atol=1e-12)


def test_dense_bf16_entry_matches_fp64_entry(orc):
    g = torch.Generator().manual_seed(3)
    q, k, v = (torch.randn(2, 65, 32, generator=g).to(torch.bfloat16) for _ in range(3))
    a = orc.dense_attn_bf16(q, k, v)
    b = orc.dense_attn(q.double().numpy(), k.double().numpy(), v.double().numpy())
    assert np.array_equal(a, b)


def test_smoothing_invariance(orc):
    g = torch.Generator().manual_seed(4)
    q = torch.randn(2, 90, 32, generator=g, dtype=torch.float64)
    k = torch.randn(2, 90, 32, generator=g, dtype=torch.float64) + 3 * torch.randn(2, 1, 32, generator=g, dtype=torch.float64)
    v = torch.randn(2, 90, 32, generator=g, dtype=torch.float64)
    mu = k.mean(dim=1, keepdim=True)
    a = orc.dense_attn(q.numpy(), k.numpy(), v.numpy())
    b = orc.dense_attn(q.numpy(), (k - mu).numpy(), v.numpy())
    np.testing.assert_allclose(a, b, rtol=0, atol=1e-12)
    # a non-constant shift must change the result (the pin is not vacuous)
    c = orc.dense_attn(q.numpy(), (k - mu * torch.arange(90, dtype=torch.float64).view(1, 90, 1) / 30).numpy(), v.numpy())
    assert np.abs(a - c).max() > 1e-3
