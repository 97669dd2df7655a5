"""Pins of the oracle's block mask (CPU only).

Reading: key blocks are ranked, per query block, by the mean-pooled block
score qbar_i . kbar_j / sqrt(d) (kbar from the smoothed keys); the k largest
are kept, ties going to the lower block index, listed in ascending order;
k = clamp(ceil(topk * Nb), 1, Nb) (sla_topk 0.05/0.1/0.15, 揭秘TurboDiffusion
教程 and "TurboDiffusion跨模态" 2.2 SLA).  Pins: the pooled means against
numpy's mean, the selection against a brute-force sort, constructed exact
ties, topk = 1, and invariance of the ranking to the smoothing shift.
"""
import numpy as np
import pytest
import torch


@pytest.mark.parametrize("nb,topk,expect", [
    (16, 0.25, 4), (512, 0.1, 52), (1182, 0.1, 119), (1182, 0.05, 60), (1182, 0.15, 178),
    (591, 0.05, 30), (591, 0.1, 60), (591, 0.15, 89), (1182, 1.0, 1182), (7, 0.01, 1), (10, 0.3, 3)])
def test_topk_count(orc, nb, topk, expect):
    assert orc.topk_count(nb, topk) == expect


def _rand(seed, BH, N, d, kbias=2.0):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(BH, N, d, generator=g).bfloat16()
    k = (torch.randn(BH, N, d, generator=g) + kbias * torch.randn(BH, 1, d, generator=g)).bfloat16()
    return q, k


@pytest.mark.parametrize("N,block", [(640, 64), (600, 64), (1000, 128), (130, 64)])
def test_pooled_means_vs_numpy(orc, N, block):
    q, k = _rand(5, 2, N, 32)
    r = orc.mask(q, k, block, 0.3)
    qf = q.float().numpy().astype(np.float64)
    kf = k.float().numpy().astype(np.float64)
    ks = kf - kf.mean(axis=1, keepdims=True)
    nb = (N + block - 1) // block
    for i in range(nb):
        sl = slice(i * block, min((i + 1) * block, N))
        np.testing.assert_allclose(r["qbar"][:, i], qf[:, sl].mean(axis=1), rtol=0, atol=2e-6)
        np.testing.assert_allclose(r["kbar"][:, i], ks[:, sl].mean(axis=1), rtol=0, atol=2e-5)


@pytest.mark.parametrize("N,block,topk", [(640, 64, 0.3), (1000, 128, 0.5), (4000, 64, 0.1)])
def test_mask_vs_bruteforce_sort(orc, N, block, topk):
    q, k = _rand(6, 2, N, 64)
    r = orc.mask(q, k, block, topk, want_scores=True)
    s = r["scores"]
    f64 = orc.block_scores_f64(q, k, block)
    assert np.abs(s - f64).max() < 1e-6          # fp32 scores follow the fp64 definition
    BH, nb, _ = s.shape
    for b in range(BH):
        for i in range(nb):
            order = sorted(range(nb), key=lambda j: (-float(s[b, i, j]), j))
            assert list(r["idx"][b, i]) == sorted(order[: r["k"]])


def test_mask_constructed_ties(orc):
    # 8 key blocks of 64 tokens, d = 16; blocks 2 and 6 are identical, so every
    # query block scores them equally; k = 3 with the tie at the boundary.
    d, block = 16, 64
    g = torch.Generator().manual_seed(7)
    base = torch.randn(8, 1, d, generator=g)
    k = base.repeat(1, block, 1)
    k = k + 0.0 * torch.randn(8, block, d, generator=g)
    k[6] = k[2]
    k = k.reshape(1, 8 * block, d)
    q = torch.randn(1, 8 * block, d, generator=g)
    qb, kb = q.bfloat16(), k.bfloat16()
    r = orc.mask(qb, kb, block, 3 / 8, want_scores=True)
    s = r["scores"][0]
    assert np.all(s[:, 2] == s[:, 6])
    for i in range(8):
        order = sorted(range(8), key=lambda j: (-float(s[i, j]), j))
        sel = set(r["idx"][0, i])
        assert sel == set(order[:3])
        if 6 in sel:
            assert 2 in sel            # never the higher index of a tie without the lower one
    # force the tie onto the boundary: query equal to block 2's key direction
    q2 = kb.reshape(8, block, d)[[2]].repeat(8, 1, 1).reshape(1, 8 * block, d).float()
    r2 = orc.mask(q2.bfloat16(), kb, block, 1 / 8, want_scores=True)
    assert np.all(r2["idx"][0, :, 0] == 2)


def test_mask_topk_one_selects_all(orc):
    q, k = _rand(8, 1, 700, 32)
    r = orc.mask(q, k, 64, 1.0)
    assert np.array_equal(r["idx"][0], np.tile(np.arange(11, dtype=np.int32), (11, 1)))


def test_mask_smoothing_invariance(orc):
    # Ranking with smoothed keys == ranking with the raw keys (a per-row shift),
    # except where two scores are within 1e-5 (near-ties), which are counted.
    q, k = _rand(9, 2, 3200, 64, kbias=3.0)
    block, topk = 64, 0.2
    r = orc.mask(q, k, block, topk)
    qf = q.double().numpy()
    kf = k.double().numpy()
    BH, N, d = qf.shape
    nb = N // block
    qb = qf.reshape(BH, nb, block, d).mean(2)
    kb = kf.reshape(BH, nb, block, d).mean(2)
    raw = np.einsum("bid,bjd->bij", qb, kb) / np.sqrt(d)
    kc = r["k"]
    near = 0
    for b in range(BH):
        for i in range(nb):
            order = sorted(range(nb), key=lambda j: (-raw[b, i, j], j))
            ref = set(order[:kc])
            got = set(r["idx"][b, i])
            if ref != got:
                kth = raw[b, i, order[kc - 1]]
                assert all(abs(raw[b, i, j] - kth) <= 1e-5 for j in ref ^ got)
                near += 1
    assert near <= 2
