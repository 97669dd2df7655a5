"""Pins of the oracle's quantised SageSLA emulation (CPU only).

 - quantisation off, topk = 1, linear off  ==  dense fp64 attention (1e-12);
 - quantised, topk = 1, linear off: cosine >= 0.999 against dense fp64;
 - closed forms: identical keys (uniform scores), identical values, the
   two-key worked example of tests/golden/worked_two_keys.json;
 - the linear branch against its per-token definition, phi against torch's
   elu + 1, and the projection's orientation (y = O_l W^T) on constant V.
Sources: 揭秘TurboDiffusion 支柱一/支柱二; TurboDiffusion跨模态 2.2 SLA.
"""
import json
import os

import numpy as np
import pytest
import torch

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _cos(a, b):
    a = a.ravel()
    b = b.ravel()
    return float(a @ b / np.sqrt((a @ a) * (b @ b)))


def _rand(seed, BH, N, d, kbias=2.0):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(BH, N, d, generator=g).bfloat16()
    k = (torch.randn(BH, N, d, generator=g) + kbias * torch.randn(BH, 1, d, generator=g)).bfloat16()
    v = torch.randn(BH, N, d, generator=g).bfloat16()
    w = (torch.randn(d, d, generator=g) / np.sqrt(d)).bfloat16()
    return q, k, v, w


@pytest.mark.parametrize("N,block", [(200, 64), (256, 128), (64, 64), (37, 64)])
def test_noquant_full_equals_dense(orc, N, block):
    q, k, v, _ = _rand(10, 2, N, 32)
    out, idx = orc.sagesla(q, k, v, None, block, 1.0, flags=orc.NOQUANT)
    ref = orc.dense_attn_bf16(q, k, v)
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)


def test_quantised_full_vs_dense_cosine(orc):
    q, k, v, _ = _rand(11, 2, 1024, 128)
    out, _ = orc.sagesla(q, k, v, None, 64, 1.0)
    ref = orc.dense_attn_bf16(q, k, v)
    assert _cos(out, ref) >= 0.999


def test_quantisation_changes_result(orc):
    q, k, v, _ = _rand(12, 1, 256, 64)
    a, _ = orc.sagesla(q, k, v, None, 64, 1.0)
    b, _ = orc.sagesla(q, k, v, None, 64, 1.0, flags=orc.NOQUANT)
    assert 1e-6 < np.abs(a - b).max() < 5e-2


@pytest.mark.parametrize("N,block,topk", [(200, 64, 0.5), (300, 128, 0.4)])
def test_identical_keys_give_mean_of_selected_values(orc, N, block, topk):
    # all keys equal -> every score in a row equal -> P = 1 -> P~ = 448 for every
    # selected valid key: O_s = mean of the dequantised V over those keys.
    q, _, v, _ = _rand(13, 1, N, 32)
    k = torch.randn(1, 1, 32).repeat(1, N, 1).bfloat16()
    out, idx = orc.sagesla(q, k, v, None, block, topk)
    qz = orc.quant(q, k, v)
    vd = orc.e4m3_decode(qz["v8"][0]) * qz["sv"][0][None, :]
    nb = (N + block - 1) // block
    for i in range(nb):
        keys = [n for j in idx[0, i] for n in range(j * block, min((j + 1) * block, N))]
        expect = vd[keys].mean(axis=0)
        for r in range(i * block, min((i + 1) * block, N)):
            np.testing.assert_allclose(out[0, r], expect, rtol=0, atol=1e-12)


def test_identical_values_pass_through(orc):
    N, d = 150, 32
    q, k, _, _ = _rand(14, 1, N, d)
    c = torch.randn(d).bfloat16()
    v = c.view(1, 1, d).repeat(1, N, 1)
    out, _ = orc.sagesla(q, k, v, None, 64, 0.5)
    qz = orc.quant(q, k, v)
    vd = orc.e4m3_decode(qz["v8"][0, 0]) * qz["sv"][0]
    np.testing.assert_allclose(out[0], np.broadcast_to(vd, (N, d)), rtol=0, atol=1e-12)
    np.testing.assert_allclose(vd, c.double().numpy(), rtol=2e-7, atol=0)


def test_worked_two_keys(orc):
    with open(os.path.join(GOLDEN, "worked_two_keys.json")) as f:
        g = json.load(f)
    d = g["d"]
    q = torch.zeros(1, 2, d)
    k = torch.zeros(1, 2, d)
    v = torch.zeros(1, 2, d)
    for (r, c, x) in g["q"]:
        q[0, r, c] = x
    for (r, c, x) in g["k"]:
        k[0, r, c] = x
    for (r, c, x) in g["v"]:
        v[0, r, c] = x
    out, idx = orc.sagesla(q.bfloat16(), k.bfloat16(), v.bfloat16(), None, 64, 1.0)
    for (r, c, num, den) in g["expect"]:
        assert abs(out[0, r, c] - num / den) < 1e-12, (r, c, out[0, r, c], num / den)


def test_phi_matches_torch_elu(orc):
    xs = np.linspace(-30, 30, 2001)
    ref = (torch.nn.functional.elu(torch.from_numpy(xs)) + 1).numpy()
    mine = np.array([orc.phi(x) for x in xs])
    # torch forms elu(x)+1 as expm1(x)+1, which cancels for x << 0: compare absolutely
    np.testing.assert_allclose(mine, ref, rtol=1e-14, atol=1e-15)
    assert all(orc.phi(x) > 0 for x in (-700.0, -50.0, 0.0))


def _linear_part(orc, q, k, v, block, topk, idx=None):
    """O_l (before the projection): out(W = I) - out(no linear branch)."""
    d = q.shape[-1]
    eye = torch.eye(d).bfloat16()
    a, idx_a = orc.sagesla(q, k, v, eye, block, topk, idx=idx)
    b, _ = orc.sagesla(q, k, v, None, block, topk, idx=idx_a)
    return a - b, idx_a


@pytest.mark.parametrize("N,block,topk", [(200, 64, 0.25), (384, 128, 0.34), (640, 64, 0.1)])
def test_linear_branch_vs_per_token_definition(orc, N, block, topk):
    q, k, v, _ = _rand(15, 1, N, 16)
    lin, idx = _linear_part(orc, q, k, v, block, topk)
    ref = orc.linear_direct(q[0].double().numpy(), k[0].double().numpy(), v[0].double().numpy(), block, idx[0])
    np.testing.assert_allclose(lin[0], ref, rtol=0, atol=1e-12)
    assert np.abs(ref).max() > 1e-3


def test_linear_branch_closed_forms(orc):
    N, d, block = 256, 16, 64
    q, _, v, w = _rand(16, 1, N, d)
    # identical keys -> uniform linear weights -> O_l = mean of v over the unselected keys
    k = torch.randn(1, 1, d).repeat(1, N, 1).bfloat16()
    lin, idx = _linear_part(orc, q, k, v, block, 0.5)
    vf = v[0].double().numpy()
    for i in range(N // block):
        un = [j for j in range(N // block) if j not in set(idx[0, i])]
        expect = vf[np.concatenate([np.arange(j * block, (j + 1) * block) for j in un])].mean(0)
        for r in range(i * block, (i + 1) * block):
            np.testing.assert_allclose(lin[0, r], expect, rtol=0, atol=1e-12)
    # topk = 1 -> no unselected block -> the linear branch contributes 0
    lin1, _ = _linear_part(orc, q, k, v, block, 1.0)
    assert np.all(lin1 == 0)
    # constant V -> O_l = c -> y = O_l W^T = W c (non-symmetric W pins the orientation)
    _, kk, _, _ = _rand(17, 1, N, d)
    c = torch.randn(d).bfloat16()
    vc = c.view(1, 1, d).repeat(1, N, 1)
    a, idx2 = orc.sagesla(q, kk, vc, w, block, 0.25)
    b, _ = orc.sagesla(q, kk, vc, None, block, 0.25, idx=idx2)
    wd = w.double().numpy()
    assert np.abs(wd - wd.T).max() > 0.1
    y = wd @ c.double().numpy()
    np.testing.assert_allclose(a[0] - b[0], np.broadcast_to(y, (N, d)), rtol=0, atol=1e-12)


def test_external_mask_and_query_selection(orc):
    q, k, v, w = _rand(18, 2, 320, 32)
    out, idx = orc.sagesla(q, k, v, w, 64, 0.4)
    # same mask passed back in -> identical result
    out2, idx2 = orc.sagesla(q, k, v, w, 64, 0.4, idx=idx)
    assert np.array_equal(idx, idx2) and np.array_equal(out, out2)
    # only query block 2 of head 1
    sel = np.zeros((2, 5), np.uint8)
    sel[1, 2] = 1
    out3, _ = orc.sagesla(q, k, v, w, 64, 0.4, qsel=sel)
    assert np.array_equal(out3[1, 128:192], out[1, 128:192])
    assert np.all(np.isnan(out3[0])) and np.all(np.isnan(out3[1, :128]))
    # a different mask changes the result
    idx_alt = idx.copy()
    idx_alt[0, 0] = [0, 3]
    if not np.array_equal(idx_alt, idx):
        out4, _ = orc.sagesla(q, k, v, w, 64, 0.4, idx=idx_alt)
        assert np.abs(out4[0, :64] - out[0, :64]).max() > 1e-4


@pytest.mark.parametrize("block,flags", [(64, 0), (128, 0), (64, 2), (128, 2)])
def test_worked_walk(orc, block, flags):
    """The walk updates the running max after every selected key block (hand-derived, golden file)."""
    with open(os.path.join(GOLDEN, "worked_walk_tiles.json")) as f:
        g = json.load(f)
    N, d = g["N"], g["d"]
    q = torch.zeros(1, N, d)
    q[0, :, 0] = g["a"]
    k = torch.zeros(1, N, d)
    k[0, 64:, 0] = 2 * g["delta"]
    v = torch.zeros(1, N, d)
    v[0, :64, :2] = torch.tensor(g["v_block0"])
    v[0, 64:, :2] = torch.tensor(g["v_block1"])
    assert flags in (0, orc.ALT_WALK128)
    out, _ = orc.sagesla(q.bfloat16(), k.bfloat16(), v.bfloat16(), None, block, 1.0, flags=flags)
    if block == 64 and flags == 0:
        # the key scale is fl32(delta/127) (scales are fp32), so c is taken with it
        c = 127 * 127 * float(np.float32(g["delta"] / 127)) / (128 * np.sqrt(d))
        assert abs(c - g["c"]) < 1e-7
        alpha = np.exp(-2 * c)
        v0, v1 = g["v_block0"], g["v_block1"]
        for ch in range(2):
            np.testing.assert_allclose(out[0, :, ch], (alpha * v0[ch] + v1[ch]) / (alpha + 1), rtol=0, atol=1e-12)
        np.testing.assert_allclose(out[0, :, 0], -0.695986, rtol=0, atol=1e-6)
        assert np.all(out[0, :, 2:] == 0)
    else:
        for (c, num, den) in g["expect_128_keys"]:
            np.testing.assert_allclose(out[0, :, c], num / den, rtol=0, atol=1e-12)
