"""GPU parity on the edge cases of the path (through the C ABI):

 - exact ties in the block mask: duplicated key blocks give bit-identical
   pooled scores, and the GPU must keep the lower block index exactly as the
   oracle does (no near-tie allowance);
 - a sequence long enough (Nb = 6250 key blocks at block 64) that the top-k
   kernel runs its four-query-rows variant, mask compared in full;
 - quantisation with an all-zero query block, an all-zero smoothed key block
   and all-zero channels (scale 1, codes 0), codes and scales bit-exact, and
   the whole call on that input against the emulation.
"""
import numpy as np
import pytest
import torch

from tests._util import MAX_ABS, MIN_COS, compare_masks, cosine, max_abs_excess

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sg():
    from sparse_bit_attention_smoothing_b200 import build
    build.build()
    import sparse_bit_attention_smoothing_b200 as s
    assert torch.cuda.is_available()
    return s


@pytest.mark.parametrize("block,topk", [(64, 0.3), (64, 0.4), (128, 0.3)])  # odd k: a tied pair is always cut
def test_mask_exact_ties_lower_index(sg, orc, block, topk):
    from sparse_bit_attention_smoothing_b200.inputs import make_inputs
    N = 16 * block
    q, k, _, _ = make_inputs(1, 2, N, 128, seed=11, outliers=True)
    # key blocks 8..15 repeat blocks 0..7 row for row: their smoothed means,
    # hence their pooled scores, are bit-identical in pairs (j, j + 8)
    k = k.clone()
    k[:, :, 8 * block:] = k[:, :, :8 * block]
    r = sg.sagesla_get_mask(q.cuda(), k.cuda(), block=block, topk=topk)
    torch.cuda.synchronize()
    o = orc.mask(q.reshape(2, N, 128), k.reshape(2, N, 128), block, topk, want_scores=True)
    sc = o["scores"]
    assert np.array_equal(sc[..., :8], sc[..., 8:])  # the construction ties every pair exactly
    gi = r["idx"].cpu().numpy().reshape(o["idx"].shape)
    assert np.array_equal(gi, o["idx"])
    # ties decided the selection somewhere: a pair split by the cut keeps its lower index
    kept = np.zeros(sc.shape, bool)
    np.put_along_axis(kept, o["idx"], True, axis=2)
    assert np.any(kept[..., :8] & ~kept[..., 8:])


def test_mask_four_row_variant_long_sequence(sg, orc):
    """Nb = 6250 (N = 400000 at block 64): above about 5800 key blocks the
    top-k kernel keeps four query rows per CTA instead of eight."""
    from sparse_bit_attention_smoothing_b200.inputs import make_inputs
    N, block, topk = 400000, 64, 0.05
    q, k, _, _ = make_inputs(1, 1, N, 128, seed=4, outliers=True)
    r = sg.sagesla_get_mask(q.cuda(), k.cuda(), block=block, topk=topk)
    torch.cuda.synchronize()
    qh, kh = q.reshape(1, N, 128), k.reshape(1, N, 128)
    o = orc.mask(qh, kh, block, topk)
    nb = o["idx"].shape[1]
    assert nb == 6250 and r["k"] == o["k"]
    s64 = orc.block_scores_f64(qh, kh, block)
    eq, near = compare_masks(r["idx"].cpu().numpy().reshape(nb, -1), o["idx"].reshape(nb, -1),
                             s64.reshape(nb, nb), o["k"])
    print(f"Nb={nb}: {eq} rows equal, {near} near-tie rows")
    assert eq + near == nb


def _zero_case():
    """B=1, H=2, N=326 (five 64-token blocks + a 6-token tail), d=128.
    Head 0: query block 1 all zero and query channel 7 all zero; keys =
    per-channel bias + a +-0.25 pattern whose mean over the sequence is 0
    and which is 0 on key block 2, so the smoothed keys of block 2 are
    exactly 0; value channel 3 all zero.  Head 1: seeded random."""
    from sparse_bit_attention_smoothing_b200.inputs import make_inputs
    N = 326
    q, k, v, w = make_inputs(1, 2, N, 128, seed=9, outliers=True)
    q, k, v = q.clone(), k.clone(), v.clone()
    g = torch.Generator().manual_seed(9)
    q[0, 0, 64:128] = 0
    q[0, 0, :, 7] = 0
    kb = torch.randint(-8, 9, (128,), generator=g).float() * 0.25
    pat = torch.zeros(N, 128)
    rows = [n for n in range(N) if not 128 <= n < 192]
    assert len(rows) % 2 == 0
    pat[rows[0::2]] = 0.25
    pat[rows[1::2]] = -0.25
    k[0, 0] = (kb + pat).bfloat16()
    v[0, 0, :, 3] = 0
    return q, k, v, w, N


def test_quant_zero_block_and_channels_bit_exact(sg, orc):
    q, k, v, _, N = _zero_case()
    r = sg.sagesla_get_quant(q.cuda(), k.cuda(), v.cuda())
    torch.cuda.synchronize()
    o = orc.quant(q.reshape(2, N, 128), k.reshape(2, N, 128), v.reshape(2, N, 128))
    g = {kk: vv.cpu().numpy().reshape((2,) + tuple(vv.shape[2:])) for kk, vv in r.items()}
    for name in ("mu", "sq", "sk", "sv", "q8", "k8", "v8"):
        assert np.array_equal(g[name], o[name]), name
    # the constructed zeros: scale 1, codes 0
    assert g["sq"][0, 1] == 1.0 and np.all(g["q8"][0, 64:128] == 0) and np.all(g["q8"][0, :, 7] == 0)
    assert g["sk"][0, 2] == 1.0 and np.all(g["k8"][0, 128:192] == 0)
    assert g["sv"][0, 3] == 1.0 and np.all(g["v8"][0, :, 3] == 0)


@pytest.mark.parametrize("block,topk", [(64, 0.4), (128, 0.5)])
def test_full_call_on_zero_case(sg, orc, block, topk):
    q, k, v, w, N = _zero_case()
    dq, dk, dv, dw = q.cuda(), k.cuda(), v.cuda(), w.cuda()
    out = sg.sagesla_attn(dq, dk, dv, dw, block=block, topk=topk)
    m = sg.sagesla_get_mask(dq, dk, block=block, topk=topk)
    torch.cuda.synchronize()
    assert sg.sync_status() == 0
    nb = (N + block - 1) // block
    emu, _ = orc.sagesla(q.reshape(2, N, 128), k.reshape(2, N, 128), v.reshape(2, N, 128), w, block, topk,
                         idx=m["idx"].cpu().numpy().reshape(2, nb, -1))
    got = out.float().cpu().numpy().reshape(2, N, 128).astype(np.float64)
    err, cos = max_abs_excess(got, emu), cosine(got, emu)
    assert err <= MAX_ABS and cos >= MIN_COS, (err, cos)
