"""Parity at the full size the benchmark times (Wan2.1-14B-720P attention: B=1,
H=40, N=75600, d=128, block 64, topk 0.1, linear branch on), in the same launch
configuration as bench.py, on sampled outputs: two heads, and in each the
first, a middle and the ragged last query block (16 of 64 rows valid), which
the oracle computes one by one.  The masks of the sampled heads are checked
whole."""
import numpy as np
import pytest
import torch

from tests._util import MAX_ABS, MIN_COS, compare_masks, cosine, max_abs_excess

pytestmark = pytest.mark.gpu

HEADS = (0, 37)


@pytest.fixture(scope="module")
def full_run():
    from sparse_bit_attention_smoothing_b200 import build
    build.build()
    import sparse_bit_attention_smoothing_b200 as sg
    from sparse_bit_attention_smoothing_b200.inputs import WAN14_720P, make_workload
    w = WAN14_720P
    q, k, v, pw = make_workload(w)
    dq, dk, dv, dw = q.cuda(), k.cuda(), v.cuda(), pw.cuda()
    out = sg.sagesla_attn(dq, dk, dv, dw, block=w.block, topk=w.topk)
    m = sg.sagesla_get_mask(dq, dk, block=w.block, topk=w.topk)
    torch.cuda.synchronize()
    assert sg.sync_status() == 0
    res = dict(w=w, q=q, k=k, v=v, pw=pw, out=out.cpu(), idx=m["idx"].cpu().numpy(), k_blocks=m["k"])
    del dq, dk, dv, dw, out
    torch.cuda.empty_cache()
    return res


def _head(t, h, N):
    return t.reshape(-1, N, 128)[h:h + 1]


@pytest.mark.parametrize("h", HEADS)
def test_full_size_mask_of_sampled_heads(orc, full_run, h):
    w, N = full_run["w"], full_run["w"].N
    qh, kh = _head(full_run["q"], h, N), _head(full_run["k"], h, N)
    o = orc.mask(qh, kh, w.block, w.topk)
    nb = o["idx"].shape[1]
    assert full_run["k_blocks"] == o["k"]
    gi = full_run["idx"].reshape(-1, nb, o["k"])[h]
    s64 = orc.block_scores_f64(qh, kh, w.block)
    eq, near = compare_masks(gi, o["idx"].reshape(nb, -1), s64.reshape(nb, nb), o["k"])
    assert eq + near == nb


@pytest.mark.parametrize("h", HEADS)
def test_full_size_sampled_query_blocks(orc, full_run, h):
    w, N = full_run["w"], full_run["w"].N
    nb = (N + w.block - 1) // w.block
    blocks = [0, nb // 2, nb - 1]
    qsel = np.zeros((1, nb), np.uint8)
    qsel[0, blocks] = 1
    idx = full_run["idx"].reshape(-1, nb, full_run["k_blocks"])[h:h + 1]
    emu, _ = orc.sagesla(_head(full_run["q"], h, N), _head(full_run["k"], h, N), _head(full_run["v"], h, N),
                         full_run["pw"], w.block, w.topk, idx=idx, qsel=qsel)
    got = full_run["out"].reshape(-1, N, 128)[h].float().numpy().astype(np.float64)
    for i in blocks:
        rows = slice(i * w.block, min(N, (i + 1) * w.block))
        g, r = got[rows], emu[0, rows]
        assert np.isfinite(r).all()
        err, cos = max_abs_excess(g, r), cosine(g, r)
        assert err <= MAX_ABS and cos >= MIN_COS, (h, i, err, cos)
