"""GPU parity of the SageAttention2++ quantisation options (sagesla_attn_opts)
against the oracle run with the same options on the GPU's own mask: one Q
scale per token and/or 4-bit Q/K codes (量子位 news, 技术解密 1).  The
default options reproduce sagesla_attn bit for bit."""
import numpy as np
import pytest
import torch

from tests._util import MAX_ABS, MIN_COS, cosine, max_abs_excess

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sg():
    from sparse_bit_attention_smoothing_b200 import build
    build.build()
    import sparse_bit_attention_smoothing_b200 as s
    assert torch.cuda.is_available()
    return s


def _case(seed, N=1000, H=2):
    from sparse_bit_attention_smoothing_b200.inputs import make_inputs
    q, k, v, w = make_inputs(1, H, N, 128, seed=seed, outliers=True)
    g = torch.Generator().manual_seed(seed)
    # token magnitudes over about two decades, so per-token scales matter
    q = (q.float() * torch.exp(torch.randn(1, H, N, 1, generator=g))).bfloat16()
    return q, k, v, w


def test_default_options_are_sagesla_attn(sg):
    q, k, v, w = _case(1)
    dq, dk, dv, dw = q.cuda(), k.cuda(), v.cuda(), w.cuda()
    a = sg.sagesla_attn(dq, dk, dv, dw, block=64, topk=0.25)
    b = sg.sagesla_attn_opts(dq, dk, dv, dw, block=64, topk=0.25, qk_bits=8, q_per_token=False)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


@pytest.mark.parametrize("bits,per_token", [(8, True), (4, False), (4, True)])
@pytest.mark.parametrize("block,topk,linear", [(64, 0.25, True), (64, 1.0, False), (128, 0.3, True)])
def test_options_vs_oracle(sg, orc, bits, per_token, block, topk, linear):
    q, k, v, w = _case(2 + bits + block)
    H, N = q.shape[1], q.shape[2]
    dq, dk, dv = q.cuda(), k.cuda(), v.cuda()
    dw = w.cuda() if linear else None
    out = sg.sagesla_attn_opts(dq, dk, dv, dw, block=block, topk=topk, qk_bits=bits, q_per_token=per_token)
    m = sg.sagesla_get_mask(dq, dk, block=block, topk=topk)
    torch.cuda.synchronize()
    assert sg.sync_status() == 0
    nb = (N + block - 1) // block
    flags = (orc.QK_INT4 if bits == 4 else 0) | (orc.Q_PER_TOKEN if per_token else 0)
    emu, _ = orc.sagesla(q.reshape(H, N, 128), k.reshape(H, N, 128), v.reshape(H, N, 128), w if linear else None,
                         block, topk, idx=m["idx"].cpu().numpy().reshape(H, nb, -1), flags=flags)
    got = out.float().cpu().numpy().reshape(H, N, 128).astype(np.float64)
    err, cos = max_abs_excess(got, emu), cosine(got, emu)
    print(f"bits={bits} per_token={per_token} block={block} topk={topk}: max-abs excess {err:.2e}, cosine {cos:.7f}")
    assert err <= MAX_ABS and cos >= MIN_COS, (err, cos)
