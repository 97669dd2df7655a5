"""GPU: q, k, v in the token-major layout [B, N, H, d] (sagesla_attn_bnhd).

The kernels that load q, k, v rows (statistics, quantiser, QK-norm sums,
linear branch) and the ones that write out (linear output, flash epilogue)
address the rows of the token-major layout in place; every other kernel works
on the tiled workspace.  The arithmetic of each row is the same, so the call
must equal sagesla_attn (or sagesla_attn_qknorm) on the tensors permuted to
[B, H, N, d], bit for bit."""
import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sg():
    from sparse_bit_attention_smoothing_b200 import build
    build.build()
    import sparse_bit_attention_smoothing_b200 as s
    assert torch.cuda.is_available()
    return s


def _tok(x):
    return x.permute(0, 2, 1, 3).contiguous()  # [B, H, N, d] <-> [B, N, H, d]


@pytest.mark.parametrize("B,H,N,block,topk,linear,norm", [
    (1, 3, 1000, 64, 0.25, True, False),   # ragged last block, linear branch
    (2, 2, 577, 128, 0.3, True, True),     # two batches, block 128, QK norm
    (1, 2, 1030, 64, 1.0, False, True),    # dense, no linear branch
    (1, 12, 32760, 64, 0.1, True, True),   # the Wan2.1-1.3B 480p shape
])
def test_token_major_equals_head_major(sg, B, H, N, block, topk, linear, norm):
    from sparse_bit_attention_smoothing_b200.inputs import make_inputs
    q, k, v, w = make_inputs(B, H, N, 128, seed=B + H + N, outliers=True)
    q, k, v, w = q.cuda(), k.cuda(), v.cuda(), (w.cuda() if linear else None)
    g = torch.Generator().manual_seed(9)
    gq = (torch.rand(H * 128, generator=g) + 0.5).bfloat16().cuda() if norm else None
    gk = (torch.rand(H * 128, generator=g) * 2 + 0.1).bfloat16().cuda() if norm else None
    if norm:
        ref = sg.sagesla_attn_qknorm(q, k, v, gq, gk, 1e-6, w, block=block, topk=topk)
    else:
        ref = sg.sagesla_attn(q, k, v, w, block=block, topk=topk)
    got = sg.sagesla_attn_bnhd(_tok(q), _tok(k), _tok(v), w, block=block, topk=topk, gamma_q=gq, gamma_k=gk)
    torch.cuda.synchronize()
    assert sg.sync_status() == 0
    assert got.shape == (B, N, H, 128)
    assert torch.equal(_tok(got), ref)


def test_one_weight_without_the_other_is_refused(sg):
    x = torch.zeros(1, 64, 1, 128, dtype=torch.bfloat16, device="cuda")
    g = torch.ones(128, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(Exception):
        sg.sagesla_attn_bnhd(x, x, x, None, gamma_q=g)
