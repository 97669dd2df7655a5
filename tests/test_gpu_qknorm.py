"""GPU parity of the QK RMSNorm fused into the path (sagesla_attn_qknorm).

The normalised q and k are never written: the per-token factors come from
one pass over q and k, and the statistics, quantisation, linear-branch
kernels apply the norm where they load a row.  Since the norm's output is
bf16 and its per-token sum is taken in fp64 (its rounding far below that of
the fp32 factor), the fused call must equal
sagesla_attn on the oracle's normalised tensors bit for bit; and that output
must match the oracle's emulation on them within the path's tolerances."""
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


def _bf16(a):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)


@pytest.mark.parametrize("B,H,N,block,topk,linear", [(1, 3, 1000, 64, 0.25, True), (2, 2, 577, 128, 0.3, True),
                                                     (1, 2, 1030, 64, 1.0, False)])
def test_fused_norm_equals_path_on_normalised_inputs(sg, orc, B, H, N, block, topk, linear):
    from sparse_bit_attention_smoothing_b200.inputs import make_inputs
    q, k, v, w = make_inputs(B, H, N, 128, seed=B + H + N, outliers=True)
    g = torch.Generator().manual_seed(5)
    gq = (torch.rand(H * 128, generator=g) + 0.5).bfloat16()
    gk = (torch.rand(H * 128, generator=g) * 2 + 0.1).bfloat16()
    qn, kn = _bf16(orc.rmsnorm_bf16(q, gq)), _bf16(orc.rmsnorm_bf16(k, gk))
    dw = w.cuda() if linear else None
    fused = sg.sagesla_attn_qknorm(q.cuda(), k.cuda(), v.cuda(), gq.cuda(), gk.cuda(), 1e-6, dw, block=block, topk=topk)
    plain = sg.sagesla_attn(qn.cuda(), kn.cuda(), v.cuda(), dw, block=block, topk=topk)
    m = sg.sagesla_get_mask(qn.cuda(), kn.cuda(), block=block, topk=topk)
    torch.cuda.synchronize()
    assert sg.sync_status() == 0
    assert torch.equal(fused, plain)
    BH, nb = B * H, (N + block - 1) // block
    emu, _ = orc.sagesla(qn.reshape(BH, N, 128), kn.reshape(BH, N, 128), v.reshape(BH, N, 128), w if linear else None,
                         block, topk, idx=m["idx"].cpu().numpy().reshape(BH, nb, -1))
    got = fused.float().cpu().numpy().reshape(BH, N, 128).astype(np.float64)
    err, cos = max_abs_excess(got, emu), cosine(got, emu)
    print(f"B={B} H={H} N={N} block={block}: max-abs excess {err:.2e}, cosine {cos:.7f}")
    assert err <= MAX_ABS and cos >= MIN_COS, (err, cos)
