"""Pins of the oracle's SageAttention2++ variants (CPU only).

量子位 news, 技术解密 1: SageAttention2++ quantises to 8 and, further, 4 bits and
calibrates the quantisation per thread.  The oracle takes these as two
options of the quantisation step: one Q scale per token (the row a softmax
thread owns) instead of per 64-token block, and Q/K codes in +-7 instead of
+-127.  The pins:
 - per-token scales equal the block scale when every row of a block has the
   block's absmax, so the variant reproduces the default path bit for bit;
 - identical keys give uniform probabilities whatever the Q/K codes, so the
   output is the mean of the dequantised values under every variant;
 - on inputs whose token magnitudes vary (one scale factor per query token),
   per-token Q scales bring the output closer to dense fp64 attention than
   per-block scales, and 4-bit codes move it further away than 8-bit ones.
"""
import numpy as np
import pytest
import torch


def _cos(a, b):
    a, b = np.asarray(a, np.float64).ravel(), np.asarray(b, np.float64).ravel()
    return float(a @ b / np.sqrt((a @ a) * (b @ b)))


def test_per_token_equals_per_block_when_every_row_has_the_block_absmax(orc):
    g = torch.Generator().manual_seed(1)
    BH, N, d = 2, 200, 128
    q = torch.randn(BH, N, d, generator=g).clamp(-2.0, 2.0)
    q[:, :, 5] = 2.5  # every row of every block has absmax 2.5 (exact in bf16)
    k = torch.randn(BH, N, d, generator=g)
    v = torch.randn(BH, N, d, generator=g)
    q, k, v = q.bfloat16(), k.bfloat16(), v.bfloat16()
    a, ia = orc.sagesla(q, k, v, None, 64, 0.5)
    b, ib = orc.sagesla(q, k, v, None, 64, 0.5, flags=orc.Q_PER_TOKEN)
    assert np.array_equal(ia, ib) and np.array_equal(a, b)


@pytest.mark.parametrize("flags", [0, 8, 16, 24])
def test_identical_keys_give_the_mean_of_the_dequantised_values(orc, flags):
    g = torch.Generator().manual_seed(2)
    BH, N, d = 1, 128, 128
    q = torch.randn(BH, N, d, generator=g).bfloat16()
    k = torch.randn(1, 1, d, generator=g).expand(BH, N, d).contiguous().bfloat16()
    v = torch.randn(BH, N, d, generator=g).bfloat16()
    out, _ = orc.sagesla(q, k, v, None, 64, 1.0, flags=flags)
    r = orc.quant(q, k, v)
    vd = orc.e4m3_decode(r["v8"][0]) * r["sv"][0][None, :]
    assert np.allclose(out[0], vd.mean(axis=0)[None, :], rtol=0, atol=1e-9)


def test_per_token_scales_help_and_int4_hurts_on_token_varying_inputs(orc):
    g = torch.Generator().manual_seed(3)
    BH, N, d = 2, 256, 128
    tok = torch.exp(torch.randn(BH, N, 1, generator=g) * 1.2)  # per-token magnitudes over ~two decades
    q = (torch.randn(BH, N, d, generator=g) * tok * 0.6).bfloat16()
    k = torch.randn(BH, N, d, generator=g).bfloat16()
    v = torch.randn(BH, N, d, generator=g).bfloat16()
    dense = orc.dense_attn_bf16(q, k, v)
    cos = {f: _cos(orc.sagesla(q, k, v, None, 64, 1.0, flags=f)[0], dense) for f in (0, 8, 16)}
    assert cos[8] > cos[0], cos
    assert cos[16] < cos[0], cos
