"""Pins of the oracle's QK RMSNorm (CPU only).

Reading ("thu-ml/TurboDiffusion" radar page §二 step 5 and 量子位 news 技术解密 4
name the DiT's own RMSNorm kernels; the pages give no formula): per token,
over the model dimension (all H heads x d channels), y = x / sqrt(mean(x^2)
+ eps) * gamma, the normalised activations rounded to bf16.  The pins:
 - the fp64 definition, to within half a bf16 ulp plus fp32 rounding;
 - eps = 0 and a constant power-of-two token: y = sign(x) * gamma exactly;
 - eps = 0: scaling a token by a power of two leaves y bit-identical;
 - tokens are independent, and the heads of one token are coupled (the
   mean runs over all H*d channels, not over one head's d).
"""
import numpy as np
import torch


def _y(orc, x, g, eps=1e-6):
    return torch.from_numpy(orc.rmsnorm_bf16(x, g, eps).view(np.int16)).view(torch.bfloat16)


def _gamma(H, d, seed=0):
    gen = torch.Generator().manual_seed(seed)
    return (torch.rand(H * d, generator=gen) + 0.5).bfloat16()


def test_fp64_definition(orc):
    gen = torch.Generator().manual_seed(1)
    B, H, N, d = 2, 3, 40, 128
    x = (torch.randn(B, H, N, d, generator=gen) * 3).bfloat16()
    g = _gamma(H, d)
    y = _y(orc, x, g).double()
    xf = x.double()
    ref = xf / (xf.pow(2).mean(dim=(1, 3), keepdim=True) + 1e-6).sqrt() * g.double().view(1, H, 1, d)
    half_ulp = torch.ldexp(torch.ones_like(ref), torch.floor(torch.log2(ref.abs().clamp_min(2.0 ** -126))).int() - 8)
    assert torch.all((y - ref).abs() <= half_ulp * (1 + 1e-5) + 1e-6 * ref.abs())


def test_constant_power_of_two_token(orc):
    B, H, N, d = 1, 2, 4, 128
    x = torch.zeros(B, H, N, d)
    for n, c in enumerate([0.25, -4.0, 1.0, -0.5]):
        x[:, :, n, :] = c
    g = _gamma(H, d, 3)
    y = _y(orc, x.bfloat16(), g, eps=0.0)
    for n, c in enumerate([0.25, -4.0, 1.0, -0.5]):
        assert torch.equal(y[0, :, n].reshape(-1), (g * (1 if c > 0 else -1)).bfloat16())


def test_power_of_two_scale_invariance(orc):
    gen = torch.Generator().manual_seed(4)
    x = torch.randn(1, 2, 30, 128, generator=gen).bfloat16()
    g = _gamma(2, 128, 5)
    assert torch.equal(_y(orc, x, g, 0.0), _y(orc, (x.float() * 8).bfloat16(), g, 0.0))


def test_tokens_independent_heads_coupled(orc):
    gen = torch.Generator().manual_seed(6)
    x = torch.randn(1, 2, 10, 128, generator=gen).bfloat16()
    g = _gamma(2, 128, 7)
    y0 = _y(orc, x, g)
    x2 = x.clone()
    x2[0, 1, 3] = (x2[0, 1, 3].float() * 3).bfloat16()  # head 1 of token 3 only
    y1 = _y(orc, x2, g)
    other = [n for n in range(10) if n != 3]
    assert torch.equal(y0[:, :, other], y1[:, :, other])  # other tokens untouched
    assert not torch.equal(y0[0, 0, 3], y1[0, 0, 3])      # head 0 of token 3 moved: one mean over both heads
