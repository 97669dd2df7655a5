"""GPU parity of the W8A8 linear layer (through the C ABI) against the oracle.

Codes and scales bit-exact (the quantiser is an integer decision taken in
fp32 on both sides); outputs within half a bf16 ulp plus the fp32
accumulation bound of the exact fp64 sum, and almost all equal to its
correctly rounded bf16.  Shapes cover a single partial tile, ragged rows,
more output tiles than SMs (the persistent loop), and sampled row blocks of
the Wan2.1-14B hidden size (x 75600 x 5120, W 5120 x 5120).
"""
import numpy as np
import pytest
import torch

from tests._util import untile_codes, w8a8_check

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sg():
    from sparse_bit_attention_smoothing_b200 import build
    build.build()
    import sparse_bit_attention_smoothing_b200 as s
    assert torch.cuda.is_available()
    return s


def _inputs(M, N, K, seed):
    g = torch.Generator().manual_seed(seed)
    x = (torch.randn(M, K, generator=g) * torch.linspace(0.2, 6.0, K)).bfloat16()  # channel-dependent ranges
    w = (torch.randn(N, K, generator=g) * 0.03).bfloat16()
    return x, w


def _dequant(q, s, rows, cols):
    return q.astype(np.float64) * np.repeat(np.repeat(s.astype(np.float64), 128, 0), 128, 1)[:rows, :cols]


@pytest.mark.parametrize("rows,cols", [(128, 128), (300, 384), (77, 256), (1000, 640)])
def test_quant_codes_and_scales_bit_exact(sg, orc, rows, cols):
    x, _ = _inputs(rows, 128, cols, rows + cols)
    x[: min(rows, 128), :128] = 0  # an all-zero block: scale 1, codes 0
    codes, scales = sg.sagesla_w8a8_quant(x.cuda())
    torch.cuda.synchronize()
    o = orc.w8a8_quant(x)
    assert np.array_equal(scales.cpu().numpy(), o["s"])
    assert np.array_equal(untile_codes(codes.cpu().numpy(), rows, cols), o["q"])
    nrb = (rows + 127) // 128
    if rows % 128:  # rows past the end are zero codes in the last tile images
        full = untile_codes(codes.cpu().numpy(), nrb * 128, cols)
        assert not full[rows:].any()


@pytest.mark.parametrize("M,N,K", [(64, 128, 128), (300, 384, 640), (2048, 1280, 256), (1000, 512, 1280)])
def test_linear_matches_oracle(sg, orc, M, N, K):
    x, w = _inputs(M, N, K, M + N + K)
    wq, sw = sg.sagesla_w8a8_quant(w.cuda())
    y = sg.sagesla_w8a8_linear(x.cuda(), wq, sw, N)
    torch.cuda.synchronize()
    assert sg.sync_status() == 0
    o = orc.w8a8_linear(x, w)
    absd = np.abs(_dequant(o["qx"], o["sx"], M, K)) @ np.abs(_dequant(o["qw"], o["sw"], N, K)).T
    frac = w8a8_check(y.float().cpu().numpy(), o["y"], absd, K // 128)
    print(f"M={M} N={N} K={K}: {frac:.5f} of outputs equal the rounded exact value")
    assert frac >= 0.99
    # the two-call form (quantise x, then the GEMM) gives the same bits
    xq, sx = sg.sagesla_w8a8_quant(x.cuda())
    y2 = sg.sagesla_w8a8_gemm(xq, sx, wq, sw, M, N, K)
    torch.cuda.synchronize()
    assert torch.equal(y, y2)


def test_wan14b_hidden_size_sampled_row_blocks(sg, orc):
    """x [75600, 5120] (the 720p token count), W [5120, 5120]; three row blocks
    (first, middle, the short last one of 80 rows) against the oracle."""
    M, N, K = 75600, 5120, 5120
    x, w = _inputs(M, N, K, 5)
    wq, sw = sg.sagesla_w8a8_quant(w.cuda())
    y = sg.sagesla_w8a8_linear(x.cuda(), wq, sw, N)
    torch.cuda.synchronize()
    assert sg.sync_status() == 0
    ow = orc.w8a8_quant(w)
    wd = np.abs(_dequant(ow["q"], ow["s"], N, K))
    for rb in (0, 295, 590):
        r0, r1 = rb * 128, min(M, rb * 128 + 128)
        ox = orc.w8a8_quant(x[r0:r1])
        yo = orc.w8a8_gemm(ox["q"], ox["s"], ow["q"], ow["s"])
        absd = np.abs(_dequant(ox["q"], ox["s"], r1 - r0, K)) @ wd.T
        frac = w8a8_check(y[r0:r1].float().cpu().numpy(), yo, absd, K // 128)
        print(f"row block {rb}: {frac:.5f} equal")
        assert frac >= 0.99
