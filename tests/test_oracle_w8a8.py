"""Pins of the oracle's W8A8 linear layer (CPU only).

"揭秘TurboDiffusion：如何让视频生成实现百倍加速？" 支柱三 and 量子位 news 技术解密 4:
weights and activations both INT8 in 128 x 128 blocks, y = x W^T.  The
oracle is pinned against things it does not compute itself:
 - unit scales: blocks whose amax is exactly 127 have scale 1 and codes equal
   to their (integer) values, so y must equal numpy's exact integer matmul;
 - any input: y must equal numpy's fp64 matmul of the dequantised operands
   (codes times their block's scale, expanded block by block), which checks
   the block indexing of both scales independently of the oracle's loops;
 - closed-form codes of a constructed block (0, +-amax, a half-way value that
   rounds to even), an all-zero block (scale 1, codes 0), a short last block
   of rows quantised over its valid rows only;
 - the quantisation error bound against the unquantised fp64 product.
"""
import numpy as np
import pytest
import torch


def bf16(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.asarray(a, np.float32)).bfloat16()


def expand(s: np.ndarray, rows: int, cols: int) -> np.ndarray:
    """Block scales [rb][cb] -> per-element [rows][cols] (128 x 128 blocks)."""
    return np.repeat(np.repeat(s.astype(np.float64), 128, axis=0), 128, axis=1)[:rows, :cols]


def test_unit_scales_give_the_integer_matmul(orc):
    g = np.random.default_rng(1)
    M, N, K = 200, 256, 384
    x = g.integers(-126, 127, (M, K)).astype(np.float32)
    w = g.integers(-126, 127, (N, K)).astype(np.float32)
    # one entry of +-127 per 128 x 128 block: amax = 127 -> scale 1, codes = values
    for a in (x, w):
        for r0 in range(0, a.shape[0], 128):
            for c0 in range(0, a.shape[1], 128):
                a[r0, c0] = 127.0 if (r0 + c0) % 256 == 0 else -127.0
    r = orc.w8a8_linear(bf16(x), bf16(w))
    assert np.all(r["sx"] == 1.0) and np.all(r["sw"] == 1.0)
    assert np.array_equal(r["qx"], x.astype(np.int8)) and np.array_equal(r["qw"], w.astype(np.int8))
    exact = x.astype(np.int64) @ w.astype(np.int64).T
    assert np.array_equal(r["y"], exact.astype(np.float64))


@pytest.mark.parametrize("M,N,K", [(130, 128, 256), (300, 384, 512), (64, 256, 128)])
def test_equals_matmul_of_the_dequantised_operands(orc, M, N, K):
    g = torch.Generator().manual_seed(M + N + K)
    x = (torch.randn(M, K, generator=g) * torch.linspace(0.1, 8.0, K)).bfloat16()  # channel-dependent ranges
    w = (torch.randn(N, K, generator=g) * 0.05).bfloat16()
    r = orc.w8a8_linear(x, w)
    xd = r["qx"].astype(np.float64) * expand(r["sx"], M, K)
    wd = r["qw"].astype(np.float64) * expand(r["sw"], N, K)
    ref = xd @ wd.T
    assert np.allclose(r["y"], ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())


def test_closed_form_codes_zero_block_and_short_last_block(orc):
    x = np.zeros((160, 256), np.float32)
    # block (0, 0): amax 2 -> scale 2/127, mult 63.5: 2 -> 127, -2 -> -127, 1 -> 63.5 -> 64 (half to even)
    x[0, 0], x[1, 1], x[2, 2], x[3, 3] = 2.0, -2.0, 1.0, 0.5  # 0.5 * 63.5 = 31.75 -> 32
    # block (0, 1) stays all zero; block (1, 0) is rows 128..159 only: its amax comes from those rows
    x[130, 5] = 4.0
    x[140, 6] = -1.0  # -1 * 31.75 = -31.75 -> -32
    r = orc.w8a8_quant(bf16(x))
    q, s = r["q"], r["s"]
    assert s.shape == (2, 2)
    assert s[0, 0] == np.float32(2.0) / np.float32(127.0)
    assert (q[0, 0], q[1, 1], q[2, 2], q[3, 3]) == (127, -127, 64, 32)
    assert s[0, 1] == 1.0 and not q[:128, 128:].any()
    assert s[1, 0] == np.float32(4.0) / np.float32(127.0)
    assert (q[130, 5], q[140, 6]) == (127, -32)
    assert s[1, 1] == 1.0


def test_quantisation_error_bound(orc):
    g = torch.Generator().manual_seed(7)
    M, N, K = 256, 256, 512
    x = torch.randn(M, K, generator=g).bfloat16()
    w = torch.randn(N, K, generator=g).bfloat16()
    r = orc.w8a8_linear(x, w)
    xf, wf = x.double().numpy(), w.double().numpy()
    ex = expand(r["sx"], M, K) / 2  # |x - x^| <= s/2 per element
    ew = expand(r["sw"], N, K) / 2
    bound = np.abs(xf) @ ew.T + ex @ np.abs(wf).T + ex @ ew.T
    err = np.abs(r["y"] - xf @ wf.T)
    assert np.all(err <= bound * (1 + 1e-9))
    assert err.max() > 0  # the quantisation is not the identity
