"""Pins of the oracle's quantisers (CPU only).

FP8 E4M3 follows the OCP 8-bit floating point spec (bias 7, 3 mantissa bits,
max 448, no infinities); the encoder is checked exhaustively against torch's
own float8_e4m3fn cast and the decoder against the spec's closed forms.  The
INT8 quantiser (symmetric, x * 127/amax, round half to even, clamp +-127) is
checked on constructed values whose codes are known in closed form.  The
smoothing mean and the per-block / per-channel scales are checked on
constructed heads.
"""
import math

import numpy as np
import pytest
import torch


def torch_e4m3_bits(x: np.ndarray) -> np.ndarray:
    return torch.from_numpy(x.astype(np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def test_e4m3_encode_exhaustive_bf16_patterns(orc):
    bits = np.arange(1 << 16, dtype=np.uint32) << 16
    x = bits.view(np.float32)
    ok = np.isfinite(x) & (np.abs(x) <= 448.0)
    x = x[ok]
    mine = orc.e4m3_encode(x)
    ref = torch_e4m3_bits(x)
    # +0 and -0 both legal; compare magnitudes for zeros
    z = (mine & 0x7F) == 0
    assert np.array_equal(mine[~z], ref[~z])
    assert np.all((ref[z] & 0x7F) == 0)


@pytest.mark.parametrize("scale", [1.0, 3.7, 448.0 / 6.31, 1e-3])
def test_e4m3_encode_random_fp32(orc, scale):
    rng = np.random.default_rng(int(scale * 1000) % 97)
    x = (rng.standard_normal(200000) * scale).astype(np.float32)
    x = x[np.abs(x) <= 448.0]
    mine = orc.e4m3_encode(x)
    ref = torch_e4m3_bits(x)
    z = (mine & 0x7F) == 0
    assert np.array_equal(mine[~z], ref[~z])


def test_e4m3_saturates(orc):
    x = np.array([448.0, 460.0, 464.0, 1e4, np.inf, -449.0, -1e30], np.float32)
    assert list(orc.e4m3_encode(x)) == [0x7E, 0x7E, 0x7E, 0x7E, 0x7E, 0xFE, 0xFE]


def test_e4m3_decode_closed_forms(orc):
    codes = np.arange(256, dtype=np.uint8)
    dec = orc.e4m3_decode(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    fin = ~np.isnan(ref)
    assert np.array_equal(np.isnan(dec), ~fin)
    assert np.array_equal(dec[fin], ref[fin])
    assert dec[0x7E] == 448.0 and dec[0x38] == 1.0 and dec[0x08] == 2.0 ** -6
    assert dec[0x01] == 2.0 ** -9 and dec[0x07] == 7 * 2.0 ** -9 and dec[0xB8] == -1.0
    assert dec[0x3C] == 1.5 and dec[0x77] == 240.0


def test_int8_code_closed_forms(orc):
    amax = np.float32(3.0)
    mult = np.float32(np.float32(127.0) / amax)
    x = np.array([3.0, -3.0, 0.0, 10.0, -10.0], np.float32)
    assert list(orc.int8_code(x, mult)) == [127, -127, 0, 127, -127]
    # exact half-way points round to even: choose mult = 1
    x = np.array([0.5, 1.5, 2.5, -0.5, -1.5, -2.5, 126.5, 127.5], np.float32)
    assert list(orc.int8_code(x, np.float32(1.0))) == [0, 2, 2, 0, -2, -2, 126, 127]
    # mult = 2: 1.25 -> 2.5 -> 2 ; 1.75 -> 3.5 -> 4
    assert list(orc.int8_code(np.array([1.25, 1.75], np.float32), np.float32(2.0))) == [2, 4]


def test_quant_head_closed_form(orc):
    # N = 70 tokens (one full 64-block + a 6-token tail), d = 8.
    N, d = 70, 8
    q = torch.zeros(1, N, d)
    q[0, 3, 2] = 2.0          # block 0 amax 2
    q[0, 5, 1] = -1.0
    q[0, 66, 4] = 0.5         # tail amax 0.5
    kb = torch.tensor([1.0, -2.0, 0.5, 4.0, 0.0, -1.0, 3.0, 2.0])
    pat = torch.zeros(N, d)
    pat[0::2, :] = 0.25
    pat[1::2, :] = -0.25      # zero mean over N=70 (35 pairs)
    k = (kb + pat).unsqueeze(0)
    v = torch.zeros(1, N, d)
    v[0, 10, 0] = -7.0
    v[0, 11, 0] = 3.5
    v[0, 69, 3] = 0.75
    r = orc.quant(q.bfloat16(), k.bfloat16(), v.bfloat16())
    assert np.array_equal(r["mu"][0], kb.numpy())            # smoothing mean = bias exactly
    assert r["sq"][0, 0] == np.float32(2.0) / np.float32(127) and r["sq"][0, 1] == np.float32(0.5) / np.float32(127)
    assert r["q8"][0, 3, 2] == 127
    assert r["q8"][0, 5, 1] == -64                           # -1 * 63.5 -> -63.5 -> even -> -64
    assert r["q8"][0, 66, 4] == 127
    assert np.all(np.abs(r["k8"][0]) == 127)                 # ks = +-0.25 everywhere -> +-127
    assert np.all(np.sign(r["k8"][0, 0::2]) == 1) and np.all(np.sign(r["k8"][0, 1::2]) == -1)
    assert r["sk"][0, 0] == np.float32(0.25) / np.float32(127)
    # V: channel 0 amax 7 -> -7 maps to -448; 3.5 maps to 224 (exact in e4m3)
    assert r["v8"][0, 10, 0] == 0xFE and orc.e4m3_decode(np.array([r["v8"][0, 11, 0]]))[0] == 224.0
    assert r["sv"][0, 0] == np.float32(7.0) / np.float32(448)
    assert r["v8"][0, 69, 3] == 0x7E and r["sv"][0, 1] == 1.0   # all-zero channel -> scale 1
    assert np.all(r["v8"][0, :, 1] == 0)
