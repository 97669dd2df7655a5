"""Shared helpers of the test suite (comparison rules; no method arithmetic)."""
import numpy as np

# Acceptance of the GPU path against the quantised emulation.
MAX_ABS = 1e-2
MIN_COS = 0.9999
# Against dense fp64 softmax attention at topk = 1 (quantisation error only).
MIN_COS_DENSE = 0.999
# A mask mismatch is accepted only when every differing block is a near-tie:
# |s_ij - s_i(k)| <= NEAR_TIE on the /sqrt(d)-scaled fp64 pooled score.
NEAR_TIE = 1e-5


def bf16_half_ulp(x):
    """Half a bf16 ulp of |x| (8 significant bits): the rounding error of a
    correctly rounded bf16 output."""
    x = np.abs(np.asarray(x, np.float64))
    e = np.floor(np.log2(np.maximum(x, 2.0 ** -126)))
    return np.ldexp(1.0, (e - 8).astype(np.int64))


def max_abs_excess(got, ref) -> float:
    """max |got - ref| beyond the bf16 rounding of the output itself.

    The output is bf16; in the x10 outlier channels |out| reaches ~15, where
    one bf16 ulp is 0.0625, so the max-abs bound is read as applying to the
    error in excess of half a bf16 ulp of the reference value."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    return float(np.max(np.abs(got - ref) - bf16_half_ulp(ref)))


def cosine(a, b) -> float:
    a = np.asarray(a, np.float64).ravel()
    b = np.asarray(b, np.float64).ravel()
    return float(a @ b / np.sqrt((a @ a) * (b @ b)))


def compare_masks(gpu_idx: np.ndarray, orc_idx: np.ndarray, scores64: np.ndarray, kc: int):
    """Returns (n_rows_equal, n_near_tie_rows); asserts on any other difference.

    gpu_idx / orc_idx [R][kc] sorted lists, scores64 [R][nb] fp64 pooled scores."""
    R = gpu_idx.shape[0]
    equal = near = 0
    for r in range(R):
        g = gpu_idx[r]
        assert np.all(np.diff(g) > 0), f"row {r}: not strictly ascending"
        assert g[0] >= 0 and g[-1] < scores64.shape[1]
        if np.array_equal(g, orc_idx[r]):
            equal += 1
            continue
        order = np.argsort(-scores64[r], kind="stable")
        kth = scores64[r, order[kc - 1]]
        diff = set(g.tolist()) ^ set(orc_idx[r].tolist())
        bad = [j for j in diff if abs(scores64[r, j] - kth) > NEAR_TIE]
        assert not bad, f"row {r}: blocks {bad} differ and are not near-ties of the k-th score"
        near += 1
    return equal, near


def untile_codes(codes: np.ndarray, rows: int, cols: int) -> np.ndarray:
    """W8A8 tile images (16 KB per 128 x 128 block, [row block][column block],
    code (r, c) at (r/8)*1024 + (c/16)*128 + (r%8)*16 + c%16) -> int8 [rows][cols]."""
    nrb, ncb = (rows + 127) // 128, cols // 128
    t = np.asarray(codes, np.uint8).view(np.int8).reshape(nrb, ncb, 16, 8, 8, 16)  # [rb][cb][r/8][c/16][r%8][c%16]
    full = t.transpose(0, 2, 4, 1, 3, 5).reshape(nrb * 128, ncb * 128)
    return full[:rows]


def w8a8_check(y_gpu, y_orc, abs_dot, nk: int):
    """W8A8 output rule: |y_gpu - y| <= half a bf16 ulp of the larger of the two
    plus the fp32 accumulation bound (nk + 2) * 2^-24 * sum |terms| (abs_dot =
    |x^| |w^|^T of the dequantised operands bounds that sum).  Returns the
    fraction of outputs equal to the correctly rounded bf16 of the exact y."""
    g = np.asarray(y_gpu, np.float64)
    y = np.asarray(y_orc, np.float64)
    tol = np.maximum(bf16_half_ulp(g), bf16_half_ulp(y)) + (nk + 2) * 2.0 ** -24 * abs_dot
    bad = np.abs(g - y) > tol
    assert not bad.any(), f"{int(bad.sum())} outputs beyond the bound, worst excess {float(np.max(np.abs(g - y) - tol))}"
    import torch
    rne = torch.from_numpy(y).to(torch.bfloat16).double().numpy()
    return float(np.mean(g == rne))
