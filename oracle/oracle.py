"""ctypes wrapper around the plain-C oracle (oracle.c).

TEST INFRASTRUCTURE ONLY: imported by tests/, by the smoke check and by the
benchmark's CPU-baseline leg.  The product library never imports or links it.
The C source states which page passage each step follows.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None

NOQUANT = 1  # test switch: no quantisation anywhere (reduction to dense)
# Alternative readings, only for measuring how far the result moves between
# readings the pages leave open (the method's reading is flags = 0).
ALT_WALK128 = 2  # running max updated once per 128 keys of the list
ALT_LSUM_P = 4  # row sum over the unquantised P instead of P~
# SageAttention2++ variants (method options, not alternative readings):
Q_PER_TOKEN = 8  # one Q scale per token instead of per 64-token block
QK_INT4 = 16     # Q and K codes in +-7 (4-bit) instead of +-127


def build(force: bool = False) -> str:
    """Compile oracle.c into oracle/liboracle.so (gcc, OpenMP, no fp contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(
            ["gcc", "-O2", "-std=c11", "-fopenmp", "-ffp-contract=off", "-fPIC", "-shared",
             "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        i, f = ctypes.c_int, ctypes.c_float
        i64 = ctypes.c_int64
        L.orc_version.restype = i
        L.orc_threads.restype = i
        L.orc_e4m3_encode.restype = ctypes.c_uint8
        L.orc_e4m3_encode.argtypes = [f]
        L.orc_e4m3_decode.restype = ctypes.c_double
        L.orc_e4m3_decode.argtypes = [ctypes.c_uint8]
        L.orc_e4m3_encode_array.argtypes = [P, P, i64]
        L.orc_e4m3_decode_array.argtypes = [P, P, i64]
        L.orc_int8_code_array.argtypes = [P, f, P, i64]
        L.orc_phi.restype = ctypes.c_double
        L.orc_phi.argtypes = [ctypes.c_double]
        L.orc_topk_count.restype = i
        L.orc_topk_count.argtypes = [i, f]
        L.orc_dense_attn.argtypes = [P, P, P, i, i, i, P]
        L.orc_dense_attn_bf16.argtypes = [P, P, P, i, i, i, P]
        L.orc_quant.argtypes = [P, P, P, i, i, i, P, P, P, P, P, P, P]
        L.orc_mask.argtypes = [P, P, i, i, i, i, f, P, P, P, P]
        L.orc_block_scores_f64.argtypes = [P, P, i, i, i, i, P]
        L.orc_sagesla.restype = i
        L.orc_sagesla.argtypes = [P, P, P, P, i, i, i, i, f, P, P, i, P, P]
        L.orc_linear_direct.argtypes = [P, P, P, i, i, i, i, P, P]
        L.orc_w8a8_quant.argtypes = [P, i, i, P, P]
        L.orc_w8a8_gemm.argtypes = [P, P, P, P, i, i, i, P]
        L.orc_rmsnorm_bf16.argtypes = [P, P, i, i, i, i, ctypes.c_double, P]
        _lib = L
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _bits(x) -> np.ndarray:
    """bf16 data -> contiguous uint16 bit patterns (accepts torch bf16 tensors or uint16 arrays)."""
    if isinstance(x, np.ndarray):
        assert x.dtype == np.uint16
        return np.ascontiguousarray(x)
    import torch
    assert x.dtype == torch.bfloat16
    return np.ascontiguousarray(x.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16))


def threads() -> int:
    return lib().orc_threads()


def e4m3_encode(x: np.ndarray) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(x.shape, np.uint8)
    lib().orc_e4m3_encode_array(_p(x), _p(out), x.size)
    return out


def e4m3_decode(c: np.ndarray) -> np.ndarray:
    c = np.ascontiguousarray(c, dtype=np.uint8)
    out = np.empty(c.shape, np.float64)
    lib().orc_e4m3_decode_array(_p(c), _p(out), c.size)
    return out


def int8_code(x: np.ndarray, mult: float) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(x.shape, np.int8)
    lib().orc_int8_code_array(_p(x), ctypes.c_float(mult), _p(out), x.size)
    return out


def phi(x: float) -> float:
    return lib().orc_phi(float(x))


def topk_count(nb: int, topk: float) -> int:
    return lib().orc_topk_count(nb, ctypes.c_float(topk))


def dense_attn(q: np.ndarray, k: np.ndarray, v: np.ndarray) -> np.ndarray:
    """fp64 dense softmax attention; q,k,v fp64 [..., N, d]."""
    q = np.ascontiguousarray(q, np.float64)
    k = np.ascontiguousarray(k, np.float64)
    v = np.ascontiguousarray(v, np.float64)
    N, d = q.shape[-2], q.shape[-1]
    BH = q.size // (N * d)
    out = np.empty(q.shape, np.float64)
    lib().orc_dense_attn(_p(q), _p(k), _p(v), BH, N, d, _p(out))
    return out


def dense_attn_bf16(q, k, v) -> np.ndarray:
    qb, kb, vb = _bits(q), _bits(k), _bits(v)
    N, d = qb.shape[-2], qb.shape[-1]
    BH = qb.size // (N * d)
    out = np.empty(qb.shape, np.float64)
    lib().orc_dense_attn_bf16(_p(qb), _p(kb), _p(vb), BH, N, d, _p(out))
    return out


def quant(q, k, v) -> dict:
    """Smoothing + INT8 Q/K (per 64-token block) + FP8 V (per channel).  Codes [BH][N][d]."""
    qb, kb, vb = _bits(q), _bits(k), _bits(v)
    N, d = qb.shape[-2], qb.shape[-1]
    BH = qb.size // (N * d)
    nq = (N + 63) // 64
    r = dict(mu=np.empty((BH, d), np.float32), q8=np.empty((BH, N, d), np.int8),
             k8=np.empty((BH, N, d), np.int8), v8=np.empty((BH, N, d), np.uint8),
             sq=np.empty((BH, nq), np.float32), sk=np.empty((BH, nq), np.float32),
             sv=np.empty((BH, d), np.float32))
    lib().orc_quant(_p(qb), _p(kb), _p(vb), BH, N, d, _p(r["mu"]), _p(r["q8"]), _p(r["k8"]),
                    _p(r["v8"]), _p(r["sq"]), _p(r["sk"]), _p(r["sv"]))
    return r


def mask(q, k, block: int, topk: float, want_scores: bool = False) -> dict:
    """Pooled means (fp32), block mask [BH][Nb][k] sorted ascending, optional fp32 scores."""
    qb, kb = _bits(q), _bits(k)
    N, d = qb.shape[-2], qb.shape[-1]
    BH = qb.size // (N * d)
    nb = (N + block - 1) // block
    kc = topk_count(nb, topk)
    r = dict(qbar=np.empty((BH, nb, d), np.float32), kbar=np.empty((BH, nb, d), np.float32),
             idx=np.empty((BH, nb, kc), np.int32),
             scores=np.empty((BH, nb, nb), np.float32) if want_scores else None, k=kc)
    lib().orc_mask(_p(qb), _p(kb), BH, N, d, block, ctypes.c_float(topk), _p(r["qbar"]),
                   _p(r["kbar"]), _p(r["idx"]), _p(r["scores"]))
    return r


def block_scores_f64(q, k, block: int) -> np.ndarray:
    qb, kb = _bits(q), _bits(k)
    N, d = qb.shape[-2], qb.shape[-1]
    BH = qb.size // (N * d)
    nb = (N + block - 1) // block
    out = np.empty((BH, nb, nb), np.float64)
    lib().orc_block_scores_f64(_p(qb), _p(kb), BH, N, d, block, _p(out))
    return out


def sagesla(q, k, v, w, block: int, topk: float, idx=None, qsel=None, flags: int = 0):
    """The quantised SageSLA path in fp64.  Returns (out fp64 [BH][N][d], idx [BH][Nb][k]).

    w: bf16 [d][d] (y = x W^T) or None for the linear branch off.
    idx: optional external mask [BH][Nb][k] (e.g. the GPU's), sorted ascending.
    qsel: optional uint8 [BH][Nb] flags; only flagged query blocks are computed
          (other rows of `out` are NaN).
    """
    qb, kb, vb = _bits(q), _bits(k), _bits(v)
    wb = None if w is None else _bits(w)
    N, d = qb.shape[-2], qb.shape[-1]
    BH = qb.size // (N * d)
    nb = (N + block - 1) // block
    kc = topk_count(nb, topk)
    if idx is not None:
        idx = np.ascontiguousarray(idx, np.int32).reshape(BH, nb, kc)
    if qsel is not None:
        qsel = np.ascontiguousarray(qsel, np.uint8).reshape(BH, nb)
    out = np.full((BH, N, d), np.nan, np.float64)
    idx_out = np.empty((BH, nb, kc), np.int32)
    rc = lib().orc_sagesla(_p(qb), _p(kb), _p(vb), _p(wb), BH, N, d, block, ctypes.c_float(topk),
                           _p(idx), _p(qsel), flags, _p(out), _p(idx_out))
    if rc < 0:
        raise ValueError("oracle: bad arguments")
    return out, idx_out


def linear_direct(q, k, v, block: int, idx: np.ndarray) -> np.ndarray:
    """Linear branch straight from its per-token definition (fp64 [N][d] inputs)."""
    q = np.ascontiguousarray(q, np.float64)
    k = np.ascontiguousarray(k, np.float64)
    v = np.ascontiguousarray(v, np.float64)
    N, d = q.shape
    idx = np.ascontiguousarray(idx, np.int32)
    kc = idx.shape[-1]
    out = np.empty((N, d), np.float64)
    lib().orc_linear_direct(_p(q), _p(k), _p(v), N, d, block, kc, _p(idx), _p(out))
    return out


# ---------------------------------------------------------------- W8A8 ----
WBLK = 128  # quantisation block of the W8A8 linear layer (128 x 128)


def w8a8_quant(a) -> dict:
    """INT8 codes [rows][cols] and fp32 scales [ceil(rows/128)][cols/128] of a bf16 matrix in 128 x 128 blocks."""
    a = _bits(a)
    rows, cols = a.shape
    assert cols % WBLK == 0
    q = np.empty((rows, cols), np.int8)
    s = np.empty(((rows + WBLK - 1) // WBLK, cols // WBLK), np.float32)
    lib().orc_w8a8_quant(_p(a), rows, cols, _p(q), _p(s))
    return {"q": q, "s": s}


def w8a8_gemm(qx, sx, qw, sw) -> np.ndarray:
    """y = sum over K blocks of s_x s_w (integer dot), fp64 [M][N]."""
    qx, qw = np.ascontiguousarray(qx, np.int8), np.ascontiguousarray(qw, np.int8)
    sx, sw = np.ascontiguousarray(sx, np.float32), np.ascontiguousarray(sw, np.float32)
    M, K = qx.shape
    N = qw.shape[0]
    assert qw.shape[1] == K and K % WBLK == 0
    y = np.empty((M, N), np.float64)
    lib().orc_w8a8_gemm(_p(qx), _p(sx), _p(qw), _p(sw), M, N, K, _p(y))
    return y


def w8a8_linear(x, w) -> dict:
    """The W8A8 layer from bf16 x [M][K] and W [N][K]: codes, scales and y (fp64)."""
    qx, qw = w8a8_quant(x), w8a8_quant(w)
    return {"qx": qx["q"], "sx": qx["s"], "qw": qw["q"], "sw": qw["s"],
            "y": w8a8_gemm(qx["q"], qx["s"], qw["q"], qw["s"])}


def rmsnorm_bf16(x, gamma, eps: float = 1e-6) -> np.ndarray:
    """QK RMSNorm over each token's H*d channels: bf16 [B][H][N][d] -> bf16 bits (uint16), same shape."""
    xb, gb = _bits(x), _bits(gamma)
    B, H, N, d = xb.shape
    assert gb.size == H * d
    y = np.empty_like(xb)
    lib().orc_rmsnorm_bf16(_p(xb), _p(gb), B, H, N, d, float(eps), _p(y))
    return y
