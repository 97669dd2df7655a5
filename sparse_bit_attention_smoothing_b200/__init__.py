"""SageSLA attention for NVIDIA B200 (sm_100a).

A thin ctypes binding over the C ABI of include/sagesla.h (libsagesla.so,
built in-tree by `build.py`).  It only marshals arguments: every step of the
path runs in the library's CUDA kernels.  Tensors are torch CUDA tensors
(device memory and streams come from PyTorch); there is no CPU fallback --
a missing library or a non-sm_100 device raises.
"""
from __future__ import annotations

import ctypes
import os

from . import inputs  # noqa: F401  (seeded synthetic inputs, no method arithmetic)

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsagesla.so")
_lib = None

ERRORS = {0: "ok", -1: "invalid argument", -2: "misaligned pointer", -3: "out of memory",
          -4: "CUDA launch error", -5: "device watchdog timeout", -6: "not an sm_100 device"}


class SageSLAError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {ERRORS.get(code, 'error')} ({code})")


EXPORTS = ["sagesla_attn", "sagesla_attn_opts", "sagesla_attn_qknorm", "sagesla_attn_bnhd", "dense_int8_attn", "sagesla_attn_host", "sagesla_get_quant", "sagesla_get_mask",
           "sagesla_smooth_stats_noalloc", "sagesla_topk_count", "sagesla_sync_status", "sagesla_strerror",
           "sagesla_release", "sagesla_profile", "sagesla_profile_read", "sagesla_watchdog_selftest",
           "sagesla_debug_flash_stall", "sagesla_w8a8_quant", "sagesla_w8a8_gemm", "sagesla_w8a8_linear"]
KERNELS = ["stats", "stats_final", "quant", "pool_topk", "linear_kv", "linear_sum", "flash", "w_tile",
           "linear_apply", "w8a8_quant", "w8a8_gemm", "rms_inv"]


def lib():
    """Load libsagesla.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: run `python -m sparse_bit_attention_smoothing_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P, i, f = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
        L.sagesla_attn.argtypes = [P, P, P, P, P, i, i, i, i, i, f, P]
        L.dense_int8_attn.argtypes = [P, P, P, P, i, i, i, i, P]
        L.sagesla_attn_opts.argtypes = [P, P, P, P, P, i, i, i, i, i, f, i, i, P]
        L.sagesla_attn_qknorm.argtypes = [P, P, P, P, P, f, P, P, i, i, i, i, i, f, P]
        L.sagesla_attn_bnhd.argtypes = [P, P, P, P, P, f, P, P, i, i, i, i, i, f, P]
        L.sagesla_attn_host.argtypes = [P, P, P, P, P, i, i, i, i, i, f, P]
        L.sagesla_get_quant.argtypes = [P, P, P, i, i, i, i, P, P, P, P, P, P, P, P]
        L.sagesla_get_mask.argtypes = [P, P, i, i, i, i, i, f, P, P, P, P, P]
        L.sagesla_smooth_stats_noalloc.argtypes = [P, P, i, i, i, i, P, P, P]
        L.sagesla_topk_count.argtypes = [i, f]
        L.sagesla_sync_status.argtypes = [P]
        L.sagesla_watchdog_selftest.argtypes = [i, P]
        L.sagesla_debug_flash_stall.argtypes = [P, P, P, P, i, i, i, i, f, i, i, ctypes.c_longlong, P]
        L.sagesla_w8a8_quant.argtypes = [P, i, i, P, P, P]
        L.sagesla_w8a8_gemm.argtypes = [P, P, P, P, P, i, i, i, P]
        L.sagesla_w8a8_linear.argtypes = [P, P, P, P, i, i, i, P]
        L.sagesla_strerror.restype = ctypes.c_char_p
        L.sagesla_strerror.argtypes = [i]
        L.sagesla_release.restype = None
        L.sagesla_profile.restype = None
        L.sagesla_profile.argtypes = [i]
        L.sagesla_profile_read.argtypes = [P, P, i]
        for name in EXPORTS:
            getattr(L, name)
        _lib = L
    return _lib


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _check(rc: int, where: str):
    if rc != 0:
        raise SageSLAError(rc, where)


def _shape(q):
    assert q.dim() == 4, "q, k, v must be [B, H, N, d]"
    return q.shape


def topk_count(nb: int, topk: float) -> int:
    return lib().sagesla_topk_count(nb, ctypes.c_float(topk))


def sagesla_attn(q, k, v, proj_w=None, out=None, block: int = 64, topk: float = 0.1, stream=None):
    """SageSLA attention.  q, k, v: bf16 CUDA [B, H, N, d]; proj_w: bf16 [d, d] or None."""
    import torch
    B, H, N, d = _shape(q)
    if out is None:
        out = torch.empty_like(q)
    _check(lib().sagesla_attn(_ptr(q), _ptr(k), _ptr(v), _ptr(proj_w), _ptr(out), B, H, N, d, block,
                              ctypes.c_float(topk), _stream(stream)), "sagesla_attn")
    return out


def sagesla_attn_opts(q, k, v, proj_w=None, out=None, block: int = 64, topk: float = 0.1, qk_bits: int = 8,
                      q_per_token: bool = False, stream=None):
    """sagesla_attn with the SageAttention2++ quantisation options: qk_bits 8 or 4 (Q/K codes in +-127 or +-7),
    q_per_token (one Q scale per token instead of per 64-token block)."""
    import torch
    B, H, N, d = _shape(q)
    if out is None:
        out = torch.empty_like(q)
    _check(lib().sagesla_attn_opts(_ptr(q), _ptr(k), _ptr(v), _ptr(proj_w), _ptr(out), B, H, N, d, block,
                                   ctypes.c_float(topk), qk_bits, 1 if q_per_token else 0, _stream(stream)),
           "sagesla_attn_opts")
    return out


def sagesla_attn_qknorm(q, k, v, gamma_q, gamma_k, eps: float = 1e-6, proj_w=None, out=None, block: int = 64,
                        topk: float = 0.1, stream=None):
    """sagesla_attn on RMS-normalised q and k (per token over H*d channels, weights gamma_q / gamma_k: bf16 [H*d]),
    the norm applied inside the kernels that load q and k."""
    import torch
    B, H, N, d = _shape(q)
    if out is None:
        out = torch.empty_like(q)
    _check(lib().sagesla_attn_qknorm(_ptr(q), _ptr(k), _ptr(v), _ptr(gamma_q), _ptr(gamma_k), ctypes.c_float(eps),
                                     _ptr(proj_w), _ptr(out), B, H, N, d, block, ctypes.c_float(topk), _stream(stream)),
           "sagesla_attn_qknorm")
    return out



def sagesla_attn_bnhd(q, k, v, proj_w=None, out=None, block: int = 64, topk: float = 0.1, gamma_q=None,
                      gamma_k=None, eps: float = 1e-6, stream=None):
    """SageSLA attention on q, k, v in the token-major layout [B, N, H, 128] (out in the same layout), read in place;
    with gamma_q / gamma_k (bf16 [H*128]) the QK RMSNorm of sagesla_attn_qknorm is fused in as well."""
    import torch
    if q.dim() != 4 or q.dtype != torch.bfloat16 or not q.is_contiguous():
        raise ValueError("q must be a contiguous bf16 [B, N, H, d] tensor")
    B, N, H, d = q.shape
    if out is None:
        out = torch.empty_like(q)
    _check(lib().sagesla_attn_bnhd(_ptr(q), _ptr(k), _ptr(v), _ptr(gamma_q), _ptr(gamma_k), ctypes.c_float(eps),
                                   _ptr(proj_w), _ptr(out), B, N, H, d, block, ctypes.c_float(topk), _stream(stream)),
           "sagesla_attn_bnhd")
    return out

def dense_int8_attn(q, k, v, out=None, stream=None):
    import torch
    B, H, N, d = _shape(q)
    if out is None:
        out = torch.empty_like(q)
    _check(lib().dense_int8_attn(_ptr(q), _ptr(k), _ptr(v), _ptr(out), B, H, N, d, _stream(stream)),
           "dense_int8_attn")
    return out


def sagesla_attn_host(q, k, v, proj_w=None, out=None, block: int = 64, topk: float = 0.1, stream=None):
    """Same on HOST tensors (pinned for asynchronous copies); returns after the result is in `out`."""
    import torch
    B, H, N, d = _shape(q)
    if out is None:
        out = torch.empty_like(q)
    _check(lib().sagesla_attn_host(_ptr(q), _ptr(k), _ptr(v), _ptr(proj_w), _ptr(out), B, H, N, d, block,
                                   ctypes.c_float(topk), _stream(stream)), "sagesla_attn_host")
    return out


def sagesla_get_quant(q, k, v, stream=None) -> dict:
    import torch
    B, H, N, d = _shape(q)
    dev = q.device
    nq = (N + 63) // 64
    r = dict(q8=torch.empty(B, H, N, d, dtype=torch.int8, device=dev),
             k8=torch.empty(B, H, N, d, dtype=torch.int8, device=dev),
             v8=torch.empty(B, H, N, d, dtype=torch.uint8, device=dev),
             sq=torch.empty(B, H, nq, dtype=torch.float32, device=dev),
             sk=torch.empty(B, H, nq, dtype=torch.float32, device=dev),
             sv=torch.empty(B, H, d, dtype=torch.float32, device=dev),
             mu=torch.empty(B, H, d, dtype=torch.float32, device=dev))
    _check(lib().sagesla_get_quant(_ptr(q), _ptr(k), _ptr(v), B, H, N, d, _ptr(r["q8"]), _ptr(r["k8"]),
                                   _ptr(r["v8"]), _ptr(r["sq"]), _ptr(r["sk"]), _ptr(r["sv"]), _ptr(r["mu"]),
                                   _stream(stream)), "sagesla_get_quant")
    return r


def sagesla_get_mask(q, k, block: int = 64, topk: float = 0.1, pooled: bool = False, stream=None) -> dict:
    import torch
    B, H, N, d = _shape(q)
    nb = (N + block - 1) // block
    kc = topk_count(nb, topk)
    dev = q.device
    r = dict(idx=torch.empty(B, H, nb, kc, dtype=torch.int32, device=dev), k=kc,
             qbar=torch.empty(B, H, nb, d, dtype=torch.float32, device=dev) if pooled else None,
             kbar=torch.empty(B, H, nb, d, dtype=torch.float32, device=dev) if pooled else None)
    kout = ctypes.c_int(0)
    _check(lib().sagesla_get_mask(_ptr(q), _ptr(k), B, H, N, d, block, ctypes.c_float(topk), _ptr(r["idx"]),
                                  _ptr(r["qbar"]), _ptr(r["kbar"]), ctypes.byref(kout), _stream(stream)),
           "sagesla_get_mask")
    assert kout.value == kc
    return r


def sagesla_smooth_stats_noalloc(k, v, mu=None, sv=None, stream=None):
    """Per-channel mean of K and FP8 scale of V, [B, H, d] fp32 each, without any device allocation by the
    library (mu / sv are allocated here by torch unless given).  Returns (mu, sv)."""
    import torch
    B, H, N, d = _shape(k)
    if mu is None:
        mu = torch.empty(B, H, d, dtype=torch.float32, device=k.device)
    if sv is None:
        sv = torch.empty(B, H, d, dtype=torch.float32, device=k.device)
    _check(lib().sagesla_smooth_stats_noalloc(_ptr(k), _ptr(v), B, H, N, d, _ptr(mu), _ptr(sv), _stream(stream)),
           "sagesla_smooth_stats_noalloc")
    return mu, sv


def sagesla_watchdog_selftest(probes: int = 1000, stream=None):
    """Make one bounded device-side wait expire on purpose (nothing faults); the next sync_status() on the stream
    then returns -5 (device watchdog timeout) and clears the flag."""
    _check(lib().sagesla_watchdog_selftest(probes, _stream(stream)), "sagesla_watchdog_selftest")


def sagesla_debug_flash_stall(q, k, v, out=None, topk: float = 0.1, grid: int = 1, stall_step: int = -1,
                              spin_limit: int = 1 << 24, stream=None):
    """sagesla_attn at block 64 without the linear branch, its flash kernel on `grid` CTAs with bounded waits of
    `spin_limit` probes; stall_step >= 0 makes CTA 0's first pipeline omit the key copies of that step, so a real
    wait of the kernel gives up (sync_status() then returns -5 once).  Returns `out`."""
    import torch
    B, H, N, d = _shape(q)
    if out is None:
        out = torch.empty_like(q)
    _check(lib().sagesla_debug_flash_stall(_ptr(q), _ptr(k), _ptr(v), _ptr(out), B, H, N, d, ctypes.c_float(topk),
                                           grid, stall_step, spin_limit, _stream(stream)),
           "sagesla_debug_flash_stall")
    return out


W8A8_BLOCK = 128


def sagesla_w8a8_quant(a, stream=None):
    """INT8 codes (tile images, uint8 [ceil(rows/128) * cols/128 * 16384]) and fp32 scales
    [ceil(rows/128), cols/128] of a bf16 CUDA matrix [rows, cols] in 128 x 128 blocks."""
    import torch
    assert a.dim() == 2 and a.dtype == torch.bfloat16 and a.is_contiguous()
    rows, cols = a.shape
    nrb, ncb = (rows + W8A8_BLOCK - 1) // W8A8_BLOCK, cols // W8A8_BLOCK
    codes = torch.empty(nrb * ncb * W8A8_BLOCK * W8A8_BLOCK, dtype=torch.uint8, device=a.device)
    scales = torch.empty(nrb, ncb, dtype=torch.float32, device=a.device)
    _check(lib().sagesla_w8a8_quant(_ptr(a), rows, cols, _ptr(codes), _ptr(scales), _stream(stream)),
           "sagesla_w8a8_quant")
    return codes, scales


def sagesla_w8a8_gemm(xq, sx, wq, sw, M: int, N: int, K: int, y=None, stream=None):
    """y = x W^T (bf16 [M, N]) from the codes and scales of x [M, K] and W [N, K]."""
    import torch
    if y is None:
        y = torch.empty(M, N, dtype=torch.bfloat16, device=xq.device)
    _check(lib().sagesla_w8a8_gemm(_ptr(xq), _ptr(sx), _ptr(wq), _ptr(sw), _ptr(y), M, N, K, _stream(stream)),
           "sagesla_w8a8_gemm")
    return y


def sagesla_w8a8_linear(x, wq, sw, N: int, y=None, stream=None):
    """The W8A8 layer: quantise x (bf16 [M, K]) and multiply by the quantised W [N, K]."""
    import torch
    M, K = x.shape
    if y is None:
        y = torch.empty(M, N, dtype=torch.bfloat16, device=x.device)
    _check(lib().sagesla_w8a8_linear(_ptr(x), _ptr(wq), _ptr(sw), _ptr(y), M, N, K, _stream(stream)),
           "sagesla_w8a8_linear")
    return y


def sync_status(stream=None) -> int:
    return lib().sagesla_sync_status(_stream(stream))


def profile(enable: bool):
    """Bracket every library kernel launch with CUDA events on its stream."""
    lib().sagesla_profile(1 if enable else 0)


def profile_read() -> dict:
    """{kernel name: (total ms, launches)} since the last read."""
    n = len(KERNELS)
    ms = (ctypes.c_double * n)()
    cnt = (ctypes.c_int * n)()
    _check(lib().sagesla_profile_read(ms, cnt, n), "sagesla_profile_read")
    return {KERNELS[i]: (ms[i], cnt[i]) for i in range(n) if cnt[i]}


def release():
    lib().sagesla_release()


def strerror(code: int) -> str:
    return lib().sagesla_strerror(code).decode()


# The C names of the utility calls, for callers that follow the header.
sagesla_topk_count = topk_count
sagesla_sync_status = sync_status
sagesla_strerror = strerror
sagesla_release = release
sagesla_profile = profile
sagesla_profile_read = profile_read
