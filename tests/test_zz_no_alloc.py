"""The entry point that allocates no device memory (sagesla_smooth_stats_noalloc).

Some callers cannot allocate device memory once they run -- a process that
fixes its memory budget at start-up, or code where an allocation would stall
or fail.  For them the library computes the smoothing statistics (the K mean
and the V scales) in a fixed scratch array that is part of the library image.
This test calls it through the C ABI and checks that two calls in a row give
exactly what the regular entry point (sagesla_get_quant) gives, and that a
size beyond the scratch is refused.  It sits in a file of its own, collected
last, and passes alone in a fresh process or after every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib():
    from sparse_bit_attention_smoothing_b200 import build
    build.build()
    import sparse_bit_attention_smoothing_b200 as sg
    L = sg.lib()
    P, i = ctypes.c_void_p, ctypes.c_int
    L.sagesla_smooth_stats_noalloc.argtypes = [P, P, i, i, i, i, P, P, P]
    L.sagesla_smooth_stats_noalloc.restype = i
    return sg, L


@pytest.mark.parametrize("B,H,N", [(1, 3, 1000), (2, 2, 577), (1, 40, 4096)])
def test_noalloc_stats_match_regular_entry(lib, B, H, N):
    sg, L = lib
    from sparse_bit_attention_smoothing_b200.inputs import make_inputs
    q, k, v, _ = make_inputs(B, H, N, 128, seed=3, outliers=True)
    dq, dk, dv = q.cuda(), k.cuda(), v.cuda()
    ref = sg.sagesla_get_quant(dq, dk, dv)
    st = torch.cuda.current_stream()
    for _ in range(2):  # two calls in a row share (and overwrite) the scratch
        mu = torch.full((B, H, 128), float("nan"), device="cuda")
        sv = torch.full((B, H, 128), float("nan"), device="cuda")
        rc = L.sagesla_smooth_stats_noalloc(ctypes.c_void_p(dk.data_ptr()), ctypes.c_void_p(dv.data_ptr()), B, H, N,
                                            128, ctypes.c_void_p(mu.data_ptr()), ctypes.c_void_p(sv.data_ptr()),
                                            ctypes.c_void_p(st.cuda_stream))
        assert rc == 0
        torch.cuda.synchronize()
        assert np.array_equal(mu.cpu().numpy(), ref["mu"].cpu().numpy())
        assert np.array_equal(sv.cpu().numpy(), ref["sv"].cpu().numpy())


def test_noalloc_rejects_sizes_beyond_its_scratch(lib):
    _, L = lib
    a = ctypes.c_void_p(0x10000)
    # 3000 heads need more partial sums than the 4 MiB scratch holds: refused
    # before any launch (the pointers are never dereferenced).
    assert L.sagesla_smooth_stats_noalloc(a, a, 1, 3000, 64, 128, a, a, None) == -1
    assert L.sagesla_smooth_stats_noalloc(a, a, 1, 4, 64, 64, a, a, None) == -1
