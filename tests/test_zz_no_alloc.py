"""The entry point that allocates no device memory (sagesla_smooth_stats_noalloc).

Some callers cannot allocate device memory once they run -- a process that
fixes its memory budget at start-up, or code where an allocation would stall
or fail.  For them the library computes the smoothing statistics (the K mean
and the V scales) in a fixed scratch array that is part of the library image.
This test calls it through the C ABI and checks that two calls in a row give
exactly what the regular entry point (sagesla_get_quant) gives -- also at the
720p shape, where the heads' partial sums do not fit the scratch at once and
run in chunks -- that a length beyond the scratch is refused, and, in a fresh
process, that device free memory is the same before and after its first call.  It sits in a file of its own, collected
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


@pytest.mark.parametrize("B,H,N", [(1, 3, 1000), (2, 2, 577), (1, 40, 4096), (1, 40, 75600)])
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
    # One head of 2 795 521 tokens needs more partial sums than the 4 MiB
    # scratch holds: refused before any launch (the pointers are never
    # dereferenced).  2 795 520 tokens is the largest length it takes.
    assert L.sagesla_smooth_stats_noalloc(a, a, 1, 1, 2795521, 128, a, a, None) == -1
    assert L.sagesla_smooth_stats_noalloc(a, a, 1, 4, 64, 64, a, a, None) == -1


_FRESH = r"""
import ctypes, os, sys
L = ctypes.CDLL(os.path.join(sys.argv[1], "sparse_bit_attention_smoothing_b200", "libsagesla.so"))
rt = ctypes.CDLL("libcudart.so.12")
P, i = ctypes.c_void_p, ctypes.c_int
L.sagesla_smooth_stats_noalloc.argtypes = [P, P, i, i, i, i, P, P, P]
B, H, N = 1, 40, 75600
nbytes = B * H * N * 128 * 2
k, v, mu, sv = P(), P(), P(), P()
for p_, n_ in ((k, nbytes), (v, nbytes), (mu, B * H * 512), (sv, B * H * 512)):
    assert rt.cudaMalloc(ctypes.byref(p_), ctypes.c_size_t(n_)) == 0
assert rt.cudaMemset(k, 0x3c, ctypes.c_size_t(nbytes)) == 0
assert rt.cudaMemset(v, 0x3c, ctypes.c_size_t(nbytes)) == 0
assert rt.cudaDeviceSynchronize() == 0
free, total = ctypes.c_size_t(), ctypes.c_size_t()
seen = []
for call in range(3):
    assert rt.cudaMemGetInfo(ctypes.byref(free), ctypes.byref(total)) == 0
    before = free.value
    assert L.sagesla_smooth_stats_noalloc(k, v, B, H, N, 128, mu, sv, None) == 0
    assert rt.cudaDeviceSynchronize() == 0
    assert rt.cudaMemGetInfo(ctypes.byref(free), ctypes.byref(total)) == 0
    seen.append(before - free.value)
print("DELTAS", seen)
"""


def test_noalloc_first_call_in_fresh_process_allocates_nothing():
    """A fresh process without torch (the library and the CUDA runtime through
    ctypes only), every module of the library loaded when
    the context is created (CUDA_MODULE_LOADING=EAGER, so the scratch array
    already exists): device free memory is unchanged across the first call and
    the two after it, at the 720p shape whose heads run in two chunks."""
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, CUDA_MODULE_LOADING="EAGER")
    r = subprocess.run([sys.executable, "-c", _FRESH, root], capture_output=True, text=True, env=env, timeout=300)
    assert r.returncode == 0, r.stdout + r.stderr
    line = [x for x in r.stdout.splitlines() if x.startswith("DELTAS")][-1]
    deltas = eval(line.split(" ", 1)[1])
    assert deltas == [0, 0, 0], deltas
