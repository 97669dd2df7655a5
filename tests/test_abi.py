"""The C-ABI library loads and exports every symbol include/sagesla.h declares;
host-side argument checks reject bad calls before any CUDA work (no GPU needed)."""
import ctypes
import os
import re
import subprocess

import pytest

from sparse_bit_attention_smoothing_b200 import build as sbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    sbuild.build()
    import sparse_bit_attention_smoothing_b200 as s
    return s.lib()


def declared_functions():
    txt = open(os.path.join(ROOT, "include", "sagesla.h")).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return sorted(set(re.findall(r"\b(?:int|void|const char\*)\s+(\w+)\s*\(", txt)))


def test_exports_every_declared_symbol(L):
    names = declared_functions()
    assert len(names) >= 9
    for n in names:
        assert hasattr(L, n), n


def test_binding_covers_every_declared_symbol():
    import sparse_bit_attention_smoothing_b200 as sg
    names = declared_functions()
    assert set(sg.EXPORTS) == set(names)
    for n in names:
        assert callable(getattr(sg, n, None)), n


def test_topk_count_matches_oracle(L, orc):
    for nb in (1, 7, 10, 16, 512, 591, 1182, 5000):
        for t in (0.01, 0.05, 0.1, 0.15, 0.25, 0.3, 0.5, 0.99, 1.0):
            assert L.sagesla_topk_count(nb, ctypes.c_float(t)) == orc.topk_count(nb, t), (nb, t)


def test_strerror(L):
    for c in (0, -1, -2, -3, -4, -5, -6, -99):
        assert isinstance(L.sagesla_strerror(c), bytes)


F = ctypes.c_float


def test_rejects_bad_arguments_without_launch(L):
    P = ctypes.c_void_p
    a = P(0x10000)
    cases = [
        (None, a, a, None, a, 1, 1, 64, 128, 64, F(0.1)),   # null q
        (a, a, a, None, a, 1, 1, 64, 64, 64, F(0.1)),       # d != 128
        (a, a, a, None, a, 1, 1, 64, 128, 32, F(0.1)),      # bad block
        (a, a, a, None, a, 1, 1, 64, 128, 64, F(0.0)),      # topk = 0
        (a, a, a, None, a, 1, 1, 64, 128, 64, F(1.5)),      # topk > 1
        (a, a, a, None, a, 1, 1, 64, 128, 64, F(float("nan"))),
        (a, a, a, None, a, 0, 1, 64, 128, 64, F(0.1)),      # B = 0
        (a, a, a, None, a, 1, 1, 0, 128, 64, F(0.1)),       # N = 0
        (a, a, a, None, a, 300, 300, 64, 128, 64, F(0.1)),  # B*H > 65535
    ]
    for c in cases:
        assert L.sagesla_attn(*c, None) == -1, c
    m = P(0x10008)
    assert L.sagesla_attn(a, m, a, None, a, 1, 1, 64, 128, 64, F(0.1), None) == -2
    assert L.sagesla_attn(a, a, a, m, a, 1, 1, 64, 128, 64, F(0.1), None) == -2
    assert L.dense_int8_attn(a, a, None, a, 1, 1, 64, 128, None) == -1
    assert L.sagesla_watchdog_selftest(0, None) == -1
    # the longest sequence: Nb <= 12288 (four score rows of the top-k kernel in 227 KB of shared memory);
    # one token more is refused before any CUDA call, the limit itself passes the argument checks
    for n_max, blk in ((786432, 64), (1572864, 128)):
        assert L.sagesla_attn(a, a, a, None, a, 1, 1, n_max + 1, 128, blk, F(0.1), None) == -1
        assert L.sagesla_attn(a, a, a, None, a, 1, 1, n_max, 128, blk, F(0.1), None) != -1
    assert L.sagesla_watchdog_selftest((1 << 20) + 1, None) == -1
    # QK RMSNorm: missing or misaligned weights, eps out of range
    assert L.sagesla_attn_qknorm(a, a, a, None, a, F(1e-6), None, a, 1, 1, 64, 128, 64, F(0.1), None) == -1
    assert L.sagesla_attn_qknorm(a, a, a, a, a, F(-1.0), None, a, 1, 1, 64, 128, 64, F(0.1), None) == -1
    assert L.sagesla_attn_qknorm(a, a, a, P(0x10008), a, F(1e-6), None, a, 1, 1, 64, 128, 64, F(0.1), None) == -2
    # token-major entry (B, N, H order): one weight without the other, eps out of range, misaligned weights, d != 128
    assert L.sagesla_attn_bnhd(a, a, a, a, None, F(1e-6), None, a, 1, 64, 1, 128, 64, F(0.1), None) == -1
    assert L.sagesla_attn_bnhd(a, a, a, a, a, F(2.0), None, a, 1, 64, 1, 128, 64, F(0.1), None) == -1
    assert L.sagesla_attn_bnhd(a, a, a, P(0x10008), a, F(1e-6), None, a, 1, 64, 1, 128, 64, F(0.1), None) == -2
    assert L.sagesla_attn_bnhd(a, a, a, None, None, F(0.0), None, a, 1, 64, 1, 64, 64, F(0.1), None) == -1
    # quantisation options out of range
    assert L.sagesla_attn_opts(a, a, a, None, a, 1, 1, 64, 128, 64, F(0.1), 5, 0, None) == -1
    assert L.sagesla_attn_opts(a, a, a, None, a, 1, 1, 64, 128, 64, F(0.1), 8, 2, None) == -1
    assert L.sagesla_attn_opts(None, a, a, None, a, 1, 1, 64, 128, 64, F(0.1), 4, 1, None) == -1
    # W8A8: shapes that are not multiples of the 128 x 128 block, null and misaligned pointers
    sp = P(0x20000)
    assert L.sagesla_w8a8_quant(a, 128, 100, a, sp, None) == -1
    assert L.sagesla_w8a8_quant(a, 0, 128, a, sp, None) == -1
    assert L.sagesla_w8a8_quant(None, 128, 128, a, sp, None) == -1
    assert L.sagesla_w8a8_quant(P(0x10008), 128, 128, a, sp, None) == -2
    assert L.sagesla_w8a8_gemm(a, sp, a, sp, a, 128, 100, 128, None) == -1
    assert L.sagesla_w8a8_gemm(a, sp, a, sp, a, 128, 128, 64, None) == -1
    assert L.sagesla_w8a8_gemm(a, sp, a, sp, P(0x10008), 128, 128, 128, None) == -2
    assert L.sagesla_w8a8_linear(None, a, sp, a, 128, 128, 128, None) == -1
    assert L.sagesla_w8a8_linear(a, a, sp, a, 0, 128, 128, None) == -1
    ll = ctypes.c_longlong
    for grid, stall, spin in ((0, -1, 1 << 14), (1, -2, 1 << 14), (1, 0, 1023), (1, 0, (1 << 24) + 1)):
        assert L.sagesla_debug_flash_stall(a, a, a, a, 1, 1, 64, 128, F(0.1), grid, stall, ll(spin), None) == -1


C_CLIENT = r"""
#include <stdio.h>
#include <string.h>
#include "sagesla.h"
int main(void) {
  /* every call below is answered by the host-side checks: no CUDA work */
  if (sagesla_topk_count(1182, 0.1f) != 119) return 1;
  if (sagesla_topk_count(16, 0.25f) != 4) return 2;
  if (sagesla_attn(NULL, NULL, NULL, NULL, NULL, 1, 1, 64, 128, 64, 0.1f, NULL) != SAGESLA_ERR_INVALID) return 3;
  if (dense_int8_attn(NULL, NULL, NULL, NULL, 1, 1, 64, 128, NULL) != SAGESLA_ERR_INVALID) return 4;
  if (strlen(sagesla_strerror(SAGESLA_ERR_MISALIGNED)) == 0) return 5;
  if (sagesla_watchdog_selftest(0, NULL) != SAGESLA_ERR_INVALID) return 6;
  puts("c client ok");
  return 0;
}
"""


def test_header_is_c99_and_the_library_links_from_c(L):
    """A plain C99 program includes the header, links against the library and
    gets the documented answers from calls that fail their argument checks."""
    import shutil
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    pkg = os.path.join(ROOT, "sparse_bit_attention_smoothing_b200")
    work = os.path.join(ROOT, "_build")  # the build directory (not tracked)
    os.makedirs(work, exist_ok=True)
    src = os.path.join(work, "c_client.c")
    with open(src, "w") as f:
        f.write(C_CLIENT)
    exe = os.path.join(work, "c_client")
    r = subprocess.run([cc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic", "-I", os.path.join(ROOT, "include"),
                        str(src), "-L", pkg, "-lsagesla", f"-Wl,-rpath,{pkg}", "-o", str(exe)],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0 and "c client ok" in r.stdout, (r.returncode, r.stdout, r.stderr)
