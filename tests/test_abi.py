"""The C-ABI library builds, loads and exports every symbol include/coda.h declares (CPU only).

No compute call is made here; host-side argument checks that return before
touching the device are exercised where they do not need a GPU.
"""

import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "coda.h")


def _declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(coda_[a-z0-9_]+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib():
    from gemm_epilogue_fusion_tmem_b200 import build
    build.build()
    return ctypes.CDLL(build.LIB_PATH)


def test_header_declares_the_entry_points():
    names = _declared_functions()
    for required in ("coda_grg_fwd", "coda_grg_bwd", "coda_swiglu_fwd", "coda_swiglu_bwd", "coda_gemm",
                     "coda_fold_gain", "coda_status_query"):
        assert required in names


def test_library_exports_every_declared_symbol(lib):
    missing = [n for n in _declared_functions() if not hasattr(lib, n)]
    assert not missing, f"declared but not exported: {missing}"


def test_status_strings(lib):
    lib.coda_status_string.restype = ctypes.c_char_p
    assert lib.coda_status_string(0) == b"ok"
    assert b"timed out" in lib.coda_status_string(7)
    assert lib.coda_status_string(99) == b"unknown status"


def test_workspace_sizes_cover_the_carved_buffers(lib):
    lib.coda_grg_fwd_workspace_bytes.restype = ctypes.c_size_t
    lib.coda_grg_bwd_workspace_bytes.restype = ctypes.c_size_t
    lib.coda_swiglu_bwd_workspace_bytes.restype = ctypes.c_size_t
    M, K, d, N = 8192, 4096, 4096, 22016
    T = -(-d // 256)
    fwd_pre = lib.coda_grg_fwd_workspace_bytes(M, K, d, N, 1)
    fwd = lib.coda_grg_fwd_workspace_bytes(M, K, d, N, 0)
    assert fwd_pre >= 256 + M * T * 4
    assert fwd >= fwd_pre + N * d * 2
    bwd = lib.coda_grg_bwd_workspace_bytes(M, K, d, N)
    assert bwd >= 256 + M * N * 2 + M * 4 + (-(-M // 128)) * 4 * d * 4
    assert lib.coda_swiglu_bwd_workspace_bytes(16384, 4096, 14336) >= 256 + 16384 * 2 * 14336 * 2


def test_argument_errors_return_before_any_device_work(lib):
    """Null pointers and unsupported shapes are rejected by host checks alone."""
    P = ctypes.c_void_p
    lib.coda_gemm.argtypes = [P, P, P, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                              P, ctypes.c_size_t, P]
    one = P(256)
    # null operand
    assert lib.coda_gemm(None, one, one, 128, 128, 64, 0, 0, one, 256, None) == 1
    # N not a multiple of 32
    assert lib.coda_gemm(one, one, one, 128, 100, 64, 0, 0, one, 256, None) == 2
    # misaligned pointer
    assert lib.coda_gemm(P(258), one, one, 128, 128, 64, 0, 0, one, 256, None) == 3
    # workspace too small
    assert lib.coda_gemm(one, one, one, 128, 128, 64, 0, 0, one, 16, None) == 4
    lib.coda_grg_fwd.argtypes = [P] * 10 + [ctypes.c_int] * 4 + [ctypes.c_float, P, ctypes.c_size_t, P]
    # eps must be positive
    assert lib.coda_grg_fwd(*([one] * 10), 128, 64, 64, 128, 0.0, one, 1 << 20, None) == 1
    # d must be a multiple of 64
    assert lib.coda_grg_fwd(*([one] * 10), 128, 64, 96, 128, 1e-6, one, 1 << 20, None) == 2


def test_empty_batch_and_negative_sizes_on_the_host(lib):
    """M = 0 is a valid empty batch: forward calls return OK without touching a
    device (row pointers may be NULL); a backward call needs its weight-gradient
    pointers; negative sizes are invalid."""
    P = ctypes.c_void_p
    one = P(256)
    lib.coda_grg_fwd.argtypes = [P] * 10 + [ctypes.c_int] * 4 + [ctypes.c_float, P, ctypes.c_size_t, P]
    nulls = [None, one, None, one, one, None, None, None, None, None]  # X, W1, R, g, W2, W2g, H, r, Y, AB
    assert lib.coda_grg_fwd(*nulls, 0, 64, 64, 128, 1e-6, None, 0, None) == 0
    assert lib.coda_grg_fwd(*nulls, 0, 64, 96, 128, 1e-6, None, 0, None) == 2   # d still checked
    assert lib.coda_grg_fwd(*nulls, 0, 64, 64, 128, 0.0, None, 0, None) == 1    # eps still checked
    assert lib.coda_grg_fwd(*nulls, -1, 64, 64, 128, 1e-6, None, 0, None) == 1
    lib.coda_grg_bwd.argtypes = [P] * 9 + [P] * 5 + [ctypes.c_int] * 4 + [P, ctypes.c_size_t, P]
    # dY, dH_in, X, W1, H, r, AB, g, W2 | dX, dR, dW1 (NULL), dW2, dg
    args = [None, None, None, one, None, None, None, one, one, None, None, None, one, one]
    assert lib.coda_grg_bwd(*args, 0, 64, 64, 128, None, 0, None) == 1
    lib.coda_gemm.argtypes = [P, P, P, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                              P, ctypes.c_size_t, P]
    assert lib.coda_gemm(None, None, None, 0, 128, 64, 0, 0, None, 0, None) == 0
    assert lib.coda_gemm(None, None, None, 128, 0, 64, 0, 0, None, 0, None) == 0
    assert lib.coda_gemm(one, one, one, -5, 128, 64, 0, 0, one, 256, None) == 1
    assert lib.coda_gemm(None, None, None, 128, 128, 0, 0, 0, None, 0, None) == 1  # K = 0 writes C: needs C
    lib.coda_swiglu_fwd.argtypes = [P] * 6 + [ctypes.c_int] * 3 + [P, ctypes.c_size_t, P]
    assert lib.coda_swiglu_fwd(None, one, one, None, None, None, 0, 64, 64, None, 0, None) == 0
    assert lib.coda_swiglu_fwd(None, one, one, None, None, None, 0, 64, 100, None, 0, None) == 2


C_CONSUMER = r"""
#include "coda.h"
#include <stdio.h>
int main(void) {
  /* host-only calls: no device is touched */
  printf("%d\n", coda_version());
  printf("%s\n", coda_status_string(CODA_ERR_WORKSPACE_TOO_SMALL));
  printf("%zu\n", coda_grg_fwd_workspace_bytes(8192, 4096, 4096, 22016, 0));
  printf("%zu\n", coda_grg_bwd_workspace_bytes(8192, 4096, 4096, 22016));
  printf("%d\n", (int)coda_grg_fwd(0, 0, 0, 0, 0, 0, 0, 0, 0, 0, 256, 512, 512, 2048, 1e-6f, 0, 0, 0));
  printf("%d\n", (int)coda_profile_arm(99, (void*)16, (void*)16));
  return 0;
}
"""


def test_header_is_plain_c_and_links_from_c(lib, tmp_path):
    """include/coda.h compiles as strict C11 and a C program links against
    libcoda.so and gets the same answers as the Python binding."""
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("gcc not available")
    from gemm_epilogue_fusion_tmem_b200 import build as Bld
    src = tmp_path / "consumer.c"
    src.write_text(C_CONSUMER)
    exe = tmp_path / "consumer"
    libdir = os.path.dirname(Bld.LIB_PATH)
    subprocess.run([gcc, "-std=c11", "-Wall", "-Wextra", "-Werror", "-pedantic", "-I", Bld.INCLUDE, str(src),
                    "-L", libdir, "-lcoda", f"-Wl,-rpath,{libdir}", "-o", str(exe)], check=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.split("\n")
    lib.coda_status_string.restype = ctypes.c_char_p
    for f in (lib.coda_grg_fwd_workspace_bytes, lib.coda_grg_bwd_workspace_bytes):
        f.restype = ctypes.c_size_t
    assert int(out[0]) == lib.coda_version()
    assert out[1] == lib.coda_status_string(4).decode()
    assert int(out[2]) == lib.coda_grg_fwd_workspace_bytes(8192, 4096, 4096, 22016, 0)
    assert int(out[3]) == lib.coda_grg_bwd_workspace_bytes(8192, 4096, 4096, 22016)
    assert int(out[4]) == 1  # null pointers: CODA_ERR_INVALID_ARG before any device work
    assert int(out[5]) == 1  # unknown kernel id
