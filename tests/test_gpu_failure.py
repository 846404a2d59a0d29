"""Device-side failure detection without a GPU fault.

A self-test kernel waits, with the bounded wait of the GEMM pipeline, on a
barrier nothing arrives on: it must give up after its limit, record
CODA_ERR_DEVICE_TIMEOUT in the workspace status word, and return.  The
context must stay usable: a GEMM afterwards runs and is correct, and a
cleared status word stays clear.
"""

import time

import pytest
import torch

from gemm_epilogue_fusion_tmem_b200 import synth
from oracle import coda_oracle as O
from tests.parity import assert_tol, f64

pytestmark = pytest.mark.gpu

CODA_ERR_DEVICE_TIMEOUT = 7


def test_bounded_wait_times_out_and_reports(cuda_lib):
    ws = cuda_lib.Workspace(4096)
    t0 = time.perf_counter()
    cuda_lib.selftest_wait_timeout(ws, 2_000_000)  # 2 ms
    st, detail = ws.query()
    elapsed = time.perf_counter() - t0
    assert st == CODA_ERR_DEVICE_TIMEOUT
    assert detail == (0x3F << 16) | (0 << 8) | 1
    assert elapsed < 10.0
    # The context is intact: clear, run real work, and the status stays clear.
    ws.clear()
    M, N, K = 256, 512, 320
    t = synth.gemm_inputs(M, N, K, seed=4)
    C = cuda_lib.gemm(t["A"].cuda(), t["B"].cuda(), M, N, K, ws=ws)
    st, detail = ws.query()
    assert st == 0 and detail == 0
    assert_tol(C, O.gemm(f64(t["A"]), f64(t["B"])), "gemm after a device timeout")


def test_status_is_sticky_until_cleared(cuda_lib):
    ws = cuda_lib.Workspace(4096)
    cuda_lib.selftest_wait_timeout(ws, 1_000)
    assert ws.query()[0] == CODA_ERR_DEVICE_TIMEOUT
    assert ws.query()[0] == CODA_ERR_DEVICE_TIMEOUT  # reading does not clear it
    ws.clear()
    assert ws.query() == (0, 0)
