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


def test_profile_hook_times_one_launch(cuda_lib):
    """The timing hook records its event pair around exactly one launch of the
    armed epilogue and then disarms: a second launch leaves the events alone,
    and a launch with another epilogue never triggers it."""
    B = cuda_lib
    M, F, K = 2048, 4096, 4096
    A = torch.randn(M, K, device="cuda").to(torch.bfloat16)
    W = (torch.randn(2 * F, K, device="cuda") * K ** -0.5).to(torch.bfloat16)
    o = B.gemm_swiglu(A, W)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
    B.profile_arm(B.EPI_XENT, ev[0], ev[1])  # another epilogue: not triggered by the SwiGLU GEMM
    B.gemm_swiglu(A, W, out=o)
    ev[2].record()
    torch.cuda.synchronize()
    assert ev[1].elapsed_time(ev[2]) > 0.01  # both recorded at arming, before the launch
    B.profile_arm(B.EPI_SWIGLU, ev[0], ev[1])
    B.gemm_swiglu(A, W, out=o)
    B.gemm_swiglu(A, W, out=o)  # the hook is one-shot: this launch records nothing
    ev[2].record()
    torch.cuda.synchronize()
    k = ev[0].elapsed_time(ev[1])
    after = ev[1].elapsed_time(ev[2])
    flops = 2.0 * M * K * 2 * F
    assert 0.005 < k < 5.0, k
    assert flops / (k / 1e3) < 3.0e15  # below any B200 bf16 rate: the pair spans the kernel
    assert after > 0.5 * k, (k, after)
    B.profile_arm(B.EPI_SWIGLU)


def test_profile_hook_times_every_kernel_of_a_step(cuda_lib):
    """Pairs armed for all nine kernels of the block's forward and backward fire
    once each, in launch order (three for the plain-store GEMMs), and bracket
    non-overlapping stretches of the stream."""
    B = cuda_lib
    M, K, d, F = 1024, 1024, 1024, 2048
    t = synth.grg_inputs(M, K, d, F, seed=12)
    dv = {k: v.cuda() for k, v in t.items()}
    ids = [B.KERNEL_FOLD_GAIN, B.EPI_RESID_RMS, B.EPI_SWIGLU,
           B.KERNEL_SWIGLU_BWD_ROWSTAT, B.EPI_DN, B.KERNEL_COL_REDUCE, B.EPI_STORE, B.EPI_STORE, B.EPI_STORE]
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in ids]
    fo = B.grg_fwd(dv["X"], dv["W1"], dv["R"], dv["g"], dv["W2"], 1e-6)  # warm: allocations, tensor maps
    bo = B.grg_bwd(dv["dY"], dv["X"], dv["W1"], fo["H"], fo["r"], fo["AB"], dv["g"], dv["W2"])
    torch.cuda.synchronize()
    for k, (x, y) in zip(ids, ev):
        B.profile_arm(k, x, y)
    B.grg_fwd(dv["X"], dv["W1"], dv["R"], dv["g"], dv["W2"], 1e-6, out=fo)
    B.grg_bwd(dv["dY"], dv["X"], dv["W1"], fo["H"], fo["r"], fo["AB"], dv["g"], dv["W2"], out=bo)
    torch.cuda.synchronize()
    B.profile_arm(0)
    for i, (x, y) in enumerate(ev):
        assert x.elapsed_time(y) > 0.0, i
        if i + 1 < len(ev):
            assert y.elapsed_time(ev[i + 1][0]) >= 0.0, i
