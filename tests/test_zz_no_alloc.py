"""The allocation-free GRG forward (coda_grg_fwd_prefolded_static) against coda_grg_fwd.

Some callers cannot allocate device memory (a framework arena that owns every
device byte, a plugin interface with no workspace, a request path that must
not allocate), so the library offers this one forward whose scratch lives in a
static device array.  It launches the same kernels with the same arguments as
coda_grg_fwd given the same pre-folded weight, so its outputs must be
identical bit for bit.  This test calls both entry points through the C ABI on
the same inputs, twice in a row with different data (the static scratch keeps
the previous call's contents), compares the outputs bit for bit, checks the
first call against the CPU oracle directly, and reads the static status word.
It runs on its own in a fresh process as well as after the other tests; its
file name makes pytest collect it last.
"""

import ctypes

import pytest
import torch

from gemm_epilogue_fusion_tmem_b200 import synth
from tests import refs

pytestmark = pytest.mark.gpu


def _static_fwd(lib, t, H, r, Y, AB, M, K, d, N, eps):
    fn = lib.coda_grg_fwd_prefolded_static
    P = ctypes.c_void_p
    fn.restype = ctypes.c_int
    fn.argtypes = [P] * 8 + [ctypes.c_int] * 4 + [ctypes.c_float, P]
    ptr = lambda x: ctypes.c_void_p(x.data_ptr())
    return fn(ptr(t["X"]), ptr(t["W1"]), ptr(t["R"]), ptr(t["W2g"]), ptr(H), ptr(r), ptr(Y), ptr(AB),
              M, K, d, N, ctypes.c_float(eps), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def _static_status(lib):
    fn = lib.coda_static_status_query
    fn.restype = ctypes.c_int
    fn.argtypes = [ctypes.c_void_p, ctypes.POINTER(ctypes.c_uint32)]
    detail = ctypes.c_uint32(0xFFFFFFFF)
    st = fn(ctypes.c_void_p(torch.cuda.current_stream().cuda_stream), ctypes.byref(detail))
    return st, detail.value


def test_static_scratch_forward_matches_workspace_forward(cuda_lib):
    lib = cuda_lib.library()
    M, K, d, F, eps = 520, 512, 768, 640, 1e-6   # ragged rows and a ragged partial-RMS tile
    N = 2 * F
    for seed in (11, 12):  # two calls in a row share the static scratch
        host = synth.grg_inputs(M, K, d, F, seed=seed)
        t = {k: v.cuda() for k, v in host.items()}
        t["W2g"] = cuda_lib.fold_gain(t["W2"], t["g"])
        ref = cuda_lib.grg_fwd(t["X"], t["W1"], t["R"], t["g"], t["W2"], eps, W2g=t["W2g"])
        H = torch.full((M, d), float("nan"), dtype=torch.bfloat16, device="cuda")
        r = torch.full((M,), float("nan"), dtype=torch.float32, device="cuda")
        Y = torch.full((M, F), float("nan"), dtype=torch.bfloat16, device="cuda")
        AB = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        st = _static_fwd(lib, t, H, r, Y, AB, M, K, d, N, eps)
        assert st == 0, f"coda_grg_fwd_prefolded_static returned {st}"
        torch.cuda.synchronize()
        for name, got in (("H", H), ("r", r), ("Y", Y), ("AB", AB)):
            assert torch.equal(got, ref[name]), f"static {name} differs from coda_grg_fwd (seed {seed})"
        assert _static_status(lib) == (0, 0)
        if seed == 11:
            refs.check_grg_fwd({"H": H, "r": r, "Y": Y, "AB": AB}, refs.grg(host, eps, bwd=False),
                               f"static fwd seed {seed}")


def test_static_scratch_forward_through_the_binding(cuda_lib):
    """The Python binding's wrapper calls the same entry point: bit-identical to
    coda_grg_fwd with the same pre-folded weight, and the status word reads 0."""
    M, K, d, F, eps = 256, 512, 512, 1024, 1e-6
    t = {k: v.cuda() for k, v in synth.grg_inputs(M, K, d, F, seed=13).items()}
    W2g = cuda_lib.fold_gain(t["W2"], t["g"])
    ref = cuda_lib.grg_fwd(t["X"], t["W1"], t["R"], t["g"], t["W2"], eps, W2g=W2g)
    got = cuda_lib.grg_fwd_prefolded_static(t["X"], t["W1"], t["R"], W2g, eps)
    assert cuda_lib.static_status() == (0, 0)
    for name in ("H", "r", "Y", "AB"):
        assert torch.equal(got[name], ref[name]), name


def test_static_scratch_forward_rejects_oversized_shapes(cuda_lib):
    lib = cuda_lib.library()
    fn = lib.coda_grg_fwd_prefolded_static
    P = ctypes.c_void_p
    fn.restype = ctypes.c_int
    fn.argtypes = [P] * 8 + [ctypes.c_int] * 4 + [ctypes.c_float, P]
    one = ctypes.c_void_p(256)
    # M * ceil(d/256) = 40000 * 32 > 2^20 partial sums: CODA_ERR_WORKSPACE_TOO_SMALL (4), nothing enqueued.
    assert fn(one, one, one, one, one, one, one, one, 40000, 64, 8192, 128, ctypes.c_float(1e-6), None) == 4
