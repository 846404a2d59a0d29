"""GPU parity at the full LLaMA-shaped workload sizes, in the launch configuration bench.py times.

Every output element of every workload is compared with both oracles: the
storage-precision fp64 oracle at the stated tolerance (each entry point on
the same inputs: a backward is also run on the saved tensors the oracle's
forward produced), and the pure fp64 oracle, for the whole forward-backward
chain, at that tolerance widened by the deviation the method's bf16 storage
points produce in that element (tests/error_model.py).  No check allows
outliers.  The host's BLAS runs each full oracle in tens of seconds.
"""

import numpy as np
import pytest
import torch

from gemm_epilogue_fusion_tmem_b200 import synth
from oracle import coda_oracle as O
from tests import refs
from tests.parity import assert_rel, f64

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

GRG_FULL = [
    # (name, M, K, d, F, eps, backward)
    ("1B", 8192, 2048, 2048, 8192, 1e-6, False),
    ("7B", 8192, 4096, 4096, 11008, 1e-6, True),
    ("70B", 4096, 8192, 8192, 28672, 1e-5, True),
]


def _host(d):
    return {k: f64(v) if v is not None else None for k, v in d.items()}


@pytest.mark.parametrize("name,M,K,d,F,eps,bwd", GRG_FULL, ids=[c[0] for c in GRG_FULL])
def test_grg_full_size(cuda_lib, name, M, K, d, F, eps, bwd):
    _grg_full(cuda_lib, name, M, K, d, F, eps, bwd, "weight")


def test_grg_full_size_activation_gain(cuda_lib):
    """The 7B block with the gain on the activation side: Hg = bf16(H*g) from
    GEMM1's epilogue feeds GEMM2 (no fold), forward and backward."""
    _grg_full(cuda_lib, "7B hg", 8192, 4096, 4096, 11008, 1e-6, True, "activation")


def _grg_full(cuda_lib, name, M, K, d, F, eps, bwd, gain):
    t = synth.grg_inputs(M, K, d, F, seed=0)
    td = {k: v.cuda() for k, v in t.items()}
    fwd = cuda_lib.grg_fwd if gain == "weight" else cuda_lib.grg_fwd_hg
    o = fwd(td["X"], td["W1"], td["R"], td["g"], td["W2"], eps)
    b = None
    if bwd:
        b = cuda_lib.grg_bwd(td["dY"], td["X"], td["W1"], o["H"], o["r"], o["AB"], td["g"], td["W2"])
    torch.cuda.synchronize()
    st, detail = cuda_lib.workspace(256).query()
    assert st == 0, f"device status {st} detail {detail:#x}"
    go = _host(o)
    gb = _host(b) if b is not None else None
    del o, b
    torch.cuda.empty_cache()
    ref = refs.grg(t, eps, gain=gain, bwd=bwd)
    refs.check_grg_fwd(go, ref, name)
    if bwd:
        si = refs.saved_inputs(ref)
        bi = cuda_lib.grg_bwd(td["dY"], td["X"], td["W1"], si["H"], si["r"], si["AB"], td["g"], td["W2"])
        torch.cuda.synchronize()
        gbi = _host(bi)
        del bi, si
        refs.check_grg_bwd(gb, gbi, ref, name)
    del td
    refs.release(ref)


def test_grg_full_size_r(cuda_lib):
    """The fp32 row scale r of the 7B forward within 1e-3 relative of both oracles."""
    M, K, d, F, eps = 8192, 4096, 4096, 11008, 1e-6
    t = synth.grg_inputs(M, K, d, F, seed=0)
    td = {k: v.cuda() for k, v in t.items()}
    o = cuda_lib.grg_fwd(td["X"], td["W1"], td["R"], td["g"], td["W2"], eps, save_ab=False)
    torch.cuda.synchronize()
    X, W1, R = (f64(t[k]) for k in ("X", "W1", "R"))
    H = X @ W1.T + R
    r_pure = 1.0 / np.sqrt(np.mean(H * H, axis=1) + eps)
    Hs = O.round_bf16(H)
    r_st = 1.0 / np.sqrt(np.mean(Hs * Hs, axis=1) + eps)
    assert_rel(o["r"], r_st, "7B r")
    assert_rel(o["r"], r_pure, "7B r (vs pure fp64)")


def test_swiglu_full_size(cuda_lib):
    M, d, F = 16384, 4096, 14336
    t = synth.swiglu_inputs(M, d, F, seed=0)
    td = {k: v.cuda() for k, v in t.items()}
    o = cuda_lib.swiglu_fwd(td["X"], td["Wgu"], td["Wdown"])
    b = cuda_lib.swiglu_bwd(td["dOut"], td["X"], td["Wgu"], td["Wdown"], o["Y"], o["AB"])
    torch.cuda.synchronize()
    go, gb = _host(o), _host(b)
    del o, b
    torch.cuda.empty_cache()
    ref = refs.swiglu(t)
    si = refs.saved_inputs(ref)
    bi = cuda_lib.swiglu_bwd(td["dOut"], td["X"], td["Wgu"], td["Wdown"], si["Y"], si["AB"])
    torch.cuda.synchronize()
    gbi = _host(bi)
    del bi, si, td
    refs.check_swiglu(go, gb, gbi, ref, "swiglu")
    refs.release(ref)


def test_mlp_block_full_size(cuda_lib):
    """The full MLP block at the 7B shape (M=8192, K=d=4096, F=11008), fwd+bwd."""
    M, K, d, F, eps = 8192, 4096, 4096, 11008, 1e-6
    t = synth.mlp_block_inputs(M, K, d, F, seed=0)
    td = {k: v.cuda() for k, v in t.items()}
    o = cuda_lib.mlp_block_fwd(td["X"], td["W1"], td["R"], td["g"], td["W2"], td["Wdown"], eps)
    b = cuda_lib.mlp_block_bwd(td["dOut"], td["X"], td["W1"], o["H"], o["r"], o["AB"], o["Y"], td["g"], td["W2"],
                               td["Wdown"])
    torch.cuda.synchronize()
    go, gb = _host(o), _host(b)
    del o, b
    torch.cuda.empty_cache()
    ref = refs.mlp_block(t, eps)
    si = refs.saved_inputs(ref)
    bi = cuda_lib.mlp_block_bwd(td["dOut"], td["X"], td["W1"], si["H"], si["r"], si["AB"], si["Y"], td["g"],
                                td["W2"], td["Wdown"])
    torch.cuda.synchronize()
    gbi = _host(bi)
    del bi, si, td
    refs.check_mlp_block(go, gb, gbi, ref, "block 7B")
    refs.release(ref)
