"""GPU parity at the full LLaMA-shaped workload sizes, in the launch configuration bench.py times.

Every output element is compared with the storage-precision fp64 oracle (the
host's BLAS runs the full oracle in tens of seconds); the 1B forward and the 7B
block are also compared with the pure fp64 oracle within the derived bound.
"""

import pytest
import torch

from gemm_epilogue_fusion_tmem_b200 import synth
from oracle import coda_oracle as O
from tests.parity import BWD_OUTLIER_FRAC, assert_pure, assert_rel, assert_tol, f64

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

GRG_FULL = [
    # (name, M, K, d, F, eps, backward, also_pure)
    ("1B", 8192, 2048, 2048, 8192, 1e-6, False, True),
    ("7B", 8192, 4096, 4096, 11008, 1e-6, True, True),
    ("70B", 4096, 8192, 8192, 28672, 1e-5, True, False),
]


@pytest.mark.parametrize("name,M,K,d,F,eps,bwd,also_pure", GRG_FULL, ids=[c[0] for c in GRG_FULL])
def test_grg_full_size(cuda_lib, name, M, K, d, F, eps, bwd, also_pure):
    t = synth.grg_inputs(M, K, d, F, seed=0)
    td = {k: v.cuda() for k, v in t.items()}
    o = cuda_lib.grg_fwd(td["X"], td["W1"], td["R"], td["g"], td["W2"], eps)
    b = None
    if bwd:
        b = cuda_lib.grg_bwd(td["dY"], td["X"], td["W1"], o["H"], o["r"], o["AB"], td["g"], td["W2"])
    torch.cuda.synchronize()
    st, detail = cuda_lib.workspace(256).query()
    assert st == 0, f"device status {st} detail {detail:#x}"
    gpu = {"H": o["H"], "Y": o["Y"], "a": o["AB"][:, :F], "b": o["AB"][:, F:]}
    gpu = {k: f64(v) for k, v in gpu.items()}
    gb = {k: f64(v) for k, v in b.items()} if b is not None else {}
    del o, b, td
    torch.cuda.empty_cache()
    X, W1, R, g, W2 = (f64(t[k]) for k in ("X", "W1", "R", "g", "W2"))
    fs = O.grg_forward_stored(X, W1, R, g, W2, eps)
    for k, v in gpu.items():
        assert_tol(v, fs[k], f"{name} {k}")
    if bwd:
        bs = O.grg_backward_stored(f64(t["dY"]), X, W1, R, g, W2, eps, fwd=fs)
        for k in ("dX", "dR", "dW1", "dW2", "dg"):
            assert_tol(gb[k], bs[k], f"{name} {k}", outlier_frac=BWD_OUTLIER_FRAC)
        del bs
    del fs
    if also_pure:
        f0 = O.grg_forward(X, W1, R, g, W2, eps)
        for k, v in gpu.items():
            assert_pure(v, f0[k], f"{name} {k}")
        if bwd:
            b0 = O.grg_backward(f64(t["dY"]), X, W1, R, g, W2, eps, fwd=f0)
            for k in ("dX", "dR", "dW1", "dW2", "dg"):
                assert_pure(gb[k], b0[k], f"{name} {k}")


def test_grg_full_size_activation_gain(cuda_lib):
    """The 7B forward with Hg = bf16(H*g) from GEMM1 feeding GEMM2 (no gain fold)."""
    M, K, d, F, eps = 8192, 4096, 4096, 11008, 1e-6
    t = synth.grg_inputs(M, K, d, F, seed=0)
    td = {k: v.cuda() for k, v in t.items()}
    o = cuda_lib.grg_fwd_hg(td["X"], td["W1"], td["R"], td["g"], td["W2"], eps)
    torch.cuda.synchronize()
    gpu = {"H": f64(o["H"]), "Y": f64(o["Y"]), "a": f64(o["AB"][:, :F]), "b": f64(o["AB"][:, F:])}
    del o, td
    X, W1, R, g, W2 = (f64(t[k]) for k in ("X", "W1", "R", "g", "W2"))
    fs = O.grg_forward_stored(X, W1, R, g, W2, eps, gain="activation")
    for k, v in gpu.items():
        assert_tol(v, fs[k], f"7B hg {k}")


def test_grg_full_size_r(cuda_lib):
    """The fp32 row scale r of the 7B forward within 1e-3 relative of both oracles."""
    M, K, d, F, eps = 8192, 4096, 4096, 11008, 1e-6
    t = synth.grg_inputs(M, K, d, F, seed=0)
    td = {k: v.cuda() for k, v in t.items()}
    o = cuda_lib.grg_fwd(td["X"], td["W1"], td["R"], td["g"], td["W2"], eps, save_ab=False)
    torch.cuda.synchronize()
    X, W1, R = (f64(t[k]) for k in ("X", "W1", "R"))
    H = X @ W1.T + R
    import numpy as np
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
    gpu = {"Y": o["Y"], "a": o["AB"][:, :F], "b": o["AB"][:, F:], "Out": o["Out"], **b}
    gpu = {k: f64(v) for k, v in gpu.items()}
    del o, b, td
    torch.cuda.empty_cache()
    X, Wgu, Wdown, dOut = (f64(t[k]) for k in ("X", "Wgu", "Wdown", "dOut"))
    fs = O.swiglu_forward_stored(X, Wgu, Wdown)
    bs = O.swiglu_backward_stored(dOut, X, Wgu, Wdown, fwd=fs)
    for k in ("Y", "a", "b", "Out"):
        assert_tol(gpu[k], fs[k], f"swiglu {k}")
    for k in ("dX", "dWgu", "dWdown"):
        assert_tol(gpu[k], bs[k], f"swiglu {k}", outlier_frac=BWD_OUTLIER_FRAC)


def test_mlp_block_full_size(cuda_lib):
    """The full MLP block at the 7B shape (M=8192, K=d=4096, F=11008), fwd+bwd."""
    from tests.parity import assert_tol as _tol
    M, K, d, F, eps = 8192, 4096, 4096, 11008, 1e-6
    t = synth.mlp_block_inputs(M, K, d, F, seed=0)
    td = {k: v.cuda() for k, v in t.items()}
    o = cuda_lib.mlp_block_fwd(td["X"], td["W1"], td["R"], td["g"], td["W2"], td["Wdown"], eps)
    b = cuda_lib.mlp_block_bwd(td["dOut"], td["X"], td["W1"], o["H"], o["r"], o["AB"], o["Y"], td["g"], td["W2"],
                               td["Wdown"])
    torch.cuda.synchronize()
    gf = {k: f64(o[k]) for k in ("Y", "Out")}
    gb = {k: f64(v) for k, v in b.items()}
    del o, b, td
    torch.cuda.empty_cache()
    X, W1, R, g, W2, Wd, dOut = (f64(t[k]) for k in ("X", "W1", "R", "g", "W2", "Wdown", "dOut"))
    fs = O.mlp_block_forward(X, W1, R, g, W2, Wd, eps, stored=True)
    for k, v in gf.items():
        _tol(v, fs[k], f"block 7B {k}")
    bs = O.mlp_block_backward(dOut, X, W1, R, g, W2, Wd, eps, stored=True, fwd=fs)
    for k in ("dX", "dR", "dW1", "dW2", "dg", "dWdown"):
        _tol(gb[k], bs[k], f"block 7B {k}", outlier_frac=BWD_OUTLIER_FRAC)
