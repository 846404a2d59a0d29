"""An empty batch (M = 0 tokens) through every entry point.

Nothing is read and no row is written; each weight gradient is a sum over
no rows, so the backward calls must write exact zeros (checked bit for bit,
over output buffers that start as garbage) and agree with the oracle run on
the same empty inputs.  A plain GEMM with an empty reduction (K = 0) writes
C = 0.
"""

import numpy as np
import pytest
import torch

from gemm_epilogue_fusion_tmem_b200 import synth
from oracle import coda_oracle as O
from tests.parity import f64

pytestmark = pytest.mark.gpu


def _cuda(d):
    return {k: v.cuda() for k, v in d.items()}


def _garbage(*shape, dtype=torch.bfloat16):
    return torch.full(shape, 7.0, dtype=dtype, device="cuda")


def _zero(t, ref, name):
    torch.cuda.synchronize()
    assert t.shape == tuple(ref.shape), name
    assert torch.count_nonzero(t).item() == 0, name
    assert np.all(ref == 0), name  # the oracle's empty sums


def test_grg_empty_batch(cuda_lib):
    M, K, d, F = 0, 256, 256, 512
    N = 2 * F
    t = synth.grg_inputs(M, K, d, F, seed=5)
    td = _cuda(t)
    o = cuda_lib.grg_fwd(td["X"], td["W1"], td["R"], td["g"], td["W2"], 1e-6)
    assert o["H"].shape == (0, d) and o["Y"].shape == (0, F) and o["AB"].shape == (0, N)
    out = {"dW1": _garbage(d, K), "dW2": _garbage(N, d), "dg": _garbage(d, dtype=torch.float32)}
    b = cuda_lib.grg_bwd(td["dY"], td["X"], td["W1"], o["H"], o["r"], o["AB"], td["g"], td["W2"], out=out)
    ref = O.grg_backward(*(f64(t[k]) for k in ("dY", "X", "W1", "R", "g", "W2")), 1e-6)
    for k in ("dW1", "dW2", "dg"):
        _zero(b[k], ref[k], f"grg {k}")
    assert b["dX"].shape == (0, K) and b["dR"].shape == (0, d)


def test_grg_unfused_and_activation_gain_empty_batch(cuda_lib):
    M, K, d, F = 0, 256, 256, 512
    N = 2 * F
    td = _cuda(synth.grg_inputs(M, K, d, F, seed=6))
    o = cuda_lib.grg_fwd_hg(td["X"], td["W1"], td["R"], td["g"], td["W2"], 1e-6)
    assert o["Y"].shape == (0, F)
    u = cuda_lib.grg_fwd_unfused(td["X"], td["W1"], td["R"], td["g"], td["W2"], 1e-6)
    out = {"dW1": _garbage(d, K), "dW2": _garbage(N, d), "dg": _garbage(d, dtype=torch.float32)}
    b = cuda_lib.grg_bwd_unfused(td["dY"], td["X"], td["W1"], u["H"], u["r"], u["AB"], u["U"], td["g"], td["W2"],
                                 out=out)
    torch.cuda.synchronize()
    for k in ("dW1", "dW2", "dg"):
        assert torch.count_nonzero(b[k]).item() == 0, k


def test_swiglu_empty_batch(cuda_lib):
    M, d, F = 0, 256, 512
    t = synth.swiglu_inputs(M, d, F, seed=7)
    td = _cuda(t)
    o = cuda_lib.swiglu_fwd(td["X"], td["Wgu"], td["Wdown"])
    assert o["Out"].shape == (0, d)
    out = {"dWgu": _garbage(2 * F, d), "dWdown": _garbage(d, F)}
    b = cuda_lib.swiglu_bwd(td["dOut"], td["X"], td["Wgu"], td["Wdown"], o["Y"], o["AB"], out=out)
    ref = O.swiglu_backward(*(f64(t[k]) for k in ("dOut", "X", "Wgu", "Wdown")))
    _zero(b["dWgu"], ref["dWgu"], "swiglu dWgu")
    _zero(b["dWdown"], ref["dWdown"], "swiglu dWdown")


def test_mlp_block_empty_batch(cuda_lib):
    M, K, d, F = 0, 256, 256, 512
    td = _cuda(synth.mlp_block_inputs(M, K, d, F, seed=8))
    o = cuda_lib.mlp_block_fwd(td["X"], td["W1"], td["R"], td["g"], td["W2"], td["Wdown"], 1e-6)
    assert o["Out"].shape == (0, d)
    out = {"dW1": _garbage(d, K), "dW2": _garbage(2 * F, d), "dg": _garbage(d, dtype=torch.float32),
           "dWdown": _garbage(d, F)}
    b = cuda_lib.mlp_block_bwd(td["dOut"], td["X"], td["W1"], o["H"], o["r"], o["AB"], o["Y"], td["g"], td["W2"],
                               td["Wdown"], out=out)
    torch.cuda.synchronize()
    for k in ("dW1", "dW2", "dg", "dWdown"):
        assert torch.count_nonzero(b[k]).item() == 0, k


def test_xent_and_rope_empty_batch(cuda_lib):
    M, d, V = 0, 256, 512
    t = synth.xent_inputs(M, d, V, seed=9)
    td = _cuda(t)
    f = cuda_lib.xent_fwd(td["X"], td["W"], td["targets"])
    assert f["loss"].shape == (0,)
    b = cuda_lib.xent_bwd(td["X"], td["W"], td["targets"], f["lse"], td["dloss"], out={"dW": _garbage(V, d)})
    ref = O.xent_backward(f64(t["dloss"]), f64(t["X"]), f64(t["W"]), t["targets"].numpy())
    _zero(b["dW"], ref["dW"], "xent dW")
    n_q, n_kv, hd = 2, 1, 64
    q = _cuda(synth.qkv_inputs(M, d, n_q, n_kv, hd, seed=10))
    Q = cuda_lib.qkv_rope_fwd(q["X"], q["Wqkv"], n_q, n_kv, hd, 16)
    assert Q.shape == (0, (n_q + 2 * n_kv) * hd)
    rb = cuda_lib.qkv_rope_bwd(q["dQKV"], q["X"], q["Wqkv"], n_q, n_kv, hd, 16,
                               out={"dW": _garbage((n_q + 2 * n_kv) * hd, d)})
    torch.cuda.synchronize()
    assert torch.count_nonzero(rb["dW"]).item() == 0


def test_gemm_empty_output_and_empty_reduction(cuda_lib):
    A0, B = torch.empty(0, 64, dtype=torch.bfloat16, device="cuda"), _garbage(128, 64)
    C0 = cuda_lib.gemm(A0, B, 0, 128, 64)
    assert C0.shape == (0, 128)
    A, Bk = torch.empty(96, 0, dtype=torch.bfloat16, device="cuda"), torch.empty(128, 0, dtype=torch.bfloat16,
                                                                               device="cuda")
    C = cuda_lib.gemm(A, Bk, 96, 128, 0, out=_garbage(96, 128))
    torch.cuda.synchronize()
    assert torch.count_nonzero(C).item() == 0
    assert np.all(O.gemm(np.zeros((96, 0)), np.zeros((128, 0))) == 0)
