"""QKV projection with the RoPE epilogue against the fp64 oracle.

The rotation angles are computed in fp32 on the GPU (pos * 2^(j * k)), as
common LLaMA implementations do; at positions below 2^13 the angle error is
below 1e-3 rad, so the bf16 bound |gpu - ref| <= 1e-2 |ref| + 1e-2 rms(ref)
holds against the fp64 angles of the oracle.  The backward's stored operand
(the inverse-rotated gradient) is bf16, compared like the block's gradients:
against pure fp64 the bound is widened by the deviation its rounding produces.
"""

import pytest
import torch

from gemm_epilogue_fusion_tmem_b200 import synth
from oracle import coda_oracle as O
from tests import error_model as E
from tests.parity import assert_pure, assert_tol, f64

pytestmark = pytest.mark.gpu

CASES = [
    # (M, d, n_q, n_kv, head_dim, seq_len, base)
    (200, 256, 2, 1, 128, 64, 10000.0),     # GQA, ragged rows, sequences wrapping inside the batch
    (256, 512, 4, 4, 64, 256, 500000.0),    # MHA, head_dim 64, LLaMA-3 base
    (512, 1024, 8, 2, 256, 512, 10000.0),
    (8192, 4096, 32, 32, 128, 2048, 10000.0),  # LLaMA-7B attention input projection
]


@pytest.mark.parametrize("M,d,nq,nkv,hd,S,base", CASES)
def test_qkv_rope_forward_backward(cuda_lib, M, d, nq, nkv, hd, S, base):
    t = synth.qkv_inputs(M, d, nq, nkv, hd, seed=M + hd)
    td = {k: v.cuda() for k, v in t.items()}
    Q = cuda_lib.qkv_rope_fwd(td["X"], td["Wqkv"], nq, nkv, hd, S, base)
    b = cuda_lib.qkv_rope_bwd(td["dQKV"], td["X"], td["Wqkv"], nq, nkv, hd, S, base)
    torch.cuda.synchronize()
    X, W, dQ = f64(t["X"]), f64(t["Wqkv"]), f64(t["dQKV"])
    f = O.qkv_rope_forward(X, W, nq, nkv, hd, S, base)
    tag = f"rope M={M} d={d} heads={nq}/{nkv}x{hd} S={S}"
    assert_tol(Q, f["QKV"], f"{tag} QKV")
    bs = O.qkv_rope_backward(dQ, X, W, nq, nkv, hd, S, base, store=O.round_bf16)
    b0 = O.qkv_rope_backward(dQ, X, W, nq, nkv, hd, S, base)
    assert_pure(Q, f["QKV"], f"{tag} QKV")
    sg = E.sigma(E.stored_operand_var(b0["dpre"], X, W))
    for k in ("dX", "dW"):
        assert_tol(b[k], bs[k], f"{tag} {k}")
        assert_pure(b[k], b0[k], f"{tag} {k}", sg[k])
