"""The full MLP block (block + down projection with residual) against the fp64 oracle.

The backward's down-projection dgrad carries the SwiGLU backward, the r scale
and the c-row partials in its epilogue; outputs are compared like the block's
(bf16 bound against the storage-precision oracle, the outlier allowance for
the deep backward chain, the derived bound against pure fp64).
"""

import pytest
import torch

from gemm_epilogue_fusion_tmem_b200 import synth
from oracle import coda_oracle as O
from tests.parity import BWD_OUTLIER_FRAC, assert_pure, assert_tol, f64

pytestmark = pytest.mark.gpu

CASES = [
    (256, 512, 512, 1024, 1e-6),
    (200, 320, 384, 320, 1e-5),
    (2048, 1024, 1024, 2816, 1e-6),
]


@pytest.mark.parametrize("M,K,d,F,eps", CASES)
def test_mlp_block_forward_backward(cuda_lib, M, K, d, F, eps):
    t = synth.mlp_block_inputs(M, K, d, F, seed=31)
    td = {k: v.cuda() for k, v in t.items()}
    o = cuda_lib.mlp_block_fwd(td["X"], td["W1"], td["R"], td["g"], td["W2"], td["Wdown"], eps)
    b = cuda_lib.mlp_block_bwd(td["dOut"], td["X"], td["W1"], o["H"], o["r"], o["AB"], o["Y"], td["g"], td["W2"],
                               td["Wdown"])
    torch.cuda.synchronize()
    X, W1, R, g, W2, Wd, dOut = (f64(t[k]) for k in ("X", "W1", "R", "g", "W2", "Wdown", "dOut"))
    fs = O.mlp_block_forward(X, W1, R, g, W2, Wd, eps, stored=True)
    f0 = O.mlp_block_forward(X, W1, R, g, W2, Wd, eps)
    tag = f"block M={M} K={K} d={d} F={F}"
    for k in ("H", "Y", "Out"):
        assert_tol(o[k], fs[k], f"{tag} {k}")
        assert_pure(o[k], f0[k], f"{tag} {k}")
    bs = O.mlp_block_backward(dOut, X, W1, R, g, W2, Wd, eps, stored=True, fwd=fs)
    b0 = O.mlp_block_backward(dOut, X, W1, R, g, W2, Wd, eps, fwd=f0)
    for k in ("dX", "dR", "dW1", "dW2", "dg", "dWdown"):
        assert_tol(b[k], bs[k], f"{tag} {k}", outlier_frac=BWD_OUTLIER_FRAC)
        assert_pure(b[k], b0[k], f"{tag} {k}")
