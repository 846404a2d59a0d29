"""The full MLP block (block + down projection with residual) against the fp64 oracle.

The backward's down-projection dgrad carries the SwiGLU backward, the r scale
and the c-row partials in its epilogue; outputs are compared like the block's
(bf16 bound against the storage-precision oracle; against pure fp64 the same
bound widened by the deviation the stored roundings produce, with no outlier
allowance).
"""

import pytest
import torch

from gemm_epilogue_fusion_tmem_b200 import synth
from tests import refs
from tests.parity import assert_tol, f64

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
    tag = f"block M={M} K={K} d={d} F={F}"
    ref = refs.mlp_block(t, eps)
    assert_tol(o["H"], ref["fs"]["H"], f"{tag} H")
    si = refs.saved_inputs(ref)
    bi = cuda_lib.mlp_block_bwd(td["dOut"], td["X"], td["W1"], si["H"], si["r"], si["AB"], si["Y"], td["g"],
                                td["W2"], td["Wdown"])
    torch.cuda.synchronize()
    refs.check_mlp_block(o, b, bi, ref, tag)
