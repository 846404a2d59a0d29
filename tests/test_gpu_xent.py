"""Cross-entropy on the LM-head GEMM (online max/sum-exp epilogue) against the fp64 oracle.

loss and lse are fp32 results of fp32-accumulated logits: |gpu - ref| <=
1e-4 |ref| + 1e-4 (fp32 accumulation over d bf16 products and fp32 exp/log
give errors near 1e-6; the bound leaves two orders of margin).  dX and dW come
from bf16-stored dlogits: the bf16 bound against the storage-precision oracle,
and against pure fp64 that bound widened by the deviation the rounding of
dlogits produces (tests/error_model.py), as for the block.
"""

import numpy as np
import pytest
import torch

from gemm_epilogue_fusion_tmem_b200 import synth
from oracle import coda_oracle as O
from tests import error_model as E
from tests.parity import assert_pure, assert_tol, f64

pytestmark = pytest.mark.gpu

CASES = [
    (200, 256, 1088),    # ragged rows, last 256-column tile ragged (64 columns)
    (1, 128, 512),
    (1024, 512, 8192),
]


def _check(o, b, t, M, d, V, tag):
    X, W, dloss = f64(t["X"]), f64(t["W"]), t["dloss"].double().numpy()
    tg = t["targets"].long().numpy()
    fwd = O.xent_forward(X, W, tg)
    for k in ("loss", "lse"):
        g = f64(o[k])
        err = np.abs(g - fwd[k])
        assert np.all(err <= 1e-4 * np.abs(fwd[k]) + 1e-4), f"{tag} {k}: max err {err.max():.3g}"
    if b is not None:
        bs = O.xent_backward(dloss, X, W, tg, fwd=fwd, store=O.round_bf16)
        b0 = O.xent_backward(dloss, X, W, tg, fwd=fwd)
        sg = E.sigma(E.stored_operand_var(b0["dlogits"], X, W))
        for k in ("dX", "dW"):
            assert_tol(b[k], bs[k], f"{tag} {k}")
            assert_pure(b[k], b0[k], f"{tag} {k}", sg[k])


@pytest.mark.parametrize("M,d,V", CASES)
def test_xent_forward_backward(cuda_lib, M, d, V):
    t = synth.xent_inputs(M, d, V, seed=M + V)
    t["targets"][0] = V - 1                       # the last column of the ragged tile
    if M > 1:
        t["targets"][1] = 0
    td = {k: v.cuda() for k, v in t.items()}
    o = cuda_lib.xent_fwd(td["X"], td["W"], td["targets"])
    b = cuda_lib.xent_bwd(td["X"], td["W"], td["targets"], o["lse"], td["dloss"])
    torch.cuda.synchronize()
    _check(o, b, t, M, d, V, f"xent M={M} d={d} V={V}")


def test_xent_out_of_range_target_gives_nan(cuda_lib):
    M, d, V = 64, 128, 256
    t = synth.xent_inputs(M, d, V, seed=3)
    t["targets"][5] = V + 7
    td = {k: v.cuda() for k, v in t.items()}
    o = cuda_lib.xent_fwd(td["X"], td["W"], td["targets"])
    torch.cuda.synchronize()
    loss = o["loss"].cpu().numpy()
    assert np.isnan(loss[5]) and np.all(np.isfinite(np.delete(loss, 5)))


@pytest.mark.slow
def test_xent_full_llama3_vocab(cuda_lib):
    """M = 8192 tokens, d = 4096, V = 128256 (LLaMA-3 vocabulary): logits never stored.

    loss and lse are compared for every row.  dX is compared on 256 sampled
    token rows and dW on 512 sampled vocabulary rows, each element against
    both oracles: the oracle's dX row i needs only row i of dlogits and its
    dW row v only column v, given the lse of every row (one fp64 logits GEMM)."""
    M, d, V = 8192, 4096, 128256
    t = synth.xent_inputs(M, d, V, seed=0)
    td = {k: v.cuda() for k, v in t.items()}
    o = cuda_lib.xent_fwd(td["X"], td["W"], td["targets"])
    b = cuda_lib.xent_bwd(td["X"], td["W"], td["targets"], o["lse"], td["dloss"])
    torch.cuda.synchronize()
    o = {k: f64(v) for k, v in o.items()}
    b = {k: f64(v) for k, v in b.items()}
    del td
    torch.cuda.empty_cache()
    X, W, dloss = f64(t["X"]), f64(t["W"]), t["dloss"].double().numpy()
    tg = t["targets"].long().numpy()
    fwd = O.xent_forward(X, W, tg)
    tag = "xent 8192x4096x128256"
    for k in ("loss", "lse"):
        err = np.abs(o[k] - fwd[k])
        assert np.all(err <= 1e-4 * np.abs(fwd[k]) + 1e-4), f"{tag} {k}: max err {err.max():.3g}"
    gen = np.random.default_rng(7)
    rows = np.sort(gen.choice(M, 256, replace=False))
    cols = np.sort(np.concatenate([gen.choice(V, 510, replace=False), [0, V - 1]]))
    # dlogits restricted to the sampled rows (all columns) and to the sampled columns (all rows)
    p_rows = np.exp(fwd["logits"][rows] - fwd["lse"][rows, None])
    p_rows[np.arange(rows.size), tg[rows]] -= 1.0
    dl_rows = p_rows * dloss[rows, None]
    p_cols = np.exp(fwd["logits"][:, cols] - fwd["lse"][:, None])
    p_cols[tg[:, None] == cols[None, :]] -= 1.0
    dl_cols = p_cols * dloss[:, None]
    del fwd
    for name, dl in (("pure", dl_rows), ("stored", O.round_bf16(dl_rows))):
        ref = dl @ W
        if name == "stored":
            assert_tol(b["dX"][rows], ref, f"{tag} dX (sampled rows)")
        else:
            sg = E.sigma(E.stored_operand_var(dl_rows, X[rows], W))["dX"]
            assert_pure(b["dX"][rows], ref, f"{tag} dX (sampled rows)", sg)
    for name, dl in (("pure", dl_cols), ("stored", O.round_bf16(dl_cols))):
        ref = dl.T @ X
        if name == "stored":
            assert_tol(b["dW"][cols], ref, f"{tag} dW (sampled rows)")
        else:
            sg = np.sqrt((E.bf16_sigma(dl_cols) ** 2).T @ X ** 2)
            assert_pure(b["dW"][cols], ref, f"{tag} dW (sampled rows)", sg)
