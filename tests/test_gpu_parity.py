"""GPU parity: the CUDA path (through the C ABI) against the fp64 CPU oracle.

Small and ragged shapes that span several tiles and a ragged tail, compared
element by element with |gpu - ref| <= 1e-2 |ref| + 1e-2 rms(ref) for bf16
outputs and 1e-3 relative for r against the oracle at the method's storage
precision (the *_stored functions: the same fp64 arithmetic with each tensor
the method stores between passes rounded to bf16), and against the pure fp64
oracle within that bound widened by the per-element deviation the storage
roundings produce (tests/error_model.py); plus structured cases whose integer
tile/row indexing is checked bit-exactly.  No check allows outliers.
"""

import numpy as np
import pytest
import torch

from gemm_epilogue_fusion_tmem_b200 import synth
from oracle import coda_oracle as O
from tests import refs
from tests.parity import assert_rel, assert_tol, f64

pytestmark = pytest.mark.gpu


def _cuda(d):
    return {k: v.cuda() for k, v in d.items()}


# ----------------------------------------------------------------------------- plain GEMM core

GEMM_CASES = [
    # (M, N, K): ragged M, ragged N tile, several k-blocks
    (200, 512, 320),
    (1, 256, 64),
    (384, 288, 4160),
    (2048, 4096, 256),  # 256 tiles > 148 SMs: persistent loop, both TMEM accumulators
    (136, 96, 200),     # reduction not a multiple of 64 (zero-filled tail), N < one tile
]


@pytest.mark.parametrize("a_mn", [False, True])
@pytest.mark.parametrize("b_mn", [False, True])
@pytest.mark.parametrize("M,N,K", GEMM_CASES)
def test_gemm_core(cuda_lib, M, N, K, a_mn, b_mn):
    if a_mn and M % 8:
        pytest.skip("MN-major A needs M % 8 == 0")
    t = synth.gemm_inputs(M, N, K, seed=M + N + K)
    A, B = t["A"], t["B"]
    Ad = A.t().contiguous().cuda() if a_mn else A.cuda()
    Bd = B.t().contiguous().cuda() if b_mn else B.cuda()
    C = cuda_lib.gemm(Ad, Bd, M, N, K, a_mn_major=a_mn, b_mn_major=b_mn)
    torch.cuda.synchronize()
    assert_tol(C, O.gemm(f64(A), f64(B)), f"gemm M={M} N={N} K={K} a_mn={a_mn} b_mn={b_mn}")


def test_gemm_ragged_reduction_mn_major(cuda_lib):
    """Reduction length not a multiple of the 64-deep stage (zero-filled tail), both MN-major."""
    M, N, K = 256, 512, 200
    t = synth.gemm_inputs(M, N, K, seed=3)
    C = cuda_lib.gemm(t["A"].t().contiguous().cuda(), t["B"].t().contiguous().cuda(), M, N, K, True, True)
    torch.cuda.synchronize()
    assert_tol(C, O.gemm(f64(t["A"]), f64(t["B"])), "gemm ragged K")


# ----------------------------------------------------------------------------- GRG forward / backward

GRG_CASES = [
    # (M, K, d, F, eps)
    (256, 512, 512, 1024, 1e-6),     # the tiny workload
    (200, 320, 384, 320, 1e-5),      # ragged M, ragged partial-RMS tile, ragged F tile, K != d
    (1, 64, 256, 128, 1e-6),         # a single token
    (2048, 1024, 1024, 2816, 1e-6),  # > 148 tiles in the gate/up GEMM
]


@pytest.mark.parametrize("M,K,d,F,eps", GRG_CASES)
def test_grg_forward(cuda_lib, M, K, d, F, eps):
    t = synth.grg_inputs(M, K, d, F, seed=1)
    td = _cuda(t)
    o = cuda_lib.grg_fwd(td["X"], td["W1"], td["R"], td["g"], td["W2"], eps)
    torch.cuda.synchronize()
    refs.check_grg_fwd(o, refs.grg(t, eps, bwd=False), f"grg_fwd M={M} K={K} d={d} F={F}")


def test_grg_forward_prefolded_weight(cuda_lib):
    M, K, d, F, eps = 256, 512, 512, 1024, 1e-6
    t = synth.grg_inputs(M, K, d, F, seed=2)
    td = _cuda(t)
    W2g = cuda_lib.fold_gain(td["W2"], td["g"])
    o = cuda_lib.grg_fwd(td["X"], td["W1"], td["R"], td["g"], td["W2"], eps, W2g=W2g)
    torch.cuda.synchronize()
    assert_tol(W2g, f64(t["W2"]) * f64(t["g"])[None, :], "W2g", rel=4e-3, rms_frac=0.0)
    refs.check_grg_fwd(o, refs.grg(t, eps, bwd=False), "grg_fwd prefolded")


@pytest.mark.parametrize("N,d", [(384, 192), (8192, 1024), (2, 4096)])
def test_fold_gain_bit_exact(cuda_lib, N, d):
    """W2g = bf16(W2 * g): the fp32 product of two bf16 values is exact, so the
    only rounding is the final round-to-nearest-even, and the kernel must match
    the oracle's rounding of the exact product bit for bit (sizes with a ragged
    last grid-stride step, several steps, and fewer vectors than threads)."""
    gen = torch.Generator().manual_seed(N + d)
    W2 = torch.randn(N, d, generator=gen).to(torch.bfloat16)
    g = (1 + 0.1 * torch.randn(d, generator=gen)).to(torch.bfloat16)
    W2g = cuda_lib.fold_gain(W2.cuda(), g.cuda())
    torch.cuda.synchronize()
    ref = O.round_bf16(f64(W2) * f64(g)[None, :])
    np.testing.assert_array_equal(f64(W2g), ref)


@pytest.mark.parametrize("with_dH_in", [False, True])
@pytest.mark.parametrize("M,K,d,F,eps", GRG_CASES)
def test_grg_backward(cuda_lib, M, K, d, F, eps, with_dH_in):
    t = synth.grg_inputs(M, K, d, F, seed=4, dH_in=with_dH_in)
    td = _cuda(t)
    o = cuda_lib.grg_fwd(td["X"], td["W1"], td["R"], td["g"], td["W2"], eps)
    b = cuda_lib.grg_bwd(td["dY"], td["X"], td["W1"], o["H"], o["r"], o["AB"], td["g"], td["W2"],
                         dH_in=td.get("dH_in"))
    torch.cuda.synchronize()
    ref = refs.grg(t, eps, dH_in=with_dH_in)
    si = refs.saved_inputs(ref)
    bi = cuda_lib.grg_bwd(td["dY"], td["X"], td["W1"], si["H"], si["r"], si["AB"], td["g"], td["W2"],
                          dH_in=td.get("dH_in"))
    torch.cuda.synchronize()
    refs.check_grg_bwd(b, bi, ref, f"grg_bwd M={M} K={K} d={d} F={F} dH_in={with_dH_in}")


def test_grg_structured_exact_indexing(cuda_lib):
    """X = 0, R one-hot v at (i, j), W2 = [I; I], g = 1 (F = d).

    Then H = R exactly, the partial sum of squares is v^2 in cell (i, j // 256)
    and 0 elsewhere (bit-exact tile/row indexing), r_i = 1/sqrt(v^2/d + eps),
    every other row has r = 1/sqrt(eps), and a = b = r H.
    """
    M, K, d, eps, v = 300, 128, 768, 1e-6, 3.0
    F = d
    X = torch.zeros(M, K, dtype=torch.bfloat16)
    W1 = synth.gemm_inputs(d, 32, K, seed=5)["A"]
    eye = torch.eye(d, dtype=torch.bfloat16)
    W2 = torch.cat([eye, eye], dim=0)
    g = torch.ones(d, dtype=torch.bfloat16)
    for (i, j) in [(0, 0), (131, 300), (299, 767), (257, 511)]:
        R = torch.zeros(M, d, dtype=torch.bfloat16)
        R[i, j] = v
        ws = cuda_lib.Workspace(cuda_lib.library().coda_grg_fwd_workspace_bytes(M, K, d, 2 * F, 0))
        o = cuda_lib.grg_fwd(X.cuda(), W1.cuda(), R.cuda(), g.cuda(), W2.cuda(), eps, ws=ws)
        torch.cuda.synchronize()
        assert torch.equal(o["H"].cpu(), R), "H must equal R bit for bit"
        T = -(-d // 256)
        P = ws.buf[256:256 + M * T * 4].view(torch.float32).view(M, T).cpu().numpy()
        expect = np.zeros((M, T), dtype=np.float32)
        expect[i, j // 256] = v * v
        np.testing.assert_array_equal(P, expect)
        r_exp = np.full(M, 1.0 / np.sqrt(eps))
        r_exp[i] = 1.0 / np.sqrt(v * v / d + eps)
        assert_rel(o["r"], r_exp, "r one-hot")
        a = f64(o["AB"][:, :F])
        b = f64(o["AB"][:, F:])
        np.testing.assert_array_equal(a, b)
        assert a[i, j] == pytest.approx(r_exp[i] * v, rel=1e-2)
        a[i, j] = 0.0
        assert not np.any(a), "only the one-hot entry may be nonzero"


def test_grg_zero_rows_forward_backward(cuda_lib):
    """Tokens whose X and R rows are zero: H = 0 there, so RMSNorm's degenerate
    case r = 1/sqrt(eps) applies, a = b = Y = 0, and the backward gives dA' = 0,
    dH = dR = 0 and dX = 0 in those rows, exactly.  Every output also matches
    the oracle at the usual tolerance."""
    M, K, d, F, eps = 256, 512, 512, 1024, 1e-6
    t = synth.grg_inputs(M, K, d, F, seed=13)
    zero = [0, 77, 255]
    t["X"][zero] = 0
    t["R"][zero] = 0
    td = _cuda(t)
    o = cuda_lib.grg_fwd(td["X"], td["W1"], td["R"], td["g"], td["W2"], eps)
    b = cuda_lib.grg_bwd(td["dY"], td["X"], td["W1"], o["H"], o["r"], o["AB"], td["g"], td["W2"])
    torch.cuda.synchronize()
    ref = refs.grg(t, eps)
    refs.check_grg_fwd(o, ref, "grg_fwd zero rows")
    si = refs.saved_inputs(ref)
    bi = cuda_lib.grg_bwd(td["dY"], td["X"], td["W1"], si["H"], si["r"], si["AB"], td["g"], td["W2"])
    torch.cuda.synchronize()
    refs.check_grg_bwd(b, bi, ref, "grg_bwd zero rows")
    r = o["r"].cpu().numpy()
    np.testing.assert_allclose(r[zero], 1.0 / np.sqrt(eps), rtol=1e-6)
    for name, v in (("H", o["H"]), ("Y", o["Y"]), ("AB", o["AB"]), ("dX", b["dX"]), ("dR", b["dR"])):
        assert torch.count_nonzero(v[zero]).item() == 0, name


# ----------------------------------------------------------------------------- SwiGLU MLP

SWIGLU_CASES = [
    (200, 256, 320),
    (512, 512, 1024),
    (1, 64, 64),
]


@pytest.mark.parametrize("M,d,F", SWIGLU_CASES)
def test_swiglu_forward_backward(cuda_lib, M, d, F):
    t = synth.swiglu_inputs(M, d, F, seed=6)
    td = _cuda(t)
    o = cuda_lib.swiglu_fwd(td["X"], td["Wgu"], td["Wdown"])
    b = cuda_lib.swiglu_bwd(td["dOut"], td["X"], td["Wgu"], td["Wdown"], o["Y"], o["AB"])
    torch.cuda.synchronize()
    ref = refs.swiglu(t)
    si = refs.saved_inputs(ref)
    bi = cuda_lib.swiglu_bwd(td["dOut"], td["X"], td["Wgu"], td["Wdown"], si["Y"], si["AB"])
    torch.cuda.synchronize()
    refs.check_swiglu(o, b, bi, ref, f"swiglu M={M} d={d} F={F}")


def test_status_word_stays_clear(cuda_lib):
    ws = cuda_lib.workspace(1 << 20)
    st, detail = ws.query()
    assert st == 0 and detail == 0, f"device status {st} detail {detail:#x}"


# ----------------------------------------------------------------------------- gain on the activation side

@pytest.mark.parametrize("M,K,d,F,eps", GRG_CASES)
def test_grg_forward_activation_gain(cuda_lib, M, K, d, F, eps):
    """coda_grg_fwd_hg: Hg = bf16(H*g) from GEMM1's epilogue feeds GEMM2 with
    the unmodified W2.  Hg is the stored H times g, rounded once: given the
    GPU's own H, it must match bf16(H*g) bit for bit (the product of two bf16
    values is exact in fp32)."""
    t = synth.grg_inputs(M, K, d, F, seed=7)
    td = _cuda(t)
    o = cuda_lib.grg_fwd_hg(td["X"], td["W1"], td["R"], td["g"], td["W2"], eps, keep_hg=True)
    b = cuda_lib.grg_bwd(td["dY"], td["X"], td["W1"], o["H"], o["r"], o["AB"], td["g"], td["W2"])
    torch.cuda.synchronize()
    tag = f"grg_fwd_hg M={M} K={K} d={d} F={F}"
    ref = refs.grg(t, eps, gain="activation")
    refs.check_grg_fwd(o, ref, tag)
    np.testing.assert_array_equal(f64(o["Hg"]), O.round_bf16(f64(o["H"]) * f64(t["g"])[None, :]))
    si = refs.saved_inputs(ref)
    bi = cuda_lib.grg_bwd(td["dY"], td["X"], td["W1"], si["H"], si["r"], si["AB"], td["g"], td["W2"])
    torch.cuda.synchronize()
    refs.check_grg_bwd(b, bi, ref, f"{tag} bwd")


def test_run_to_run_bit_reproducible(cuda_lib):
    """Partials + fixed-order reduces (no atomics): two runs give identical bits."""
    M, K, d, F, eps = 2048, 1024, 1024, 2816, 1e-6
    t = synth.grg_inputs(M, K, d, F, seed=9, dH_in=True)
    td = _cuda(t)
    outs = []
    for _ in range(2):
        o = cuda_lib.grg_fwd(td["X"], td["W1"], td["R"], td["g"], td["W2"], eps)
        b = cuda_lib.grg_bwd(td["dY"], td["X"], td["W1"], o["H"], o["r"], o["AB"], td["g"], td["W2"],
                             dH_in=td["dH_in"])
        torch.cuda.synchronize()
        outs.append({k: v.clone() for k, v in {**o, **b}.items()})
    for k in outs[0]:
        assert torch.equal(outs[0][k], outs[1][k]), f"{k} differs between runs"


def test_rows_are_independent_under_permutation(cuda_lib):
    """Permuting token rows permutes every row-local output bit for bit (row i of
    H, r, Y, AB, dX, dR depends on row i only); the weight gradients, sums over
    rows, agree within the bf16 bound."""
    M, K, d, F, eps = 640, 512, 768, 640, 1e-6
    t = synth.grg_inputs(M, K, d, F, seed=13)
    perm = torch.randperm(M, generator=torch.Generator().manual_seed(1))
    tp = dict(t)
    for k in ("X", "R", "dY"):
        tp[k] = t[k][perm].contiguous()
    res = []
    for src in (t, tp):
        td = _cuda(src)
        o = cuda_lib.grg_fwd(td["X"], td["W1"], td["R"], td["g"], td["W2"], eps)
        b = cuda_lib.grg_bwd(td["dY"], td["X"], td["W1"], o["H"], o["r"], o["AB"], td["g"], td["W2"])
        torch.cuda.synchronize()
        res.append({k: v.cpu() for k, v in {**o, **b}.items()})
    a, p = res
    for k in ("H", "r", "Y", "AB", "dX", "dR"):
        assert torch.equal(a[k][perm], p[k]), f"{k}: row results depend on row position"
    for k in ("dW1", "dW2", "dg"):
        assert_tol(p[k], f64(a[k]), f"{k} under row permutation")
