"""The unfused comparison sequence, and the fused path's error against it.

The unfused calls run the block operator by operator (every intermediate in
HBM).  They are checked against the pure fp64 oracle within the stated bound
widened by the deviation their own bf16 intermediates produce
(tests/error_model.py), and the fused path's error must be comparable or smaller:
the pages report the reparameterisation's numerical error as comparable to the
PyTorch reference and sometimes smaller, thanks to the mainloop's fp32
accumulator (kucoin.com (ru) CODA article, section «Результаты эксперимента»).
The comparison is rms error against the pure fp64 oracle, fused <= 1.5x
unfused (the factor is a chosen allowance, not a figure from the pages).
"""

import numpy as np
import pytest
import torch

from gemm_epilogue_fusion_tmem_b200 import synth
from oracle import coda_oracle as O
from tests import error_model as E
from tests.parity import assert_pure, f64

pytestmark = pytest.mark.gpu

CASES = [
    (256, 512, 512, 1024, 1e-6),
    (200, 320, 384, 320, 1e-5),
    (2048, 1024, 1024, 2816, 1e-6),
]


def _rms_err(gpu, ref):
    g = f64(gpu)
    return float(np.sqrt(np.mean((g - ref) ** 2)))


@pytest.mark.parametrize("M,K,d,F,eps", CASES)
def test_unfused_matches_oracle_and_fused_error_is_comparable(cuda_lib, M, K, d, F, eps):
    t = synth.grg_inputs(M, K, d, F, seed=21, dH_in=True)
    td = {k: v.cuda() for k, v in t.items()}
    fu = cuda_lib.grg_fwd(td["X"], td["W1"], td["R"], td["g"], td["W2"], eps)
    bu = cuda_lib.grg_bwd(td["dY"], td["X"], td["W1"], fu["H"], fu["r"], fu["AB"], td["g"], td["W2"],
                          dH_in=td["dH_in"])
    uf = cuda_lib.grg_fwd_unfused(td["X"], td["W1"], td["R"], td["g"], td["W2"], eps)
    ub = cuda_lib.grg_bwd_unfused(td["dY"], td["X"], td["W1"], uf["H"], uf["r"], uf["AB"], uf["U"], td["g"],
                                  td["W2"], dH_in=td["dH_in"])
    torch.cuda.synchronize()
    X, W1, R, g, W2, dY, dH_in = (f64(t[k]) for k in ("X", "W1", "R", "g", "W2", "dY", "dH_in"))
    fwd = O.grg_forward(X, W1, R, g, W2, eps)
    bwd = O.grg_backward(dY, X, W1, R, g, W2, eps, dH_in=dH_in, fwd=fwd)
    tag = f"M={M} K={K} d={d} F={F}"
    unf = {"H": uf["H"], "Y": uf["Y"], "a": uf["AB"][:, :F], "b": uf["AB"][:, F:], **ub}
    fus = {"H": fu["H"], "Y": fu["Y"], "a": fu["AB"][:, :F], "b": fu["AB"][:, F:], **bu}
    ref = {**{k: fwd[k] for k in ("H", "Y", "a", "b")}, **{k: bwd[k] for k in ("dX", "dR", "dW1", "dW2", "dg")}}
    sg = E.sigma(E.grg_unfused_var(fwd, bwd, X, W1, g, W2, dY))
    for k, v in unf.items():
        assert_pure(v, ref[k], f"unfused {tag} {k}", sg[k])
    np.testing.assert_allclose(f64(uf["r"]), fwd["r"], rtol=1e-3)
    for k in ref:
        e_f, e_u = _rms_err(fus[k], ref[k]), _rms_err(unf[k], ref[k])
        rms = float(np.sqrt(np.mean(ref[k] ** 2)))
        assert e_f <= 1.5 * e_u + 1e-4 * rms, f"{tag} {k}: fused rms error {e_f:.3g} vs unfused {e_u:.3g}"


@pytest.mark.parametrize("M,d,F", [(200, 256, 320), (512, 512, 1024)])
def test_swiglu_unfused_matches_oracle_and_fused_error_is_comparable(cuda_lib, M, d, F):
    t = synth.swiglu_inputs(M, d, F, seed=22)
    td = {k: v.cuda() for k, v in t.items()}
    fo = cuda_lib.swiglu_fwd(td["X"], td["Wgu"], td["Wdown"])
    fb = cuda_lib.swiglu_bwd(td["dOut"], td["X"], td["Wgu"], td["Wdown"], fo["Y"], fo["AB"])
    uo = cuda_lib.swiglu_fwd_unfused(td["X"], td["Wgu"], td["Wdown"])
    ub = cuda_lib.swiglu_bwd_unfused(td["dOut"], td["X"], td["Wgu"], td["Wdown"], uo["Y"], uo["AB"])
    torch.cuda.synchronize()
    X, Wgu, Wdown, dOut = (f64(t[k]) for k in ("X", "Wgu", "Wdown", "dOut"))
    fwd = O.swiglu_forward(X, Wgu, Wdown)
    bwd = O.swiglu_backward(dOut, X, Wgu, Wdown, fwd=fwd)
    ref = {"Y": fwd["Y"], "Out": fwd["Out"], "dX": bwd["dX"], "dWgu": bwd["dWgu"], "dWdown": bwd["dWdown"]}
    unf = {"Y": uo["Y"], "Out": uo["Out"], **ub}
    fus = {"Y": fo["Y"], "Out": fo["Out"], **fb}
    tag = f"swiglu M={M} d={d} F={F}"
    sg = E.sigma(E.swiglu_unfused_var(fwd, bwd, X, Wgu, Wdown, dOut))
    for k, v in unf.items():
        assert_pure(v, ref[k], f"unfused {tag} {k}", sg[k])
    for k in ref:
        e_f, e_u = _rms_err(fus[k], ref[k]), _rms_err(unf[k], ref[k])
        rms = float(np.sqrt(np.mean(ref[k] ** 2)))
        assert e_f <= 1.5 * e_u + 1e-4 * rms, f"{tag} {k}: fused rms error {e_f:.3g} vs unfused {e_u:.3g}"
