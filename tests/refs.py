"""Reference results for the GPU parity tests: the pure fp64 oracle, the
storage-precision oracle and the per-element sigma of the pure comparison,
with the checks that apply them to one call's outputs (test infrastructure)."""

from __future__ import annotations

import numpy as np

from oracle import coda_oracle as O
from tests import error_model as E
from tests.parity import assert_pure, assert_rel, assert_tol, f64

GRG_BWD_KEYS = ("dX", "dR", "dW1", "dW2", "dg")


def grg(t: dict, eps: float, gain: str = "weight", bwd: bool = True, dH_in: bool = False) -> dict:
    """Oracle results and sigmas for the GRG block on the host inputs t (bf16 tensors)."""
    X, W1, R, g, W2 = (f64(t[k]) for k in ("X", "W1", "R", "g", "W2"))
    f0 = O.grg_forward(X, W1, R, g, W2, eps)
    fs = O.grg_forward_stored(X, W1, R, g, W2, eps, gain=gain)
    vf = E.grg_forward_var(f0, g, W2, gain)
    ref = {"f0": f0, "fs": fs, "sf": E.sigma(vf)}
    if bwd:
        dY = f64(t["dY"])
        dh = f64(t["dH_in"]) if dH_in else None
        b0 = O.grg_backward(dY, X, W1, R, g, W2, eps, dH_in=dh, fwd=f0)
        ref["b0"] = b0
        ref["bs"] = O.grg_backward_stored(dY, X, W1, R, g, W2, eps, dH_in=dh, fwd=fs)
        ref["sb"] = E.sigma(E.grg_backward_var(f0, b0, vf, dY, X, W1, g, W2))
    return ref


def check_grg_fwd(o: dict, ref: dict, tag: str) -> None:
    """H, Y, a, b against both oracles; r within 1e-3 relative of both."""
    f0, fs, sf = ref["f0"], ref["fs"], ref["sf"]
    F = f0["a"].shape[1]
    gpu = {"H": o["H"], "Y": o["Y"], "a": o["AB"][:, :F], "b": o["AB"][:, F:]} if o.get("AB") is not None \
        else {"H": o["H"], "Y": o["Y"]}
    for k, v in gpu.items():
        v = f64(v)
        assert_tol(v, fs[k], f"{tag} {k}")
        assert_pure(v, f0[k], f"{tag} {k}", sf[k])
    assert_rel(o["r"], fs["r"], f"{tag} r")
    assert_rel(o["r"], f0["r"], f"{tag} r (vs pure fp64)")


def check_grg_bwd(b: dict, ref: dict, tag: str) -> None:
    for k in GRG_BWD_KEYS:
        v = f64(b[k])
        assert_tol(v, ref["bs"][k], f"{tag} {k}")
        assert_pure(v, ref["b0"][k], f"{tag} {k}", ref["sb"][k])


def swiglu(t: dict) -> dict:
    X, Wgu, Wdown, dOut = (f64(t[k]) for k in ("X", "Wgu", "Wdown", "dOut"))
    f0 = O.swiglu_forward(X, Wgu, Wdown)
    b0 = O.swiglu_backward(dOut, X, Wgu, Wdown, fwd=f0)
    fs = O.swiglu_forward_stored(X, Wgu, Wdown)
    bs = O.swiglu_backward_stored(dOut, X, Wgu, Wdown, fwd=fs)
    return {"f0": f0, "b0": b0, "fs": fs, "bs": bs, "s": E.sigma(E.swiglu_var(f0, b0, X, Wgu, Wdown, dOut))}


def check_swiglu(o: dict, b: dict, ref: dict, tag: str) -> None:
    F = ref["f0"]["a"].shape[1]
    gpu = {"Y": o["Y"], "a": o["AB"][:, :F], "b": o["AB"][:, F:], "Out": o["Out"],
           "dX": b["dX"], "dWgu": b["dWgu"], "dWdown": b["dWdown"]}
    for k, v in gpu.items():
        v = f64(v)
        src_s, src_0 = (ref["fs"], ref["f0"]) if k in ref["f0"] else (ref["bs"], ref["b0"])
        assert_tol(v, src_s[k], f"{tag} {k}")
        assert_pure(v, src_0[k], f"{tag} {k}", ref["s"][k])


def mlp_block(t: dict, eps: float) -> dict:
    X, W1, R, g, W2, Wd, dOut = (f64(t[k]) for k in ("X", "W1", "R", "g", "W2", "Wdown", "dOut"))
    f0 = O.mlp_block_forward(X, W1, R, g, W2, Wd, eps)
    b0 = O.mlp_block_backward(dOut, X, W1, R, g, W2, Wd, eps, fwd=f0)
    fs = O.mlp_block_forward(X, W1, R, g, W2, Wd, eps, stored=True)
    bs = O.mlp_block_backward(dOut, X, W1, R, g, W2, Wd, eps, stored=True, fwd=fs)
    s = E.sigma(E.mlp_block_var(f0, b0, g, W2, Wd, dOut, b0["dY"], X, W1))
    return {"f0": f0, "b0": b0, "fs": fs, "bs": bs, "s": s}


def check_mlp_block(o: dict, b: dict, ref: dict, tag: str) -> None:
    for k in ("Y", "Out"):
        v = f64(o[k])
        assert_tol(v, ref["fs"][k], f"{tag} {k}")
        assert_pure(v, ref["f0"][k], f"{tag} {k}", ref["s"][k])
    for k in GRG_BWD_KEYS + ("dWdown",):
        v = f64(b[k])
        assert_tol(v, ref["bs"][k], f"{tag} {k}")
        assert_pure(v, ref["b0"][k], f"{tag} {k}", ref["s"][k])


def release(*dicts) -> None:
    """Drop large arrays early (full-size checks hold several GB of float64)."""
    for d in dicts:
        if isinstance(d, dict):
            d.clear()


__all__ = ["grg", "check_grg_fwd", "check_grg_bwd", "swiglu", "check_swiglu", "mlp_block", "check_mlp_block",
           "release", "np"]
