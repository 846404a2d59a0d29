"""Reference results for the GPU parity tests: the pure fp64 oracle, the
storage-precision oracle and the per-element sigma of the pure comparison,
with the checks that apply them to one call's outputs (test infrastructure).

Two checks per output, both without outlier allowance:

* the whole chain (the GPU forward, then the GPU backward on the GPU's own
  saved tensors) against the pure fp64 oracle, at the stated bound widened by
  the deviation the bf16 storage points produce (tests/error_model.py);
* each entry point against the storage-precision oracle at the stated bound,
  on the same inputs: a backward entry point is given the saved tensors (H,
  r, [a|b], Y) that the storage-precision oracle's forward produced.  Fed the
  GPU's own saved tensors instead, the backward would inherit rounding flips:
  fp32 accumulation in GEMM1 rounds about 0.2% of H to the other bf16
  neighbour than fp64 does, which moves a and b enough to flip about 5% of
  the saved a, b and, through them, about a quarter of dR.
"""

from __future__ import annotations

import numpy as np
import torch

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
        ref["sb"] = E.sigma(E.grg_backward_var(f0, b0, vf, dY, X, W1, g, W2))
        # The backward entry point's saved inputs, as the storage-precision
        # forward produced them (r passed in fp32, the entry point's type).
        fin = {"H": fs["H"], "r": fs["r"].astype(np.float32).astype(np.float64), "a_s": fs["a_s"],
               "b_s": fs["b_s"]}
        ref["bwd_in"] = {"H": fin["H"], "r": fin["r"], "AB": np.concatenate([fin["a_s"], fin["b_s"]], axis=1)}
        ref["bs"] = O.grg_backward_stored(dY, X, W1, R, g, W2, eps, dH_in=dh, fwd=fin)
    return ref


def saved_inputs(ref: dict, device="cuda") -> dict:
    """The storage oracle's saved forward tensors as the backward entry point's
    inputs: bf16 H, [a|b] (and Y), fp32 r, on the device."""
    out = {}
    for k, v in ref["bwd_in"].items():
        dt = torch.float32 if k == "r" else torch.bfloat16
        out[k] = torch.from_numpy(np.ascontiguousarray(v)).to(dt).to(device)
    return out


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


def check_grg_bwd(b: dict, b_saved: dict, ref: dict, tag: str) -> None:
    """b: the backward on the GPU's own saved tensors (against the pure oracle);
    b_saved: the backward on the storage oracle's saved tensors (against the
    storage oracle)."""
    for k in GRG_BWD_KEYS:
        assert_tol(f64(b_saved[k]), ref["bs"][k], f"{tag} {k}")
        assert_pure(f64(b[k]), ref["b0"][k], f"{tag} {k}", ref["sb"][k])


def swiglu(t: dict) -> dict:
    X, Wgu, Wdown, dOut = (f64(t[k]) for k in ("X", "Wgu", "Wdown", "dOut"))
    f0 = O.swiglu_forward(X, Wgu, Wdown)
    b0 = O.swiglu_backward(dOut, X, Wgu, Wdown, fwd=f0)
    fs = O.swiglu_forward_stored(X, Wgu, Wdown)
    bs = O.swiglu_backward_stored(dOut, X, Wgu, Wdown, fwd=fs)
    bwd_in = {"Y": fs["Y_s"], "AB": np.concatenate([fs["a_s"], fs["b_s"]], axis=1)}
    return {"f0": f0, "b0": b0, "fs": fs, "bs": bs, "bwd_in": bwd_in,
            "s": E.sigma(E.swiglu_var(f0, b0, X, Wgu, Wdown, dOut))}


def check_swiglu(o: dict, b: dict, b_saved: dict, ref: dict, tag: str) -> None:
    F = ref["f0"]["a"].shape[1]
    fwd = {"Y": o["Y"], "a": o["AB"][:, :F], "b": o["AB"][:, F:], "Out": o["Out"]}
    for k, v in fwd.items():
        v = f64(v)
        assert_tol(v, ref["fs"][k], f"{tag} {k}")
        assert_pure(v, ref["f0"][k], f"{tag} {k}", ref["s"][k])
    for k in ("dX", "dWgu", "dWdown"):
        assert_tol(f64(b_saved[k]), ref["bs"][k], f"{tag} {k}")
        assert_pure(f64(b[k]), ref["b0"][k], f"{tag} {k}", ref["s"][k])


def mlp_block(t: dict, eps: float) -> dict:
    X, W1, R, g, W2, Wd, dOut = (f64(t[k]) for k in ("X", "W1", "R", "g", "W2", "Wdown", "dOut"))
    f0 = O.mlp_block_forward(X, W1, R, g, W2, Wd, eps)
    b0 = O.mlp_block_backward(dOut, X, W1, R, g, W2, Wd, eps, fwd=f0)
    fs = O.mlp_block_forward(X, W1, R, g, W2, Wd, eps, stored=True)
    fin = dict(fs)
    fin["r"] = fs["r"].astype(np.float32).astype(np.float64)
    bs = O.mlp_block_backward(dOut, X, W1, R, g, W2, Wd, eps, stored=True, fwd=fin)
    s = E.sigma(E.mlp_block_var(f0, b0, g, W2, Wd, dOut, b0["dY"], X, W1))
    bwd_in = {"H": fs["H"], "r": fin["r"], "AB": np.concatenate([fs["a_s"], fs["b_s"]], axis=1),
              "Y": O.round_bf16(fs["Y"])}
    return {"f0": f0, "b0": b0, "fs": fs, "bs": bs, "s": s, "bwd_in": bwd_in}


def check_mlp_block(o: dict, b: dict, b_saved: dict, ref: dict, tag: str) -> None:
    for k in ("Y", "Out"):
        v = f64(o[k])
        assert_tol(v, ref["fs"][k], f"{tag} {k}")
        assert_pure(v, ref["f0"][k], f"{tag} {k}", ref["s"][k])
    for k in GRG_BWD_KEYS + ("dWdown",):
        assert_tol(f64(b_saved[k]), ref["bs"][k], f"{tag} {k}")
        assert_pure(f64(b[k]), ref["b0"][k], f"{tag} {k}", ref["s"][k])


def release(*dicts) -> None:
    """Drop large arrays early (full-size checks hold several GB of float64)."""
    for d in dicts:
        if isinstance(d, dict):
            d.clear()


__all__ = ["grg", "saved_inputs", "check_grg_fwd", "check_grg_bwd", "swiglu", "check_swiglu", "mlp_block",
           "check_mlp_block", "release"]
