"""Per-element error bounds for comparing the CUDA path with the pure fp64 oracle.

Test infrastructure (numpy only; no kernel and no oracle code).  The CUDA path
stores some tensors in bf16 between its GEMM-epilogue programs; each such
rounding perturbs every result downstream of it.  This module propagates
those perturbations to first order through the block's algebra, evaluated at
the pure oracle's values, and returns for every output element the standard
deviation sigma of the deviation they cause.  A GPU result then matches the
pure fp64 oracle when

    |gpu - ref| <= 1e-2 |ref| + 1e-2 rms(ref) + Z_TAIL * sigma

elementwise (tests/parity.py), i.e. the stated bf16 tolerance widened by
exactly what the stored roundings in that output's chain can account for.

Model.  Rounding x to bf16 (8 significant bits, to nearest) leaves an error
spread evenly over one unit in the last place, so its standard deviation is
ulp(x) / sqrt(12) with ulp(x) = 2^(e-8) for x = m 2^e, 0.5 <= |m| < 1 (and
no error where x is a bf16 value already).
Roundings of different elements are independent, so variances add: through a
contraction C = A B^T the variance is sigma_A^2 (B^2)^T + A^2 (sigma_B^2)^T,
and through an elementwise map it is the squared partial derivatives times the
input variances.  fp32 accumulation error (about 2^-24 sqrt(K) relative) is
negligible beside a bf16 unit and is not modelled.  tests/test_error_model.py
checks the model against the storage-precision oracle, which performs the
same roundings exactly: the deviations it predicts must have unit rms.
"""

from __future__ import annotations

import numpy as np

Z_TAIL = 7.0  # a normal deviate beyond 7 sigma has probability 2.6e-12 per element


def bf16_sigma(x) -> np.ndarray:
    """Standard deviation of the error of rounding x to bfloat16: ulp(x) / sqrt(12),
    and 0 where x is a bfloat16 value already (zeros, copied bf16 inputs)."""
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)
    exact = np.rint(m * 256.0) == m * 256.0
    return np.where(exact, 0.0, np.ldexp(1.0, e - 8)) / np.sqrt(12.0)


def _sig(x):
    out = np.empty_like(x)
    p = x >= 0
    out[p] = 1.0 / (1.0 + np.exp(-x[p]))
    q = np.exp(x[~p])
    out[~p] = q / (1.0 + q)
    return out


def _silu_derivs(a):
    """silu(a), silu'(a), silu''(a) with silu(a) = a sigmoid(a)."""
    s = _sig(a)
    d1 = s * (1.0 + a * (1.0 - s))
    d2 = s * (1.0 - s) * (2.0 + a * (1.0 - 2.0 * s))
    return a * s, d1, d2


def _mm_var(va, b2t):
    """Variance of (A @ B) from the variance of A and the squares of B.  A
    variance needs only a few significant digits, so the product runs in
    float32 (twice as fast as float64 in BLAS)."""
    return (np.asarray(va, dtype=np.float32) @ np.asarray(b2t, dtype=np.float32)).astype(np.float64)


def _swiglu_fwd_var(a, b, va, vb):
    """Variance of Y = silu(a) b from the variances of a and b."""
    s0, s1, _ = _silu_derivs(a)
    return (s1 * b) ** 2 * va + s0 ** 2 * vb


def _swiglu_bwd_var(dY, a, b, vdY, va, vb):
    """Variances of da = dY b silu'(a) and db = dY silu(a)."""
    s0, s1, s2 = _silu_derivs(a)
    vda = (b * s1) ** 2 * vdY + (dY * s1) ** 2 * vb + (dY * b * s2) ** 2 * va
    vdb = s0 ** 2 * vdY + (dY * s1) ** 2 * va
    return vda, vdb


# ----------------------------------------------------------------------------- fused block

def grg_forward_var(f0, g, W2, gain: str = "weight") -> dict:
    """Variances of the forward outputs.  Stored on the way: H (GEMM1's
    epilogue), W2g = bf16(W2 diag g) or Hg = bf16(H diag g) (GEMM2's operands)."""
    H, r = f0["H"], f0["r"]
    F = W2.shape[0] // 2
    vH = bf16_sigma(H) ** 2
    if gain == "weight":
        W2g = W2 * g[None, :]
        vZ = _mm_var(vH, (W2g ** 2).T) + _mm_var(H ** 2, (bf16_sigma(W2g) ** 2).T)
    else:
        vHg = vH * (g ** 2)[None, :] + bf16_sigma(H * g[None, :]) ** 2
        vZ = _mm_var(vHg, (W2 ** 2).T)
    vA = vZ * (r ** 2)[:, None]
    va, vb = vA[:, :F], vA[:, F:]
    return {"H": vH, "A": vA, "a": va, "b": vb, "Y": _swiglu_fwd_var(f0["a"], f0["b"], va, vb)}


def grg_backward_var(f0, b0, vf, dY, X, W1, g, W2, vdY=None) -> dict:
    """Variances of the backward outputs.  Stored on the way: the saved a, b,
    the r-scaled gradient dZ = bf16(r dA) (the operand of the dn and dW2
    GEMMs) and dR = bf16(dH) (the operand of the dX and dW1 GEMMs)."""
    H, r, a, b = f0["H"], f0["r"], f0["a"], f0["b"]
    d = H.shape[1]
    vas = vf["a"] + bf16_sigma(a) ** 2
    vbs = vf["b"] + bf16_sigma(b) ** 2
    vdY = np.zeros_like(dY) if vdY is None else vdY
    vda, vdb = _swiglu_bwd_var(dY, a, b, vdY, vas, vbs)
    dA = b0["dA"]
    dZ = dA * r[:, None]
    vdZ = np.concatenate([vda, vdb], axis=1) * (r ** 2)[:, None] + bf16_sigma(dZ) ** 2
    del vda, vdb
    P = dZ @ W2                                     # = r du
    vP = _mm_var(vdZ, W2 ** 2)
    c = (r ** 2 / d) * np.sum(dA * f0["A"], axis=1)
    vH = vf["H"]
    vdH = vP * (g ** 2)[None, :] + (c ** 2)[:, None] * vH
    dH = b0["dH"]
    vdRs = vdH + bf16_sigma(dH) ** 2
    out = {"dR": vdH, "dX": _mm_var(vdRs, W1 ** 2), "dW1": _mm_var(vdRs.T, X ** 2)}
    out["dW2"] = (_mm_var(vdZ.T, H ** 2) + _mm_var((dZ ** 2).T, vH)) * (g ** 2)[None, :]
    out["dg"] = np.sum(H ** 2 * vP + P ** 2 * vH, axis=0)
    return out


# ----------------------------------------------------------------------------- SwiGLU MLP

def swiglu_var(f0, b0, X, Wgu, Wdown, dOut) -> dict:
    """Variances of the MLP's outputs.  Stored on the way: Y (the down GEMM's
    operand), the saved a, b, and dA (the gate/up GEMM's adjoint operand)."""
    a, b, Y = f0["a"], f0["b"], f0["Y"]
    vYs = bf16_sigma(Y) ** 2
    out = {"a": np.zeros_like(a), "b": np.zeros_like(b), "Y": np.zeros_like(Y),
           "Out": _mm_var(vYs, (Wdown ** 2).T)}
    vda, vdb = _swiglu_bwd_var(b0["dY"], a, b, 0.0, bf16_sigma(a) ** 2, bf16_sigma(b) ** 2)
    vdA = np.concatenate([vda, vdb], axis=1) + bf16_sigma(b0["dA"]) ** 2
    out["dX"] = _mm_var(vdA, Wgu ** 2)
    out["dWgu"] = _mm_var(vdA.T, X ** 2)
    out["dWdown"] = _mm_var((dOut ** 2).T, vYs)
    return out


def mlp_block_var(f0, b0, g, W2, Wdown, dOut, dY, X, W1) -> dict:
    """The block followed by Out = Y Wdown^T + H: Y is stored for the down
    GEMM, whose epilogue reads the stored H; the backward is the block's with
    dY = dOut Wdown (never stored) and dH_in = dOut."""
    vf = grg_forward_var(f0, g, W2)
    vYs = vf["Y"] + bf16_sigma(f0["Y"]) ** 2
    out = {"Y": vf["Y"], "Out": _mm_var(vYs, (Wdown ** 2).T) + vf["H"]}
    out.update(grg_backward_var(f0, b0, vf, dY, X, W1, g, W2))
    out["dWdown"] = _mm_var((dOut ** 2).T, vYs)
    return out


# ----------------------------------------------------------------------------- LM head, RoPE

def stored_operand_var(G, X, W) -> dict:
    """A backward whose only stored tensor is the GEMM operand G (dlogits of the
    cross-entropy, the unrotated dpre of RoPE): dX = bf16(G) W, dW = bf16(G)^T X."""
    vG = bf16_sigma(G) ** 2
    return {"dX": _mm_var(vG, W ** 2), "dW": _mm_var(vG.T, X ** 2)}


# ----------------------------------------------------------------------------- unfused sequences

def grg_unfused_var(f0, b0, X, W1, g, W2, dY) -> dict:
    """The operator-by-operator sequence stores T = X W1^T, H, U = r H g, the
    GEMM output AB, Y, dA, du = dA W2 and dH, each in bf16."""
    H, r, u, a, b = f0["H"], f0["r"], f0["u"], f0["a"], f0["b"]
    F = W2.shape[0] // 2
    d = H.shape[1]
    vH = bf16_sigma(H) ** 2 + bf16_sigma(X @ W1.T) ** 2
    vU = vH * ((r[:, None] * g[None, :]) ** 2) + bf16_sigma(u) ** 2
    vA = _mm_var(vU, (W2 ** 2).T)
    va, vb = vA[:, :F], vA[:, F:]
    vas, vbs = va + bf16_sigma(a) ** 2, vb + bf16_sigma(b) ** 2
    out = {"H": vH, "a": va, "b": vb, "Y": _swiglu_fwd_var(a, b, vas, vbs)}
    vda, vdb = _swiglu_bwd_var(dY, a, b, 0.0, vas, vbs)
    dA, du, dH = b0["dA"], b0["du"], b0["dH"]
    vdA = np.concatenate([vda, vdb], axis=1) + bf16_sigma(dA) ** 2
    vdu = _mm_var(vdA, W2 ** 2) + bf16_sigma(du) ** 2
    coef = (r ** 3 / d) * np.sum(du * g[None, :] * H, axis=1)
    vdH = vdu * ((r[:, None] * g[None, :]) ** 2) + (coef ** 2)[:, None] * vH
    vdHs = vdH + bf16_sigma(dH) ** 2
    out["dR"] = vdH
    out["dX"] = _mm_var(vdHs, W1 ** 2)
    out["dW1"] = _mm_var(vdHs.T, X ** 2)
    out["dW2"] = _mm_var(vdA.T, u ** 2) + _mm_var((dA ** 2).T, vU)
    out["dg"] = np.sum((H * r[:, None]) ** 2 * vdu + (du * r[:, None]) ** 2 * vH, axis=0)
    return out


def swiglu_unfused_var(f0, b0, X, Wgu, Wdown, dOut) -> dict:
    """The MLP operator by operator: the GEMM output AB, Y, dY and dA stored in bf16."""
    a, b, Y = f0["a"], f0["b"], f0["Y"]
    vas, vbs = bf16_sigma(a) ** 2, bf16_sigma(b) ** 2
    vY = _swiglu_fwd_var(a, b, vas, vbs)
    vYs = vY + bf16_sigma(Y) ** 2
    out = {"Y": vY, "Out": _mm_var(vYs, (Wdown ** 2).T)}
    dY = b0["dY"]
    vda, vdb = _swiglu_bwd_var(dY, a, b, bf16_sigma(dY) ** 2, vas, vbs)
    vdA = np.concatenate([vda, vdb], axis=1) + bf16_sigma(b0["dA"]) ** 2
    out["dX"] = _mm_var(vdA, Wgu ** 2)
    out["dWgu"] = _mm_var(vdA.T, X ** 2)
    out["dWdown"] = _mm_var((dOut ** 2).T, vYs)
    return out


def sigma(var: dict) -> dict:
    """Standard deviations from a dict of variances."""
    return {k: np.sqrt(v) for k, v in var.items()}
