"""Shared helpers for GPU-vs-oracle parity checks (no method arithmetic here)."""

from __future__ import annotations

import numpy as np
import torch

# Tolerances: bf16 outputs |gpu - ref| <= 1e-2 |ref| + 1e-2 rms(ref) elementwise;
# the fp32 RMSNorm row scale r within 1e-3 relative.
BF16_REL = 1e-2
BF16_RMS = 1e-2
R_REL = 1e-3

# Backward outputs downstream of the stored bf16 operands (dA' scaled by r, then
# dH) may differ from the storage-precision oracle in a few elements: a value of
# H within fp32 accumulation error of a bf16 rounding midpoint rounds one way on
# the GPU and the other in fp64, which moves r_i by ~1e-5 and re-rounds part of
# row i's stored operands.  At most a 1e-5 fraction of elements may exceed the
# bound, none by more than 2x.
BWD_OUTLIER_FRAC = 1e-5


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def assert_tol(gpu, ref, name: str, rel: float = BF16_REL, rms_frac: float = BF16_RMS,
               outlier_frac: float = 0.0, outlier_factor: float = 2.0) -> dict:
    """Elementwise |gpu - ref| <= rel |ref| + rms_frac rms(ref).

    outlier_frac > 0 admits at most ceil(outlier_frac * size) elements above the
    bound, none above outlier_factor times it (used only for backward outputs
    that sit behind three stored bf16 operands; see BWD_OUTLIER_FRAC)."""
    g = f64(gpu) if isinstance(gpu, torch.Tensor) else np.asarray(gpu, dtype=np.float64)
    r = np.asarray(ref, dtype=np.float64)
    assert g.shape == r.shape, f"{name}: shape {g.shape} vs {r.shape}"
    assert np.all(np.isfinite(g)), f"{name}: non-finite values in GPU output"
    rms = float(np.sqrt(np.mean(r * r))) if r.size else 0.0
    err = np.abs(g - r)
    bound = rel * np.abs(r) + rms_frac * rms
    bad = err > bound
    n_bad = int(bad.sum())
    if n_bad and outlier_frac > 0 and n_bad <= int(np.ceil(outlier_frac * bad.size)) \
            and np.all(err <= outlier_factor * bound):
        bad = np.zeros_like(bad)
    if np.any(bad):
        idx = np.unravel_index(np.argmax(err - bound), err.shape)
        raise AssertionError(
            f"{name}: {int(bad.sum())}/{bad.size} elements out of tolerance; worst at {idx}: "
            f"gpu={g[idx]:.6g} ref={r[idx]:.6g} |err|={err[idx]:.3g} bound={bound[idx]:.3g} (rms(ref)={rms:.3g})")
    return {"max_abs": float(err.max()) if err.size else 0.0, "rms_ref": rms,
            "rel_rms_err": float(np.sqrt(np.mean(err * err)) / rms) if rms > 0 else 0.0}


def assert_rel(gpu, ref, name: str, rel: float = R_REL) -> None:
    g = f64(gpu) if isinstance(gpu, torch.Tensor) else np.asarray(gpu, dtype=np.float64)
    r = np.asarray(ref, dtype=np.float64)
    e = np.abs(g - r) / np.maximum(np.abs(r), 1e-30)
    assert np.all(e <= rel), f"{name}: max relative error {e.max():.3e} > {rel}"


# Against the pure-fp64 oracle (no storage rounding) the bf16 storage of the
# method's intermediates adds deviations of a few units of 2^-8 relative, which
# SwiGLU amplifies by up to ~|b|: elementwise 1e-2 |ref| + 1e-1 rms(ref), and an
# rms deviation below 1e-2 rms(ref).
PURE_RMS_BOUND = 1e-1
PURE_RMS_ERR = 1e-2


def assert_pure(gpu, ref, name: str) -> None:
    assert_tol(gpu, ref, name + " (vs pure fp64)", rel=BF16_REL, rms_frac=PURE_RMS_BOUND)
    g = f64(gpu) if isinstance(gpu, torch.Tensor) else np.asarray(gpu, dtype=np.float64)
    r = np.asarray(ref, dtype=np.float64)
    rms = float(np.sqrt(np.mean(r * r)))
    e = float(np.sqrt(np.mean((g - r) ** 2)))
    assert e <= PURE_RMS_ERR * rms, f"{name}: rms deviation {e:.3g} > {PURE_RMS_ERR} * rms(ref) {rms:.3g}"
