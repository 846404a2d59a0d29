"""Shared helpers for GPU-vs-oracle parity checks (no method arithmetic here).

Two comparisons, both elementwise and without any allowance for outliers:

* against the storage-precision oracle (the *_stored functions, which round
  to bf16 exactly the tensors the method stores between its GEMM-epilogue
  programs): the stated tolerance, |gpu - ref| <= 1e-2 |ref| + 1e-2 rms(ref)
  for bf16 outputs and 1e-3 relative for the fp32 row scale r;
* against the pure fp64 oracle (no rounding anywhere): the same bound plus
  Z_TAIL times the per-element standard deviation that the method's bf16
  storage points produce in that output (tests/error_model.py).

Every check records its worst |err| / bound and the number of elements above
the bound; tests/conftest.py prints them at the end of the session and, when
CODA_PARITY_REPORT names a file, writes them there as JSON lines.
"""

from __future__ import annotations

import numpy as np
import torch

from tests.error_model import Z_TAIL

BF16_REL = 1e-2
BF16_RMS = 1e-2
R_REL = 1e-3

REPORT: list = []


def f64(t) -> np.ndarray:
    if isinstance(t, torch.Tensor):
        return t.detach().to("cpu", torch.float64).numpy()
    return np.asarray(t, dtype=np.float64)


def _check(gpu, ref, name: str, rel: float, rms_frac: float, sigma=None, kind: str = "stored") -> dict:
    g = f64(gpu)
    r = np.asarray(ref, dtype=np.float64)
    assert g.shape == r.shape, f"{name}: shape {g.shape} vs {r.shape}"
    assert np.all(np.isfinite(g)), f"{name}: non-finite values in GPU output"
    rms = float(np.sqrt(np.mean(r * r))) if r.size else 0.0
    err = np.abs(g - r)
    bound = rel * np.abs(r) + rms_frac * rms
    if sigma is not None:
        bound = bound + Z_TAIL * np.asarray(sigma, dtype=np.float64)
    with np.errstate(divide="ignore", invalid="ignore"):
        ratio = np.where(bound > 0, err / bound, np.where(err > 0, np.inf, 0.0))
    n_bad = int(np.count_nonzero(ratio > 1.0))
    worst = float(ratio.max()) if ratio.size else 0.0
    rec = {"check": name, "kind": kind, "n": int(r.size), "worst_ratio": round(worst, 4), "above_bound": n_bad,
           "rel_rms_err": float(np.sqrt(np.mean(err * err)) / rms) if rms > 0 else 0.0}
    REPORT.append(rec)
    if n_bad:
        idx = np.unravel_index(int(np.argmax(ratio)), ratio.shape)
        raise AssertionError(
            f"{name}: {n_bad}/{r.size} elements out of tolerance; worst at {idx}: gpu={g[idx]:.6g} "
            f"ref={r[idx]:.6g} |err|={err[idx]:.3g} bound={bound[idx]:.3g} (rms(ref)={rms:.3g})")
    return rec


def assert_tol(gpu, ref, name: str, rel: float = BF16_REL, rms_frac: float = BF16_RMS) -> dict:
    """Elementwise |gpu - ref| <= rel |ref| + rms_frac rms(ref) (against the storage-precision oracle)."""
    return _check(gpu, ref, name, rel, rms_frac, None, "stored")


def assert_pure(gpu, ref, name: str, sigma=None) -> dict:
    """Elementwise |gpu - ref| <= 1e-2 |ref| + 1e-2 rms(ref) + Z_TAIL sigma against
    the pure fp64 oracle; sigma is the error model's per-element deviation of
    this output (None where the chain stores nothing in bf16)."""
    return _check(gpu, ref, name + " (vs pure fp64)", BF16_REL, BF16_RMS, sigma, "pure")


def assert_rel(gpu, ref, name: str, rel: float = R_REL) -> dict:
    g = f64(gpu)
    r = np.asarray(ref, dtype=np.float64)
    e = np.abs(g - r) / np.maximum(np.abs(r), 1e-30)
    worst = float(e.max() / rel) if e.size else 0.0
    n_bad = int(np.count_nonzero(e > rel))
    REPORT.append({"check": name, "kind": "relative", "n": int(r.size), "worst_ratio": round(worst, 4),
                   "above_bound": n_bad, "rel_rms_err": float(np.sqrt(np.mean(e * e))) if e.size else 0.0})
    assert n_bad == 0, f"{name}: max relative error {e.max():.3e} > {rel}"
    return REPORT[-1]
