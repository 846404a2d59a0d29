"""Pins for tests/error_model.py, the per-element deviation model behind the
pure-oracle bound (CPU only).

The model claims that the bf16 storage points of a dataflow move each output
element by a deviation of standard deviation sigma.  Each test here runs the
same dataflow with the roundings actually applied (the storage-precision
oracle, or the operator-by-operator chain written out below) and checks that
(stored - pure) / sigma has unit rms and stays far inside Z_TAIL: a model that
forgot a storage point, mis-scaled a derivative or dropped a term of a
contraction's variance fails this.
"""

import numpy as np
import pytest
import torch

from oracle import coda_oracle as O
from tests import error_model as E


def _assert_unit(stored, pure, sig, name, lo=0.85, covered=0.9):
    """(stored - pure) / sigma has rms in (lo, 1.15) and stays below Z_TAIL - 1;
    where sigma is 0 (no rounding reaches the element) the two agree exactly
    up to float64 round-off."""
    stored, pure, sig = (np.asarray(x, dtype=np.float64) for x in (stored, pure, sig))
    m = sig > 0
    assert m.mean() > covered, f"{name}: sigma is zero on {1 - m.mean():.1%} of the elements"
    scale = float(np.abs(pure).max())
    assert np.all(np.abs(stored[~m] - pure[~m]) <= 1e-12 * scale), f"{name}: deviation where sigma = 0"
    z = (stored[m] - pure[m]) / sig[m]
    rms, mx = float(np.sqrt(np.mean(z * z))), float(np.abs(z).max())
    assert lo < rms < 1.15, f"{name}: rms of (stored - pure) / sigma is {rms:.3f}"
    assert mx < E.Z_TAIL - 1.0, f"{name}: max |z| {mx:.2f}"


def test_bf16_sigma_closed_form_and_library_rounding():
    assert E.bf16_sigma(1.0 + 2.0 ** -9) == 2.0 ** -7 / np.sqrt(12.0)
    assert E.bf16_sigma(-3.0 - 2.0 ** -9) == 2.0 ** -6 / np.sqrt(12.0)
    assert E.bf16_sigma(0.0) == 0.0 and E.bf16_sigma(1.0) == 0.0 and E.bf16_sigma(1.0 + 2.0 ** -7) == 0.0
    gen = torch.Generator().manual_seed(3)
    # float32 inputs: torch rounds float32 -> bfloat16 once, to nearest even
    x = torch.randn(400000, generator=gen) * torch.exp(torch.randn(400000, generator=gen))
    err = (x.to(torch.bfloat16).to(torch.float64) - x.to(torch.float64)).numpy()
    sig = E.bf16_sigma(x.to(torch.float64).numpy())
    assert np.all(err[sig == 0] == 0)
    z = err[sig > 0] / sig[sig > 0]
    assert abs(np.sqrt(np.mean(z * z)) - 1.0) < 0.01
    assert np.abs(z).max() <= np.sqrt(3.0) + 1e-12   # uniform over one ulp: at most sqrt(12) / 2


def _grg_inputs(seed, M=192, K=256, d=384, F=320):
    rng = np.random.default_rng(seed)
    bf = O.round_bf16
    return dict(X=bf(rng.standard_normal((M, K))), R=bf(rng.standard_normal((M, d))),
                W1=bf(rng.standard_normal((d, K)) / np.sqrt(K)), W2=bf(rng.standard_normal((2 * F, d)) / np.sqrt(d)),
                g=bf(1 + 0.1 * rng.standard_normal(d)), dY=bf(rng.standard_normal((M, F))),
                dH_in=bf(rng.standard_normal((M, d))))


@pytest.mark.parametrize("gain", ["weight", "activation"])
def test_grg_model_matches_the_storage_oracle(gain):
    p = _grg_inputs(1)
    eps = 1e-6
    args = (p["X"], p["W1"], p["R"], p["g"], p["W2"], eps)
    f0 = O.grg_forward(*args)
    fs = O.grg_forward_stored(*args, gain=gain)
    b0 = O.grg_backward(p["dY"], *args, dH_in=p["dH_in"], fwd=f0)
    bs = O.grg_backward_stored(p["dY"], *args, dH_in=p["dH_in"], fwd=fs)
    vf = E.grg_forward_var(f0, p["g"], p["W2"], gain)
    vb = E.grg_backward_var(f0, b0, vf, p["dY"], p["X"], p["W1"], p["g"], p["W2"])
    for k in ("a", "b", "Y"):
        _assert_unit(fs[k], f0[k], np.sqrt(vf[k]), f"{gain} {k}")
    _assert_unit(fs["H"], f0["H"], np.sqrt(vf["H"]), f"{gain} H")
    for k in ("dX", "dR", "dW1", "dW2", "dg"):
        _assert_unit(bs[k], b0[k], np.sqrt(vb[k]), f"{gain} {k}")


def test_swiglu_and_block_models_match_the_storage_oracle():
    rng = np.random.default_rng(2)
    bf = O.round_bf16
    M, d, F, K = 192, 256, 320, 128
    X = bf(rng.standard_normal((M, d)))
    Wgu, Wd = bf(rng.standard_normal((2 * F, d)) / np.sqrt(d)), bf(rng.standard_normal((d, F)) / np.sqrt(F))
    dOut = bf(rng.standard_normal((M, d)))
    f0 = O.swiglu_forward(X, Wgu, Wd)
    b0 = O.swiglu_backward(dOut, X, Wgu, Wd, fwd=f0)
    fs = O.swiglu_forward_stored(X, Wgu, Wd)
    bs = O.swiglu_backward_stored(dOut, X, Wgu, Wd, fwd=fs)
    v = E.swiglu_var(f0, b0, X, Wgu, Wd, dOut)
    _assert_unit(fs["Out"], f0["Out"], np.sqrt(v["Out"]), "swiglu Out")
    for k in ("dX", "dWgu", "dWdown"):
        _assert_unit(bs[k], b0[k], np.sqrt(v[k]), f"swiglu {k}")
    # the block with the down projection
    p = _grg_inputs(4, M=M, K=K, d=d, F=F)
    eps = 1e-6
    a = (p["X"], p["W1"], p["R"], p["g"], p["W2"], Wd, eps)
    g0 = O.mlp_block_forward(*a)
    c0 = O.mlp_block_backward(dOut, *a, fwd=g0)
    gs = O.mlp_block_forward(*a, stored=True)
    cs = O.mlp_block_backward(dOut, *a, stored=True, fwd=gs)
    vb = E.mlp_block_var(g0, c0, p["g"], p["W2"], Wd, dOut, c0["dY"], p["X"], p["W1"])
    for k in ("Y", "Out"):
        _assert_unit(gs[k], g0[k], np.sqrt(vb[k]), f"block {k}")
    for k in ("dX", "dR", "dW1", "dW2", "dg", "dWdown"):
        _assert_unit(cs[k], c0[k], np.sqrt(vb[k]), f"block {k}")


def test_stored_operand_model_xent_and_rope():
    rng = np.random.default_rng(5)
    bf = O.round_bf16
    M, d, V = 160, 128, 640
    X, W = bf(rng.standard_normal((M, d))), bf(rng.standard_normal((V, d)) / np.sqrt(d))
    tg = rng.integers(0, V, M)
    dl = bf(rng.standard_normal(M))
    f = O.xent_forward(X, W, tg)
    b0 = O.xent_backward(dl, X, W, tg, fwd=f)
    bs = O.xent_backward(dl, X, W, tg, fwd=f, store=O.round_bf16)
    v = E.stored_operand_var(b0["dlogits"], X, W)
    # One dlogits element per row is dloss (p - 1) with p ~ 1/V: it lies within
    # a fraction p of the bf16 value -dloss, so its rounding error is smaller
    # than a uniform one and the model overestimates it (a conservative bound).
    for k in ("dX", "dW"):
        _assert_unit(bs[k], b0[k], np.sqrt(v[k]), f"xent {k}", lo=0.6)
    Wq = bf(rng.standard_normal((6 * 64, d)) / np.sqrt(d))
    dQ = bf(rng.standard_normal((M, 6 * 64)))
    r0 = O.qkv_rope_backward(dQ, X, Wq, 2, 2, 64, 50, 10000.0)
    rs = O.qkv_rope_backward(dQ, X, Wq, 2, 2, 64, 50, 10000.0, store=O.round_bf16)
    v = E.stored_operand_var(r0["dpre"], X, Wq)
    # the v heads' gradient is copied, not rotated: its weight-gradient rows
    # (a third of dW here) carry no rounding at all
    for k in ("dX", "dW"):
        _assert_unit(rs[k], r0[k], np.sqrt(v[k]), f"rope {k}", covered=0.6)


def _sigmoid(x):
    return 1.0 / (1.0 + np.exp(-x))


def test_unfused_models_match_the_operator_by_operator_chain():
    """The unfused sequence written out with every intermediate rounded where
    the operator-by-operator kernels store it."""
    p = _grg_inputs(6)
    bf = O.round_bf16
    eps = 1e-6
    X, W1, R, g, W2, dY = p["X"], p["W1"], p["R"], p["g"], p["W2"], p["dY"]
    F = W2.shape[0] // 2
    d = R.shape[1]
    T = bf(X @ W1.T)
    H = bf(T + R)
    r = 1.0 / np.sqrt(np.mean(H * H, axis=1) + eps)
    U = bf(H * r[:, None] * g[None, :])
    AB = bf(U @ W2.T)
    a, b = AB[:, :F], AB[:, F:]
    s = _sigmoid(a)
    Y = a * s * b
    da = dY * b * s * (1 + a * (1 - s))
    db = dY * a * s
    dA = bf(np.concatenate([da, db], axis=1))
    du = bf(dA @ W2)
    dW2 = dA.T @ U
    dg = np.sum(du * H * r[:, None], axis=0)
    coef = r ** 3 / d * np.sum(du * g[None, :] * H, axis=1)
    dH = r[:, None] * du * g[None, :] - coef[:, None] * H
    dRs = bf(dH)
    st = {"H": H, "a": (U @ W2.T)[:, :F], "b": (U @ W2.T)[:, F:], "Y": Y, "dR": dH, "dX": dRs @ W1,
          "dW1": dRs.T @ X, "dW2": dW2, "dg": dg}
    f0 = O.grg_forward(X, W1, R, g, W2, eps)
    b0 = O.grg_backward(dY, X, W1, R, g, W2, eps, fwd=f0)
    v = E.grg_unfused_var(f0, b0, X, W1, g, W2, dY)
    ref = {**{k: f0[k] for k in ("H", "a", "b", "Y")}, **{k: b0[k] for k in ("dR", "dX", "dW1", "dW2", "dg")}}
    for k in st:
        _assert_unit(st[k], ref[k], np.sqrt(v[k]), f"unfused {k}")
