"""Pins for the CPU oracle, independent of the oracle's own code (CPU only).

Each test checks the oracle against something other than itself: a
hand-derived worked example (tests/golden), closed forms, invariants of
RMSNorm and SwiGLU, central finite differences of the scalar loss, torch fp64
library routines (rms_norm, linear, silu, autograd), and brute-force loops on
tiny inputs.  A plausible slip in the oracle (eps outside the root, the mean
over a tile instead of d, gate/up swapped, a dropped RMSNorm backward term, a
transposed weight gradient) fails at least one of them.
"""

import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as Fn

from oracle import coda_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _ev(expr, **env):
    return eval(expr, {"exp": math.exp, "sqrt": math.sqrt, "__builtins__": {}}, env)


# ----------------------------------------------------------------------------- worked example

def _hand():
    with open(os.path.join(GOLDEN, "grg_hand_example.json")) as f:
        return json.load(f)


def test_hand_example_forward():
    ex = _hand()
    inp = {k: np.array(v, dtype=np.float64) for k, v in ex["inputs"].items()}
    for key, eps in (("eps0", 0.0), ("eps1", 1.0)):
        f = O.grg_forward(inp["X"], inp["W1"], inp["R"], inp["g"], inp["W2"], eps)
        exp = ex["expected"][key]
        assert f["r"][0] == pytest.approx(_ev(exp["r"]), rel=1e-15)
        assert f["a"][0, 0] == pytest.approx(_ev(exp["a"]), rel=1e-15)
        assert f["b"][0, 0] == pytest.approx(_ev(exp["b"]), rel=1e-15)
        assert f["Y"][0, 0] == pytest.approx(_ev(exp["Y"]), rel=1e-14)
        if "H" in exp:
            np.testing.assert_array_equal(f["H"][0], [_ev(e) for e in exp["H"]])


def test_hand_example_backward():
    ex = _hand()
    inp = {k: np.array(v, dtype=np.float64) for k, v in ex["inputs"].items()}
    e = ex["expected"]["bwd_eps0"]
    s = _ev(e["s"])
    da = _ev(e["da"], s=s)
    db = _ev(e["db"], s=s)
    env = {"da": da, "db": db}
    b = O.grg_backward(inp["dY"], inp["X"], inp["W1"], inp["R"], inp["g"], inp["W2"], 0.0)
    np.testing.assert_allclose(b["dA"][0], [da, db], rtol=1e-14)
    np.testing.assert_allclose(b["dH"][0], [_ev(x, **env) for x in e["dH"]], rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(b["dX"][0], [_ev(x, **env) for x in e["dH"]], rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(b["dW1"], [[_ev(x, **env) for x in row] for row in e["dW1"]], rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(b["dW2"], [[_ev(x, **env) for x in row] for row in e["dW2"]], rtol=1e-14)
    np.testing.assert_allclose(b["dg"], [_ev(x, **env) for x in e["dg"]], rtol=1e-14)


# ----------------------------------------------------------------------------- closed forms

def test_constant_rows_closed_form_r():
    """X = 0 and R_i = c_i * ones  =>  H_i = c_i, r_i = 1/sqrt(c_i^2 + eps).

    Distinguishes eps inside vs outside the root and mean over d vs a sum.
    """
    M, K, d, F = 5, 8, 12, 3
    c = np.array([0.5, -1.0, 2.0, 3.0, 1e-3])
    R = c[:, None] * np.ones((1, d))
    X = np.zeros((M, K))
    rng = np.random.default_rng(1)
    W1 = rng.standard_normal((d, K))
    W2 = rng.standard_normal((2 * F, d))
    g = 1 + 0.1 * rng.standard_normal(d)
    for eps in (1e-6, 0.25):
        f = O.grg_forward(X, W1, R, g, W2, eps)
        np.testing.assert_allclose(f["r"], 1.0 / np.sqrt(c * c + eps), rtol=1e-14)


def test_zero_rows_degenerate_case():
    """A row with X_i = 0 and R_i = 0 has H_i = 0: r_i = 1/sqrt(eps) exactly
    (the RMSNorm degenerate case), Y_i = 0, and its gradients dH_i = dX_i = 0
    (a = b = 0 makes da = db = 0).  The other rows are unaffected: they equal
    the oracle run on those rows alone (rows are independent), and the weight
    gradients get nothing from the zero row."""
    rng = np.random.default_rng(21)
    M, K, d, F, eps = 4, 6, 8, 5, 1e-4
    X, R = rng.standard_normal((M, K)), rng.standard_normal((M, d))
    X[2], R[2] = 0.0, 0.0
    W1, W2 = rng.standard_normal((d, K)), rng.standard_normal((2 * F, d))
    g, dY = 1 + 0.1 * rng.standard_normal(d), rng.standard_normal((M, F))
    f = O.grg_forward(X, W1, R, g, W2, eps)
    b = O.grg_backward(dY, X, W1, R, g, W2, eps, fwd=f)
    assert f["r"][2] == 1.0 / math.sqrt(eps)
    assert not np.any(f["Y"][2]) and not np.any(b["dX"][2]) and not np.any(b["dR"][2])
    keep = [0, 1, 3]
    f3 = O.grg_forward(X[keep], W1, R[keep], g, W2, eps)
    b3 = O.grg_backward(dY[keep], X[keep], W1, R[keep], g, W2, eps, fwd=f3)
    np.testing.assert_allclose(f["Y"][keep], f3["Y"], rtol=1e-13, atol=1e-13)
    for k in ("dW1", "dW2", "dg"):
        np.testing.assert_allclose(b[k], b3[k], rtol=1e-12, atol=1e-12)


def test_unit_rms_rows_when_gain_is_one():
    """g = 1: mean_j n_ij^2 = ms_i / (ms_i + eps); exactly 1 at eps = 0."""
    rng = np.random.default_rng(2)
    M, K, d, F = 7, 16, 24, 5
    X, R = rng.standard_normal((M, K)), rng.standard_normal((M, d))
    W1, W2 = rng.standard_normal((d, K)), rng.standard_normal((2 * F, d))
    g = np.ones(d)
    f0 = O.grg_forward(X, W1, R, g, W2, 0.0)
    np.testing.assert_allclose(np.mean(f0["n"] ** 2, axis=1), 1.0, rtol=1e-13)
    eps = 0.3
    f1 = O.grg_forward(X, W1, R, g, W2, eps)
    ms = np.mean(f1["H"] ** 2, axis=1)
    np.testing.assert_allclose(np.mean(f1["n"] ** 2, axis=1), ms / (ms + eps), rtol=1e-13)


def test_scale_invariance_at_zero_eps():
    """RMSNorm(alpha H) = RMSNorm(H) when eps = 0, so Y is unchanged by scaling X and R."""
    rng = np.random.default_rng(3)
    M, K, d, F = 4, 8, 8, 6
    X, R = rng.standard_normal((M, K)), rng.standard_normal((M, d))
    W1, W2 = rng.standard_normal((d, K)), rng.standard_normal((2 * F, d))
    g = 1 + 0.1 * rng.standard_normal(d)
    y1 = O.grg_forward(X, W1, R, g, W2, 0.0)["Y"]
    y2 = O.grg_forward(3.5 * X, W1, 3.5 * R, g, W2, 0.0)["Y"]
    np.testing.assert_allclose(y1, y2, rtol=1e-12, atol=1e-14)


def test_row_scale_commutes_with_second_gemm():
    """The CODA identity: diag(r) (H (diag(g) W2^T)) equals RMSNorm(H)*g times W2^T.

    The oracle computes the right-hand side in textbook order; the test
    evaluates the left-hand side (r deferred past the GEMM, g folded into W2).
    """
    rng = np.random.default_rng(4)
    M, K, d, F = 9, 12, 16, 10
    X, R = rng.standard_normal((M, K)), rng.standard_normal((M, d))
    W1, W2 = rng.standard_normal((d, K)), rng.standard_normal((2 * F, d))
    g = 1 + 0.1 * rng.standard_normal(d)
    f = O.grg_forward(X, W1, R, g, W2, 1e-5)
    W2g = W2 * g[None, :]
    lhs = f["r"][:, None] * (f["H"] @ W2g.T)
    np.testing.assert_allclose(lhs, f["A"], rtol=1e-12, atol=1e-12)


def test_gate_up_order_closed_form():
    """F = d, W2 = [I; 2I], g = 1: a = n, b = 2n, Y = silu(n) * 2n (gate = first F rows)."""
    rng = np.random.default_rng(5)
    M, K, d = 6, 8, 8
    X, R = rng.standard_normal((M, K)), rng.standard_normal((M, d))
    W1 = rng.standard_normal((d, K))
    W2 = np.concatenate([np.eye(d), 2 * np.eye(d)], axis=0)
    f = O.grg_forward(X, W1, R, np.ones(d), W2, 1e-6)
    n = f["n"]
    np.testing.assert_allclose(f["Y"], n / (1 + np.exp(-n)) * 2 * n, rtol=1e-13, atol=1e-15)


def test_silu_special_values():
    assert O.silu(0.0) == 0.0
    assert O.silu(1.0) == pytest.approx(1 / (1 + math.exp(-1)), rel=1e-15)
    x = np.linspace(-40, 40, 161)
    np.testing.assert_allclose(O.silu(x) - O.silu(-x), x, atol=1e-13)  # silu(x) - silu(-x) = x
    assert O.silu(-745.0) == pytest.approx(-745.0 * math.exp(-745.0), rel=1e-6, abs=1e-300)
    assert O.silu(800.0) == 800.0


def test_partial_sumsq_one_hot_and_totals():
    """One-hot H puts v^2 in exactly one (row, tile) cell; tiles sum to d * ms."""
    M, d, w = 3, 10, 4  # ragged last tile of width 2
    for (i, j, v) in [(0, 0, 3.0), (1, 5, -2.0), (2, 9, 0.5)]:
        H = np.zeros((M, d))
        H[i, j] = v
        P = O.partial_sumsq(H, w)
        assert P.shape == (M, 3)
        expect = np.zeros_like(P)
        expect[i, j // w] = v * v
        np.testing.assert_array_equal(P, expect)
    rng = np.random.default_rng(6)
    H = rng.standard_normal((M, d))
    np.testing.assert_allclose(O.partial_sumsq(H, w).sum(axis=1), np.einsum("ij,ij->i", H, H), rtol=1e-14)


def test_gemm_brute_force():
    rng = np.random.default_rng(7)
    A, B = rng.standard_normal((3, 5)), rng.standard_normal((4, 5))
    C = O.gemm(A, B)
    for i in range(3):
        for j in range(4):
            s = 0.0
            for k in range(5):
                s += A[i, k] * B[j, k]
            assert C[i, j] == pytest.approx(s, rel=1e-13, abs=1e-14)


# ----------------------------------------------------------------------------- finite differences

def _grg_loss(p, dY, dH_in, eps):
    f = O.grg_forward(p["X"], p["W1"], p["R"], p["g"], p["W2"], eps)
    return float(np.sum(dY * f["Y"]) + np.sum(dH_in * f["H"]))


def _fd_check(loss_fn, params, grads, names, h_rel=1e-6, tol=2e-6):
    for name in names:
        x = params[name]
        num = np.zeros_like(x)
        it = np.nditer(x, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            h = h_rel * max(1.0, abs(x[idx]))
            old = x[idx]
            x[idx] = old + h
            lp = loss_fn(params)
            x[idx] = old - h
            lm = loss_fn(params)
            x[idx] = old
            num[idx] = (lp - lm) / (2 * h)
        scale = max(1.0, float(np.max(np.abs(num))))
        err = float(np.max(np.abs(num - grads[name])))
        assert err <= tol * scale, f"d{name}: max |fd - oracle| = {err:.3e} (scale {scale:.3e})"


def test_grg_backward_finite_differences():
    rng = np.random.default_rng(8)
    M, K, d, F = 3, 5, 6, 4
    p = {
        "X": rng.standard_normal((M, K)),
        "W1": rng.standard_normal((d, K)) / np.sqrt(K),
        "R": rng.standard_normal((M, d)),
        "g": 1 + 0.1 * rng.standard_normal(d),
        "W2": rng.standard_normal((2 * F, d)) / np.sqrt(d),
    }
    dY = rng.standard_normal((M, F))
    dH_in = rng.standard_normal((M, d))
    eps = 0.1  # large enough that a dropped eps term would show
    b = O.grg_backward(dY, p["X"], p["W1"], p["R"], p["g"], p["W2"], eps, dH_in=dH_in)
    grads = {"X": b["dX"], "W1": b["dW1"], "R": b["dR"], "g": b["dg"], "W2": b["dW2"]}
    _fd_check(lambda q: _grg_loss(q, dY, dH_in, eps), p, grads, ["X", "W1", "R", "g", "W2"])


def test_swiglu_backward_finite_differences():
    rng = np.random.default_rng(9)
    M, d, F = 3, 5, 4
    p = {
        "X": rng.standard_normal((M, d)),
        "Wgu": rng.standard_normal((2 * F, d)) / np.sqrt(d),
        "Wdown": rng.standard_normal((d, F)) / np.sqrt(F),
    }
    dOut = rng.standard_normal((M, d))

    def loss(q):
        return float(np.sum(dOut * O.swiglu_forward(q["X"], q["Wgu"], q["Wdown"])["Out"]))

    b = O.swiglu_backward(dOut, p["X"], p["Wgu"], p["Wdown"])
    grads = {"X": b["dX"], "Wgu": b["dWgu"], "Wdown": b["dWdown"]}
    _fd_check(loss, p, grads, ["X", "Wgu", "Wdown"])


# ----------------------------------------------------------------------------- library cross-check

def test_torch_fp64_library_crosscheck_grg():
    """torch CPU fp64: linear + rms_norm(weight=g) + linear + silu, autograd for the backward."""
    torch.manual_seed(10)
    M, K, d, F, eps = 16, 32, 48, 40, 1e-5
    X = torch.randn(M, K, dtype=torch.float64, requires_grad=True)
    W1 = (torch.randn(d, K, dtype=torch.float64) / K ** 0.5).requires_grad_()
    R = torch.randn(M, d, dtype=torch.float64, requires_grad=True)
    g = (1 + 0.1 * torch.randn(d, dtype=torch.float64)).requires_grad_()
    W2 = (torch.randn(2 * F, d, dtype=torch.float64) / d ** 0.5).requires_grad_()
    dY = torch.randn(M, F, dtype=torch.float64)
    dH_in = torch.randn(M, d, dtype=torch.float64)
    H = Fn.linear(X, W1) + R
    H.retain_grad()
    A = Fn.linear(Fn.rms_norm(H, (d,), weight=g, eps=eps), W2)
    Y = Fn.silu(A[:, :F]) * A[:, F:]
    ((Y * dY).sum() + (H * dH_in).sum()).backward()

    npy = lambda t: t.detach().numpy()
    f = O.grg_forward(npy(X), npy(W1), npy(R), npy(g), npy(W2), eps)
    np.testing.assert_allclose(f["H"], npy(H), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(f["A"], npy(A), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(f["Y"], npy(Y), rtol=1e-12, atol=1e-12)
    b = O.grg_backward(npy(dY), npy(X), npy(W1), npy(R), npy(g), npy(W2), eps, dH_in=npy(dH_in), fwd=f)
    for mine, ref in (("dX", X), ("dW1", W1), ("dR", R), ("dg", g), ("dW2", W2)):
        np.testing.assert_allclose(b[mine], ref.grad.numpy(), rtol=1e-10, atol=1e-11, err_msg=mine)


def test_torch_fp64_library_crosscheck_swiglu():
    torch.manual_seed(11)
    M, d, F = 16, 32, 24
    X = torch.randn(M, d, dtype=torch.float64, requires_grad=True)
    Wgu = (torch.randn(2 * F, d, dtype=torch.float64) / d ** 0.5).requires_grad_()
    Wdown = (torch.randn(d, F, dtype=torch.float64) / F ** 0.5).requires_grad_()
    dOut = torch.randn(M, d, dtype=torch.float64)
    A = Fn.linear(X, Wgu)
    Out = Fn.linear(Fn.silu(A[:, :F]) * A[:, F:], Wdown)
    (Out * dOut).sum().backward()
    npy = lambda t: t.detach().numpy()
    f = O.swiglu_forward(npy(X), npy(Wgu), npy(Wdown))
    np.testing.assert_allclose(f["Out"], npy(Out), rtol=1e-12, atol=1e-12)
    b = O.swiglu_backward(npy(dOut), npy(X), npy(Wgu), npy(Wdown), fwd=f)
    for mine, ref in (("dX", X), ("dWgu", Wgu), ("dWdown", Wdown)):
        np.testing.assert_allclose(b[mine], ref.grad.numpy(), rtol=1e-10, atol=1e-11, err_msg=mine)


def test_row_locality_of_forward_and_row_gradients():
    """Permuting token rows permutes H, r, Y, dX, dR and leaves the weight gradients unchanged."""
    rng = np.random.default_rng(12)
    M, K, d, F = 6, 8, 8, 4
    X, R = rng.standard_normal((M, K)), rng.standard_normal((M, d))
    W1, W2 = rng.standard_normal((d, K)), rng.standard_normal((2 * F, d))
    g = 1 + 0.1 * rng.standard_normal(d)
    dY = rng.standard_normal((M, F))
    perm = rng.permutation(M)
    b0 = O.grg_backward(dY, X, W1, R, g, W2, 1e-6)
    b1 = O.grg_backward(dY[perm], X[perm], W1, R[perm], g, W2, 1e-6)
    np.testing.assert_allclose(b1["dX"], b0["dX"][perm], rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(b1["dW2"], b0["dW2"], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(b1["dg"], b0["dg"], rtol=1e-12, atol=1e-12)


# ----------------------------------------------------------------------------- storage precision

def test_round_bf16_matches_library_conversion_and_ties():
    """round_bf16 equals torch's float32 -> bfloat16 conversion (round to nearest even)."""
    gen = torch.Generator().manual_seed(13)
    x = torch.randn(200000, generator=gen, dtype=torch.float32) * torch.exp(torch.randn(200000, generator=gen) * 4)
    ref = x.to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(O.round_bf16(x.double().numpy()), ref)
    # Hand ties: the bf16 spacing at 1 is 2^-7, so 1 + 2^-8 is halfway and goes to even (1.0);
    # 1 + 3*2^-8 is halfway between 1 + 2^-7 (odd) and 1 + 2^-6 (even).
    np.testing.assert_array_equal(O.round_bf16([1 + 2 ** -8, 1 + 3 * 2 ** -8, -(1 + 2 ** -8), 0.0, 3.0]),
                                  [1.0, 1 + 2 ** -6, -1.0, 0.0, 3.0])


def _ident(x):
    return x


def test_stored_functions_reduce_to_textbook_without_rounding():
    rng = np.random.default_rng(14)
    M, K, d, F, eps = 9, 16, 24, 10, 1e-5
    X, R = rng.standard_normal((M, K)), rng.standard_normal((M, d))
    W1, W2 = rng.standard_normal((d, K)) / 4, rng.standard_normal((2 * F, d)) / 5
    g = 1 + 0.1 * rng.standard_normal(d)
    dY, dH_in = rng.standard_normal((M, F)), rng.standard_normal((M, d))
    f0 = O.grg_forward(X, W1, R, g, W2, eps)
    for gain in ("weight", "activation"):
        f1 = O.grg_forward_stored(X, W1, R, g, W2, eps, store=_ident, gain=gain)
        for k in ("H", "r", "a", "b", "Y"):
            np.testing.assert_allclose(f1[k], f0[k], rtol=1e-12, atol=1e-12, err_msg=f"{gain} {k}")
    with pytest.raises(ValueError):
        O.grg_forward_stored(X, W1, R, g, W2, eps, gain="neither")
    b0 = O.grg_backward(dY, X, W1, R, g, W2, eps, dH_in=dH_in)
    b1 = O.grg_backward_stored(dY, X, W1, R, g, W2, eps, dH_in=dH_in, store=_ident)
    for k in ("dX", "dR", "dW1", "dW2", "dg"):
        np.testing.assert_allclose(b1[k], b0[k], rtol=1e-11, atol=1e-11, err_msg=k)
    Wgu, Wdown, dOut = rng.standard_normal((2 * F, d)) / 5, rng.standard_normal((d, F)) / 3, rng.standard_normal((M, d))
    s0 = O.swiglu_forward(R, Wgu, Wdown)
    s1 = O.swiglu_forward_stored(R, Wgu, Wdown, store=_ident)
    np.testing.assert_allclose(s1["Out"], s0["Out"], rtol=1e-12, atol=1e-12)
    t0 = O.swiglu_backward(dOut, R, Wgu, Wdown)
    t1 = O.swiglu_backward_stored(dOut, R, Wgu, Wdown, store=_ident)
    for k in ("dX", "dWgu", "dWdown"):
        np.testing.assert_allclose(t1[k], t0[k], rtol=1e-12, atol=1e-12, err_msg=k)


def test_stored_rounding_is_small_and_present():
    """bf16 storage moves results by about the bf16 unit (2^-8), not more, not zero."""
    rng = np.random.default_rng(15)
    M, K, d, F, eps = 64, 64, 64, 64, 1e-6
    X, R = rng.standard_normal((M, K)), rng.standard_normal((M, d))
    W1, W2 = rng.standard_normal((d, K)) / 8, rng.standard_normal((2 * F, d)) / 8
    g = 1 + 0.1 * rng.standard_normal(d)
    f0 = O.grg_forward(X, W1, R, g, W2, eps)
    f1 = O.grg_forward_stored(X, W1, R, g, W2, eps)
    assert np.array_equal(f1["H"], O.round_bf16(f0["H"]))
    rel = np.sqrt(np.mean((f1["A"] - f0["A"]) ** 2)) / np.sqrt(np.mean(f0["A"] ** 2))
    assert 1e-4 < rel < 2 ** -8


def _placement(case):
    with open(os.path.join(GOLDEN, "storage_placement.json")) as f:
        c = json.load(f)["cases"][case]
    inp = {k: (np.array(v, dtype=np.float64) if isinstance(v, list) else float(v)) for k, v in c["inputs"].items()}
    return inp, c


def _evx(e):
    return np.array([_evx(x) for x in e]) if isinstance(e, list) else \
        eval(e, {"exp": math.exp, "sqrt": math.sqrt, "__builtins__": {}})


def test_storage_placement_H_rounded_before_r():
    """H on a bf16 midpoint: the stored H (ties to even) feeds r, so r = 1
    exactly; computing r from the unrounded H, or rounding ties away from
    zero, gives r < 1 (tests/golden/storage_placement.json, H_midpoint)."""
    p, c = _placement("H_midpoint")
    f = O.grg_forward_stored(p["X"], p["W1"], p["R"], p["g"], p["W2"], p["eps"])
    e = c["expected"]
    np.testing.assert_array_equal(f["H"][0], _evx(e["H"]))
    for k in ("r",):
        assert f[k][0] == _evx(e[k])
    for k in ("a", "b"):
        assert f[k][0, 0] == _evx(e[k])
    assert f["Y"][0, 0] == pytest.approx(_evx(e["Y"]), rel=1e-15)
    # the textbook oracle keeps the exact H, and its r differs from the stored one
    f0 = O.grg_forward(p["X"], p["W1"], p["R"], p["g"], p["W2"], p["eps"])
    assert f0["r"][0] == pytest.approx(_evx(c["textbook"]["r"]), rel=1e-15)
    assert f0["r"][0] < f["r"][0]


def test_storage_placement_Y_from_unrounded_pre_activations():
    """a = 1 + 2^-8 sits on a bf16 midpoint: Y is computed from the unrounded
    a, while the saved a_s is rounded (to 1) (a_midpoint)."""
    p, c = _placement("a_midpoint")
    f = O.grg_forward_stored(p["X"], p["W1"], p["R"], p["g"], p["W2"], p["eps"])
    e = c["expected"]
    assert f["a"][0, 0] == _evx(e["a"])
    assert f["a_s"][0, 0] == _evx(e["a_s"]) and f["b_s"][0, 0] == _evx(e["b_s"])
    assert f["Y"][0, 0] == pytest.approx(_evx(e["Y"]), rel=1e-15)
    assert abs(f["Y"][0, 0] - float(O.silu(1.0))) > 1e-3


def test_storage_placement_gemm2_adjoint_reads_r_scaled_gradient():
    """r = 1/3: the backward rounds dZ = r [da, db] (171/512), not [da, db]
    (which is exact at 1), and every weight and input gradient follows from
    that operand (dZ_row_scale_third)."""
    p, c = _placement("dZ_row_scale_third")
    f = O.grg_forward_stored(p["X"], p["W1"], p["R"], p["g"], p["W2"], p["eps"])
    b = O.grg_backward_stored(p["dY"], p["X"], p["W1"], p["R"], p["g"], p["W2"], p["eps"], fwd=f)
    e = c["expected"]
    np.testing.assert_array_equal(b["dZ"][0], _evx(e["dZ"]))
    np.testing.assert_array_equal(b["dW2"], _evx(e["dW2"]))
    np.testing.assert_array_equal(b["dg"], _evx(e["dg"]))
    np.testing.assert_array_equal(b["dR"][0], _evx(e["dR"]))
    np.testing.assert_array_equal(b["dX"][0], _evx(e["dX"]))
    np.testing.assert_array_equal(b["dW1"], _evx(e["dW1"]))
    b0 = O.grg_backward(p["dY"], p["X"], p["W1"], p["R"], p["g"], p["W2"], p["eps"])
    np.testing.assert_allclose(b0["dR"][0], [1 / 3, -1 / 3], rtol=1e-15)
    np.testing.assert_allclose(b0["dW2"], [[1, 1], [0, 0]], rtol=1e-15, atol=1e-300)


def test_storage_placement_activation_gain_from_stored_H():
    """With the gain on the activation side, Hg = bf16(stored H * g) = 1.5, not
    bf16(exact H * g) = 1.5078125; the folded-weight placement gives the same
    a, b, Y here (activation_gain_from_stored_H)."""
    p, c = _placement("activation_gain_from_stored_H")
    e = c["expected"]
    for gain in ("activation", "weight"):
        f = O.grg_forward_stored(p["X"], p["W1"], p["R"], p["g"], p["W2"], p["eps"], gain=gain)
        assert f["a"][0, 0] == _evx(e["a"]) and f["b"][0, 0] == _evx(e["b"]), gain
        assert f["Y"][0, 0] == pytest.approx(_evx(e["Y"]), rel=1e-15)


# ----------------------------------------------------------------------------- cross-entropy

def test_xent_uniform_logits_closed_form():
    """W = 0 gives equal logits: loss = log V for every target, softmax = 1/V."""
    M, d, V = 5, 8, 37
    X = np.random.default_rng(16).standard_normal((M, d))
    W = np.zeros((V, d))
    t = np.array([0, 3, 36, 10, 10])
    f = O.xent_forward(X, W, t)
    np.testing.assert_allclose(f["loss"], np.log(V), rtol=1e-15)
    b = O.xent_backward(np.ones(M), X, W, t, fwd=f)
    expect = np.full((M, V), 1.0 / V)
    expect[np.arange(M), t] -= 1.0
    np.testing.assert_allclose(b["dlogits"], expect, rtol=1e-14, atol=1e-16)


def test_xent_matches_torch_cross_entropy_and_autograd():
    torch.manual_seed(17)
    M, d, V = 12, 16, 50
    X = torch.randn(M, d, dtype=torch.float64, requires_grad=True)
    W = (torch.randn(V, d, dtype=torch.float64) / 2).requires_grad_()
    t = torch.randint(0, V, (M,))
    dloss = torch.rand(M, dtype=torch.float64)
    loss = Fn.cross_entropy(Fn.linear(X, W), t, reduction="none")
    (loss * dloss).sum().backward()
    f = O.xent_forward(X.detach().numpy(), W.detach().numpy(), t.numpy())
    np.testing.assert_allclose(f["loss"], loss.detach().numpy(), rtol=1e-12)
    b = O.xent_backward(dloss.numpy(), X.detach().numpy(), W.detach().numpy(), t.numpy(), fwd=f)
    np.testing.assert_allclose(b["dX"], X.grad.numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(b["dW"], W.grad.numpy(), rtol=1e-10, atol=1e-12)


def test_xent_shift_invariance_and_finite_differences():
    """Adding a constant to a row's logits leaves the loss unchanged (a bias column
    of X with a constant W column); the backward matches central differences."""
    rng = np.random.default_rng(18)
    M, d, V = 4, 6, 9
    X, W = rng.standard_normal((M, d)), rng.standard_normal((V, d))
    t = np.array([1, 8, 0, 4])
    Xb = np.concatenate([X, np.ones((M, 1))], axis=1)
    Wb = np.concatenate([W, np.full((V, 1), 5.0)], axis=1)
    np.testing.assert_allclose(O.xent_forward(Xb, Wb, t)["loss"], O.xent_forward(X, W, t)["loss"], rtol=1e-12)
    dloss = rng.standard_normal(M)
    b = O.xent_backward(dloss, X, W, t)
    p = {"X": X.copy(), "W": W.copy()}
    _fd_check(lambda q: float(np.sum(dloss * O.xent_forward(q["X"], q["W"], t)["loss"])), p,
              {"X": b["dX"], "W": b["dW"]}, ["X", "W"])


# ----------------------------------------------------------------------------- RoPE

def test_rope_closed_forms():
    """head_dim 2: the single pair turns by exactly pos radians (base^0 = 1); pos 0 is the identity."""
    x = np.array([[1.0, 0.0], [1.0, 0.0], [0.0, 2.0], [3.0, -1.0]])
    pos = np.array([0, 1, 2, 0])
    y = O.rope_rotate(x, pos, head_dim=2, base=10000.0)
    np.testing.assert_allclose(y[0], [1.0, 0.0], atol=1e-15)
    np.testing.assert_allclose(y[1], [np.cos(1.0), np.sin(1.0)], rtol=1e-15)
    np.testing.assert_allclose(y[2], [-2.0 * np.sin(2.0), 2.0 * np.cos(2.0)], rtol=1e-14)
    np.testing.assert_allclose(y[3], [3.0, -1.0], atol=1e-15)
    # Second frequency of head_dim 4 with base 100: 100^(-2/4) = 0.1 rad per position.
    z = O.rope_rotate(np.array([[0.0, 1.0, 0.0, 0.0]]), np.array([5]), head_dim=4, base=100.0)
    np.testing.assert_allclose(z[0], [0.0, np.cos(0.5), 0.0, np.sin(0.5)], atol=1e-15)


def test_rope_preserves_norms_and_inverse_undoes_it():
    rng = np.random.default_rng(19)
    M, heads, hd = 9, 3, 8
    x = rng.standard_normal((M, heads * hd))
    pos = rng.integers(0, 4096, M)
    y = O.rope_rotate(x, pos, hd, 10000.0)
    for h in range(heads):
        np.testing.assert_allclose(np.linalg.norm(y[:, h * hd:(h + 1) * hd], axis=1),
                                   np.linalg.norm(x[:, h * hd:(h + 1) * hd], axis=1), rtol=1e-13)
    np.testing.assert_allclose(O.rope_rotate(y, pos, hd, 10000.0, inverse=True), x, atol=1e-12)


def test_rope_relative_position_property():
    """<RoPE(q, m), RoPE(k, n)> depends on m - n only: RoPE's defining property."""
    rng = np.random.default_rng(20)
    hd = 16
    q, k = rng.standard_normal((1, hd)), rng.standard_normal((1, hd))
    dots = []
    for m, n in [(7, 3), (104, 100), (4004, 4000)]:
        qm = O.rope_rotate(q, np.array([m]), hd, 10000.0)
        kn = O.rope_rotate(k, np.array([n]), hd, 10000.0)
        dots.append(float((qm @ kn.T)[0, 0]))
    np.testing.assert_allclose(dots, dots[0], rtol=1e-10)


def test_qkv_rope_backward_finite_differences():
    rng = np.random.default_rng(21)
    M, d, nq, nkv, hd, S = 5, 6, 2, 1, 4, 3
    p = {"X": rng.standard_normal((M, d)), "W": rng.standard_normal(((nq + 2 * nkv) * hd, d))}
    dQ = rng.standard_normal((M, (nq + 2 * nkv) * hd))
    b = O.qkv_rope_backward(dQ, p["X"], p["W"], nq, nkv, hd, S, 50.0)
    _fd_check(lambda q: float(np.sum(dQ * O.qkv_rope_forward(q["X"], q["W"], nq, nkv, hd, S, 50.0)["QKV"])),
              p, {"X": b["dX"], "W": b["dW"]}, ["X", "W"])
    # v columns pass through unrotated.
    f = O.qkv_rope_forward(p["X"], p["W"], nq, nkv, hd, S, 50.0)
    np.testing.assert_array_equal(f["QKV"][:, (nq + nkv) * hd:], f["pre"][:, (nq + nkv) * hd:])


# ----------------------------------------------------------------------------- full MLP block

def test_mlp_block_finite_differences():
    rng = np.random.default_rng(22)
    M, K, d, F, eps = 3, 5, 6, 4, 0.05
    p = {
        "X": rng.standard_normal((M, K)),
        "W1": rng.standard_normal((d, K)) / np.sqrt(K),
        "R": rng.standard_normal((M, d)),
        "g": 1 + 0.1 * rng.standard_normal(d),
        "W2": rng.standard_normal((2 * F, d)) / np.sqrt(d),
        "Wdown": rng.standard_normal((d, F)) / np.sqrt(F),
    }
    dOut = rng.standard_normal((M, d))

    def loss(q):
        return float(np.sum(dOut * O.mlp_block_forward(q["X"], q["W1"], q["R"], q["g"], q["W2"], q["Wdown"],
                                                        eps)["Out"]))

    b = O.mlp_block_backward(dOut, p["X"], p["W1"], p["R"], p["g"], p["W2"], p["Wdown"], eps)
    grads = {"X": b["dX"], "W1": b["dW1"], "R": b["dR"], "g": b["dg"], "W2": b["dW2"], "Wdown": b["dWdown"]}
    _fd_check(loss, p, grads, list(grads))


def test_mlp_block_stored_reduces_to_textbook():
    rng = np.random.default_rng(23)
    M, K, d, F, eps = 6, 8, 12, 10, 1e-5
    X, R = rng.standard_normal((M, K)), rng.standard_normal((M, d))
    W1, W2 = rng.standard_normal((d, K)) / 3, rng.standard_normal((2 * F, d)) / 3
    Wd, g = rng.standard_normal((d, F)) / 3, 1 + 0.1 * rng.standard_normal(d)
    dOut = rng.standard_normal((M, d))
    f0 = O.mlp_block_forward(X, W1, R, g, W2, Wd, eps)
    f1 = O.mlp_block_forward(X, W1, R, g, W2, Wd, eps, stored=True, store=_ident)
    np.testing.assert_allclose(f1["Out"], f0["Out"], rtol=1e-12, atol=1e-12)
    b0 = O.mlp_block_backward(dOut, X, W1, R, g, W2, Wd, eps, fwd=f0)
    b1 = O.mlp_block_backward(dOut, X, W1, R, g, W2, Wd, eps, stored=True, store=_ident, fwd=f1)
    for k in ("dX", "dR", "dW1", "dW2", "dg", "dWdown"):
        np.testing.assert_allclose(b1[k], b0[k], rtol=1e-11, atol=1e-11, err_msg=k)
