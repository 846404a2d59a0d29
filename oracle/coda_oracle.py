"""CPU oracle for the CODA GEMM-Residual-RMSNorm-GEMM block and the SwiGLU MLP.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
module.  The product path (the CUDA library and its Python binding) never calls
it and shares no code with it.

Everything here is the plain, unfused definition of what the fused kernels must
reach, evaluated in float64 with numpy on the bf16-rounded inputs (the caller
converts bf16 tensors to float64 arrays; that conversion is exact).  Matrix
products use ``numpy.matmul`` (BLAS) as a library primitive; nothing is blocked,
fused or reordered beyond the textbook order of operations.

Sources (the pages give no formulas; see each function for the reading taken):

* toolin.ai, "CODA：LLMと初心者が光速のGPUカーネルを書けるようにする",
  section 核心の洞察 (core insight): a GEMM-RMSNorm-GEMM block, whose RMSNorm
  row scale r commutes with the following GEMM.
* kucoin.com (ru), "CODA: новое исследование ...", section
  «В «Финале» спрятаны сокровища»: the block is GEMM -> residual add -> RMS
  normalisation -> GEMM; the first GEMM's epilogue emits per-tile partial
  mean squares which a light reduction combines.
* same pages, the five-primitive table (toolin.ai §組み合わせ可能な5種類の「積み木」;
  kucoin (ru) §Пять «кирпичиков»): residual add and activation (SwiGLU) are
  elementwise epilogue transforms.
* toolin.ai §実験結果 and kucoin (ru) §Результаты эксперимента: the backward of
  GEMM-Residual-PartialRMS-GEMM and of SwiGLU are the measured kernels.

Readings taken where the pages are silent:
eps sits inside the root, r_i = 1/sqrt(mean_j H_ij^2 + eps), the mean runs over
the full hidden width d; the first F rows of the gate/up weight are the gate
(silu input) and the last F the up projection; weights use the [out, in]
layout, so the pages' "X*W1" is ``X @ W1.T``; the scalar loss whose gradient the
backward returns is <dY, Y> + <dH_in, H>.

Parity pins: every function here is pinned by tests in
``tests/test_oracle_pins.py`` (closed forms, a hand-derived worked example in
``tests/golden/``, central finite differences, and torch fp64 library routines).
"""

from __future__ import annotations

import numpy as np

__all__ = [
    "silu",
    "grg_forward",
    "grg_backward",
    "partial_sumsq",
    "swiglu_forward",
    "swiglu_backward",
    "gemm",
    "round_bf16",
    "grg_forward_stored",
    "grg_backward_stored",
    "swiglu_forward_stored",
    "swiglu_backward_stored",
    "xent_forward",
    "xent_backward",
    "rope_angles",
    "rope_rotate",
    "qkv_rope_forward",
    "qkv_rope_backward",
    "mlp_block_forward",
    "mlp_block_backward",
]


def _f64(x) -> np.ndarray:
    return np.asarray(x, dtype=np.float64)


def _sigmoid(x: np.ndarray) -> np.ndarray:
    # Two-branch logistic so that neither branch overflows.
    out = np.empty_like(x)
    pos = x >= 0
    out[pos] = 1.0 / (1.0 + np.exp(-x[pos]))
    ex = np.exp(x[~pos])
    out[~pos] = ex / (1.0 + ex)
    return out


def silu(x) -> np.ndarray:
    """silu(x) = x * sigmoid(x), the gate nonlinearity of SwiGLU."""
    x = _f64(x)
    return x * _sigmoid(x)


def gemm(A, B) -> np.ndarray:
    """C = A @ B.T in float64 (weights in [out, in] layout)."""
    return _f64(A) @ _f64(B).T


def partial_sumsq(H, tile_width: int) -> np.ndarray:
    """Per-tile partial sums of squares of H.

    P[i, t] = sum over j in [t*w, (t+1)*w) of H[i, j]**2, with w = tile_width
    and the last tile ragged when d is not a multiple of w.  This is the
    "partial RMS" that the first GEMM's epilogue emits (kucoin (ru)
    §«В «Финале» спрятаны сокровища»; toolin.ai five-primitive table, row
    "tile-wise reduction: local mean square").
    """
    H = _f64(H)
    M, d = H.shape
    T = -(-d // tile_width)
    P = np.zeros((M, T), dtype=np.float64)
    for t in range(T):
        blk = H[:, t * tile_width:(t + 1) * tile_width]
        P[:, t] = np.sum(blk * blk, axis=1)
    return P


def grg_forward(X, W1, R, g, W2, eps: float) -> dict:
    """GEMM -> residual -> RMSNorm(gain g) -> GEMM -> SwiGLU, unfused.

    Shapes: X [M, K], W1 [d, K], R [M, d], g [d], W2 [2F, d].
    Steps in textbook order (toolin.ai §核心の洞察; kucoin (ru)
    §«В «Финале» спрятаны сокровища»):
      H  = X W1^T + R                      (GEMM1 + residual add)
      ms = mean_j H_ij^2 ;  r = 1/sqrt(ms + eps)
      n  = diag(r) H ;  u = n * g          (RMSNorm with gain)
      A  = u W2^T ;  a = A[:, :F], b = A[:, F:]
      Y  = silu(a) * b                     (SwiGLU)
    Returns every intermediate so that tests can compare each saved tensor.
    """
    X, W1, R, g, W2 = map(_f64, (X, W1, R, g, W2))
    H = X @ W1.T + R
    d = H.shape[1]
    ms = np.sum(H * H, axis=1) / d
    r = 1.0 / np.sqrt(ms + eps)
    n = H * r[:, None]
    u = n * g[None, :]
    A = u @ W2.T
    F = W2.shape[0] // 2
    a = A[:, :F]
    b = A[:, F:]
    Y = silu(a) * b
    return {"H": H, "ms": ms, "r": r, "n": n, "u": u, "A": A, "a": a, "b": b, "Y": Y}


def _swiglu_grads(dY, a, b):
    """d(silu(a)*b)/da and /db contracted with dY (chain rule, by hand)."""
    s = _sigmoid(a)
    dsilu = s * (1.0 + a * (1.0 - s))  # derivative of a*sigmoid(a)
    da = dY * b * dsilu
    db = dY * a * s
    return da, db


def grg_backward(dY, X, W1, R, g, W2, eps: float, dH_in=None, fwd: dict | None = None) -> dict:
    """Gradients of L = <dY, Y> + <dH_in, H> for the block of grg_forward.

    Textbook reverse-mode, one step at a time (no fused identities):
      da, db from SwiGLU;  dA = [da | db]
      dW2 = dA^T u ;  du = dA W2 ;  dg_j = sum_i du_ij n_ij ;  dn = du * g
      RMSNorm:  n_ij = H_ij r_i with r_i = (ms_i + eps)^(-1/2), ms_i = mean_j H_ij^2
                dH = r * dn - (r^3 / d) * (sum_k dn_ik H_ik) * H   (+ dH_in)
      dR = dH ;  dX = dH W1 ;  dW1 = dH^T X
    The pages name this backward (toolin.ai §実験結果: GEMM-Residual-PartialRMS-GEMM
    backward; kucoin (ru) §Результаты эксперимента) but print no formula; the
    chain rule above is the plain definition.
    """
    if fwd is None:
        fwd = grg_forward(X, W1, R, g, W2, eps)
    dY, X, W1, g, W2 = map(_f64, (dY, X, W1, g, W2))
    H, r, n, u, a, b = fwd["H"], fwd["r"], fwd["n"], fwd["u"], fwd["a"], fwd["b"]
    d = H.shape[1]
    da, db = _swiglu_grads(dY, a, b)
    dA = np.concatenate([da, db], axis=1)
    dW2 = dA.T @ u
    du = dA @ W2
    dg = np.sum(du * n, axis=0)
    dn = du * g[None, :]
    dr = np.sum(dn * H, axis=1)               # dL/dr_i
    dms = dr * (-0.5) * r ** 3                # dr/dms = -1/2 (ms+eps)^(-3/2)
    dH = dn * r[:, None] + (dms[:, None] * (2.0 / d)) * H
    if dH_in is not None:
        dH = dH + _f64(dH_in)
    dX = dH @ W1
    dW1 = dH.T @ X
    return {"dA": dA, "da": da, "db": db, "du": du, "dn": dn, "dH": dH, "dR": dH,
            "dX": dX, "dW1": dW1, "dW2": dW2, "dg": dg}


def swiglu_forward(X, Wgu, Wdown) -> dict:
    """SwiGLU MLP: A = X Wgu^T, Y = silu(a) * b, Out = Y Wdown^T.

    Shapes: X [M, d], Wgu [2F, d] (gate rows first), Wdown [d, F].
    SwiGLU as an elementwise epilogue transform (toolin.ai five-primitive
    table, "activation"; kucoin (ru) §«В «Финале» спрятаны сокровища", SwiGLU
    named among the reparameterised operations).
    """
    X, Wgu, Wdown = map(_f64, (X, Wgu, Wdown))
    A = X @ Wgu.T
    F = Wgu.shape[0] // 2
    a = A[:, :F]
    b = A[:, F:]
    Y = silu(a) * b
    Out = Y @ Wdown.T
    return {"A": A, "a": a, "b": b, "Y": Y, "Out": Out}


def swiglu_backward(dOut, X, Wgu, Wdown, fwd: dict | None = None) -> dict:
    """Gradients of L = <dOut, Out> for swiglu_forward (chain rule by hand).

      dY = dOut Wdown ;  dWdown = dOut^T Y
      da, db from SwiGLU ;  dA = [da | db]
      dWgu = dA^T X ;  dX = dA Wgu
    SwiGLU backward is one of the measured kernels (toolin.ai §実験結果).
    """
    if fwd is None:
        fwd = swiglu_forward(X, Wgu, Wdown)
    dOut, X, Wgu, Wdown = map(_f64, (dOut, X, Wgu, Wdown))
    dY = dOut @ Wdown
    dWdown = dOut.T @ fwd["Y"]
    da, db = _swiglu_grads(dY, fwd["a"], fwd["b"])
    dA = np.concatenate([da, db], axis=1)
    dWgu = dA.T @ X
    dX = dA @ Wgu
    return {"dY": dY, "dA": dA, "da": da, "db": db, "dWgu": dWgu, "dWdown": dWdown, "dX": dX}


# ----------------------------------------------------------------------------- storage precision
#
# The same definitions evaluated at the precision of the method's dataflow:
# every tensor that crosses HBM between two GEMM-epilogue programs is bf16
# there, so the functions below round (with ``store``, default round to
# nearest bf16, ties to even) exactly those tensors and nothing else.  Which
# tensors those are follows from the pages, not from any kernel:
#
# (S1) A GEMM's operands are bf16 tensors in HBM.  In the forward these are
#      H, which GEMM1's epilogue stores and GEMM2 reads back (toolin.ai
#      §核心の洞察 and kucoin (ru) §«В «Финале» спрятаны сокровища»: H goes to
#      memory, the RMSNorm scale r does not), the gain-folded weight
#      W2g = bf16(diag(g) W2) (the fold of the RMSNorm gain into the second
#      GEMM's weight), or, with the gain on the activation side, Hg, and in the
#      MLP the down projection's operand Y.
# (S2) The saved activations a and b are stored for the backward (the
#      matrix-tile store primitive, "saving activations for the backward", in
#      the five-primitive table of both pages).
# (S3) The backward of a GEMM-epilogue program is again a GEMM with an
#      epilogue (kucoin (ru) §«В «Финале» спрятаны сокровища»: a block-local
#      forward epilogue gives a backward of the same structure).  Its GEMMs are
#      the adjoint of the forward GEMM, and the operand they read is the
#      gradient at the forward GEMM's raw output, before that GEMM's epilogue
#      transform.  GEMM2's epilogue applies r (the pages defer r to it), so
#      GEMM2's adjoint reads dZ = diag(r) dA, the gradient of Z = H W2g^T with
#      A = diag(r) Z; GEMM1's epilogue adds the residual, so GEMM1's adjoint
#      reads dH (which is the output dR, stored bf16); the MLP's gate/up GEMM
#      has no row scale, so its adjoint reads dA itself.
#
# Everything else stays float64: r, the SwiGLU output Y computed from the
# unrounded a and b, the RMSNorm backward's row term.  With store = identity
# every function here reduces to the textbook one above (pinned), and the
# placement of each rounding is pinned by hand-derived cases in
# tests/golden/ (a value of H on a bf16 midpoint, a pre-activation on a
# midpoint, a row scale r = 1/3 that moves the rounding of dZ).


def round_bf16(x) -> np.ndarray:
    """Round float64 values to the nearest bfloat16 (8 significant bits), ties to even.

    x = m * 2**e with 0.5 <= |m| < 1; keeping 8 significant bits means rounding
    m * 2**8 to an integer (numpy.rint rounds halves to even).  Values stay in
    bf16's normal range here (|x| between 1e-30 and 1e30), so no exponent
    clamping is needed; zeros pass through.
    """
    x = _f64(x)
    m, e = np.frexp(x)
    return np.ldexp(np.rint(m * 256.0) / 256.0, e)


def _ident(x):
    return x


def grg_forward_stored(X, W1, R, g, W2, eps: float, store=round_bf16, gain: str = "weight") -> dict:
    """grg_forward at the precision of the method's dataflow (S1, S2 above).

      H    = store(X W1^T + R)                 GEMM1's epilogue stores H (S1)
      r    = 1/sqrt(mean_j H_ij^2 + eps)       from the H that GEMM2 reads
      gain = "weight":     Z = H W2g^T,  W2g = store(W2 diag(g))      (S1, the fold)
      gain = "activation": Z = Hg W2^T,  Hg  = store(H diag(g))       (S1, gain on H)
      A    = diag(r) Z                         r applied after GEMM2 (the pages' identity)
      a, b = A[:, :F], A[:, F:];  Y = silu(a) * b      (from the unrounded a, b)
      a_s, b_s = store(a), store(b)            saved for the backward (S2)
    """
    X, W1, R, g, W2 = map(_f64, (X, W1, R, g, W2))
    H = store(X @ W1.T + R)
    d = H.shape[1]
    ms = np.sum(H * H, axis=1) / d
    r = 1.0 / np.sqrt(ms + eps)
    if gain == "weight":
        Z = H @ store(W2 * g[None, :]).T
    elif gain == "activation":
        Z = store(H * g[None, :]) @ W2.T
    else:
        raise ValueError(f"gain must be 'weight' or 'activation', got {gain!r}")
    A = r[:, None] * Z
    F = W2.shape[0] // 2
    a, b = A[:, :F], A[:, F:]
    Y = silu(a) * b
    return {"H": H, "r": r, "A": A, "a": a, "b": b, "a_s": store(a), "b_s": store(b), "Y": Y}


def grg_backward_stored(dY, X, W1, R, g, W2, eps: float, dH_in=None, store=round_bf16,
                        fwd: dict | None = None) -> dict:
    """grg_backward at the precision of the method's dataflow (S2, S3 above).

    The chain rule of grg_backward, fed by the stored H and the saved a_s, b_s,
    with two bf16 operands on the way:
      dA  = [da | db] from SwiGLU at (dY, a_s, b_s)
      dZ  = store(diag(r) dA)              gradient at GEMM2's raw output (S3)
      dW2 = g * (dZ^T H);  du = dZ W2 / r;  dg = sum_i du * n;  dn = du * g
      dH  = r dn - (r^3/d)(sum_k dn H) H (+ dH_in);   dR = dH
      dX  = store(dR) W1;  dW1 = store(dR)^T X   GEMM1's adjoint reads the stored dR (S3)
    """
    if fwd is None:
        fwd = grg_forward_stored(X, W1, R, g, W2, eps, store)
    dY, X, W1, g, W2 = map(_f64, (dY, X, W1, g, W2))
    H, r, a, b = fwd["H"], fwd["r"], fwd["a_s"], fwd["b_s"]
    d = H.shape[1]
    n = H * r[:, None]
    u = n * g[None, :]
    da, db = _swiglu_grads(dY, a, b)
    dZ = store(np.concatenate([da, db], axis=1) * r[:, None])
    dA = dZ / r[:, None]                  # the stored operand in units of the textbook dA
    dW2 = dA.T @ u
    du = dA @ W2
    dg = np.sum(du * n, axis=0)
    dn = du * g[None, :]
    dr = np.sum(dn * H, axis=1)
    dH = dn * r[:, None] + (dr * (-0.5) * r ** 3)[:, None] * (2.0 / d) * H
    if dH_in is not None:
        dH = dH + _f64(dH_in)
    dRs = store(dH)
    return {"dZ": dZ, "dA": dA, "dH": dH, "dR": dH, "dX": dRs @ W1, "dW1": dRs.T @ X, "dW2": dW2, "dg": dg}


def swiglu_forward_stored(X, Wgu, Wdown, store=round_bf16) -> dict:
    """swiglu_forward with the down projection reading the stored Y (S1) and
    a, b saved stored (S2)."""
    X, Wgu, Wdown = map(_f64, (X, Wgu, Wdown))
    A = X @ Wgu.T
    F = Wgu.shape[0] // 2
    a, b = A[:, :F], A[:, F:]
    Y = silu(a) * b
    Ys = store(Y)
    return {"A": A, "a": a, "b": b, "a_s": store(a), "b_s": store(b), "Y": Y, "Y_s": Ys, "Out": Ys @ Wdown.T}


def swiglu_backward_stored(dOut, X, Wgu, Wdown, store=round_bf16, fwd: dict | None = None) -> dict:
    """swiglu_backward fed by the stored Y, a, b, with the gate/up GEMM's
    adjoint reading the stored gradient at its output, dA = [da | db] (S3)."""
    if fwd is None:
        fwd = swiglu_forward_stored(X, Wgu, Wdown, store)
    dOut, X, Wgu, Wdown = map(_f64, (dOut, X, Wgu, Wdown))
    dY = dOut @ Wdown
    da, db = _swiglu_grads(dY, fwd["a_s"], fwd["b_s"])
    dA = store(np.concatenate([da, db], axis=1))
    return {"dY": dY, "dA": dA, "dWdown": dOut.T @ fwd["Y_s"], "dWgu": dA.T @ X, "dX": dA @ Wgu}


# ----------------------------------------------------------------------------- cross-entropy

def xent_forward(X, W, targets) -> dict:
    """Cross-entropy of the LM-head GEMM, textbook order.

      logits = X W^T              (X [M, d], W [V, d])
      lse_i  = log sum_j exp(logits_ij)          (max-shifted for range)
      loss_i = lse_i - logits_i,t_i
    The pages name cross-entropy among the operations rewritten as
    GEMM-epilogue programs, via a tile-wise log-sum-exp and the online
    max / sum-exp statistics (toolin.ai five-primitive table, rows "tile-wise
    reduction" and "stateful transform"; kucoin (ru) «В «Финале» спрятаны
    сокровища»).  The oracle is the plain definition, not the tiled form.
    """
    X, W = _f64(X), _f64(W)
    t = np.asarray(targets, dtype=np.int64)
    logits = X @ W.T
    m = np.max(logits, axis=1)
    lse = m + np.log(np.sum(np.exp(logits - m[:, None]), axis=1))
    loss = lse - logits[np.arange(X.shape[0]), t]
    return {"logits": logits, "lse": lse, "loss": loss}


def xent_backward(dloss, X, W, targets, fwd: dict | None = None, store=None) -> dict:
    """Gradients of L = sum_i dloss_i loss_i (chain rule by hand):
      dlogits_ij = dloss_i (softmax_ij - [j == t_i]);  dX = dlogits W;  dW = dlogits^T X.
    store: optional rounding of dlogits where the method stores it (bf16)
    before the two GEMMs read it; None keeps float64.
    """
    if fwd is None:
        fwd = xent_forward(X, W, targets)
    X, W, dloss = _f64(X), _f64(W), _f64(dloss)
    t = np.asarray(targets, dtype=np.int64)
    p = np.exp(fwd["logits"] - fwd["lse"][:, None])
    p[np.arange(X.shape[0]), t] -= 1.0
    dlogits = p * dloss[:, None]
    if store is not None:
        dlogits = store(dlogits)
    return {"dlogits": dlogits, "dX": dlogits @ W, "dW": dlogits.T @ X}


# ----------------------------------------------------------------------------- rotary position embedding

def rope_angles(seq_len: int, head_dim: int, base: float) -> np.ndarray:
    """angle[pos, j] = pos * base^(-2j / head_dim), j in [0, head_dim / 2)."""
    j = np.arange(head_dim // 2, dtype=np.float64)
    inv_freq = base ** (-2.0 * j / head_dim)
    return np.arange(seq_len, dtype=np.float64)[:, None] * inv_freq[None, :]


def rope_rotate(x, positions, head_dim: int, base: float, inverse: bool = False) -> np.ndarray:
    """Rotate each head of x [M, heads*head_dim]: the pair (j, j + head_dim/2)
    of a head at position p turns by p * base^(-2j/head_dim) (the
    rotate-half pairing); inverse=True turns by the negative angle."""
    x = _f64(x)
    M, W = x.shape
    half = head_dim // 2
    ang = np.asarray(positions, dtype=np.float64)[:, None] * \
        (base ** (-2.0 * np.arange(half, dtype=np.float64) / head_dim))[None, :]
    if inverse:
        ang = -ang
    c, s = np.cos(ang), np.sin(ang)
    out = np.empty_like(x)
    for h in range(W // head_dim):
        x1 = x[:, h * head_dim:h * head_dim + half]
        x2 = x[:, h * head_dim + half:(h + 1) * head_dim]
        out[:, h * head_dim:h * head_dim + half] = x1 * c - x2 * s
        out[:, h * head_dim + half:(h + 1) * head_dim] = x2 * c + x1 * s
    return out


def qkv_rope_forward(X, Wqkv, n_q: int, n_kv: int, head_dim: int, seq_len: int, base: float) -> dict:
    """QKV projection followed by RoPE on the q and k heads, unfused.

      QKV = X Wqkv^T, columns [q heads | k heads | v heads] (n_q, n_kv, n_kv heads)
      q, k rotated at position pos = token index mod seq_len; v unchanged.
    RoPE is one of the elementwise transforms the pages place in a GEMM
    epilogue (toolin.ai five-primitive table, row "elementwise transform";
    kucoin (ru) «В «Финале» спрятаны сокровища»).
    """
    X, Wqkv = _f64(X), _f64(Wqkv)
    pre = X @ Wqkv.T
    pos = np.arange(X.shape[0]) % seq_len
    nqk = (n_q + n_kv) * head_dim
    out = pre.copy()
    out[:, :nqk] = rope_rotate(pre[:, :nqk], pos, head_dim, base)
    return {"pre": pre, "QKV": out}


def qkv_rope_backward(dQKV, X, Wqkv, n_q: int, n_kv: int, head_dim: int, seq_len: int, base: float,
                      store=None) -> dict:
    """Gradients of <dQKV, QKV>: the inverse rotation of the q/k gradient, then
    dX = dPre Wqkv and dW = dPre^T X (store: optional rounding of dPre, which
    the method stores as bf16 before the GEMMs read it)."""
    dQKV, X, Wqkv = _f64(dQKV), _f64(X), _f64(Wqkv)
    pos = np.arange(X.shape[0]) % seq_len
    nqk = (n_q + n_kv) * head_dim
    dpre = dQKV.copy()
    dpre[:, :nqk] = rope_rotate(dQKV[:, :nqk], pos, head_dim, base, inverse=True)
    if store is not None:
        dpre = store(dpre)
    return {"dpre": dpre, "dX": dpre @ Wqkv, "dW": dpre.T @ X}


# ----------------------------------------------------------------------------- full MLP block

def mlp_block_forward(X, W1, R, g, W2, Wdown, eps: float, stored: bool = False, store=round_bf16) -> dict:
    """The block followed by the down projection and its residual:

      (H, r, a, b, Y) = the GEMM-Residual-RMSNorm-GEMM-SwiGLU forward
      Out = Y Wdown^T + H               (Wdown [d, F]; the next block's residual stream)
    The pages name residual add and SwiGLU among the epilogue transforms of
    the same family of GEMMs (toolin.ai five-primitive table).  With
    stored=True the GEMM-RMSNorm-GEMM part follows grg_forward_stored and the
    down GEMM reads the stored Y and the stored H.
    """
    Wdown = _f64(Wdown)
    if stored:
        f = grg_forward_stored(X, W1, R, g, W2, eps, store)
        out = store(f["Y"]) @ Wdown.T + f["H"]
    else:
        f = grg_forward(X, W1, R, g, W2, eps)
        out = f["Y"] @ Wdown.T + f["H"]
    return {**f, "Out": out}


def mlp_block_backward(dOut, X, W1, R, g, W2, Wdown, eps: float, stored: bool = False, store=round_bf16,
                       fwd: dict | None = None) -> dict:
    """Gradients of <dOut, Out> for mlp_block_forward by the chain rule:
      dY = dOut Wdown;  dWdown = dOut^T Y;  the residual passes dOut to H,
      then the block's backward with upstream (dY, dH_in = dOut).
    """
    if fwd is None:
        fwd = mlp_block_forward(X, W1, R, g, W2, Wdown, eps, stored, store)
    dOut, Wdown = _f64(dOut), _f64(Wdown)
    dY = dOut @ Wdown
    Ys = store(fwd["Y"]) if stored else fwd["Y"]
    dWdown = dOut.T @ Ys
    if stored:
        b = grg_backward_stored(dY, X, W1, R, g, W2, eps, dH_in=dOut, store=store, fwd=fwd)
    else:
        b = grg_backward(dY, X, W1, R, g, W2, eps, dH_in=dOut, fwd=fwd)
    return {**b, "dY": dY, "dWdown": dWdown}
