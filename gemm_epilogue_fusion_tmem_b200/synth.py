"""Seeded synthetic inputs shared by the tests, the smoke check and the bench.

This module draws random tensors and nothing else: it holds none of the
block's arithmetic.  Every tensor is drawn in float32 from one CPU
``torch.Generator`` and rounded to bfloat16 (round to nearest even), so the
CUDA path and the CPU oracle read the very same bf16 values.

Distributions (LLaMA-shaped synthetic data): activations X, R ~ N(0, 1);
weights ~ N(0, 1/fan_in) with fan_in the input width of that projection;
RMSNorm gain g = 1 + 0.1 N(0, 1); upstream gradients ~ N(0, 1).
"""

from __future__ import annotations

from dataclasses import dataclass

import torch


@dataclass(frozen=True)
class GRGShape:
    """GEMM-Residual-RMSNorm-GEMM(+SwiGLU) block: X[M,K] W1[d,K] R[M,d] W2[2F,d]."""
    name: str
    M: int
    K: int
    d: int
    F: int
    eps: float
    backward: bool = True

    @property
    def N(self) -> int:
        return 2 * self.F

    def flops(self, backward: bool | None = None) -> float:
        """Dense-contraction FLOPs: 2MKd + 2MdN forward, twice that backward."""
        bwd = self.backward if backward is None else backward
        fwd = 2.0 * self.M * self.K * self.d + 2.0 * self.M * self.d * self.N
        return fwd * (3.0 if bwd else 1.0)


@dataclass(frozen=True)
class SwiGLUShape:
    """SwiGLU MLP: X[M,d], Wgu[2F,d], Wdown[d,F]."""
    name: str
    M: int
    d: int
    F: int

    def flops(self, backward: bool = True) -> float:
        fwd = 2.0 * self.M * self.d * 2 * self.F + 2.0 * self.M * self.F * self.d
        return fwd * (3.0 if backward else 1.0)


# The LLaMA-shaped workloads (hidden sizes of 1B, 7B and 70B models).
TINY = GRGShape("tiny", M=256, K=512, d=512, F=1024, eps=1e-6)
GRG_1B = GRGShape("1B", M=8192, K=2048, d=2048, F=8192, eps=1e-6, backward=False)
GRG_7B = GRGShape("7B", M=8192, K=4096, d=4096, F=11008, eps=1e-6)
GRG_70B = GRGShape("70B", M=4096, K=8192, d=8192, F=28672, eps=1e-5)
SWIGLU_MLP = SwiGLUShape("swiglu", M=16384, d=4096, F=14336)

GRG_SHAPES = {s.name: s for s in (TINY, GRG_1B, GRG_7B, GRG_70B)}


def _normal(gen: torch.Generator, shape, std: float = 1.0, mean: float = 0.0) -> torch.Tensor:
    t = torch.randn(*shape, generator=gen, dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    if mean != 0.0:
        t.add_(mean)
    return t.to(torch.bfloat16)


def grg_inputs(M: int, K: int, d: int, F: int, seed: int = 0, dH_in: bool = False) -> dict:
    """Inputs of the GRG block, drawn in the fixed order X, R, W1, W2, g, dY (, dH_in)."""
    gen = torch.Generator().manual_seed(seed)
    out = {
        "X": _normal(gen, (M, K)),
        "R": _normal(gen, (M, d)),
        "W1": _normal(gen, (d, K), std=K ** -0.5),
        "W2": _normal(gen, (2 * F, d), std=d ** -0.5),
        "g": _normal(gen, (d,), std=0.1, mean=1.0),
        "dY": _normal(gen, (M, F)),
    }
    if dH_in:
        out["dH_in"] = _normal(gen, (M, d))
    return out


def swiglu_inputs(M: int, d: int, F: int, seed: int = 0) -> dict:
    """Inputs of the SwiGLU MLP, drawn in the fixed order X, Wgu, Wdown, dOut."""
    gen = torch.Generator().manual_seed(seed)
    return {
        "X": _normal(gen, (M, d)),
        "Wgu": _normal(gen, (2 * F, d), std=d ** -0.5),
        "Wdown": _normal(gen, (d, F), std=F ** -0.5),
        "dOut": _normal(gen, (M, d)),
    }


def gemm_inputs(M: int, N: int, K: int, seed: int = 0) -> dict:
    """A[M,K], B[N,K] ~ N(0,1) bf16 for plain-GEMM checks."""
    gen = torch.Generator().manual_seed(seed)
    return {"A": _normal(gen, (M, K)), "B": _normal(gen, (N, K), std=K ** -0.5)}


def xent_inputs(M: int, d: int, V: int, seed: int = 0) -> dict:
    """LM-head inputs drawn in the order X, W, targets, dloss: X ~ N(0,1), W ~ N(0, 1/d),
    targets uniform in [0, V) (int32), dloss ~ U(0, 1) / M (fp32)."""
    gen = torch.Generator().manual_seed(seed)
    X = _normal(gen, (M, d))
    W = _normal(gen, (V, d), std=d ** -0.5)
    targets = torch.randint(0, V, (M,), generator=gen, dtype=torch.int64).to(torch.int32)
    dloss = torch.rand(M, generator=gen, dtype=torch.float32) / M
    return {"X": X, "W": W, "targets": targets, "dloss": dloss}


XENT_LM_HEAD = {"name": "xent", "M": 8192, "d": 4096, "V": 128256}


def qkv_inputs(M: int, d: int, n_q: int, n_kv: int, head_dim: int, seed: int = 0) -> dict:
    """QKV projection inputs drawn in the order X, Wqkv, dQKV: X ~ N(0,1),
    Wqkv ~ N(0, 1/d) with rows [q heads | k heads | v heads], dQKV ~ N(0,1)."""
    gen = torch.Generator().manual_seed(seed)
    ncols = (n_q + 2 * n_kv) * head_dim
    return {"X": _normal(gen, (M, d)), "Wqkv": _normal(gen, (ncols, d), std=d ** -0.5),
            "dQKV": _normal(gen, (M, ncols))}


# LLaMA-7B attention input projection: 32 query and 32 key/value heads of 128, sequences of 2048.
QKV_ROPE_7B = {"name": "rope", "M": 8192, "d": 4096, "n_q": 32, "n_kv": 32, "head_dim": 128, "seq_len": 2048,
               "base": 10000.0}


def mlp_block_inputs(M: int, K: int, d: int, F: int, seed: int = 0) -> dict:
    """Full MLP block inputs: those of grg_inputs (X, R, W1, W2, g, dY drawn first, in that
    order) then Wdown ~ N(0, 1/F) and dOut ~ N(0, 1); dY is dropped (the block's upstream
    gradient is dOut)."""
    t = grg_inputs(M, K, d, F, seed=seed)
    gen = torch.Generator().manual_seed(seed + 7919)
    t.pop("dY")
    t["Wdown"] = _normal(gen, (d, F), std=F ** -0.5)
    t["dOut"] = _normal(gen, (M, d))
    return t
