"""Python binding of the C-ABI library (argument marshalling only).

Every step of the path runs in the CUDA kernels of ``libcoda.so``; this module
checks tensor dtypes/devices/contiguity, allocates outputs and the workspace
with torch (device memory and streams are all torch is used for), and passes
raw device pointers plus ``torch.cuda.current_stream()`` to the C entry points
of the same names.  There is no CPU fallback: if the library is missing or the
device is not sm_100, calls raise.  Each call into an entry point that enqueues
GPU work is wrapped in an NVTX range of the entry point's name.
"""

from __future__ import annotations

import ctypes
import os
import threading

import torch

from .build import LIB_PATH

_c_void_p = ctypes.c_void_p
_c_int = ctypes.c_int
_c_size_t = ctypes.c_size_t
_c_float = ctypes.c_float

CODA_ERR_INVALID_ARG = 1
CODA_ERR_DEVICE_TIMEOUT = 7


class CodaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = int(status)
        super().__init__(f"{where}: {_status_string(status)} (status {status})")


_lib = None
_lib_lock = threading.Lock()


def library() -> ctypes.CDLL:
    """Load libcoda.so (built in-tree by gemm_epilogue_fusion_tmem_b200.build)."""
    global _lib
    if _lib is not None:
        return _lib
    with _lib_lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"CUDA library not built ({LIB_PATH}); run `python -m gemm_epilogue_fusion_tmem_b200.build`")
        lib = ctypes.CDLL(LIB_PATH)
        P, I, S, F = _c_void_p, _c_int, _c_size_t, _c_float
        sig = {
            "coda_status_string": (ctypes.c_char_p, [I]),
            "coda_version": (I, []),
            "coda_status_clear": (I, [P, P]),
            "coda_status_query": (I, [P, P, ctypes.POINTER(ctypes.c_uint32)]),
            "coda_set_wait_limit_ns": (None, [ctypes.c_uint64]),
            "coda_selftest_wait_timeout": (I, [P, ctypes.c_uint64, P]),
            "coda_profile_arm": (I, [I, P, P]),
            "coda_gemm_workspace_bytes": (S, []),
            "coda_gemm": (I, [P, P, P, I, I, I, I, I, P, S, P]),
            "coda_fold_gain": (I, [P, P, P, I, I, P]),
            "coda_gemm_swiglu": (I, [P, P, P, P, P, I, I, I, P, S, P]),
            "coda_grg_fwd_workspace_bytes": (S, [I, I, I, I, I]),
            "coda_grg_fwd": (I, [P, P, P, P, P, P, P, P, P, P, I, I, I, I, F, P, S, P]),
            "coda_grg_bwd_workspace_bytes": (S, [I, I, I, I]),
            "coda_grg_bwd": (I, [P, P, P, P, P, P, P, P, P, P, P, P, P, P, I, I, I, I, P, S, P]),
            "coda_swiglu_fwd_workspace_bytes": (S, [I, I, I]),
            "coda_swiglu_fwd": (I, [P, P, P, P, P, P, I, I, I, P, S, P]),
            "coda_swiglu_bwd_workspace_bytes": (S, [I, I, I]),
            "coda_swiglu_bwd": (I, [P, P, P, P, P, P, P, P, P, I, I, I, P, S, P]),
            "coda_grg_fwd_hg_workspace_bytes": (S, [I, I, I, I, I]),
            "coda_grg_fwd_hg": (I, [P] * 10 + [I, I, I, I, F, P, S, P]),
            "coda_xent_fwd_workspace_bytes": (S, [I, I, I]),
            "coda_xent_fwd": (I, [P, P, P, P, P, I, I, I, P, S, P]),
            "coda_xent_bwd_workspace_bytes": (S, [I, I, I]),
            "coda_xent_bwd": (I, [P, P, P, P, P, P, P, I, I, I, P, S, P]),
            "coda_qkv_rope_fwd": (I, [P, P, P, I, I, I, I, I, I, F, P, S, P]),
            "coda_qkv_rope_bwd_workspace_bytes": (S, [I, I, I, I, I]),
            "coda_qkv_rope_bwd": (I, [P, P, P, P, P, I, I, I, I, I, I, F, P, S, P]),
            "coda_mlp_block_fwd_workspace_bytes": (S, [I, I, I, I]),
            "coda_mlp_block_fwd": (I, [P] * 11 + [I, I, I, I, F, P, S, P]),
            "coda_mlp_block_bwd_workspace_bytes": (S, [I, I, I, I]),
            "coda_mlp_block_bwd": (I, [P] * 16 + [I, I, I, I, P, S, P]),
            "coda_swiglu_fwd_unfused": (I, [P, P, P, P, P, P, I, I, I, P, S, P]),
            "coda_swiglu_bwd_unfused_workspace_bytes": (S, [I, I, I]),
            "coda_swiglu_bwd_unfused": (I, [P, P, P, P, P, P, P, P, P, I, I, I, P, S, P]),
            "coda_grg_fwd_unfused_workspace_bytes": (S, [I, I, I, I]),
            "coda_grg_fwd_unfused": (I, [P] * 10 + [I, I, I, I, F, P, S, P]),
            "coda_grg_bwd_unfused_workspace_bytes": (S, [I, I, I, I]),
            "coda_grg_bwd_unfused": (I, [P] * 15 + [I, I, I, I, P, S, P]),
            "coda_grg_fwd_prefolded_static": (I, [P] * 8 + [I, I, I, I, F, P]),
            "coda_static_status_query": (I, [P, ctypes.POINTER(ctypes.c_uint32)]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
            if name not in _UNRANGED and not name.endswith("_workspace_bytes"):
                setattr(lib, name, _Ranged(fn, name))
        _lib = lib
        return lib


# Host-side entry points that enqueue no GPU work get no NVTX range.
_UNRANGED = {"coda_status_string", "coda_version", "coda_set_wait_limit_ns", "coda_profile_arm",
             "coda_status_query", "coda_static_status_query"}


class _Ranged:
    """A C entry point called inside an NVTX range of its own name, so profilers
    (ncu --nvtx, Nsight Systems) attribute each call's kernels to it.  Without
    a profiler attached the push and pop do nothing."""

    __slots__ = ("_fn", "_name")

    def __init__(self, fn, name):
        self._fn, self._name = fn, name

    def __call__(self, *args):
        torch.cuda.nvtx.range_push(self._name)
        try:
            return self._fn(*args)
        finally:
            torch.cuda.nvtx.range_pop()

    def __getattr__(self, key):
        return getattr(self._fn, key)

    def __setattr__(self, key, value):
        # restype / argtypes set by a caller go to the ctypes function itself
        if key in self.__slots__:
            object.__setattr__(self, key, value)
        else:
            setattr(self._fn, key, value)


def _status_string(status: int) -> str:
    try:
        return library().coda_status_string(int(status)).decode()
    except Exception:  # pragma: no cover - only when the library cannot load
        return "unknown"


def _check(status: int, where: str) -> None:
    if status != 0:
        raise CodaError(status, where)


def _ptr(t: torch.Tensor | None):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _req(t: torch.Tensor, name: str, dtype=torch.bfloat16, shape=None) -> torch.Tensor:
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (no CPU path exists)")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    return t


# ------------------------------------------------------------------ workspace

class Workspace:
    """A caller-owned device workspace whose first 256 bytes are the status word."""

    def __init__(self, nbytes: int, device=None):
        self.buf = torch.zeros(max(int(nbytes), 256), dtype=torch.uint8, device=device or "cuda")

    @property
    def nbytes(self) -> int:
        return self.buf.numel()

    def ptr(self):
        return ctypes.c_void_p(self.buf.data_ptr())

    def clear(self) -> None:
        _check(library().coda_status_clear(self.ptr(), _stream()), "coda_status_clear")

    def query(self) -> tuple[int, int]:
        """Synchronise the current stream and return (status, detail)."""
        detail = ctypes.c_uint32(0)
        st = library().coda_status_query(self.ptr(), _stream(), ctypes.byref(detail))
        return int(st), int(detail.value)


_ws_cache: dict = {}


def workspace(nbytes: int, device=None) -> Workspace:
    """Per-device cached workspace grown on demand (zeroed when (re)allocated)."""
    dev = torch.device(device or "cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    ws = _ws_cache.get(dev)
    if ws is None or ws.nbytes < nbytes:
        ws = Workspace(nbytes, dev)
        _ws_cache[dev] = ws
    return ws


def set_wait_limit_ns(ns: int) -> None:
    library().coda_set_wait_limit_ns(int(ns))


# Kernel ids of the timing hook (coda_profile_arm): GEMMs by epilogue, light passes from 16.
EPI_STORE, EPI_RESID_RMS, EPI_SWIGLU, EPI_DN, EPI_SWIGLU_BWD, EPI_XENT, EPI_XENT_BWD, EPI_ROPE = range(8)
(KERNEL_FOLD_GAIN, KERNEL_RMS_ROWREDUCE, KERNEL_SWIGLU_BWD_ROWSTAT, KERNEL_COL_REDUCE, KERNEL_ROWCOEF_REDUCE,
 KERNEL_XENT_REDUCE, KERNEL_ROPE_UNROTATE) = range(16, 23)


def profile_arm(kernel: int, start=None, stop=None) -> None:
    """Arm a one-shot torch.cuda.Event pair around the next launch, from this
    thread, of the kernel `kernel` names (EPI_* or KERNEL_*); pairs armed for
    the same kernel fire on its successive launches.  No events disarms all."""
    def handle(ev):
        if ev is None:
            return None
        if ev.cuda_event == 0:  # torch creates the CUDA event at its first record
            ev.record()
        return ctypes.c_void_p(ev.cuda_event)

    _check(library().coda_profile_arm(int(kernel), handle(start), handle(stop)), "coda_profile_arm")


def selftest_wait_timeout(ws: Workspace, limit_ns: int) -> None:
    """Launch the bounded-wait self-test (a wait that must time out) on the current stream."""
    _check(library().coda_selftest_wait_timeout(ws.ptr(), int(limit_ns), _stream()), "coda_selftest_wait_timeout")


# ------------------------------------------------------------------ entry points

def gemm(A: torch.Tensor, B: torch.Tensor, M: int, N: int, K: int, a_mn_major: bool = False,
         b_mn_major: bool = False, out: torch.Tensor | None = None, ws: Workspace | None = None) -> torch.Tensor:
    """C[M,N] = op(A) op(B)^T (bf16 out, fp32 accumulate); see coda_gemm in include/coda.h."""
    lib = library()
    _req(A, "A", shape=(K, M) if a_mn_major else (M, K))
    _req(B, "B", shape=(K, N) if b_mn_major else (N, K))
    C = out if out is not None else torch.empty(M, N, dtype=torch.bfloat16, device=A.device)
    _req(C, "C", shape=(M, N))
    ws = ws or workspace(lib.coda_gemm_workspace_bytes(), A.device)
    _check(lib.coda_gemm(_ptr(A), _ptr(B), _ptr(C), M, N, K, int(a_mn_major), int(b_mn_major),
                         ws.ptr(), ws.nbytes, _stream()), "coda_gemm")
    return C


def gemm_swiglu(A, Wgu, r=None, save_ab: bool = True, out: dict | None = None,
                ws: Workspace | None = None) -> dict:
    """Y = silu(r*(A Wgu^T)_gate) * (r*(A Wgu^T)_up), AB = [a | b]; see coda_gemm_swiglu."""
    lib = library()
    M, K = A.shape
    F = Wgu.shape[0] // 2
    _req(A, "A"), _req(Wgu, "Wgu", shape=(2 * F, K))
    if r is not None:
        _req(r, "r", torch.float32, (M,))
    o = dict(out or {})
    if "Y" not in o:
        o["Y"] = torch.empty(M, F, dtype=torch.bfloat16, device=A.device)
    if save_ab:
        if "AB" not in o:
            o["AB"] = torch.empty(M, 2 * F, dtype=torch.bfloat16, device=A.device)
    ws = ws or workspace(lib.coda_gemm_workspace_bytes(), A.device)
    _check(lib.coda_gemm_swiglu(_ptr(A), _ptr(Wgu), _ptr(r), _ptr(o["Y"]), _ptr(o.get("AB") if save_ab else None),
                                M, K, F, ws.ptr(), ws.nbytes, _stream()), "coda_gemm_swiglu")
    return o


def fold_gain(W2: torch.Tensor, g: torch.Tensor, out: torch.Tensor | None = None) -> torch.Tensor:
    """W2g = W2 * g (per column), bf16; see coda_fold_gain."""
    N, d = W2.shape
    _req(W2, "W2")
    _req(g, "g", shape=(d,))
    W2g = out if out is not None else torch.empty_like(W2)
    _req(W2g, "W2g", shape=(N, d))
    _check(library().coda_fold_gain(_ptr(W2), _ptr(g), _ptr(W2g), d, N, _stream()), "coda_fold_gain")
    return W2g


def grg_fwd(X, W1, R, g, W2, eps: float, W2g=None, save_ab: bool = True, out: dict | None = None,
            ws: Workspace | None = None) -> dict:
    """Fused GEMM-Residual-PartialRMS-GEMM-SwiGLU forward; returns H, r, Y, AB."""
    lib = library()
    M, K = X.shape
    d = W1.shape[0]
    N = W2.shape[0]
    F = N // 2
    _req(X, "X"), _req(W1, "W1", shape=(d, K)), _req(R, "R", shape=(M, d))
    _req(g, "g", shape=(d,)), _req(W2, "W2", shape=(N, d))
    if W2g is not None:
        _req(W2g, "W2g", shape=(N, d))
    o = dict(out or {})
    dev = X.device
    if "H" not in o:
        o["H"] = torch.empty(M, d, dtype=torch.bfloat16, device=dev)
    if "r" not in o:
        o["r"] = torch.empty(M, dtype=torch.float32, device=dev)
    if "Y" not in o:
        o["Y"] = torch.empty(M, F, dtype=torch.bfloat16, device=dev)
    if save_ab and "AB" not in o:
        o["AB"] = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
    _req(o["H"], "H", shape=(M, d)), _req(o["r"], "r", torch.float32, (M,)), _req(o["Y"], "Y", shape=(M, F))
    AB = o.get("AB") if save_ab else None
    if AB is not None:
        _req(AB, "AB", shape=(M, N))
    need = lib.coda_grg_fwd_workspace_bytes(M, K, d, N, int(W2g is not None))
    ws = ws or workspace(need, dev)
    _check(lib.coda_grg_fwd(_ptr(X), _ptr(W1), _ptr(R), _ptr(g), _ptr(W2), _ptr(W2g), _ptr(o["H"]),
                            _ptr(o["r"]), _ptr(o["Y"]), _ptr(AB), M, K, d, N, float(eps),
                            ws.ptr(), ws.nbytes, _stream()), "coda_grg_fwd")
    return o


def grg_fwd_prefolded_static(X, W1, R, W2g, eps: float, save_ab: bool = True, out: dict | None = None) -> dict:
    """The forward for callers that cannot allocate device memory: the same
    kernels as grg_fwd given a pre-folded W2g, with the scratch in the
    library's static device array (no workspace).  Outputs are allocated here
    unless passed in `out`; a caller that must not allocate passes them all.
    Calls that overlap on the GPU share the static array and must be
    serialised.  Returns H, r, Y, AB."""
    lib = library()
    M, K = X.shape
    d = W1.shape[0]
    N = W2g.shape[0]
    F = N // 2
    _req(X, "X"), _req(W1, "W1", shape=(d, K)), _req(R, "R", shape=(M, d)), _req(W2g, "W2g", shape=(N, d))
    o = dict(out or {})
    dev = X.device
    for k, shape, dt in (("H", (M, d), torch.bfloat16), ("r", (M,), torch.float32), ("Y", (M, F), torch.bfloat16)):
        if k not in o:
            o[k] = torch.empty(*shape, dtype=dt, device=dev)
        _req(o[k], k, dt, shape)
    if save_ab and "AB" not in o:
        o["AB"] = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
    AB = o.get("AB") if save_ab else None
    if AB is not None:
        _req(AB, "AB", shape=(M, N))
    _check(lib.coda_grg_fwd_prefolded_static(_ptr(X), _ptr(W1), _ptr(R), _ptr(W2g), _ptr(o["H"]), _ptr(o["r"]),
                                             _ptr(o["Y"]), _ptr(AB), M, K, d, N, float(eps), _stream()),
           "coda_grg_fwd_prefolded_static")
    return o


def static_status() -> tuple[int, int]:
    """Synchronise the current stream and return (status, detail) of the last
    grg_fwd_prefolded_static call on the current device."""
    detail = ctypes.c_uint32(0)
    st = library().coda_static_status_query(_stream(), ctypes.byref(detail))
    return int(st), int(detail.value)


def grg_fwd_hg(X, W1, R, g, W2, eps: float, save_ab: bool = True, keep_hg: bool = False, out: dict | None = None,
               ws: Workspace | None = None) -> dict:
    """Forward with the gain on the activation side (Hg = H*g from GEMM1's epilogue); returns H, r, Y, AB (, Hg)."""
    lib = library()
    M, K = X.shape
    d = W1.shape[0]
    N = W2.shape[0]
    F = N // 2
    _req(X, "X"), _req(W1, "W1", shape=(d, K)), _req(R, "R", shape=(M, d))
    _req(g, "g", shape=(d,)), _req(W2, "W2", shape=(N, d))
    o = dict(out or {})
    dev = X.device
    want = [("H", (M, d), torch.bfloat16), ("r", (M,), torch.float32), ("Y", (M, F), torch.bfloat16)]
    if save_ab:
        want.append(("AB", (M, N), torch.bfloat16))
    if keep_hg:
        want.append(("Hg", (M, d), torch.bfloat16))
    for k, shape, dt in want:
        if k not in o:
            o[k] = torch.empty(*shape, dtype=dt, device=dev)
        _req(o[k], k, dt, shape)
    Hg = o.get("Hg") if keep_hg else None
    ws = ws or workspace(lib.coda_grg_fwd_hg_workspace_bytes(M, K, d, N, int(Hg is not None)), dev)
    _check(lib.coda_grg_fwd_hg(_ptr(X), _ptr(W1), _ptr(R), _ptr(g), _ptr(W2), _ptr(o["H"]), _ptr(Hg), _ptr(o["r"]),
                               _ptr(o["Y"]), _ptr(o.get("AB") if save_ab else None), M, K, d, N, float(eps),
                               ws.ptr(), ws.nbytes, _stream()), "coda_grg_fwd_hg")
    return o


def grg_bwd(dY, X, W1, H, r, AB, g, W2, dH_in=None, out: dict | None = None, ws: Workspace | None = None) -> dict:
    """Fused backward of the block; returns dX, dR, dW1, dW2, dg."""
    lib = library()
    M, K = X.shape
    d = W1.shape[0]
    N = W2.shape[0]
    F = N // 2
    _req(dY, "dY", shape=(M, F)), _req(X, "X"), _req(W1, "W1", shape=(d, K)), _req(H, "H", shape=(M, d))
    _req(r, "r", torch.float32, (M,)), _req(AB, "AB", shape=(M, N)), _req(g, "g", shape=(d,))
    _req(W2, "W2", shape=(N, d))
    if dH_in is not None:
        _req(dH_in, "dH_in", shape=(M, d))
    o = dict(out or {})
    dev = X.device
    for k, shape, dt in (("dX", (M, K), torch.bfloat16), ("dR", (M, d), torch.bfloat16),
                         ("dW1", (d, K), torch.bfloat16), ("dW2", (N, d), torch.bfloat16),
                         ("dg", (d,), torch.float32)):
        if k not in o:
            o[k] = torch.empty(*shape, dtype=dt, device=dev)
    ws = ws or workspace(lib.coda_grg_bwd_workspace_bytes(M, K, d, N), dev)
    _check(lib.coda_grg_bwd(_ptr(dY), _ptr(dH_in), _ptr(X), _ptr(W1), _ptr(H), _ptr(r), _ptr(AB), _ptr(g),
                            _ptr(W2), _ptr(o["dX"]), _ptr(o["dR"]), _ptr(o["dW1"]), _ptr(o["dW2"]), _ptr(o["dg"]),
                            M, K, d, N, ws.ptr(), ws.nbytes, _stream()), "coda_grg_bwd")
    return o


def swiglu_fwd(X, Wgu, Wdown, save_ab: bool = True, out: dict | None = None, ws: Workspace | None = None) -> dict:
    """SwiGLU MLP forward; returns Y, AB, Out."""
    lib = library()
    M, d = X.shape
    F = Wgu.shape[0] // 2
    _req(X, "X"), _req(Wgu, "Wgu", shape=(2 * F, d)), _req(Wdown, "Wdown", shape=(d, F))
    o = dict(out or {})
    dev = X.device
    if "Y" not in o:
        o["Y"] = torch.empty(M, F, dtype=torch.bfloat16, device=dev)
    if save_ab:
        if "AB" not in o:
            o["AB"] = torch.empty(M, 2 * F, dtype=torch.bfloat16, device=dev)
    if "Out" not in o:
        o["Out"] = torch.empty(M, d, dtype=torch.bfloat16, device=dev)
    ws = ws or workspace(lib.coda_swiglu_fwd_workspace_bytes(M, d, F), dev)
    _check(lib.coda_swiglu_fwd(_ptr(X), _ptr(Wgu), _ptr(Wdown), _ptr(o["Y"]), _ptr(o.get("AB") if save_ab else None),
                               _ptr(o["Out"]), M, d, F, ws.ptr(), ws.nbytes, _stream()), "coda_swiglu_fwd")
    return o


def swiglu_bwd(dOut, X, Wgu, Wdown, Y, AB, out: dict | None = None, ws: Workspace | None = None) -> dict:
    """SwiGLU MLP backward; returns dX, dWgu, dWdown."""
    lib = library()
    M, d = X.shape
    F = Wgu.shape[0] // 2
    _req(dOut, "dOut", shape=(M, d)), _req(X, "X"), _req(Wgu, "Wgu", shape=(2 * F, d))
    _req(Wdown, "Wdown", shape=(d, F)), _req(Y, "Y", shape=(M, F)), _req(AB, "AB", shape=(M, 2 * F))
    o = dict(out or {})
    dev = X.device
    if "dX" not in o:
        o["dX"] = torch.empty(M, d, dtype=torch.bfloat16, device=dev)
    if "dWgu" not in o:
        o["dWgu"] = torch.empty(2 * F, d, dtype=torch.bfloat16, device=dev)
    if "dWdown" not in o:
        o["dWdown"] = torch.empty(d, F, dtype=torch.bfloat16, device=dev)
    ws = ws or workspace(lib.coda_swiglu_bwd_workspace_bytes(M, d, F), dev)
    _check(lib.coda_swiglu_bwd(_ptr(dOut), _ptr(X), _ptr(Wgu), _ptr(Wdown), _ptr(Y), _ptr(AB), _ptr(o["dX"]),
                               _ptr(o["dWgu"]), _ptr(o["dWdown"]), M, d, F, ws.ptr(), ws.nbytes, _stream()),
           "coda_swiglu_bwd")
    return o


# ------------------------------------------------------------------ unfused comparison sequence

def grg_fwd_unfused(X, W1, R, g, W2, eps: float, out: dict | None = None, ws: Workspace | None = None) -> dict:
    """Operator-by-operator forward (measurement/comparison only); returns H, r, Y, AB, U."""
    lib = library()
    M, K = X.shape
    d = W1.shape[0]
    N = W2.shape[0]
    F = N // 2
    _req(X, "X"), _req(W1, "W1", shape=(d, K)), _req(R, "R", shape=(M, d))
    _req(g, "g", shape=(d,)), _req(W2, "W2", shape=(N, d))
    o = dict(out or {})
    dev = X.device
    for k, shape, dt in (("H", (M, d), torch.bfloat16), ("r", (M,), torch.float32), ("Y", (M, F), torch.bfloat16),
                         ("AB", (M, N), torch.bfloat16), ("U", (M, d), torch.bfloat16)):
        if k not in o:
            o[k] = torch.empty(*shape, dtype=dt, device=dev)
        _req(o[k], k, dt, shape)
    ws = ws or workspace(lib.coda_grg_fwd_unfused_workspace_bytes(M, K, d, N), dev)
    _check(lib.coda_grg_fwd_unfused(_ptr(X), _ptr(W1), _ptr(R), _ptr(g), _ptr(W2), _ptr(o["H"]), _ptr(o["r"]),
                                    _ptr(o["Y"]), _ptr(o["AB"]), _ptr(o["U"]), M, K, d, N, float(eps),
                                    ws.ptr(), ws.nbytes, _stream()), "coda_grg_fwd_unfused")
    return o


def grg_bwd_unfused(dY, X, W1, H, r, AB, U, g, W2, dH_in=None, out: dict | None = None,
                    ws: Workspace | None = None) -> dict:
    """Operator-by-operator backward (measurement/comparison only); returns dX, dR, dW1, dW2, dg."""
    lib = library()
    M, K = X.shape
    d = W1.shape[0]
    N = W2.shape[0]
    F = N // 2
    _req(dY, "dY", shape=(M, F)), _req(X, "X"), _req(W1, "W1", shape=(d, K)), _req(H, "H", shape=(M, d))
    _req(r, "r", torch.float32, (M,)), _req(AB, "AB", shape=(M, N)), _req(U, "U", shape=(M, d))
    _req(g, "g", shape=(d,)), _req(W2, "W2", shape=(N, d))
    if dH_in is not None:
        _req(dH_in, "dH_in", shape=(M, d))
    o = dict(out or {})
    dev = X.device
    for k, shape, dt in (("dX", (M, K), torch.bfloat16), ("dR", (M, d), torch.bfloat16),
                         ("dW1", (d, K), torch.bfloat16), ("dW2", (N, d), torch.bfloat16),
                         ("dg", (d,), torch.float32)):
        if k not in o:
            o[k] = torch.empty(*shape, dtype=dt, device=dev)
    ws = ws or workspace(lib.coda_grg_bwd_unfused_workspace_bytes(M, K, d, N), dev)
    _check(lib.coda_grg_bwd_unfused(_ptr(dY), _ptr(dH_in), _ptr(X), _ptr(W1), _ptr(H), _ptr(r), _ptr(AB), _ptr(U),
                                    _ptr(g), _ptr(W2), _ptr(o["dX"]), _ptr(o["dR"]), _ptr(o["dW1"]), _ptr(o["dW2"]),
                                    _ptr(o["dg"]), M, K, d, N, ws.ptr(), ws.nbytes, _stream()),
           "coda_grg_bwd_unfused")
    return o


# ------------------------------------------------------------------ cross-entropy on the LM head

def xent_fwd(X, W, targets, out: dict | None = None, ws: Workspace | None = None) -> dict:
    """Per-row cross-entropy of X W^T without materialising the logits; returns loss, lse (fp32 [M])."""
    lib = library()
    M, d = X.shape
    V = W.shape[0]
    _req(X, "X"), _req(W, "W", shape=(V, d)), _req(targets, "targets", torch.int32, (M,))
    o = dict(out or {})
    for k in ("loss", "lse"):
        if k not in o:
            o[k] = torch.empty(M, dtype=torch.float32, device=X.device)
        _req(o[k], k, torch.float32, (M,))
    ws = ws or workspace(lib.coda_xent_fwd_workspace_bytes(M, d, V), X.device)
    _check(lib.coda_xent_fwd(_ptr(X), _ptr(W), _ptr(targets), _ptr(o["loss"]), _ptr(o["lse"]), M, d, V,
                             ws.ptr(), ws.nbytes, _stream()), "coda_xent_fwd")
    return o


def xent_bwd(X, W, targets, lse, dloss, out: dict | None = None, ws: Workspace | None = None) -> dict:
    """Gradients of sum_i dloss_i loss_i; returns dX [M,d], dW [V,d] (bf16)."""
    lib = library()
    M, d = X.shape
    V = W.shape[0]
    _req(X, "X"), _req(W, "W", shape=(V, d)), _req(targets, "targets", torch.int32, (M,))
    _req(lse, "lse", torch.float32, (M,)), _req(dloss, "dloss", torch.float32, (M,))
    o = dict(out or {})
    if "dX" not in o:
        o["dX"] = torch.empty(M, d, dtype=torch.bfloat16, device=X.device)
    if "dW" not in o:
        o["dW"] = torch.empty(V, d, dtype=torch.bfloat16, device=X.device)
    ws = ws or workspace(lib.coda_xent_bwd_workspace_bytes(M, d, V), X.device)
    _check(lib.coda_xent_bwd(_ptr(X), _ptr(W), _ptr(targets), _ptr(lse), _ptr(dloss), _ptr(o["dX"]), _ptr(o["dW"]),
                             M, d, V, ws.ptr(), ws.nbytes, _stream()), "coda_xent_bwd")
    return o


# ------------------------------------------------------------------ QKV projection with RoPE

def qkv_rope_fwd(X, Wqkv, n_q: int, n_kv: int, head_dim: int, seq_len: int, base: float = 10000.0,
                 out: torch.Tensor | None = None, ws: Workspace | None = None) -> torch.Tensor:
    """QKV = X Wqkv^T with RoPE on the q and k heads applied in the GEMM epilogue."""
    lib = library()
    M, d = X.shape
    ncols = (n_q + 2 * n_kv) * head_dim
    _req(X, "X"), _req(Wqkv, "Wqkv", shape=(ncols, d))
    Q = out if out is not None else torch.empty(M, ncols, dtype=torch.bfloat16, device=X.device)
    _req(Q, "QKV", shape=(M, ncols))
    ws = ws or workspace(lib.coda_gemm_workspace_bytes(), X.device)
    _check(lib.coda_qkv_rope_fwd(_ptr(X), _ptr(Wqkv), _ptr(Q), M, d, n_q, n_kv, head_dim, seq_len, float(base),
                                 ws.ptr(), ws.nbytes, _stream()), "coda_qkv_rope_fwd")
    return Q


def qkv_rope_bwd(dQKV, X, Wqkv, n_q: int, n_kv: int, head_dim: int, seq_len: int, base: float = 10000.0,
                 out: dict | None = None, ws: Workspace | None = None) -> dict:
    """Backward of qkv_rope_fwd; returns dX, dW."""
    lib = library()
    M, d = X.shape
    ncols = (n_q + 2 * n_kv) * head_dim
    _req(dQKV, "dQKV", shape=(M, ncols)), _req(X, "X"), _req(Wqkv, "Wqkv", shape=(ncols, d))
    o = dict(out or {})
    if "dX" not in o:
        o["dX"] = torch.empty(M, d, dtype=torch.bfloat16, device=X.device)
    if "dW" not in o:
        o["dW"] = torch.empty(ncols, d, dtype=torch.bfloat16, device=X.device)
    ws = ws or workspace(lib.coda_qkv_rope_bwd_workspace_bytes(M, d, n_q, n_kv, head_dim), X.device)
    _check(lib.coda_qkv_rope_bwd(_ptr(dQKV), _ptr(X), _ptr(Wqkv), _ptr(o["dX"]), _ptr(o["dW"]), M, d, n_q, n_kv,
                                 head_dim, seq_len, float(base), ws.ptr(), ws.nbytes, _stream()), "coda_qkv_rope_bwd")
    return o


# ------------------------------------------------------------------ full MLP block

def mlp_block_fwd(X, W1, R, g, W2, Wdown, eps: float, out: dict | None = None, ws: Workspace | None = None) -> dict:
    """Block forward plus the down projection with the residual epilogue; returns H, r, Y, AB, Out."""
    lib = library()
    M, K = X.shape
    d = W1.shape[0]
    N = W2.shape[0]
    F = N // 2
    _req(X, "X"), _req(W1, "W1", shape=(d, K)), _req(R, "R", shape=(M, d)), _req(g, "g", shape=(d,))
    _req(W2, "W2", shape=(N, d)), _req(Wdown, "Wdown", shape=(d, F))
    o = dict(out or {})
    for k, shape, dt in (("H", (M, d), torch.bfloat16), ("r", (M,), torch.float32), ("Y", (M, F), torch.bfloat16),
                         ("AB", (M, N), torch.bfloat16), ("Out", (M, d), torch.bfloat16)):
        if k not in o:
            o[k] = torch.empty(*shape, dtype=dt, device=X.device)
        _req(o[k], k, dt, shape)
    ws = ws or workspace(lib.coda_mlp_block_fwd_workspace_bytes(M, K, d, F), X.device)
    _check(lib.coda_mlp_block_fwd(_ptr(X), _ptr(W1), _ptr(R), _ptr(g), _ptr(W2), _ptr(Wdown), _ptr(o["H"]),
                                  _ptr(o["r"]), _ptr(o["Y"]), _ptr(o["AB"]), _ptr(o["Out"]), M, K, d, F, float(eps),
                                  ws.ptr(), ws.nbytes, _stream()), "coda_mlp_block_fwd")
    return o


def mlp_block_bwd(dOut, X, W1, H, r, AB, Y, g, W2, Wdown, out: dict | None = None,
                  ws: Workspace | None = None) -> dict:
    """Backward of the full block; returns dX, dR, dW1, dW2, dg, dWdown."""
    lib = library()
    M, K = X.shape
    d = W1.shape[0]
    N = W2.shape[0]
    F = N // 2
    _req(dOut, "dOut", shape=(M, d)), _req(X, "X"), _req(W1, "W1", shape=(d, K)), _req(H, "H", shape=(M, d))
    _req(r, "r", torch.float32, (M,)), _req(AB, "AB", shape=(M, N)), _req(Y, "Y", shape=(M, F))
    _req(g, "g", shape=(d,)), _req(W2, "W2", shape=(N, d)), _req(Wdown, "Wdown", shape=(d, F))
    o = dict(out or {})
    for k, shape, dt in (("dX", (M, K), torch.bfloat16), ("dR", (M, d), torch.bfloat16),
                         ("dW1", (d, K), torch.bfloat16), ("dW2", (N, d), torch.bfloat16),
                         ("dg", (d,), torch.float32), ("dWdown", (d, F), torch.bfloat16)):
        if k not in o:
            o[k] = torch.empty(*shape, dtype=dt, device=X.device)
    ws = ws or workspace(lib.coda_mlp_block_bwd_workspace_bytes(M, K, d, F), X.device)
    _check(lib.coda_mlp_block_bwd(_ptr(dOut), _ptr(X), _ptr(W1), _ptr(H), _ptr(r), _ptr(AB), _ptr(Y), _ptr(g),
                                  _ptr(W2), _ptr(Wdown), _ptr(o["dX"]), _ptr(o["dR"]), _ptr(o["dW1"]), _ptr(o["dW2"]),
                                  _ptr(o["dg"]), _ptr(o["dWdown"]), M, K, d, F, ws.ptr(), ws.nbytes, _stream()),
           "coda_mlp_block_bwd")
    return o


def swiglu_fwd_unfused(X, Wgu, Wdown, out: dict | None = None, ws: Workspace | None = None) -> dict:
    """The SwiGLU MLP forward operator by operator (measurement only); returns Y, AB, Out."""
    lib = library()
    M, d = X.shape
    F = Wgu.shape[0] // 2
    _req(X, "X"), _req(Wgu, "Wgu", shape=(2 * F, d)), _req(Wdown, "Wdown", shape=(d, F))
    o = dict(out or {})
    for k, shape in (("Y", (M, F)), ("AB", (M, 2 * F)), ("Out", (M, d))):
        if k not in o:
            o[k] = torch.empty(*shape, dtype=torch.bfloat16, device=X.device)
    ws = ws or workspace(lib.coda_gemm_workspace_bytes(), X.device)
    _check(lib.coda_swiglu_fwd_unfused(_ptr(X), _ptr(Wgu), _ptr(Wdown), _ptr(o["Y"]), _ptr(o["AB"]), _ptr(o["Out"]),
                                       M, d, F, ws.ptr(), ws.nbytes, _stream()), "coda_swiglu_fwd_unfused")
    return o


def swiglu_bwd_unfused(dOut, X, Wgu, Wdown, Y, AB, out: dict | None = None, ws: Workspace | None = None) -> dict:
    """The SwiGLU MLP backward operator by operator (measurement only); returns dX, dWgu, dWdown."""
    lib = library()
    M, d = X.shape
    F = Wgu.shape[0] // 2
    _req(dOut, "dOut", shape=(M, d)), _req(Y, "Y", shape=(M, F)), _req(AB, "AB", shape=(M, 2 * F))
    o = dict(out or {})
    for k, shape in (("dX", (M, d)), ("dWgu", (2 * F, d)), ("dWdown", (d, F))):
        if k not in o:
            o[k] = torch.empty(*shape, dtype=torch.bfloat16, device=X.device)
    ws = ws or workspace(lib.coda_swiglu_bwd_unfused_workspace_bytes(M, d, F), X.device)
    _check(lib.coda_swiglu_bwd_unfused(_ptr(dOut), _ptr(X), _ptr(Wgu), _ptr(Wdown), _ptr(Y), _ptr(AB), _ptr(o["dX"]),
                                       _ptr(o["dWgu"]), _ptr(o["dWdown"]), M, d, F, ws.ptr(), ws.nbytes, _stream()),
           "coda_swiglu_bwd_unfused")
    return o
