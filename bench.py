#!/usr/bin/env python
"""Throughput of the fused GEMM-Residual-RMSNorm-GEMM(+SwiGLU) block on B200.

One step = one pass of the whole hot path over one batch of synthetic
LLaMA-shaped input: for the GRG workloads the gain fold, GEMM1 + residual +
partial RMS, GEMM2 + r (reduced from the partials in its epilogue) + SwiGLU,
and (fwd+bwd workloads) the
SwiGLU backward + row statistic, the dn GEMM, the dg column reduce, the dW2,
dX and dW1 GEMMs.  All of it runs in libcoda.so through the C ABI.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload 7B|70B|1B|swiglu|tiny|xent|rope|block7B]
  python bench.py --impl reference ...   (the fp64 CPU oracle on the host cores)

Prints one JSON line on rank 0.  Under torchrun each rank runs an independent
replica on its own GPU (the block has no exchange step on one GPU's worth of
tokens); value = all ranks' FLOPs / max-over-ranks device time.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "fused GEMM-RMSNorm-GEMM fwd+bwd TFLOP/s and % of B200 bf16 tensor peak"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
DENSE_BF16_FLOP_PER_SM_CLK = 8192  # tcgen05 dense bf16: 4096 multiply-adds per SM per clock
INTERLEAVED = ("10 rounds of alternating bursts of at least 5 steps each, the order swapped every round, "
               "median ms per step of each")

WORKLOADS = {
    "tiny": ("grg", dict(M=256, K=512, d=512, F=1024, eps=1e-6), True),
    "1B": ("grg", dict(M=8192, K=2048, d=2048, F=8192, eps=1e-6), False),
    "7B": ("grg", dict(M=8192, K=4096, d=4096, F=11008, eps=1e-6), True),
    "70B": ("grg", dict(M=4096, K=8192, d=8192, F=28672, eps=1e-5), True),
    "swiglu": ("swiglu", dict(M=16384, d=4096, F=14336), True),
    "xent": ("xent", dict(M=8192, d=4096, V=128256), True),
    "block7B": ("block", dict(M=8192, K=4096, d=4096, F=11008, eps=1e-6), True),
    "rope": ("rope", dict(M=8192, d=4096, n_q=32, n_kv=32, head_dim=128, seq_len=2048, base=10000.0), True),
}


def _args():
    p = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=100)
    p.add_argument("--warmup", type=int, default=3)
    p.add_argument("--impl", choices=["coda", "reference"], default="coda")
    p.add_argument("--workload", choices=sorted(WORKLOADS), default="7B")
    p.add_argument("--no-cpu-baseline", action="store_true", help="skip the timed oracle sample")
    p.add_argument("--no-e2e", action="store_true", help="skip the host-buffer end-to-end measurement")
    p.add_argument("--no-unfused", action="store_true", help="skip timing the unfused comparison sequence")
    p.add_argument("--no-extra", action="store_true", help="skip timing the 70B shape beside the 7B headline")
    p.add_argument("--only", choices=["fused", "activation_gain", "unfused"], default=None,
                   help="profiling aid: run the warm-up steps and then exactly one step of this path, "
                        "print its kernel launches per step and exit (no timing, no JSON contract line)")
    return p.parse_args()


def _peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return json.load(f), "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def _flops(kind, s, bwd):
    if kind == "block":  # the block plus the down projection
        fwd = 2.0 * s["M"] * s["K"] * s["d"] + 2.0 * s["M"] * s["d"] * 2 * s["F"] + 2.0 * s["M"] * s["F"] * s["d"]
        return fwd * (3.0 if bwd else 1.0)
    if kind == "rope":
        return 2.0 * s["M"] * s["d"] * (s["n_q"] + 2 * s["n_kv"]) * s["head_dim"] * (3.0 if bwd else 1.0)
    if kind == "xent":  # logits GEMM forward, dX and dW backward (the backward's recompute is not counted)
        return 2.0 * s["M"] * s["d"] * s["V"] * (3.0 if bwd else 1.0)
    if kind == "grg":
        fwd = 2.0 * s["M"] * s["K"] * s["d"] + 2.0 * s["M"] * s["d"] * 2 * s["F"]
    else:
        fwd = 2.0 * s["M"] * s["d"] * 2 * s["F"] + 2.0 * s["M"] * s["F"] * s["d"]
    return fwd * (3.0 if bwd else 1.0)


def _describe(name, kind, s, bwd):
    if kind == "grg":
        what = f"GEMM-Residual-RMSNorm-GEMM-SwiGLU {name} {'fwd+bwd' if bwd else 'fwd'}"
    elif kind == "xent":
        what = "LM-head cross-entropy fwd+bwd (LLaMA-3 vocabulary)"
    elif kind == "rope":
        what = "QKV projection with RoPE epilogue fwd+bwd (LLaMA-7B attention)"
    elif kind == "block":
        what = f"full MLP block (GEMM-Residual-RMSNorm-GEMM-SwiGLU + down projection + residual) {name} fwd+bwd"
    else:
        what = "SwiGLU MLP fwd+bwd"
    return {"workload": what, **s, "tokens": s["M"]}


# ----------------------------------------------------------------------------- CPU oracle timing

def _blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


def _oracle_step(kind, s, bwd, inputs, rows):
    """The fp64 oracle over the first `rows` tokens of the workload (forward row-local,
    weight gradients summed over those rows only)."""
    from oracle import coda_oracle as O
    if kind == "block":
        X, R, dOut = inputs["X"][:rows], inputs["R"][:rows], inputs["dOut"][:rows]
        fwd = O.mlp_block_forward(X, inputs["W1"], R, inputs["g"], inputs["W2"], inputs["Wdown"], s["eps"])
        if bwd:
            O.mlp_block_backward(dOut, X, inputs["W1"], R, inputs["g"], inputs["W2"], inputs["Wdown"], s["eps"],
                                 fwd=fwd)
        return
    if kind == "rope":
        X = inputs["X"][:rows]
        a = (s["n_q"], s["n_kv"], s["head_dim"], s["seq_len"], s["base"])
        O.qkv_rope_forward(X, inputs["Wqkv"], *a)
        if bwd:
            O.qkv_rope_backward(inputs["dQKV"][:rows], X, inputs["Wqkv"], *a)
        return
    if kind == "xent":
        X, t, dl = inputs["X"][:rows], inputs["targets"][:rows], inputs["dloss"][:rows]
        fwd = O.xent_forward(X, inputs["W"], t)
        if bwd:
            O.xent_backward(dl, X, inputs["W"], t, fwd=fwd)
        return
    if kind == "grg":
        X, R, dY = inputs["X"][:rows], inputs["R"][:rows], inputs["dY"][:rows]
        fwd = O.grg_forward(X, inputs["W1"], R, inputs["g"], inputs["W2"], s["eps"])
        if bwd:
            O.grg_backward(dY, X, inputs["W1"], R, inputs["g"], inputs["W2"], s["eps"], fwd=fwd)
    else:
        X, dOut = inputs["X"][:rows], inputs["dOut"][:rows]
        fwd = O.swiglu_forward(X, inputs["Wgu"], inputs["Wdown"])
        if bwd:
            O.swiglu_backward(dOut, X, inputs["Wgu"], inputs["Wdown"], fwd=fwd)


def _oracle_inputs(kind, s):
    """Seeded inputs in float64 for the oracle (first rows only are used)."""
    import torch
    from gemm_epilogue_fusion_tmem_b200 import synth
    if kind == "grg":
        t = synth.grg_inputs(s["M"], s["K"], s["d"], s["F"], seed=0)
    elif kind == "rope":
        t = synth.qkv_inputs(s["M"], s["d"], s["n_q"], s["n_kv"], s["head_dim"], seed=0)
    elif kind == "block":
        t = synth.mlp_block_inputs(s["M"], s["K"], s["d"], s["F"], seed=0)
    elif kind == "xent":
        t = synth.xent_inputs(s["M"], s["d"], s["V"], seed=0)
        out = {k: v.to(torch.float64).numpy() for k, v in t.items() if k != "targets"}
        out["targets"] = t["targets"].long().numpy()
        return out
    else:
        t = synth.swiglu_inputs(s["M"], s["d"], s["F"], seed=0)
    return {k: v.to(torch.float64).numpy() for k, v in t.items()}


def cpu_baseline(kind, s, bwd, inputs=None, target_s=12.0):
    inputs = inputs if inputs is not None else _oracle_inputs(kind, s)
    # Probe on a few rows to size the bounded sample.
    probe = min(64, s["M"])
    t0 = time.perf_counter()
    _oracle_step(kind, s, bwd, inputs, probe)
    dt = max(time.perf_counter() - t0, 1e-3)
    rate = _flops(kind, dict(s, M=probe), bwd) / dt
    rows = max(probe, min(s["M"], int(target_s * rate / _flops(kind, dict(s, M=1), bwd))))
    t0 = time.perf_counter()
    _oracle_step(kind, s, bwd, inputs, rows)
    dt = time.perf_counter() - t0
    fl = _flops(kind, dict(s, M=rows), bwd)
    return {"value": fl / dt / 1e12, "unit": "TFLOP/s", "cores": _blas_threads(), "kind": "oracle",
            "sample": f"fp64 numpy oracle, unfused textbook {'fwd+bwd' if bwd else 'fwd'} on the first {rows} "
                      f"of {s['M']} tokens with the full weights ({fl / 1e12:.3f} TFLOP in {dt:.1f} s)"}


# ----------------------------------------------------------------------------- clocks

CLOCK_FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
                "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
                "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")


class ClockSampler:
    """Samples this process's GPU while the `with` block runs: SM clock, its
    maximum, power and the active clock-event reasons.  Every 10 ms through
    NVML on a thread (the device found by its UUID), so that even a region of
    a few tens of milliseconds gets several samples; every 50 ms through
    nvidia-smi when NVML cannot read the device.  Only reads counters."""

    # NVML clock-event reason bits, named as nvidia-smi names them.
    REASON_BITS = (("hw_slowdown", 0x8), ("hw_thermal_slowdown", 0x40), ("sw_thermal_slowdown", 0x20),
                   ("sw_power_cap", 0x4))

    def __init__(self, device_index: int, interval_s: float = 0.01):
        self.idx = device_index
        self.interval = interval_s
        self.proc = None
        self.thread = None
        self.rows = []  # (sm MHz, max sm MHz, power W, reason bits) per NVML sample
        self.out = ""

    def _nvml_handle(self):
        import pynvml
        pynvml.nvmlInit()
        try:
            import torch
            u = str(torch.cuda.get_device_properties(self.idx).uuid)
            return pynvml.nvmlDeviceGetHandleByUUID(u if u.startswith("GPU-") else "GPU-" + u)
        except Exception:
            ids = [x.strip() for x in os.environ.get("CUDA_VISIBLE_DEVICES", "").split(",") if x.strip()]
            phys = int(ids[self.idx]) if self.idx < len(ids) and ids[self.idx].isdigit() else self.idx
            return pynvml.nvmlDeviceGetHandleByIndex(phys)

    def _nvml_sample(self):
        import pynvml
        h = self.handle
        self.rows.append((float(pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)),
                          float(pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)),
                          pynvml.nvmlDeviceGetPowerUsage(h) / 1000.0,
                          int(pynvml.nvmlDeviceGetCurrentClocksEventReasons(h))))

    def _loop(self):
        while not self.stop.wait(self.interval):
            try:
                self._nvml_sample()
            except Exception:
                return

    def __enter__(self):
        try:
            self.handle = self._nvml_handle()
            self._nvml_sample()  # raises here, before any thread starts, when NVML cannot read the device
            self.stop = threading.Event()
            self.thread = threading.Thread(target=self._loop, daemon=True)
            self.thread.start()
            return self
        except Exception:
            self.thread, self.rows = None, []
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.idx}", f"--query-gpu={CLOCK_FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            time.sleep(0.3)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.thread is not None:
            self.stop.set()
            self.thread.join(timeout=2)
            try:
                self._nvml_sample()
            except Exception:
                pass
            return
        self.out = ""
        if self.proc is not None:
            time.sleep(0.2)
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                self.out = ""

    def summary(self):
        sm, mx, pw, reasons = [], [], [], set()
        for c, m, p, bits in self.rows:
            sm.append(c)
            mx.append(m)
            pw.append(p)
            reasons.update(n for n, b in self.REASON_BITS if bits & b)
        names = [n for n, _ in self.REASON_BITS]
        for line in (self.out or "").splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
                pw.append(float(f[3]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        # Median over the samples taken under load (power above 30% of the highest seen).
        hot = [c for c, p in zip(sm, pw) if p >= 0.3 * max(pw)] or sm
        return {"sm_mhz": statistics.median(hot), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm), "samples_under_load": len(hot), "power_w_max": max(pw),
                "source": "nvml" if self.rows else "nvidia-smi"}


# ----------------------------------------------------------------------------- traffic record

def _kernel_source_hash():
    """Hash of the CUDA sources' code (comments and whitespace removed), so a
    recorded ncu traffic figure stays valid across comment-only edits and is
    dropped once any code changes."""
    import re
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "gemm_epilogue_fusion_tmem_b200", "csrc")
    for name in sorted(os.listdir(csrc)):
        if name.endswith((".cu", ".cuh")):
            with open(os.path.join(csrc, name), encoding="utf-8") as f:
                code = f.read()
            code = re.sub(r"/\*.*?\*/", "", code, flags=re.S)
            code = re.sub(r"//[^\n]*", "", code)
            h.update(re.sub(r"\s+", "", code).encode())
    return h.hexdigest()[:16]


def _recorded_traffic(kernel: str, workload: str):
    """DRAM bytes per launch recorded from an ncu capture, if taken on the current kernel source."""
    path = os.path.join(ROOT, "profiles", "traffic.txt")
    try:
        with open(path) as f:
            for line in f:
                parts = line.split()
                if len(parts) >= 4 and parts[0] == kernel and parts[1] == workload:
                    return float(parts[2]) if parts[3] == _kernel_source_hash() else None
    except OSError:
        pass
    return None


# ----------------------------------------------------------------------------- ranks (replicas)

def dist_env():
    """(rank, world, local_rank) from the torchrun environment (1 process when absent)."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def max_over_ranks(x: float, device, world: int) -> float:
    """The largest value of x over all ranks (every rank gets it)."""
    if world <= 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_throughput(flops_per_step: float, steps: int, world: int, max_ms: float) -> float:
    """Whole-job TFLOP/s: every rank runs its own replica of the workload, the
    job's time is the slowest rank's (weak scaling, no data-path collective)."""
    return flops_per_step * steps * world / (max_ms / 1e3) / 1e12


# ----------------------------------------------------------------------------- the CUDA arm

def _setup(kind, s, bwd, device):
    import torch
    from gemm_epilogue_fusion_tmem_b200 import synth
    if kind == "grg":
        host = synth.grg_inputs(s["M"], s["K"], s["d"], s["F"], seed=0)
        if not bwd:
            host.pop("dY")
    elif kind == "xent":
        host = synth.xent_inputs(s["M"], s["d"], s["V"], seed=0)
    elif kind == "rope":
        host = synth.qkv_inputs(s["M"], s["d"], s["n_q"], s["n_kv"], s["head_dim"], seed=0)
    elif kind == "block":
        host = synth.mlp_block_inputs(s["M"], s["K"], s["d"], s["F"], seed=0)
    else:
        host = synth.swiglu_inputs(s["M"], s["d"], s["F"], seed=0)
    dev = {k: v.to(device) for k, v in host.items()}
    return host, dev


def _make_step(kind, s, bwd, dev):
    """Returns (step, outputs, launches_per_step, result_keys)."""
    import torch
    from gemm_epilogue_fusion_tmem_b200 import binding as B
    lib = B.library()
    M = s["M"]
    if kind == "grg":
        K, d, F = s["K"], s["d"], s["F"]
        N = 2 * F
        ws = B.Workspace(max(lib.coda_grg_fwd_workspace_bytes(M, K, d, N, 0),
                             lib.coda_grg_bwd_workspace_bytes(M, K, d, N)), dev["X"].device)
        fo = {"H": torch.empty(M, d, dtype=torch.bfloat16, device=dev["X"].device),
              "r": torch.empty(M, dtype=torch.float32, device=dev["X"].device),
              "Y": torch.empty(M, F, dtype=torch.bfloat16, device=dev["X"].device),
              "AB": torch.empty(M, N, dtype=torch.bfloat16, device=dev["X"].device)}
        bo = {}
        if bwd:
            bo = {"dX": torch.empty(M, K, dtype=torch.bfloat16, device=dev["X"].device),
                  "dR": torch.empty(M, d, dtype=torch.bfloat16, device=dev["X"].device),
                  "dW1": torch.empty(d, K, dtype=torch.bfloat16, device=dev["X"].device),
                  "dW2": torch.empty(N, d, dtype=torch.bfloat16, device=dev["X"].device),
                  "dg": torch.empty(d, dtype=torch.float32, device=dev["X"].device)}

        def fwd_only():
            B.grg_fwd(dev["X"], dev["W1"], dev["R"], dev["g"], dev["W2"], s["eps"], out=fo, ws=ws)

        def bwd_only():
            B.grg_bwd(dev["dY"], dev["X"], dev["W1"], fo["H"], fo["r"], fo["AB"], dev["g"], dev["W2"], out=bo, ws=ws)

        def step():
            fwd_only()
            if bwd:
                bwd_only()

        step.fwd, step.bwd = fwd_only, (bwd_only if bwd else None)
        outs = {**fo, **bo}
        keys = ["Y", "dX", "dR", "dW1", "dW2", "dg"] if bwd else ["Y", "H", "r"]
        return step, outs, (9 if bwd else 3), keys, ws
    if kind == "block":
        K, d, F = s["K"], s["d"], s["F"]
        ws = B.Workspace(max(lib.coda_mlp_block_fwd_workspace_bytes(M, K, d, F),
                             lib.coda_mlp_block_bwd_workspace_bytes(M, K, d, F)), dev["X"].device)
        fo = B.mlp_block_fwd(dev["X"], dev["W1"], dev["R"], dev["g"], dev["W2"], dev["Wdown"], s["eps"], ws=ws)
        bo = B.mlp_block_bwd(dev["dOut"], dev["X"], dev["W1"], fo["H"], fo["r"], fo["AB"], fo["Y"], dev["g"],
                             dev["W2"], dev["Wdown"], ws=ws)

        def bstep():
            B.mlp_block_fwd(dev["X"], dev["W1"], dev["R"], dev["g"], dev["W2"], dev["Wdown"], s["eps"], out=fo, ws=ws)
            B.mlp_block_bwd(dev["dOut"], dev["X"], dev["W1"], fo["H"], fo["r"], fo["AB"], fo["Y"], dev["g"],
                            dev["W2"], dev["Wdown"], out=bo, ws=ws)

        return bstep, {**fo, **bo}, 12, ["Out", "dX", "dR", "dW1", "dW2", "dg", "dWdown"], ws
    if kind == "rope":
        a = (s["n_q"], s["n_kv"], s["head_dim"], s["seq_len"], s["base"])
        ws = B.Workspace(lib.coda_qkv_rope_bwd_workspace_bytes(M, s["d"], s["n_q"], s["n_kv"], s["head_dim"]),
                         dev["X"].device)
        q = B.qkv_rope_fwd(dev["X"], dev["Wqkv"], *a, ws=ws)
        bo = B.qkv_rope_bwd(dev["dQKV"], dev["X"], dev["Wqkv"], *a, ws=ws)

        def rstep():
            B.qkv_rope_fwd(dev["X"], dev["Wqkv"], *a, out=q, ws=ws)
            B.qkv_rope_bwd(dev["dQKV"], dev["X"], dev["Wqkv"], *a, out=bo, ws=ws)

        return rstep, {"QKV": q, **bo}, 4, ["QKV", "dX", "dW"], ws
    if kind == "xent":
        d, V = s["d"], s["V"]
        ws = B.Workspace(max(lib.coda_xent_fwd_workspace_bytes(M, d, V), lib.coda_xent_bwd_workspace_bytes(M, d, V)),
                         dev["X"].device)
        fo = B.xent_fwd(dev["X"], dev["W"], dev["targets"], ws=ws)
        bo = B.xent_bwd(dev["X"], dev["W"], dev["targets"], fo["lse"], dev["dloss"], ws=ws)

        def xstep():
            B.xent_fwd(dev["X"], dev["W"], dev["targets"], out=fo, ws=ws)
            B.xent_bwd(dev["X"], dev["W"], dev["targets"], fo["lse"], dev["dloss"], out=bo, ws=ws)

        return xstep, {**fo, **bo}, 5, ["loss", "dX", "dW"], ws
    d, F = s["d"], s["F"]
    ws = B.Workspace(lib.coda_swiglu_bwd_workspace_bytes(M, d, F), dev["X"].device)
    fo = B.swiglu_fwd(dev["X"], dev["Wgu"], dev["Wdown"], ws=ws)
    bo = B.swiglu_bwd(dev["dOut"], dev["X"], dev["Wgu"], dev["Wdown"], fo["Y"], fo["AB"], ws=ws)

    def fwd_only():
        B.swiglu_fwd(dev["X"], dev["Wgu"], dev["Wdown"], out=fo, ws=ws)

    def bwd_only():
        B.swiglu_bwd(dev["dOut"], dev["X"], dev["Wgu"], dev["Wdown"], fo["Y"], fo["AB"], out=bo, ws=ws)

    def step():
        fwd_only()
        bwd_only()

    step.fwd, step.bwd = fwd_only, bwd_only
    outs = {**fo, **bo}
    return step, outs, 6, ["Out", "dX", "dWgu", "dWdown"], ws


def _make_unfused_step(kind, s, bwd, dev):
    """The same work run operator by operator (every intermediate in HBM)."""
    import torch
    from gemm_epilogue_fusion_tmem_b200 import binding as B
    lib = B.library()
    if kind == "swiglu":
        M, d, F = s["M"], s["d"], s["F"]
        ws = B.Workspace(lib.coda_swiglu_bwd_unfused_workspace_bytes(M, d, F), dev["X"].device)
        fo = B.swiglu_fwd_unfused(dev["X"], dev["Wgu"], dev["Wdown"], ws=ws)
        bo = B.swiglu_bwd_unfused(dev["dOut"], dev["X"], dev["Wgu"], dev["Wdown"], fo["Y"], fo["AB"], ws=ws)

        def fwd_only():
            B.swiglu_fwd_unfused(dev["X"], dev["Wgu"], dev["Wdown"], out=fo, ws=ws)

        def bwd_only():
            B.swiglu_bwd_unfused(dev["dOut"], dev["X"], dev["Wgu"], dev["Wdown"], fo["Y"], fo["AB"], out=bo, ws=ws)

        launches = 3 + 5
    else:
        M, K, d, F = s["M"], s["K"], s["d"], s["F"]
        N = 2 * F
        ws = B.Workspace(max(lib.coda_grg_fwd_unfused_workspace_bytes(M, K, d, N),
                             lib.coda_grg_bwd_unfused_workspace_bytes(M, K, d, N)), dev["X"].device)
        fo = B.grg_fwd_unfused(dev["X"], dev["W1"], dev["R"], dev["g"], dev["W2"], s["eps"], ws=ws)
        bo = {}
        if bwd:
            bo = B.grg_bwd_unfused(dev["dY"], dev["X"], dev["W1"], fo["H"], fo["r"], fo["AB"], fo["U"], dev["g"],
                                   dev["W2"], ws=ws)

        def fwd_only():
            B.grg_fwd_unfused(dev["X"], dev["W1"], dev["R"], dev["g"], dev["W2"], s["eps"], out=fo, ws=ws)

        def bwd_only():
            B.grg_bwd_unfused(dev["dY"], dev["X"], dev["W1"], fo["H"], fo["r"], fo["AB"], fo["U"], dev["g"],
                              dev["W2"], out=bo, ws=ws)

        launches = 5 + (8 if bwd else 0)

    def step():
        fwd_only()
        if bwd:
            bwd_only()

    step.fwd, step.bwd = fwd_only, (bwd_only if bwd else None)
    return step, launches, ws


def _time_loop(fn, steps, warmup, device, world, barrier):
    """Device time of `steps` calls of fn (CUDA events on the current stream), max over ranks."""
    import torch
    for _ in range(max(warmup, 3) if warmup is not None else 0):
        fn()
    torch.cuda.synchronize()
    st = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    e0.record(st)
    for _ in range(steps):
        fn()
    e1.record(st)
    torch.cuda.synchronize()
    barrier()
    return max_over_ranks(e0.elapsed_time(e1), device, world)


def _time_interleaved(fa, fb, steps, warmup, device, world, barrier, rounds=10):
    """Median ms per call of fa and of fb, timed in alternating bursts of at
    least 5 calls, the order swapped every round (fa fb, fb fa, ...), so that
    both see the same thermal and power-cap drift and neither always runs
    first; each burst is max over ranks."""
    import statistics
    per = max(5, steps // 4)
    for _ in range(max(warmup, 3)):
        fa()
        fb()
    ta, tb = [], []
    for i in range(rounds):
        order = ((fa, ta), (fb, tb)) if i % 2 == 0 else ((fb, tb), (fa, ta))
        for fn, acc in order:
            acc.append(_time_loop(fn, per, None, device, world, barrier) / per)
    return statistics.median(ta), statistics.median(tb)


def _make_hg_step(s, bwd, dev, outs, device):
    """The GRG step with the gain on the activation side (coda_grg_fwd_hg: GEMM1's
    epilogue stores Hg = bf16(H g), GEMM2 reads the unfolded W2), writing into
    the same output buffers as the folded-gain step."""
    from gemm_epilogue_fusion_tmem_b200 import binding as B
    lib = B.library()
    hws = B.Workspace(max(lib.coda_grg_fwd_hg_workspace_bytes(s["M"], s["K"], s["d"], 2 * s["F"], 0),
                          lib.coda_grg_bwd_workspace_bytes(s["M"], s["K"], s["d"], 2 * s["F"])), device)
    hf = {k: outs[k] for k in ("H", "r", "Y", "AB")}
    hb = {k: outs[k] for k in ("dX", "dR", "dW1", "dW2", "dg")} if bwd else {}

    def hstep():
        B.grg_fwd_hg(dev["X"], dev["W1"], dev["R"], dev["g"], dev["W2"], s["eps"], out=hf, ws=hws)
        if bwd:
            B.grg_bwd(dev["dY"], dev["X"], dev["W1"], hf["H"], hf["r"], hf["AB"], dev["g"], dev["W2"], out=hb,
                      ws=hws)

    return hstep, hws


def _in_step_kernel_ms(step, epi, steps):
    """Mean duration of the first launch with epilogue `epi` in each of `steps`
    back-to-back steps (the library's event hook on the launching stream)."""
    import torch
    from gemm_epilogue_fusion_tmem_b200 import binding as B
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    torch.cuda.synchronize()
    for x, y in ev:
        B.profile_arm(epi, x, y)
        step()
    torch.cuda.synchronize()
    B.profile_arm(epi)
    return sum(x.elapsed_time(y) for x, y in ev) / steps


def grg_extra(name, a, device, world, barrier):
    """Another GRG workload timed in the same run (the 70B shape beside the 7B
    headline): the step with the folded gain, with the gain on the activation
    side, and the unfused sequence, in alternating bursts (medians), plus the
    gate/up GEMM's in-step launch time against the burst peak."""
    import torch
    kind, s, bwd = WORKLOADS[name]
    host, dev = _setup(kind, s, bwd, device)
    del host
    step, outs, launches, _, ws = _make_step(kind, s, bwd, dev)
    hstep, hws = _make_hg_step(s, bwd, dev, outs, device)
    ustep, ulaunch, uws = _make_unfused_step(kind, s, bwd, dev)
    flops = _flops(kind, s, bwd)
    f_ms, u_ms = _time_interleaved(step, ustep, a.steps, a.warmup, device, world, barrier)
    h_ms, u2_ms = _time_interleaved(hstep, ustep, a.steps, a.warmup, device, world, barrier)
    fd, ud = _time_interleaved(step.fwd, ustep.fwd, a.steps, a.warmup, device, world, barrier)
    peaks, src = _peaks()
    burst = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    k_flops = 2.0 * s["M"] * s["d"] * 2 * s["F"]
    kh = _in_step_kernel_ms(hstep, DOMINANT_EPI[kind], max(a.steps, 5))
    kf = _in_step_kernel_ms(step, DOMINANT_EPI[kind], max(a.steps, 5))
    status, detail = ws.query()
    if status != 0:
        raise SystemExit(f"bench.py: device status {status} detail {detail:#x} in the {name} extra")
    rate = lambda ms: round(replica_throughput(flops, 1, world, ms), 2)  # noqa: E731
    out = {"config": _describe(name, kind, s, bwd), "flops_per_step": flops,
           "timing": INTERLEAVED,
           "fused_folded_gain": {"ms_per_step": round(f_ms, 4), "value": rate(f_ms),
                                 "frac_of_burst": round(rate(f_ms) / world / burst, 4),
                                 "unfused_ms_per_step": round(u_ms, 4), "speedup_vs_unfused": round(u_ms / f_ms, 4),
                                 "fwd": {"fused_ms": round(fd, 4), "unfused_ms": round(ud, 4),
                                         "speedup": round(ud / fd, 4)},
                                 "gate_up_gemm_in_step_ms": round(kf, 4),
                                 "gate_up_gemm_frac_of_burst": round(k_flops / (kf / 1e3) / 1e12 / burst, 4)},
           "fused_activation_gain": {"ms_per_step": round(h_ms, 4), "value": rate(h_ms),
                                     "frac_of_burst": round(rate(h_ms) / world / burst, 4),
                                     "unfused_ms_per_step": round(u2_ms, 4),
                                     "speedup_vs_unfused": round(u2_ms / h_ms, 4),
                                     "gate_up_gemm_in_step_ms": round(kh, 4),
                                     "gate_up_gemm_frac_of_burst": round(k_flops / (kh / 1e3) / 1e12 / burst, 4)},
           "unfused": {"value": rate(u_ms), "gpu_launches_per_step": ulaunch},
           "peak": {"bf16_burst_tflops": burst, "source": src},
           "unit": "TFLOP/s"}
    del ws, hws, uws, outs, dev, step, hstep, ustep
    torch.cuda.empty_cache()
    return out


def epilogue_ab(kind, s, dev, outs, a, device, world, barrier):
    """The dominant gate/up GEMM with its r + SwiGLU epilogue against a plain
    store of the same [M, 2F] product (same operands, same kernel, epilogue
    swapped), in alternating bursts with the SM clock sampled in each: the
    epilogue's cost at equal clocks is time x MHz."""
    import torch
    from gemm_epilogue_fusion_tmem_b200 import binding as B
    if kind not in ("grg", "block", "swiglu"):
        return None
    if kind in ("grg", "block"):
        A, W, r = outs["H"], dev["W2"], outs["r"]
    else:
        A, W, r = dev["X"], dev["Wgu"], None
    M, K, F = s["M"], s["d"], s["F"]
    o = {"Y": torch.empty(M, F, dtype=torch.bfloat16, device=device),
         "AB": torch.empty(M, 2 * F, dtype=torch.bfloat16, device=device)}
    C = torch.empty(M, 2 * F, dtype=torch.bfloat16, device=device)
    fused = lambda: B.gemm_swiglu(A, W, r, out=o)  # noqa: E731
    plain = lambda: B.gemm(A, W, M, 2 * F, K, out=C)  # noqa: E731
    for _ in range(3):
        fused()
        plain()
    # Bursts of about 250 ms, long enough for several 50 ms clock samples.
    per = max(10, int(250.0 / max(_time_loop(fused, 3, None, device, world, barrier) / 3, 1e-3)))
    tf, tp, cf, cp = [], [], [], []
    for _ in range(4):
        with ClockSampler(device.index) as c1:
            tf.append(_time_loop(fused, per, None, device, world, barrier) / per)
        with ClockSampler(device.index) as c2:
            tp.append(_time_loop(plain, per, None, device, world, barrier) / per)
        cf.append(c1.summary().get("sm_mhz"))
        cp.append(c2.summary().get("sm_mhz"))
    med = statistics.median
    mf, mp = med(tf), med(tp)
    out = {"swiglu_ms": round(mf, 4), "plain_store_ms": round(mp, 4), "ratio": round(mf / mp, 4),
           "timing": f"4 alternating bursts of {per} launches each, medians"}
    cf, cp = [x for x in cf if x], [x for x in cp if x]
    if cf and cp:
        out["sm_mhz"] = {"swiglu": med(cf), "plain_store": med(cp)}
        out["ratio_at_equal_clock"] = round(mf * med(cf) / (mp * med(cp)), 4)
    return out


def _grg_kernels(s, bwd):
    """The block's kernels in launch order with their algorithmic work per launch:
    (hook id, name, bound, amount) with FLOPs for tensor-bound GEMMs and
    compulsory HBM bytes for the light passes."""
    M, K, d, F = s["M"], s["K"], s["d"], s["F"]
    N = 2 * F
    ks = [(16, "fold_gain (W2g = W2 diag g)", "hbm", 4.0 * N * d + 2.0 * d),
          (1, "GEMM1 + residual + partial sums", "tensor", 2.0 * M * K * d),
          (2, "GEMM2 + r (from the partial sums) + SwiGLU", "tensor", 2.0 * M * d * N)]
    if bwd:
        rows = -(-M // 256) * 256 // 32  # dg partial rows: one per 32 output rows
        ks += [(18, "SwiGLU bwd + row coefficient", "hbm", 2.0 * M * F + 4.0 * M * N + 8.0 * M),
               (3, "dn GEMM + RMSNorm correction + dg partials", "tensor", 2.0 * M * N * d),
               (19, "column reduce -> dg", "hbm", 4.0 * rows * d + 4.0 * d),
               (0, "dW2 = g (dA'^T H)", "tensor", 2.0 * N * d * M),
               (0, "dX = dH W1", "tensor", 2.0 * M * K * d),
               (0, "dW1 = dH^T X", "tensor", 2.0 * d * K * M)]
    return ks


def _kernel_breakdown(kind, s, bwd, step, reps=10):
    """Every kernel of the block's step timed through the library's event hook
    over `reps` extra steps (outside the timed region: the events take the
    place of the PDL overlap at every boundary), against the measured peaks.
    The steps run right after the headline region and last well under a
    second, so the GEMMs are compared with the burst bf16 peak, as the
    headline's roofline is."""
    if kind != "grg":
        return None
    import torch
    from gemm_epilogue_fusion_tmem_b200 import binding as B
    peaks, src = _peaks()
    hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    tc = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    ks = _grg_kernels(s, bwd)
    ev = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in ks]
          for _ in range(reps)]
    torch.cuda.synchronize()
    for r in range(reps):
        for (kid, _, _, _), (x, y) in zip(ks, ev[r]):
            B.profile_arm(kid, x, y)
        step()
    torch.cuda.synchronize()
    B.profile_arm(0)
    out = []
    for i, (kid, name, bound, amount) in enumerate(ks):
        ms = sum(ev[r][i][0].elapsed_time(ev[r][i][1]) for r in range(reps)) / reps
        if bound == "tensor":
            ach = amount / (ms / 1e3) / 1e12
            out.append({"kernel": name, "ms": round(ms, 4), "bound": "tensor", "TFLOP": round(amount / 1e12, 4),
                        "achieved_TFLOP/s": round(ach, 1), "frac": round(ach / tc, 4)})
        else:
            ach = amount / (ms / 1e3) / 1e9
            out.append({"kernel": name, "ms": round(ms, 4), "bound": "hbm", "MB": round(amount / 1e6, 2),
                        "achieved_GB/s": round(ach, 1), "frac": round(ach / hbm, 4)})
    return {"steps": reps, "peaks": f"{src}: burst bf16 {tc} TFLOP/s, HBM copy {hbm} GB/s",
            "note": "each kernel inside its own CUDA-event pair (no PDL overlap at its boundaries)",
            "kernels": out, "sum_ms": round(sum(k["ms"] for k in out), 4)}


# Epilogue of the dominant GEMM per workload kind (the launch the timing hook arms).
DOMINANT_EPI = {"grg": 2, "swiglu": 2, "block": 2, "xent": 5, "rope": 7}


def _dominant_kernel(kind, s, dev, outs, reps=20):
    """Time the dominant kernel alone, launched through its entry point with the
    library's event hook around the kernel: the gate/up GEMM with the r + SwiGLU
    epilogue (cross-entropy: the logits GEMM with its online max / sum-exp
    epilogue; RoPE: the QKV GEMM with its rotary epilogue).
    Returns (name, mean launch ms, FLOPs per launch)."""
    import torch
    from gemm_epilogue_fusion_tmem_b200 import binding as B
    if kind == "rope":
        a = (s["n_q"], s["n_kv"], s["head_dim"], s["seq_len"], s["base"])
        q = outs["QKV"]
        call = lambda: B.qkv_rope_fwd(dev["X"], dev["Wqkv"], *a, out=q)  # noqa: E731
        name, flops = "qkv_rope", 2.0 * s["M"] * s["d"] * (s["n_q"] + 2 * s["n_kv"]) * s["head_dim"]
    elif kind == "xent":
        lib = B.library()
        M, d, V = s["M"], s["d"], s["V"]
        ws = B.Workspace(lib.coda_xent_fwd_workspace_bytes(M, d, V), dev["X"].device)
        o = {}
        call = lambda: B.xent_fwd(dev["X"], dev["W"], dev["targets"], out=o, ws=ws)  # noqa: E731
        name, flops = "xent_logits", 2.0 * M * d * V
    else:
        if kind in ("grg", "block"):
            A, W, r = outs["H"], dev["W2"], outs["r"]  # same shape and work as GEMM2 on W2g
        else:
            A, W, r = dev["X"], dev["Wgu"], None
        M, K, F = s["M"], s["d"], s["F"]
        o = {"Y": torch.empty(M, F, dtype=torch.bfloat16, device=A.device),
             "AB": torch.empty(M, 2 * F, dtype=torch.bfloat16, device=A.device)}
        call = lambda: B.gemm_swiglu(A, W, r, out=o)  # noqa: E731
        name, flops = "gemm_swiglu", 2.0 * M * K * 2 * F
    call()  # allocates the outputs on the first call
    for _ in range(2):
        call()
    st = torch.cuda.current_stream()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
    torch.cuda.synchronize()
    for x, y in ev:
        B.profile_arm(DOMINANT_EPI[kind], x, y)
        call()
    torch.cuda.synchronize()
    B.profile_arm(DOMINANT_EPI[kind])
    return name, sum(x.elapsed_time(y) for x, y in ev) / reps, flops


def _e2e_pipelined(kind, s, bwd, host, dev, step, outs, result_keys, flops, a, device, world, barrier):
    import torch
    dev2 = {k: torch.empty_like(v) for k, v in dev.items()}
    for k in dev2:
        dev2[k].copy_(dev[k])
    step2, outs2, _, _, ws2 = _make_step(kind, s, bwd, dev2)
    bufs = [(dev, step, outs), (dev2, step2, outs2)]
    pin_in = {k: v.pin_memory() for k, v in host.items()}
    pin_out = [{k: torch.empty(outs[k].shape, dtype=outs[k].dtype, pin_memory=True) for k in result_keys}
               for _ in range(2)]
    h2d = sum(v.numel() * v.element_size() for v in pin_in.values())
    d2h = sum(v.numel() * v.element_size() for v in pin_out[0].values())
    comp = torch.cuda.current_stream()
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_done = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]

    def run(n):
        for i in range(n):
            b = i % 2
            d, st, o = bufs[b]
            with torch.cuda.stream(s_in):
                if i >= 2:
                    s_in.wait_event(ev_done[b])      # step i-2 has finished reading these inputs
                for k, v in pin_in.items():
                    d[k].copy_(v, non_blocking=True)
                ev_in[b].record(s_in)
            comp.wait_event(ev_in[b])
            if i >= 2:
                comp.wait_event(ev_out[b])           # step i-2's results have been read back
            st()
            ev_done[b].record(comp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_done[b])
                for k in result_keys:
                    pin_out[b][k].copy_(o[k], non_blocking=True)
                ev_out[b].record(s_out)

    run(4)
    torch.cuda.synchronize()
    n_e2e = max(4, min(a.steps, 20))
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    t0.record(s_in)
    comp.wait_event(t0)
    run(n_e2e)
    t1.record(s_out)
    torch.cuda.synchronize()
    barrier()
    te = max_over_ranks(t0.elapsed_time(t1), device, world)
    del ws2
    return {"value": round(replica_throughput(flops, n_e2e, world, te), 2), "unit": "TFLOP/s",
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h), "steps": n_e2e,
            "ms_per_step": round(te / n_e2e, 3),
            "how": "pinned host inputs copied in and results (the step's outputs) copied out every step; "
                   "double-buffered, copies on their own streams overlapping the neighbouring steps' compute"}


def run_coda(a):
    import torch
    import torch.distributed as dist
    kind, s, bwd = WORKLOADS[a.workload]
    rank, world, local = dist_env()
    if not torch.cuda.is_available():
        raise SystemExit("bench.py: no CUDA device (the library has no CPU path)")
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=device)

    def barrier():
        if world > 1:
            dist.barrier()

    host, dev = _setup(kind, s, bwd, device)
    step, outs, launches, result_keys, ws = _make_step(kind, s, bwd, dev)
    flops = _flops(kind, s, bwd)

    from gemm_epilogue_fusion_tmem_b200 import binding as B
    for _ in range(max(a.warmup, 3)):
        step()
    torch.cuda.synchronize()
    # The dominant kernel alone, on a warm but not power-limited GPU (context
    # for the roofline; the reported fraction is the in-step one below).
    kname, k_alone_ms, k_flops = _dominant_kernel(kind, s, dev, outs)
    st = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    # One event pair per timed step around the dominant kernel's launch,
    # recorded by the library on the stream it launches on.
    kev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(a.steps)]
    for x, y in kev:
        x.record(st)
        y.record(st)
    k_epi = DOMINANT_EPI[kind]
    with ClockSampler(local) as clk:
        barrier()
        torch.cuda.synchronize()
        e0.record(st)
        for i in range(a.steps):
            B.profile_arm(k_epi, *kev[i])
            step()
        e1.record(st)
        torch.cuda.synchronize()
        barrier()
    B.profile_arm(k_epi)
    ms_total = e0.elapsed_time(e1)
    k_ms = sum(x.elapsed_time(y) for x, y in kev) / a.steps
    status, detail = ws.query()
    if status != 0:
        raise SystemExit(f"bench.py: device status {status} detail {detail:#x}")

    # The same step with L2 flushed before each one (a 256 MiB write between
    # steps, outside the per-step event pair): context for the unflushed
    # headline, whose inputs already exceed L2.
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=device)
    n_fl = max(5, min(a.steps, 20))
    fev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n_fl)]
    for x, y in fev:
        flush.fill_(1)
        x.record(st)
        step()
        y.record(st)
    torch.cuda.synchronize()
    fl_ms = max_over_ranks(sum(x.elapsed_time(y) for x, y in fev), device, world)
    l2_flushed = {"ms_per_step": round(fl_ms / n_fl, 4),
                  "value": round(replica_throughput(flops, n_fl, world, fl_ms), 2), "steps": n_fl,
                  "how": "256 MiB write before each step, each step timed by its own event pair"}
    del flush
    ws_bytes = sum(v.numel() * v.element_size() for v in list(dev.values()) + list(outs.values()))
    l2_note = (f"inputs larger than L2 (step tensors {ws_bytes / 1e9:.2f} GB > 126 MB L2), no flush"
               if ws_bytes > 126e6 else
               f"step tensors ({ws_bytes / 1e6:.0f} MB) fit in L2: warm-cache figure; see l2_flushed")
    ms_max = max_over_ranks(ms_total, device, world)
    value = replica_throughput(flops, a.steps, world, ms_max)

    # The same step once the power cap has settled: about two seconds of
    # back-to-back steps, then the same number of steps timed again (the
    # headline region above starts right after the warm-up, a short burst).
    n_pre = max(1, int(2000.0 / max(ms_total / a.steps, 1e-3)))
    n_set = max(a.steps, int(1000.0 / max(ms_total / a.steps, 1e-3)))  # at least a second, for clock samples
    kev_s = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n_set)]
    with ClockSampler(local) as clk_settled:
        for _ in range(n_pre):
            step()
        torch.cuda.synchronize()
        barrier()
        s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s0.record(st)
        for i in range(n_set):
            B.profile_arm(k_epi, *kev_s[i])
            step()
        s1.record(st)
        torch.cuda.synchronize()
        barrier()
    B.profile_arm(k_epi)
    settled_ms = max_over_ranks(s0.elapsed_time(s1), device, world)
    k_set_ms = sum(x.elapsed_time(y) for x, y in kev_s) / n_set
    settled = {"ms_per_step": round(settled_ms / n_set, 4),
               "value": round(replica_throughput(flops, n_set, world, settled_ms), 2), "steps": n_set,
               "after_steps": n_pre, "clocks": clk_settled.summary(),
               "dominant_kernel_ms": round(k_set_ms, 4),
               "how": f"{n_pre} untimed back-to-back steps (about 2 s), then {n_set} steps (about 1 s) timed "
                      f"like the headline"}

    # The activation-side gain variant (Hg from GEMM1's epilogue, no gain fold).
    variants = {}
    if kind == "grg":
        from gemm_epilogue_fusion_tmem_b200 import binding as B
        lib = B.library()
        hstep, hws = _make_hg_step(s, bwd, dev, outs, device)
        f_ms, h_ms = _time_interleaved(step, hstep, a.steps, a.warmup, device, world, barrier)
        variants["activation_gain"] = {"ms_per_step": round(h_ms, 4),
                                       "value": round(replica_throughput(flops, 1, world, h_ms), 2),
                                       "fused_ms_per_step": round(f_ms, 4),
                                       "timing": INTERLEAVED + " (against the folded-gain step)",
                                       "what": "coda_grg_fwd_hg: GEMM1 stores H*g, GEMM2 reads W2 unfolded"}
        del hws

    # The same step captured once in a CUDA graph and replayed (no per-launch
    # host overhead), timed in alternating bursts with the eager step.
    try:
        graph = torch.cuda.CUDAGraph()
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            with torch.cuda.graph(graph, stream=side):
                step()
        torch.cuda.current_stream().wait_stream(side)
        e_ms, g_ms = _time_interleaved(step, graph.replay, a.steps, a.warmup, device, world, barrier)
        variants["cuda_graph"] = {"ms_per_step": round(g_ms, 4),
                                  "value": round(replica_throughput(flops, 1, world, g_ms), 2),
                                  "eager_ms_per_step": round(e_ms, 4),
                                  "timing": INTERLEAVED + " (against the eager step)",
                                  "what": "the same step captured once with torch.cuda.graph and replayed"}
        del graph
    except RuntimeError as err:  # capture not possible: report it instead of a number
        variants["cuda_graph"] = {"error": str(err)[:200]}

    # The unfused comparison sequence, timed the same way right after, and
    # both paths split into forward and backward (the pages compare each
    # direction separately).
    unfused = None
    if kind in ("grg", "swiglu") and not a.no_unfused:
        ustep, ulaunch, uws = _make_unfused_step(kind, s, bwd, dev)
        # Fused and unfused in alternating bursts (medians), so drift under the
        # power cap does not favour whichever runs first.
        f_ms, u_ms = _time_interleaved(step, ustep, a.steps, a.warmup, device, world, barrier)
        unfused = {"ms_per_step": round(u_ms, 4),
                   "value": round(replica_throughput(flops, 1, world, u_ms), 2), "unit": "TFLOP/s",
                   "fused_ms_per_step": round(f_ms, 4), "fused_speedup": round(u_ms / f_ms, 4),
                   "gpu_launches_per_step": ulaunch, "timing": INTERLEAVED,
                   "what": "same GEMM kernels with plain stores; residual add, RMSNorm, SwiGLU and their backward "
                           "as separate HBM-round-trip kernels"}
        for dname in ("fwd", "bwd"):
            ff, uf = getattr(step, dname, None), getattr(ustep, dname, None)
            if ff is None or uf is None:
                continue
            fd, ud = _time_interleaved(ff, uf, a.steps, a.warmup, device, world, barrier)
            unfused[dname] = {"fused_ms": round(fd, 4), "unfused_ms": round(ud, 4), "speedup": round(ud / fd, 4)}
        del uws

    # Roofline of the dominant kernel: its average launch duration inside the
    # timed steps.  The timed region is a short burst unless it runs for more
    # than a second, so the burst peak is the denominator then (the sustained
    # one, a seconds-long loop under the power cap, otherwise).  Beside it the
    # same kernel timed alone, and the fraction of the dense bf16 rate at the
    # SM clock measured under load in the timed region.
    peaks, peaks_src = _peaks()
    achieved = k_flops / (k_ms / 1e3) / 1e12
    burst = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    sustained = float(peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))
    long_region = ms_total > 1000.0
    peak = sustained if long_region else burst
    alone = k_flops / (k_alone_ms / 1e3) / 1e12
    clk_head = clk.summary()
    sms = torch.cuda.get_device_properties(device).multi_processor_count
    # The headline region (about 0.1 s at the driver's 20 steps) holds too few
    # 50 ms clock samples under load to know its clock; the settled region
    # (a second or more) does, so the clock-normalised fraction is taken there.
    clk_set = settled["clocks"]
    set_mhz = clk_set.get("sm_mhz") if clk_set.get("samples_under_load", 0) >= 5 else None
    at_clock = (sms * DENSE_BF16_FLOP_PER_SM_CLK * set_mhz * 1e6 / 1e12) if set_mhz else None
    achieved_set = k_flops / (settled["dominant_kernel_ms"] / 1e3) / 1e12
    roofline = {"bound": "tensor", "kernel": kname, "achieved": round(achieved, 1), "peak": peak,
                "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
                "traffic": _recorded_traffic(kname, a.workload),
                "peak_source": (f"{peaks_src} {'sustained' if long_region else 'burst'} bf16 "
                                f"(timed region {ms_total:.0f} ms: "
                                f"{'longer' if long_region else 'shorter'} than 1 s)"),
                "launch_ms": round(k_ms, 4), "launches_timed": a.steps,
                "flops_per_launch": k_flops,
                "clock_normalised": None if at_clock is None else {
                    "region": "settled", "launch_ms": settled["dominant_kernel_ms"],
                    "achieved": round(achieved_set, 1), "sm_mhz": set_mhz, "sms": sms,
                    "dense_bf16_at_clock": round(at_clock, 1), "frac": round(achieved_set / at_clock, 4),
                    "how": f"the kernel's mean launch time in the settled steps against {sms} SMs x "
                           f"{DENSE_BF16_FLOP_PER_SM_CLK} dense bf16 FLOP per SM clock x the median SM clock "
                           f"sampled under load there"},
                "alone": {"launch_ms": round(k_alone_ms, 4), "achieved": round(alone, 1), "peak": burst,
                          "frac": round(alone / burst, 4),
                          "peak_source": f"{peaks_src} burst bf16 (kernel timed alone, after warm-up)"}}

    # The dominant kernel's epilogue against a plain store of the same product.
    epi_ab = epilogue_ab(kind, s, dev, outs, a, device, world, barrier)
    if epi_ab is not None:
        roofline["epilogue_vs_plain_store"] = epi_ab

    # Every kernel of the step timed on its own (light passes in GB/s against HBM).
    breakdown = _kernel_breakdown(kind, s, bwd, step)

    # End to end through the public API with host buffers: every step copies its
    # inputs from pinned host memory and its results back, inside the timed
    # region.  Inputs and outputs are double-buffered and the copies run on their
    # own streams, so step i's compute overlaps step i+1's upload and step i-1's
    # download (the way a training loop feeds a GPU).
    e2e = None
    if not a.no_e2e:
        e2e = _e2e_pipelined(kind, s, bwd, host, dev, step, outs, result_keys, flops, a, device, world, barrier)

    # The 70B shape timed in the same run beside the 7B headline.
    extra = {}
    if a.workload == "7B" and not a.no_extra:
        extra["70B"] = grg_extra("70B", a, device, world, barrier)

    cpu = None
    if rank == 0 and world == 1 and not a.no_cpu_baseline:
        cpu = cpu_baseline(kind, s, bwd)

    if rank == 0:
        per_gpu = value / world
        line = {
            "metric": METRIC,
            "value": round(value, 2),
            "unit": "TFLOP/s",
            "n_gpus": world,
            "steps": a.steps,
            "warmup": max(a.warmup, 3),
            "ms_per_step": round(ms_max / a.steps, 4),
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": "bf16",
            "data": "synthetic",
            "config": {**_describe(a.workload, kind, s, bwd), "parallelism": f"replicas x{world}",
                       "l2": l2_note,
                       "l2_flushed": l2_flushed,
                       "flops_per_step": flops, "timed_region_ms": round(ms_max, 2),
                       "frac_of_bf16_peak": {"burst": round(per_gpu / burst, 4),
                                             "sustained": round(per_gpu / sustained, 4),
                                             "source": peaks_src}},
            "roofline": roofline,
            "settled": settled,
            "kernels": breakdown,
            "extra": extra or None,
            "cpu_baseline": cpu,
            "unfused": unfused,
            "variants": variants or None,
            "e2e": e2e,
            "gpu_launches": launches * a.steps,
            "clocks": clk_head,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


def run_reference(a):
    """The reference arm: the fp64 CPU oracle on the host cores, bounded samples of the workload.
    Under torchrun only rank 0 runs it; the other ranks return without work."""
    rank, world, _ = dist_env()
    if rank != 0:
        return None
    kind, s, bwd = WORKLOADS[a.workload]
    inputs = _oracle_inputs(kind, s)
    probe = min(64, s["M"])
    t0 = time.perf_counter()
    _oracle_step(kind, s, bwd, inputs, probe)
    rate = _flops(kind, dict(s, M=probe), bwd) / max(time.perf_counter() - t0, 1e-3)
    # Each step a sample sized for about 2 s (less when many steps are asked
    # for) so the whole run stays within about two minutes.
    per_step_s = min(2.0, 120.0 / max(1, a.steps + a.warmup))
    rows = max(probe, min(s["M"], int(per_step_s * rate / _flops(kind, dict(s, M=1), bwd))))
    for _ in range(a.warmup):
        _oracle_step(kind, s, bwd, inputs, rows)
    t0 = time.perf_counter()
    for _ in range(a.steps):
        _oracle_step(kind, s, bwd, inputs, rows)
    dt = time.perf_counter() - t0
    fl = _flops(kind, dict(s, M=rows), bwd)
    value = fl * a.steps / dt / 1e12
    sample = (f"fp64 numpy oracle, unfused textbook {'fwd+bwd' if bwd else 'fwd'} on the first {rows} of "
              f"{s['M']} tokens with the full weights per step")
    line = {
        "metric": METRIC, "value": round(value, 4), "unit": "TFLOP/s", "n_gpus": world, "steps": a.steps,
        "warmup": a.warmup, "ms_per_step": round(dt / a.steps * 1e3, 2), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
        "config": {**_describe(a.workload, kind, s, bwd), "parallelism": "host cores", "sample_rows": rows},
        "cpu_baseline": {"value": round(value, 4), "unit": "TFLOP/s", "cores": _blas_threads(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(value, 4), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return line


def run_only(a):
    """One step of one path after the warm-up steps, for a profiler's launch list:
    the captured launches are those after warmup x launches-per-step."""
    import torch
    kind, s, bwd = WORKLOADS[a.workload]
    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    host, dev = _setup(kind, s, bwd, device)
    del host
    if a.only == "unfused":
        step, launches, ws = _make_unfused_step(kind, s, bwd, dev)
    else:
        step, outs, launches, _, ws = _make_step(kind, s, bwd, dev)
        if a.only == "activation_gain":
            step, ws = _make_hg_step(s, bwd, dev, outs, device)
            launches -= 1  # no gain fold
    for _ in range(a.warmup):
        step()
    step()
    torch.cuda.synchronize()
    status, detail = ws.query()
    if status != 0:
        raise SystemExit(f"bench.py --only: device status {status} detail {detail:#x}")
    print(json.dumps({"only": a.only, "workload": a.workload, "warmup": a.warmup,
                      "launches_per_step": launches}), flush=True)


def main():
    a = _args()
    if a.impl == "reference":
        run_reference(a)
    elif a.only is not None:
        run_only(a)
    else:
        run_coda(a)


if __name__ == "__main__":
    main()
