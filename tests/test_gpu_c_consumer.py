"""The C ABI driven from plain C on the GPU.

tests/c_consumer_grg.c allocates with cudaMalloc, runs coda_grg_fwd and
coda_grg_bwd on the legacy default stream and writes its inputs and outputs to
a file.  The same inputs through the Python binding must give the same bits
(one library, deterministic kernels), and the C program's forward output must
match the fp64 oracle at the usual tolerance.
"""

import os
import shutil
import subprocess

import numpy as np
import pytest
import torch

from oracle import coda_oracle as O
from tests.parity import assert_tol, f64

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))
M, K, D, F = 512, 512, 512, 1024
N = 2 * F


def _cuda_root():
    nvcc = shutil.which("nvcc")
    return os.path.dirname(os.path.dirname(nvcc)) if nvcc else "/usr/local/cuda"


def test_c_program_matches_the_binding_bit_for_bit(cuda_lib, tmp_path):
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("gcc not available")
    from gemm_epilogue_fusion_tmem_b200 import build as Bld
    cuda = _cuda_root()
    exe = tmp_path / "c_consumer_grg"
    libdir = os.path.dirname(Bld.LIB_PATH)
    subprocess.run([gcc, "-std=c11", "-Wall", "-Wextra", "-Werror", "-I", Bld.INCLUDE, "-I", f"{cuda}/include",
                    os.path.join(HERE, "c_consumer_grg.c"), "-L", libdir, "-lcoda", f"-Wl,-rpath,{libdir}",
                    "-L", f"{cuda}/lib64", "-lcudart", f"-Wl,-rpath,{cuda}/lib64", "-lm", "-o", str(exe)], check=True)
    out = tmp_path / "grg.bin"
    r = subprocess.run([str(exe), str(out)], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0 and r.stdout.strip() == "ok", r.stdout + r.stderr

    raw = np.fromfile(out, dtype=np.uint8)
    pos = 0

    def take(shape, dtype):
        nonlocal pos
        n = int(np.prod(shape)) * torch.tensor([], dtype=dtype).element_size()
        t = torch.from_numpy(raw[pos:pos + n].copy()).view(dtype).reshape(shape)
        pos += n
        return t

    bf, f32 = torch.bfloat16, torch.float32
    inp = {"X": take((M, K), bf), "R": take((M, D), bf), "W1": take((D, K), bf), "W2": take((N, D), bf),
           "g": take((D,), bf), "dY": take((M, F), bf)}
    c_out = {"H": take((M, D), bf), "r": take((M,), f32), "Y": take((M, F), bf), "AB": take((M, N), bf),
             "dX": take((M, K), bf), "dR": take((M, D), bf), "dW1": take((D, K), bf), "dW2": take((N, D), bf),
             "dg": take((D,), f32)}
    assert pos == raw.size

    td = {k: v.cuda() for k, v in inp.items()}
    fo = cuda_lib.grg_fwd(td["X"], td["W1"], td["R"], td["g"], td["W2"], 1e-6)
    bo = cuda_lib.grg_bwd(td["dY"], td["X"], td["W1"], fo["H"], fo["r"], fo["AB"], td["g"], td["W2"])
    torch.cuda.synchronize()
    for k, v in {**fo, **bo}.items():
        bits = torch.int16 if v.dtype == bf else torch.int32
        assert torch.equal(v.cpu().view(bits), c_out[k].view(bits)), k

    fs = O.grg_forward_stored(*(f64(inp[k]) for k in ("X", "W1", "R", "g", "W2")), 1e-6)
    assert_tol(c_out["Y"], fs["Y"], "C program Y")
    assert_tol(c_out["H"], fs["H"], "C program H")
