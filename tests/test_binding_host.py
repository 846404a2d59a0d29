"""Host-side behaviour of the Python binding (CPU only, no compute call).

There is no CPU path: CPU tensors, wrong dtypes and wrong shapes are refused
before anything reaches the library's compute entry points, and every entry
point the binding names is exported by the built library.
"""

import ctypes
import os
import re

import pytest
import torch

from gemm_epilogue_fusion_tmem_b200 import binding as B


def _bf(*s):
    return torch.zeros(*s, dtype=torch.bfloat16)


def test_library_loads_and_binds_every_entry_point():
    lib = B.library()
    for name in ("coda_grg_fwd", "coda_grg_bwd", "coda_swiglu_fwd", "coda_swiglu_bwd", "coda_gemm",
                 "coda_gemm_swiglu", "coda_grg_fwd_hg", "coda_xent_fwd", "coda_xent_bwd", "coda_qkv_rope_fwd",
                 "coda_qkv_rope_bwd", "coda_mlp_block_fwd", "coda_mlp_block_bwd", "coda_grg_fwd_unfused",
                 "coda_grg_bwd_unfused", "coda_selftest_wait_timeout"):
        assert getattr(lib, name).restype is not None or name == "coda_set_wait_limit_ns"


def test_cpu_tensors_are_refused():
    X, W1, R, g, W2 = _bf(256, 512), _bf(512, 512), _bf(256, 512), _bf(512), _bf(2048, 512)
    with pytest.raises(ValueError, match="CUDA tensor"):
        B.grg_fwd(X, W1, R, g, W2, 1e-6)
    with pytest.raises(ValueError, match="CUDA tensor"):
        B.gemm(X, W1, 256, 512, 512)
    with pytest.raises(ValueError, match="CUDA tensor"):
        B.xent_fwd(X, _bf(1024, 512), torch.zeros(256, dtype=torch.int32))


def test_wrong_dtype_and_shape_are_refused():
    X = torch.zeros(4, 8)  # float32 on CPU: the device check fires first
    with pytest.raises(ValueError):
        B._req(X, "X")
    with pytest.raises(TypeError):
        B._req("not a tensor", "X")


def test_status_strings_round_trip():
    assert B._status_string(0) == "ok"
    assert "timed out" in B._status_string(B.CODA_ERR_DEVICE_TIMEOUT)
    err = B.CodaError(3, "coda_gemm")
    assert err.status == 3 and "16-byte" in str(err)


def test_profile_hook_argument_checks():
    """coda_profile_arm validates its arguments and its table without touching the GPU."""
    import ctypes
    lib = B.library()
    fake = ctypes.c_void_p(1)  # never recorded: nothing is launched in this process
    try:
        for bad in (-1, 8, 15, 23, 99):
            assert lib.coda_profile_arm(bad, fake, fake) == B.CODA_ERR_INVALID_ARG, bad
        assert lib.coda_profile_arm(B.EPI_SWIGLU, fake, None) == B.CODA_ERR_INVALID_ARG
        assert lib.coda_profile_arm(B.EPI_SWIGLU, None, fake) == B.CODA_ERR_INVALID_ARG
        ids = list(range(8)) + list(range(16, 23))
        for k in ids:
            assert lib.coda_profile_arm(k, fake, fake) == 0, k
        assert lib.coda_profile_arm(B.EPI_STORE, fake, fake) == 0  # 16th pair: the table is full
        assert lib.coda_profile_arm(B.EPI_STORE, fake, fake) == B.CODA_ERR_INVALID_ARG
    finally:
        assert lib.coda_profile_arm(0, None, None) == 0  # disarm all
    assert lib.coda_profile_arm(B.EPI_STORE, fake, fake) == 0  # room again after disarming
    assert lib.coda_profile_arm(0, None, None) == 0
    assert (B.EPI_STORE, B.EPI_SWIGLU, B.EPI_ROPE, B.KERNEL_FOLD_GAIN, B.KERNEL_ROPE_UNROTATE) == (0, 2, 7, 16, 22)


def test_oracle_and_product_path_share_no_code():
    """The package never imports the oracle and the oracle never imports the
    package (only the seeded input generator, which holds none of the method's
    arithmetic, is shared through the tests); bench.py touches the oracle only
    inside its CPU legs."""
    import ast
    import os
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    pkg = os.path.join(root, "gemm_epilogue_fusion_tmem_b200")

    def imports(path):
        tree = ast.parse(open(path, encoding="utf-8").read())
        out = []
        for node in ast.walk(tree):
            if isinstance(node, ast.Import):
                out += [a.name for a in node.names]
            elif isinstance(node, ast.ImportFrom) and node.module:
                out.append(node.module)
        return out

    for name in os.listdir(pkg):
        if name.endswith(".py"):
            assert not any(m.split(".")[0] == "oracle" for m in imports(os.path.join(pkg, name))), name
    for name in os.listdir(os.path.join(root, "oracle")):
        if name.endswith(".py"):
            mods = imports(os.path.join(root, "oracle", name))
            assert not any(m.startswith("gemm_epilogue_fusion_tmem_b200") for m in mods), name
            assert not any(m in ("torch", "ctypes") for m in mods), name
    # bench.py: oracle imports only inside the CPU-leg functions
    tree = ast.parse(open(os.path.join(root, "bench.py"), encoding="utf-8").read())
    for fn in [n for n in tree.body if isinstance(n, ast.FunctionDef)]:
        uses = any(isinstance(x, ast.ImportFrom) and x.module and x.module.startswith("oracle") for x in ast.walk(fn))
        if uses:
            assert fn.name in ("_oracle_step", "_oracle_inputs", "cpu_baseline", "run_reference"), fn.name
    assert not any(isinstance(x, (ast.Import, ast.ImportFrom)) and "oracle" in ast.dump(x) for x in tree.body)


def test_missing_library_fails_loudly(tmp_path):
    """Without the built CUDA library the binding raises; there is no fallback."""
    import subprocess
    import sys
    code = (
        "import sys; sys.path.insert(0, %r)\n"
        "from gemm_epilogue_fusion_tmem_b200 import binding as B\n"
        "B.LIB_PATH = %r\n"
        "try:\n"
        "    B.library()\n"
        "except RuntimeError as e:\n"
        "    print('raised', 'not built' in str(e))\n"
    ) % (os.path.dirname(os.path.dirname(os.path.abspath(__file__))), str(tmp_path / "absent.so"))
    out = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=120).stdout
    assert out.strip() == "raised True", out


def _header_prototypes():
    """(return type, name, [parameter declarations]) of every function include/coda.h declares."""
    src = open(os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "coda.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    src = re.sub(r"//[^\n]*", "", src)
    src = "\n".join(line for line in src.splitlines() if not line.strip().startswith("#"))
    out = []
    for ret, name, args in re.findall(r"([A-Za-z_][\w\s*]*?)\b(coda_\w+)\s*\(([^)]*)\)\s*;", src):
        params = [a for a in (x.strip() for x in args.split(",")) if a and a != "void"]
        out.append((ret, name, params))
    return out


def _c_kind(decl: str) -> str:
    """Kind of a C type (or of a declaration 'type name'): ptr, int, float, u64 or void."""
    if "*" in decl:
        return "ptr"
    words = [w for w in decl.split() if w != "const"]
    base = words[0] if words else ""
    return {"int": "int", "int32_t": "int", "coda_status": "int", "float": "float", "size_t": "u64",
            "uint64_t": "u64", "void": "void"}.get(base, base)


def _py_kind(t) -> str:
    if t is None:
        return "void"
    if t in (ctypes.c_void_p, ctypes.c_char_p) or (isinstance(t, type) and issubclass(t, ctypes._Pointer)):
        return "ptr"
    if t is ctypes.c_int:
        return "int"
    if t is ctypes.c_float:
        return "float"
    if t in (ctypes.c_size_t, ctypes.c_uint64):
        return "u64"
    return repr(t)


def test_signatures_match_the_header():
    """Every prototype in include/coda.h has a ctypes signature in the binding
    with the same number and kinds of arguments and the same kind of result,
    so the binding cannot drift from the C ABI unnoticed."""
    protos = _header_prototypes()
    names = {n for _, n, _ in protos}
    assert len(protos) >= 40 and {"coda_grg_fwd", "coda_grg_bwd", "coda_swiglu_fwd", "coda_swiglu_bwd"} <= names
    grg = next(p for _, n, p in protos if n == "coda_grg_fwd")
    assert len(grg) == 18 and _c_kind(grg[14]) == "float"  # the parser sees eps as the 15th argument
    lib = B.library()
    for ret, name, params in protos:
        fn = getattr(lib, name)
        assert fn.argtypes is not None, f"{name}: no ctypes signature"
        want = [_c_kind(p if p.endswith("*") else p.rsplit(" ", 1)[0]) for p in params]
        assert [_py_kind(t) for t in fn.argtypes] == want, name
        assert _py_kind(fn.restype) == _c_kind(ret), name
