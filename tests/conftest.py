import json
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU and the built CUDA library")
    config.addinivalue_line("markers", "slow: full-size workload check (seconds to minutes)")


@pytest.fixture(scope="session")
def cuda_lib():
    """The built C-ABI library, loaded through the Python binding (GPU tests only)."""
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from gemm_epilogue_fusion_tmem_b200 import binding
    return binding


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """Worst |err| / bound and the count above the bound of every parity check run."""
    from tests.parity import REPORT
    if not REPORT:
        return
    tr = terminalreporter
    tr.section("parity: worst |err| / bound per check (above_bound must be 0)")
    for rec in REPORT:
        tr.write_line(f"{rec['worst_ratio']:8.4f}  above={rec['above_bound']:<4d} n={rec['n']:<10d} "
                      f"[{rec['kind']}] {rec['check']}")
    path = os.environ.get("CODA_PARITY_REPORT")
    if path:
        with open(path, "a") as f:
            for rec in REPORT:
                f.write(json.dumps(rec) + "\n")
