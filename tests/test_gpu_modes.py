"""The GEMM's alternate launch modes stay correct.

CODA_CTA_PAIR=0 selects one 128-row tile per CTA (cta_group::1) instead of the
CTA-pair tiles; CODA_PDL=0 turns programmatic dependent launch off.  Both are
read once per process, so each mode runs a subset of the parity suite in a
child process.
"""

import os
import subprocess
import sys

import pytest

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SUBSET = "gemm_core or test_grg_forward or test_grg_backward or swiglu or activation_gain"


@pytest.mark.parametrize("env", [{"CODA_CTA_PAIR": "0"}, {"CODA_PDL": "0"}], ids=["one_cta_tiles", "no_pdl"])
def test_parity_subset_in_mode(cuda_lib, env):
    r = subprocess.run([sys.executable, "-m", "pytest", "tests/test_gpu_parity.py", "tests/test_gpu_block.py",
                        "-m", "gpu", "-q", "-x", "-p", "no:cacheprovider", "-k", SUBSET],
                       cwd=ROOT, env={**os.environ, **env}, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-2000:]
