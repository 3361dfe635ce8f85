"""The bounds-checked build (libaurora_muon_checked.so, AURORA_MUON_CHECKED=1).

No memory sanitizer runs on this pool, so the library also exists in a
build whose kernels test every global access against the extent of the
buffer it addresses, skip an access that falls outside and record
MUON_ERR_BOUNDS.  Each test runs in a fresh process that loads that build:
  * the self-test shows the mechanism records a failed test (it touches no
    memory) and that reading the status clears it;
  * the GPU parity suites (every entry point against the float64 oracle on
    small and ragged shapes: 3 x 5, 129 x 65, 1 x 40, 33 x 7, rows not a
    multiple of 8, ...) and the degenerate-step and AdamW tests pass on it,
    with no failed index test after any of them (tests/conftest.py)."""
import os
import subprocess
import sys

import pytest

torch = pytest.importorskip("torch")
pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
ENV = dict(os.environ, AURORA_MUON_CHECKED="1")

SELFTEST = r"""
import sys
sys.path.insert(0, %r)
import torch
from aurora_orthogonalised_optimizer_b200 import _abi as A
assert A.build_checked(), "not the checked build"
torch.cuda.init()
assert A.last_device_status() == A.MUON_OK
assert A.selftest_bounds_check() == A.MUON_OK
assert A.last_device_status() == A.MUON_ERR_BOUNDS
assert A.last_check_line() // 100000 == 1       # the self-test sits in elementwise.cu
assert A.last_device_status() == A.MUON_OK      # reading cleared it
print("checked selftest ok")
""" % ROOT


def test_checked_build_records_a_failed_index_test():
    r = subprocess.run([sys.executable, "-c", SELFTEST], env=ENV, cwd=ROOT, capture_output=True, text=True,
                       timeout=600)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-3000:]
    assert "checked selftest ok" in r.stdout


def test_parity_suites_pass_on_the_checked_build():
    cmd = [sys.executable, "-m", "pytest", "-q", "-x", "-m", "gpu", "-p", "no:cacheprovider",
           "tests/test_gpu_parity.py", "tests/test_gpu_degenerate.py", "tests/test_gpu_adamw.py"]
    r = subprocess.run(cmd, env=ENV, cwd=ROOT, capture_output=True, text=True, timeout=1800)
    assert r.returncode == 0, r.stdout[-4000:] + r.stderr[-2000:]
