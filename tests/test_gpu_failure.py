"""Failure detection on the device without a fault: a bounded wait that runs
out records MUON_ERR_TIMEOUT in the status word, the kernel returns, the
host reads (and clears) the status, and the context keeps working."""
import numpy as np
import pytest

import oracle.muon_oracle as O
from tests.helpers import f64, rel_fro

torch = pytest.importorskip("torch")
pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

from aurora_orthogonalised_optimizer_b200 import _abi as A  # noqa: E402


def test_bounded_wait_times_out_and_context_stays_usable():
    assert A.last_device_status() == A.MUON_OK                 # clean start
    assert A.selftest_wait_timeout(2_000_000) == A.MUON_OK     # ~1-2 ms of waiting
    assert A.last_device_status() == A.MUON_ERR_TIMEOUT        # the wait gave up and said so
    assert A.last_device_status() == A.MUON_OK                 # reading clears the word
    # the context still runs real work correctly
    x = np.random.default_rng(3).standard_normal((96, 160)).astype(np.float32)
    cfg = A.Config(gemm_mode=A.MUON_GEMM_BF16)
    out = [torch.empty((96, 160), dtype=torch.float32, device="cuda")]
    A.ns_polar(cfg, [torch.from_numpy(x).cuda()], out, A.make_workspace(cfg, [(96, 160)]))
    torch.cuda.synchronize()
    assert A.last_device_status() == A.MUON_OK
    assert rel_fro(f64(out[0]), O.newton_schulz(x.astype(np.float64))) <= 3e-2
