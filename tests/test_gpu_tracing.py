"""Tracing (muon_profile_enable / muon_profile_read): one step of a small
Aurora stack records every kernel class of the path, and the per-kind split
of the tensor-core GEMM launches adds up to the ns_gemm_tc class."""
import pytest

import workloads as WL

torch = pytest.importorskip("torch")
pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

from aurora_orthogonalised_optimizer_b200 import _abi as A  # noqa: E402


def test_profile_classes_and_gemm_kinds():
    shapes = [(256, 128), (192, 320), (128, 128)]
    wl = WL.custom("trace", 5, shapes, WL.aurora_stack(), WL.BF16, WL.BF16)
    W, G = WL.generate_torch(wl, None, 0)
    p = [w.cuda() for w in W]
    g = [x.cuda() for x in G]
    m = [torch.zeros(s, dtype=torch.float32, device="cuda") for s in shapes]
    cfg = A.Config.from_step_config(wl.cfg, gemm_mode=A.MUON_GEMM_BF16, param_dtype=A.MUON_BF16,
                                    grad_dtype=A.MUON_BF16)
    ws = A.make_workspace(cfg, shapes)
    A.profile_enable(True)
    A.muon_step(cfg, p, g, m, None, ws)
    torch.cuda.synchronize()
    prof = A.profile_read()
    A.profile_enable(False)
    for cls in ("ns_gemm_tc", "prologue", "power_iter", "aurora_rows", "reductions", "epilogue"):
        assert prof[cls]["launches"] > 0, cls
        assert prof[cls]["ms"] > 0.0, cls
    kinds = [prof["tc_kind_gram"], prof["tc_kind_square"], prof["tc_kind_update"]]
    # one launch of each kind per Newton-Schulz step and polar
    assert kinds[0]["launches"] == kinds[1]["launches"] == kinds[2]["launches"]
    assert sum(k["launches"] for k in kinds) == prof["ns_gemm_tc"]["launches"]
    assert abs(sum(k["flops"] for k in kinds) - prof["ns_gemm_tc"]["flops"]) <= 1e-6 * prof["ns_gemm_tc"]["flops"]
    assert prof["ns_gemm_simt"]["launches"] == 0
