"""Degenerate inputs on the GPU path: a step with g = 0 from zero momentum
must stay finite and leave W exactly as it was (the oracle gives V = 0), in
both GEMM modes, for wide, tall and square matrices (the tall ones take the
bf16 fast paths of the prologue and epilogue)."""
import pytest

torch = pytest.importorskip("torch")
pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

from aurora_orthogonalised_optimizer_b200 import _abi as A  # noqa: E402


@pytest.mark.parametrize("mode", [A.MUON_GEMM_BF16, A.MUON_GEMM_FP32])
def test_zero_gradient_step_is_a_no_op(mode):
    shapes = [(256, 128), (96, 160), (64, 64), (1024, 192)]
    dt = torch.bfloat16 if mode == A.MUON_GEMM_BF16 else torch.float32
    cfg = A.Config(gemm_mode=mode, param_dtype=A.dtype_code(torch.empty(0, dtype=dt)),
                   grad_dtype=A.dtype_code(torch.empty(0, dtype=dt)))
    gen = torch.Generator(device="cuda").manual_seed(3)
    p = [(torch.randn(s, device="cuda", generator=gen) * 0.02).to(dt) for s in shapes]
    p0 = [t.clone() for t in p]
    g = [torch.zeros(s, dtype=dt, device="cuda") for s in shapes]
    m = [torch.zeros(s, dtype=torch.float32, device="cuda") for s in shapes]
    v = [torch.full(s, float("nan"), dtype=torch.float32, device="cuda") for s in shapes]
    A.muon_step(cfg, p, g, m, v, A.make_workspace(cfg, shapes))
    torch.cuda.synchronize()
    assert A.last_device_status() == A.MUON_OK
    for a, b, vv, mm in zip(p, p0, v, m):
        assert torch.isfinite(vv).all()
        assert (vv == 0).all()
        assert (mm == 0).all()
        assert torch.equal(a, b)
