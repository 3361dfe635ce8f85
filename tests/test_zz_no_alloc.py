"""opnorm_normalize_noalloc: the operator-norm normalisation for callers that
cannot allocate device memory where they need it (code under a framework whose
memory manager owns the whole device, loops that must not enter the allocator
after start-up).  Its scratch is a static array inside the library, so it
takes no workspace.  Its output must match the workspace entry point
opnorm_normalize within the tolerance the other operator-norm tests use, on
two calls in a row (the second call reuses the static array the first call
left behind), and the float64 oracle run on the same stored input values.
This file is collected last on purpose."""
import ctypes as C

import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

import oracle.muon_oracle as O  # noqa: E402
from aurora_orthogonalised_optimizer_b200 import _abi as A  # noqa: E402

TOL = 1e-5          # fp32 inputs, as in the operator-norm parity test
ORACLE_TOL = 1e-5   # fp32 arithmetic on the stored values against float64


def _inputs(shapes, seed, dtype):
    rng = np.random.default_rng(seed)
    return [torch.from_numpy(rng.standard_normal(s).astype(np.float32)).to(dtype).cuda() for s in shapes]


def _reference(cfg, ins):
    outs = [torch.empty(t.shape, dtype=torch.float32, device="cuda") for t in ins]
    sig = torch.zeros(len(ins), dtype=torch.float32, device="cuda")
    A.opnorm_normalize(cfg, ins, outs, sig, A.make_workspace(cfg, [t.shape for t in ins]))
    return outs, sig


def _noalloc(cfg, ins):
    outs = [torch.full(t.shape, float("nan"), dtype=torch.float32, device="cuda") for t in ins]
    sig = torch.full((len(ins),), float("nan"), dtype=torch.float32, device="cuda")
    A.opnorm_normalize_noalloc(cfg, ins, outs, sig)     # goes through the C ABI; no workspace
    return outs, sig


def _compare(cfg, ins):
    ro, rs = _reference(cfg, ins)
    no, ns = _noalloc(cfg, ins)
    torch.cuda.synchronize()
    assert A.last_device_status() == A.MUON_OK
    assert torch.allclose(ns, rs, rtol=TOL, atol=0), (ns, rs)
    for a, b in zip(no, ro):
        rel = (a.double() - b.double()).norm() / b.double().norm()
        assert rel.item() <= TOL, rel.item()
    # directly against the oracle: the power iteration runs in fp32 on the
    # stored values, so both dtypes meet the fp32 bound
    for k, t in enumerate(ins):
        x = t.double().cpu().numpy()
        N, s = O.scale_to_unit_operator_norm(x, cfg.power_iters)
        assert abs(ns[k].item() - s) <= ORACLE_TOL * s, (t.shape, ns[k].item(), s)
        got = no[k].double().cpu().numpy()
        assert np.linalg.norm(got - N) <= ORACLE_TOL * np.linalg.norm(N), t.shape


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_noalloc_matches_workspace_entry_on_two_calls_in_a_row(dtype):
    # staging precision of the workspace entry = the input's own precision
    cfg = A.Config(gemm_mode=A.MUON_GEMM_FP32 if dtype == torch.float32 else A.MUON_GEMM_BF16, power_iters=5)
    first = _inputs([(256, 128), (100, 300), (64, 64), (1, 9), (517, 33)], 1, dtype)
    second = _inputs([(1024, 3072), (3072, 1024), (33, 7)], 2, dtype)
    _compare(cfg, first)
    _compare(cfg, second)
    _compare(cfg, first)        # and back: nothing left over from a larger call leaks in


def test_noalloc_rejects_requests_beyond_its_static_scratch():
    cfg = A.Config()
    lib = A.load()
    sh = A._shapes([(1 << 17, 1 << 17)])           # 2 x 128K floats of vectors > 1 MiB
    ptrs = (C.c_void_p * 1)(0x7f0000000000)         # never dereferenced: rejected on the host
    code = lib.opnorm_normalize_noalloc(C.byref(cfg.to_c()), 1, sh, ptrs, A.MUON_F32, None, None, None)
    assert code == A.MUON_ERR_UNSUPPORTED
