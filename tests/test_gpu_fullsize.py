"""Full-size parity of the 3.8B matrix sets (168 matrices, 2.82 G parameters)
in the launch configuration the bench times: one muon_step call over every
matrix per step, tensor-core Newton-Schulz, for all 3 steps each set states.

* Sampled outputs: one fc (12288 x 3072, tall), one proj (3072 x 12288,
  wide), one q (3072 x 3072, square) and k / v (1024 x 3072) of the first
  and last layer follow the float64 oracle's own trajectory (its weights and
  momentum carried from step to step); at every step the update V is within
  3e-2 relative Frobenius error and the momentum within 1e-6.  From step 2 on
  the momentum is non-zero, so the Nesterov blend u is not a multiple of the
  gradient and the operands of the polar and of the contra term are told
  apart.
* Properties that hold for every matrix at any size, checked on all 168 at
  every step:
  - momentum: m = m_prev + (1 - mu)(g - m_prev) up to fp32 rounding;
  - the parameter add: W_new = W - lr V up to the bf16 rounding of W_new
    and the fp32 rounding of the product and the difference;
  - the update is finite and (Aurora stack) ||V||_F / ||W||_F >= TARGET_UW.
"""
import numpy as np
import pytest

import oracle.muon_oracle as O
import workloads as WL
from tests.helpers import f64, rel_fro

torch = pytest.importorskip("torch")
pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

from aurora_orthogonalised_optimizer_b200 import _abi as A  # noqa: E402


def _check_all(wl, p, w_prev, g, m, m_prev, v):
    """Properties every matrix meets after one step, whatever its size."""
    mu, lr = wl.cfg.mu, wl.cfg.lr
    for k in range(wl.n):
        assert torch.isfinite(v[k]).all(), ("V not finite", k)
        want_m = m_prev[k].double() + (1.0 - mu) * (g[k].double() - m_prev[k].double())
        em = ((m[k].double() - want_m).norm() / want_m.norm()).item()
        assert em <= 1e-6, ("momentum", k, em)
        w0 = w_prev[k].double()
        step = lr * v[k].double()
        want = w0 - step
        # bf16 rounding of W_new plus the fp32 rounding of lr * V and of the subtraction
        half_ulp = torch.ldexp(torch.ones_like(want), torch.frexp(want.abs().clamp_min(1e-30))[1] - 9)
        bound = 1.01 * half_ulp + 2.0 ** -23 * (step.abs() + want.abs())
        err = (p[k].double() - want).abs()
        assert bool((err <= bound).all()), ("param add", k, (err / bound).max().item())
        if wl.cfg.target_uw > 0:
            assert (v[k].norm() / w0.norm()).item() >= wl.cfg.target_uw * (1 - 1e-5)


def _run_full(wl, sample):
    cfg = A.Config.from_step_config(wl.cfg, gemm_mode=A.MUON_GEMM_BF16, param_dtype=A.MUON_BF16,
                                    grad_dtype=A.MUON_BF16)
    W, _ = WL.generate_torch(wl, None, 0, threads=16, want_g=False)
    p = [w.cuda() for w in W]
    del W
    m = [torch.zeros(s, dtype=torch.float32, device="cuda") for s in wl.shapes]
    v = [torch.empty(s, dtype=torch.float32, device="cuda") for s in wl.shapes]
    ws = A.make_workspace(cfg, wl.shapes)
    Wn, _, _ = WL.generate(wl, sample)
    oW = {k: WL.to_f64(Wn[j], WL.BF16) for j, k in enumerate(sample)}
    oM = {k: np.zeros(wl.shapes[k]) for k in sample}
    assert wl.steps == 3
    for st in range(wl.steps):
        _, G = WL.generate_torch(wl, None, st, threads=16, want_w=False)
        g = [x.cuda() for x in G]
        del G
        w_prev = [t.clone() for t in p]
        m_prev = [t.clone() for t in m]
        A.muon_step(cfg, p, g, m, v, ws)
        torch.cuda.synchronize()
        assert A.last_device_status() == A.MUON_OK
        _check_all(wl, p, w_prev, g, m, m_prev, v)
        del w_prev, m_prev, g
        for k in sample:
            gk = WL.to_f64(WL.grad(wl, k, st), WL.BF16)
            oW[k], oM[k], V = O.step(oW[k], gk, oM[k], wl.cfg, WL.BF16)
            ev = rel_fro(f64(v[k]), V)
            assert ev <= 3e-2, ("V", st, k, wl.shapes[k], ev)
            assert rel_fro(f64(m[k]), oM[k]) <= 1e-6, ("m", st, k)


# fc of layer 0 (tall: transposed into the X orientation; two Aurora polars),
# proj of layer 13 (wide, two polars), q of layer 27 (square, one polar),
# k of layer 0 and v of layer 27 (1024 x 3072, the Aurora wide path)
SAMPLE = [1, 4, 6 * 13 + 5, 6 * 27, 6 * 27 + 2]


def test_llama_3p8b_aurora_stack_full_size_three_steps():
    _run_full(WL.llama_3p8b_aurora(), SAMPLE)


def test_llama_3p8b_plain_muon_full_size_three_steps():
    _run_full(WL.llama_3p8b_plain(), SAMPLE)


def _run_sampled_trajectory(wl, sample, gemm_mode=A.MUON_GEMM_BF16, tol=3e-2):
    """All matrices of the workload stepped together (one call per step, as the
    bench does); the sampled ones follow the oracle's own trajectory."""
    pdt = A.MUON_BF16 if wl.param_dtype == WL.BF16 else A.MUON_F32
    gdt = A.MUON_BF16 if wl.grad_dtype == WL.BF16 else A.MUON_F32
    cfg = A.Config.from_step_config(wl.cfg, gemm_mode=gemm_mode, param_dtype=pdt, grad_dtype=gdt)
    W, _ = WL.generate_torch(wl, None, 0, threads=16, want_g=False)
    p = [w.cuda() for w in W]
    m = [torch.zeros(s, dtype=torch.float32, device="cuda") for s in wl.shapes]
    v = [torch.empty(s, dtype=torch.float32, device="cuda") for s in wl.shapes]
    ws = A.make_workspace(cfg, wl.shapes)
    Wn, _, _ = WL.generate(wl, sample)
    oW = {k: WL.to_f64(Wn[j], wl.param_dtype) for j, k in enumerate(sample)}
    oM = {k: np.zeros(wl.shapes[k]) for k in sample}
    for st in range(wl.steps):
        _, G = WL.generate_torch(wl, None, st, threads=16, want_w=False)
        g = [x.cuda() for x in G]
        A.muon_step(cfg, p, g, m, v, ws)
        torch.cuda.synchronize()
        assert A.last_device_status() == A.MUON_OK
        for k in sample:
            gk = WL.to_f64(WL.grad(wl, k, st), wl.grad_dtype)
            oW[k], oM[k], V = O.step(oW[k], gk, oM[k], wl.cfg, wl.param_dtype)
            ev = rel_fro(f64(v[k]), V)
            assert ev <= tol, ("V", st, k, wl.shapes[k], ev)
            assert rel_fro(f64(m[k]), oM[k]) <= 1e-6, ("m", st, k)


def test_gpt2_124m_all_72_matrices_five_steps():
    """GPT-2 124M set, plain Muon, mu 0.90, lr 0.04: all 72 matrices per call,
    5 steps; layers 0 and 11 against the oracle at every step."""
    wl = WL.gpt2_124m_plain()
    _run_sampled_trajectory(wl, list(range(6)) + list(range(66, 72)))


def test_aurora_sweep_all_128_matrices():
    """Aurora sweep (32 each of 1024x4096, 4096x1024, 2048^2, 768x3072), full
    stack, fp32 params/grads: all 128 per call, one of each shape sampled."""
    wl = WL.aurora_shape_sweep()
    _run_sampled_trajectory(wl, [5, 37, 69, 101])
