"""GPU parity of the fused auxiliary AdamW against the float64 oracle.

Tolerances: exp_avg / exp_avg_sq 1e-6 relative (fp32 state arithmetic);
params: |dp_gpu - dp_oracle| <= 1e-5 (|dp_oracle| + rms(dp_oracle)) + the
storage rounding of
the new parameter (half a bf16 ulp for bf16) + 4 fp32 ulps of |p| (the
kernel's fp32 decay product and subtraction)."""
import numpy as np
import pytest

import oracle.muon_oracle as O
import workloads as WL
from tests.helpers import bf16_half_ulp, f64, rel_fro, to_dev

torch = pytest.importorskip("torch")
pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

from aurora_orthogonalised_optimizer_b200 import _abi as A  # noqa: E402


def _check(wl, indices, steps):
    P = [WL.aux_param(wl, i) for i in indices]
    p = [to_dev(x, wl.param_dtype) for x in P]
    m = [torch.zeros(wl.shapes[i], dtype=torch.float32, device="cuda") for i in indices]
    v = [torch.zeros(wl.shapes[i], dtype=torch.float32, device="cuda") for i in indices]
    lrs = [wl.lrs[i] for i in indices]
    oP = [WL.to_f64(x, wl.param_dtype) for x in P]
    oM = [np.zeros(wl.shapes[i]) for i in indices]
    oV = [np.zeros(wl.shapes[i]) for i in indices]
    for st in range(1, steps + 1):
        G = [WL.aux_grad(wl, i, st) for i in indices]
        g = [to_dev(x, wl.grad_dtype) for x in G]
        before = [f64(t) for t in p]
        A.adamw_step(p, g, m, v, st, lrs, wl.beta1, wl.beta2, wl.eps, wl.weight_decay)
        torch.cuda.synchronize()
        for k in range(len(indices)):
            pn, mn, vn = O.adamw_step(oP[k], WL.to_f64(G[k], wl.grad_dtype), oM[k], oV[k], lrs[k], wl.beta1,
                                      wl.beta2, wl.eps, wl.weight_decay, st)
            assert rel_fro(f64(m[k]), mn) <= 1e-6, ("m", st, k)
            assert rel_fro(f64(v[k]), vn) <= 1e-6, ("v", st, k)
            dp_or = pn - oP[k]
            dp = f64(p[k]) - before[k]
            # storage rounding of the new parameter, plus the fp32 rounding of the
            # decay product and of the subtraction (a few ulps of |p|)
            rnd = (bf16_half_ulp(pn) if wl.param_dtype == WL.BF16 else 0.0) + 4 * 2.0 ** -24 * (
                np.abs(pn) + np.abs(before[k]))
            scale = np.abs(dp_or) + np.sqrt(np.mean(dp_or ** 2))   # element update + the tensor's rms update
            assert np.all(np.abs(dp - dp_or) <= 1e-5 * scale + 1.01 * rnd + 1e-30), ("p", st, k)
            # the oracle continues from the stored (rounded) parameter, like the GPU
            oP[k] = before[k] + dp
            oM[k], oV[k] = mn, vn


@pytest.mark.parametrize("pdt", [WL.BF16, WL.F32])
def test_adamw_mixed_sizes(pdt):
    shapes = [(1,), (7,), (33,), (1000,), (4097,), (128, 129), (8192,), (3, 8193)]
    lrs = [0.01, 0.3, 1.0 / 320, 0.01, 0.3, 0.05, 0.01, 0.3]
    wl = WL.AuxWorkload("mixed", 7, shapes, lrs, param_dtype=pdt, grad_dtype=pdt, weight_decay=0.1)
    _check(wl, range(len(shapes)), 3)


def test_adamw_3p8b_aux_sampled():
    """The 3.8B non-matrix set's own tensors: token embedding, one value table, gains, scalars."""
    wl = WL.llama_3p8b_aux()
    _check(wl, [0, 5, 16, 17, 18, 19], 2)
