"""torch.optim front-ends on the GPU: one MuonAurora + FusedAdamW training
step matches the float64 oracle (with the momentum warm-up and WSD schedule
applied on the host), and a 2 + 3 step run resumed from state_dict() equals
5 straight steps bit for bit."""
import numpy as np
import pytest

import oracle.muon_oracle as O
import workloads as WL
from tests.helpers import f64, rel_fro

torch = pytest.importorskip("torch")
pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

from aurora_orthogonalised_optimizer_b200.optim import FusedAdamW, MuonAurora  # noqa: E402
from aurora_orthogonalised_optimizer_b200 import schedules as S  # noqa: E402


def _model(seed=0):
    g = torch.Generator().manual_seed(seed)
    mats = [torch.randn(s, generator=g) * 0.02 for s in [(192, 64), (64, 192), (128, 128)]]
    vecs = [torch.randn(s, generator=g) * 0.02 for s in [(64,), (1,), (300, 8)]]
    return [m.cuda().to(torch.bfloat16) for m in mats], [v.cuda().to(torch.bfloat16) for v in vecs]


def _grads(params, step, seed=1):
    g = torch.Generator().manual_seed(seed * 1000 + step)
    return [(torch.randn(p.shape, generator=g) * 1e-2).cuda().to(p.dtype) for p in params]


def _run(mats, vecs, steps, start=0, opt_state=None):
    mats = [torch.nn.Parameter(m.clone()) for m in mats]
    vecs = [torch.nn.Parameter(v.clone()) for v in vecs]
    T = 10
    muon = MuonAurora(mats, lr=0.0375, momentum_warmup=(4, 0.85, 0.95),
                      lr_schedule=lambda k: S.wsd_multiplier(k, T, 0.7))
    adam = FusedAdamW(vecs, lr=0.01, lr_schedule=lambda k: S.wsd_multiplier(k, T, 0.7))
    if opt_state is not None:
        muon.load_state_dict(opt_state[0])
        adam.load_state_dict(opt_state[1])
    for st in range(start, start + steps):
        for p, g in zip(mats, _grads(mats, st)):
            p.grad = g
        for p, g in zip(vecs, _grads(vecs, st, seed=2)):
            p.grad = g
        muon.step()
        adam.step()
    torch.cuda.synchronize()
    return [m.detach() for m in mats], [v.detach() for v in vecs], (muon.state_dict(), adam.state_dict())


def test_optimizers_match_oracle_for_two_steps():
    mats, vecs = _model()
    out_m, out_v, _ = _run(mats, vecs, 2)
    cfg = WL.aurora_stack()
    oW = [f64(m) for m in mats]
    oM = [np.zeros(m.shape) for m in mats]
    oP = [f64(v) for v in vecs]
    oA = [np.zeros(v.shape) for v in vecs]
    oS = [np.zeros(v.shape) for v in vecs]
    for st in range(2):
        mult = S.wsd_multiplier(st, 10, 0.7)
        cfg.mu = S.momentum_warmup(st, 4, 0.85, 0.95)
        cfg.lr = 0.0375 * mult
        for k, g in enumerate(_grads(mats, st)):
            oW[k], oM[k], _ = O.step(oW[k], f64(g), oM[k], cfg, "bf16")
        for k, g in enumerate(_grads(vecs, st, seed=2)):
            p, oA[k], oS[k] = O.adamw_step(oP[k], f64(g), oA[k], oS[k], 0.01 * mult, 0.8, 0.95, 1e-10, 0.0, st + 1)
            oP[k] = O.round_to_bf16(p)
    for k in range(len(mats)):
        dw = f64(out_m[k]) - f64(mats[k])
        assert rel_fro(dw, oW[k] - f64(mats[k])) <= 3e-2 + 2 ** -8 * np.linalg.norm(oW[k]) / np.linalg.norm(dw)
    for k in range(len(vecs)):
        dv = f64(out_v[k]) - f64(vecs[k])
        want = oP[k] - f64(vecs[k])
        assert np.linalg.norm(dv - want) <= 1e-2 * np.linalg.norm(want) + np.linalg.norm(2 ** -8 * np.abs(oP[k]))


def test_resume_from_state_dict_is_bitwise_identical():
    mats, vecs = _model(3)
    full_m, full_v, _ = _run(mats, vecs, 5)
    half_m, half_v, state = _run(mats, vecs, 2)
    res_m, res_v, _ = _run(half_m, half_v, 3, start=2, opt_state=state)
    for a, b in zip(full_m + full_v, res_m + res_v):
        assert torch.equal(a, b)
