"""The sharded optimizer step reproduces the one-call step (one GPU).

The modded-nanogpt 2024-11-10 record write-up (训练管线与系统实现 / 四路优化器分工)
runs Muon data-parallel: each matrix is updated by one rank and the updates
are then exchanged.  Here ownership comes from the LPT plan, every rank's
parameters live in its slice of a [world, shard] flat buffer, and the
exchange is an all-gather of the slices.  With one GPU the ranks are
emulated in one process: each rank has its own copy of the flat buffer,
steps only the matrices it owns (one muon_step over that subset, as
bench.py --gpus N does), and the exchange is the all-gather's copy of every
owner's slice into every rank's buffer.  No kernel waits on another rank.

Checks, for world sizes 2 and 3 over three steps of the GPT-2 shapes with
the full Aurora + Contra-Muon + u/w-floor stack (bf16 params and grads):
  * the update V of every matrix equals the one-call step's within 1e-5
    relative Frobenius error (the item split of the power iteration follows
    the call's total size, so only the fp32 summation order of sigma-hat
    may differ);
  * after the exchange every rank holds, for every matrix, the parameters of
    the one-call step up to that difference: elementwise within one bf16
    unit in the last place plus lr |dV| and the fp32 rounding of W - lr V
    (near W = lr V the rounded result is tiny and its ulp tells nothing);
  * the momentum of every owned matrix matches the one-call step within 1e-6;
  * one matrix of each rank follows the float64 oracle within 3e-2 (V).
"""
import numpy as np
import pytest

import oracle.muon_oracle as O
import workloads as WL
from aurora_orthogonalised_optimizer_b200 import sharding as SH
from tests.helpers import f64, rel_fro

torch = pytest.importorskip("torch")
pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

from aurora_orthogonalised_optimizer_b200 import _abi as A  # noqa: E402


def _bf16_ulp(x: torch.Tensor) -> torch.Tensor:
    """One bf16 unit in the last place at |x| (x in float64)."""
    return torch.ldexp(torch.ones_like(x), torch.frexp(x.abs().clamp_min(1e-30))[1] - 8)


def _param_budget(w0, dw0, w1, ws, v1, dv, lr):
    """Largest difference of two bf16 parameters each rounded from its own
    W0 - lr V (the two W0 differ by dw0, the two V by dv)."""
    return (_bf16_ulp(torch.maximum(w1.abs(), ws.abs())) + dw0.abs() + lr * dv.abs()
            + 2.0 ** -22 * (w0.abs() + lr * v1.abs()))


@pytest.mark.parametrize("world", [2, 3])
def test_sharded_step_matches_one_call_step(world):
    wl = WL.custom("gpt2_shapes_aurora_stack", 11, WL.gpt2_124m_shapes(), WL.aurora_stack(), WL.BF16, WL.BF16,
                   w_std=WL.fan_in_std(WL.gpt2_124m_shapes()), grad_kind="row_lognormal", grad_base=1e-3,
                   grad_sigma=0.5, steps=3)
    shapes = wl.shapes
    cfg = A.Config.from_step_config(wl.cfg, gemm_mode=A.MUON_GEMM_BF16, param_dtype=A.MUON_BF16,
                                    grad_dtype=A.MUON_BF16)
    owned = SH.lpt_partition(SH.step_costs(shapes, wl.cfg.ns_steps, wl.cfg.aurora, wl.cfg.pp_iterations), world)
    assert sorted(i for o in owned for i in o) == list(range(wl.n))
    assert all(owned)
    lay = SH.flat_layout(shapes, owned)

    W, _ = WL.generate_torch(wl, None, 0, threads=8, want_g=False)
    # one-call reference
    p1 = [w.cuda() for w in W]
    m1 = [torch.zeros(s, dtype=torch.float32, device="cuda") for s in shapes]
    v1 = [torch.empty(s, dtype=torch.float32, device="cuda") for s in shapes]
    ws1 = A.make_workspace(cfg, shapes)
    # the ranks: one flat buffer each, all holding every parameter
    flats = [torch.empty(lay.total_elems, dtype=torch.bfloat16, device="cuda") for _ in range(world)]
    views = [SH.views(f, lay, shapes) for f in flats]
    for r in range(world):
        for i in range(wl.n):
            views[r][i].copy_(p1[i])
    mom = {i: torch.zeros(shapes[i], dtype=torch.float32, device="cuda") for i in range(wl.n)}
    upd = {i: torch.empty(shapes[i], dtype=torch.float32, device="cuda") for i in range(wl.n)}
    wss = [A.make_workspace(cfg, [shapes[i] for i in owned[r]]) for r in range(world)]
    sample = [owned[r][len(owned[r]) // 2] for r in range(world)]      # one matrix per rank
    Wn, _, _ = WL.generate(wl, sample)
    oW = {k: WL.to_f64(Wn[j], WL.BF16) for j, k in enumerate(sample)}
    oM = {k: np.zeros(shapes[k]) for k in sample}

    for st in range(wl.steps):
        _, G = WL.generate_torch(wl, None, st, threads=8, want_w=False)
        g = [x.cuda() for x in G]
        w0 = [t.clone() for t in p1]
        w0s = [[t.clone() for t in views[r]] for r in range(world)]
        A.muon_step(cfg, p1, g, m1, v1, ws1)
        for r in range(world):
            ids = owned[r]
            A.muon_step(cfg, [views[r][i] for i in ids], [g[i] for i in ids], [mom[i] for i in ids],
                        [upd[i] for i in ids], wss[r])
        # the exchange: every owner's slice lands in every rank's buffer
        for r in range(world):
            src = flats[r].narrow(0, r * lay.shard_elems, lay.shard_elems)
            for q in range(world):
                if q != r:
                    flats[q].narrow(0, r * lay.shard_elems, lay.shard_elems).copy_(src)
        torch.cuda.synchronize()
        assert A.last_device_status() == A.MUON_OK
        for i in range(wl.n):
            ev = rel_fro(f64(upd[i]), f64(v1[i]))
            assert ev <= 1e-5, ("V", st, world, i, shapes[i], ev)
            want = p1[i].double()
            dv = upd[i].double() - v1[i].double()
            for r in range(world):
                got = views[r][i].double()
                w0d = w0[i].double()
                budget = _param_budget(w0d, w0s[r][i].double() - w0d, want, got, v1[i].double(), dv, wl.cfg.lr)
                ratio = ((got - want).abs() / budget).max().item()
                assert ratio <= 1.0, ("params", st, world, r, i, shapes[i], ratio)
            em = ((mom[i] - m1[i]).double().norm() / m1[i].double().norm()).item()
            assert em <= 1e-6, ("momentum", st, i, em)
        for k in sample:
            gk = WL.to_f64(WL.grad(wl, k, st), WL.BF16)
            oW[k], oM[k], V = O.step(oW[k], gk, oM[k], wl.cfg, WL.BF16)
            assert rel_fro(f64(upd[k]), V) <= 3e-2, ("V", st, k, shapes[k])
