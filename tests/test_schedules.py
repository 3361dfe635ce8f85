"""Host-side schedules: closed forms at the points the pages state."""
import math

import pytest

import oracle.muon_oracle as O
from aurora_orthogonalised_optimizer_b200 import schedules as S


def test_momentum_warmup_matches_page_and_oracle():
    assert S.momentum_warmup(0) == pytest.approx(0.85)
    assert S.momentum_warmup(250) == pytest.approx(0.90)
    assert S.momentum_warmup(500) == pytest.approx(0.95)
    assert S.momentum_warmup(10_000) == pytest.approx(0.95)
    for k in (0, 1, 17, 499, 500, 501, 3000):
        assert S.momentum_warmup(k) == pytest.approx(O.momentum_warmup(k), abs=1e-15)


def test_wsd_multiplier():
    T = 3200
    assert S.wsd_multiplier(0, T) == 1.0
    assert S.wsd_multiplier(int(0.3 * T) - 1, T) == 1.0          # stable phase: first 1 - 0.7
    assert S.wsd_multiplier(int(0.65 * T), T) == pytest.approx(0.5)   # halfway through the cool-down
    assert S.wsd_multiplier(T, T) == 0.0
    xs = [S.wsd_multiplier(k, T) for k in range(T + 1)]
    assert all(a >= b for a, b in zip(xs, xs[1:]))               # monotone non-increasing


def test_warmdown_multiplier_record_values():
    # 3000 iterations, warm-down over the last 900, no warm-up
    assert S.warmdown_multiplier(0, 3000, 900) == 1.0
    assert S.warmdown_multiplier(2099, 3000, 900) == 1.0
    assert S.warmdown_multiplier(2100, 3000, 900) == pytest.approx(1.0)
    assert S.warmdown_multiplier(2550, 3000, 900) == pytest.approx(0.5)
    assert S.warmdown_multiplier(3000, 3000, 900) == 0.0
    assert S.warmdown_multiplier(4, 100, 10, warmup_iters=10) == pytest.approx(0.5)


def test_optimizer_state_dict_keeps_fp32_state_for_bf16_params():
    """torch's load_state_dict would cast the fp32 momentum / moments to the
    parameters' bf16; the front-ends must hand the library fp32 state back."""
    torch = pytest.importorskip("torch")
    from aurora_orthogonalised_optimizer_b200.optim import FusedAdamW, MuonAurora
    val = 1.0 + 2.0 ** -12                      # not representable in bf16
    for cls, keys in ((MuonAurora, ["momentum_buffer"]), (FusedAdamW, ["exp_avg", "exp_avg_sq"])):
        p = torch.nn.Parameter(torch.zeros(4, 4, dtype=torch.bfloat16))
        o = cls([p])
        for k in keys:
            o.state[p][k] = torch.full((4, 4), val, dtype=torch.float32)
        o.param_groups[0]["step"] = 7
        o2 = cls([torch.nn.Parameter(torch.zeros(4, 4, dtype=torch.bfloat16))])
        o2.load_state_dict(o.state_dict())
        q = o2.param_groups[0]["params"][0]
        assert o2.param_groups[0]["step"] == 7
        for k in keys:
            assert o2.state[q][k].dtype == torch.float32
            assert bool((o2.state[q][k] == val).all())


def test_muon_optimizer_rejects_non_matrices_and_weight_decay():
    torch = pytest.importorskip("torch")
    from aurora_orthogonalised_optimizer_b200.optim import MuonAurora
    with pytest.raises(ValueError):
        MuonAurora([torch.nn.Parameter(torch.zeros(5))])
    with pytest.raises(ValueError):
        MuonAurora([torch.nn.Parameter(torch.zeros(5, 5))], weight_decay=0.1)
