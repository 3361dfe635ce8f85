"""GPU parity of every C-ABI entry point against the float64 oracle.

Tolerances (relative Frobenius error per matrix):
  update V:  3e-2 with bf16 GEMM operands (MUON_GEMM_BF16, MUON_GEMM_BF16_SIMT),
             1e-4 with fp32 GEMMs (MUON_GEMM_FP32);
  momentum:  1e-6;
  W_new:     |dW_gpu - dW_oracle| <= tol_V * lr |V| + the storage rounding of W_new.
"""
import math

import numpy as np
import pytest

import oracle.muon_oracle as O
import workloads as WL
from tests.helpers import bf16_half_ulp, f64, rel_fro, to_dev

torch = pytest.importorskip("torch")
pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

from aurora_orthogonalised_optimizer_b200 import _abi as A  # noqa: E402

MODES = {"bf16": A.MUON_GEMM_BF16, "fp32": A.MUON_GEMM_FP32, "bf16simt": A.MUON_GEMM_BF16_SIMT}
TOL_V = {A.MUON_GEMM_BF16: 3e-2, A.MUON_GEMM_BF16_SIMT: 3e-2, A.MUON_GEMM_FP32: 1e-4}
TOL_M = 1e-6


def gauss(shape, seed, scale=1.0):
    return (np.random.default_rng(seed).standard_normal(shape) * scale).astype(np.float32)


def run_polar(cfg, mats, aurora=False):
    ins = [torch.from_numpy(m).cuda() for m in mats]
    outs = [torch.empty(m.shape, dtype=torch.float32, device="cuda") for m in mats]
    ws = A.make_workspace(cfg, [m.shape for m in mats])
    A.ns_polar(cfg, ins, outs, ws, aurora=aurora)
    torch.cuda.synchronize()
    assert A.last_device_status() == A.MUON_OK
    return [f64(o) for o in outs]


# ------------------------------------------------------------------ Newton-Schulz
NS_SHAPES = [(256, 128), (128, 256), (96, 96), (3, 5), (129, 65), (300, 700), (700, 300), (384, 384),
             (260, 1030), (1, 40), (1000, 8)]


@pytest.mark.parametrize("mode", list(MODES))
def test_ns_polar_matches_oracle(mode):
    cfg = A.Config(gemm_mode=MODES[mode])
    mats = [gauss(s, 100 + i) for i, s in enumerate(NS_SHAPES)]
    got = run_polar(cfg, mats)
    for m, g in zip(mats, got):
        want = O.newton_schulz(m.astype(np.float64), 12, 2.0, -1.5, 0.5, 1e-7)
        assert rel_fro(g, want) <= TOL_V[cfg.gemm_mode], (m.shape, rel_fro(g, want))


@pytest.mark.parametrize("mode", list(MODES))
@pytest.mark.parametrize("coef", [(0.0, 1.0, 0.0), (0.0, 0.0, 1.0), (1.0, 0.0, 0.0), (2.0, -1.5, 0.5),
                                  (3.4445, -4.7750, 2.0315)])
def test_ns_single_step_isolates_each_gemm(mode, coef):
    """One step with (a,b,c) = (0,1,0) -> A X, (0,0,1) -> A^2 X, (1,0,0) -> X."""
    a, b, c = coef
    cfg = A.Config(gemm_mode=MODES[mode], ns_steps=1, ns_a=a, ns_b=b, ns_c=c)
    mats = [gauss((300, 700), 7), gauss((700, 300), 8), gauss((257, 257), 9), gauss((100, 2000), 10)]
    got = run_polar(cfg, mats)
    tol = 1e-5 if cfg.gemm_mode == A.MUON_GEMM_FP32 else 1.5e-2
    for m, g in zip(mats, got):
        want = O.newton_schulz(m.astype(np.float64), 1, a, b, c, 1e-7)
        assert rel_fro(g, want) <= tol, (m.shape, coef, rel_fro(g, want))


@pytest.mark.parametrize("mode", list(MODES))
@pytest.mark.parametrize("coef", [(0.0, 1.0, 0.0), (0.0, 0.0, 1.0)])
@pytest.mark.parametrize("s,k", [(300, 200), (257, 40), (64, 1000), (520, 520)])
def test_symmetric_gemm_blocks_exactly_symmetric(s, k, coef, mode):
    """X = [M | I] (s x (k + s)): one step with (a, b, c) = (0, 1, 0) returns
    A X, whose last s columns are the stored Gram matrix A = X Xᵀ times the
    stored scale of I (one non-zero product per output element); with
    (0, 0, 1) they are the stored square A·A.  The tensor-core kernel writes
    each off-diagonal 32 x 32 block of these symmetric products once directly
    and once transposed, and completes each diagonal block from its upper
    half, so that block of the output must be exactly symmetric, and each of
    its elements close to the float64 product.  The SIMT kernel (fp32 and
    bf16 storage) runs the upper triangle of its 128 x 128 tiles and mirrors
    each stored element."""
    a, b, c = coef
    cfg = A.Config(gemm_mode=MODES[mode], ns_steps=1, ns_a=a, ns_b=b, ns_c=c)
    X = np.concatenate([gauss((s, k), 31 + s), np.eye(s, dtype=np.float32)], axis=1)
    got = run_polar(cfg, [X])[0][:, k:]
    assert np.array_equal(got, got.T), np.argwhere(got != got.T)[:5]
    want = O.newton_schulz(X.astype(np.float64), 1, a, b, c, 1e-7)[:, k:]
    tol = 1e-5 if mode == "fp32" else 1e-2
    assert np.max(np.abs(got - want)) <= tol * np.max(np.abs(want)), np.max(np.abs(got - want))


@pytest.mark.parametrize("mode", list(MODES))
def test_ns_quintic_five_steps(mode):
    cfg = A.Config(gemm_mode=MODES[mode], ns_steps=5, ns_a=3.4445, ns_b=-4.7750, ns_c=2.0315)
    mats = [gauss((768, 768), 11), gauss((768, 3072), 12), gauss((3072, 768), 13)]
    got = run_polar(cfg, mats)
    for m, g in zip(mats, got):
        want = O.newton_schulz(m.astype(np.float64), 5, 3.4445, -4.7750, 2.0315, 1e-7)
        assert rel_fro(g, want) <= TOL_V[cfg.gemm_mode], (m.shape, rel_fro(g, want))


# ------------------------------------------------------------------ Aurora
@pytest.mark.parametrize("mode", list(MODES))
def test_aurora_polar_matches_oracle(mode):
    cfg = A.Config(gemm_mode=MODES[mode])
    shapes = [(256, 128), (128, 256), (96, 96), (130, 520), (520, 130), (33, 7)]
    mats = [gauss(s, 200 + i) * np.exp(np.random.default_rng(300 + i).standard_normal((s[0], 1))).astype(np.float32)
            for i, s in enumerate(shapes)]
    got = run_polar(cfg, mats, aurora=True)
    for m, g in zip(mats, got):
        want = O.aurora_orthogonalize(m.astype(np.float64), 2, 0.5, 1e-7)
        assert rel_fro(g, want) <= TOL_V[cfg.gemm_mode], (m.shape, rel_fro(g, want))


@pytest.mark.parametrize("pp", [1, 3])
@pytest.mark.parametrize("mode", ["fp32", "bf16"])
def test_aurora_pp_iterations(pp, mode):
    """pp polars per matrix.  In the tensor-core mode each D update reads the
    column sums of U^2 that the last update GEMM of the previous polar wrote
    per 32-row block; the shapes leave partial row blocks (80, 130 and 33
    rows in the X orientation) and rows that are not whole 32-column chunks
    (200, 520)."""
    cfg = A.Config(gemm_mode=MODES[mode], pp_iterations=pp, pp_beta=0.5)
    mats = [gauss((200, 80), 21), gauss((80, 200), 22), gauss((130, 520), 23), gauss((2000, 33), 24)]
    got = run_polar(cfg, mats, aurora=True)
    for m, g in zip(mats, got):
        want = O.aurora_orthogonalize(m.astype(np.float64), pp, 0.5, 1e-7)
        assert rel_fro(g, want) <= TOL_V[cfg.gemm_mode], (m.shape, rel_fro(g, want))


# ------------------------------------------------------------------ operator norm
@pytest.mark.parametrize("mode", ["fp32", "bf16"])
def test_opnorm_normalize_matches_oracle(mode):
    cfg = A.Config(gemm_mode=MODES[mode])
    shapes = [(256, 128), (100, 300), (64, 64), (1, 9), (9, 1), (517, 33)]
    mats = [gauss(s, 400 + i) for i, s in enumerate(shapes)]
    ins = [torch.from_numpy(m).cuda() for m in mats]
    outs = [torch.empty(m.shape, dtype=torch.float32, device="cuda") for m in mats]
    sig = torch.zeros(len(mats), dtype=torch.float32, device="cuda")
    ws = A.make_workspace(cfg, shapes)
    A.opnorm_normalize(cfg, ins, outs, sig, ws)
    torch.cuda.synchronize()
    tol = 1e-5 if mode == "fp32" else 1e-2
    for i, m in enumerate(mats):
        N, s = O.scale_to_unit_operator_norm(m.astype(np.float64), 5)
        assert abs(sig[i].item() - s) <= tol * s, (m.shape, sig[i].item(), s)
        assert rel_fro(f64(outs[i]), N) <= tol


@pytest.mark.parametrize("mode", ["fp32", "bf16"])
def test_opnorm_fused_pass_team_widths_items_and_fallback(mode):
    """The power iteration reads each row of the s x l orientation once per
    iteration when l (padded to 8) is at most 12288 (bf16 staging) or 8192
    (fp32), with 1 to 16 warps per row; longer rows take the two-pass path.
    Shapes cover every team width, rows split over several items, ragged l,
    both orientations, and the first length past each limit."""
    cfg = A.Config(gemm_mode=MODES[mode])
    shapes = [(300, 1000), (5, 2040), (4000, 7), (2000, 300), (3, 8190), (8192, 2), (8200, 2), (2, 8201)]
    if mode == "bf16":
        shapes += [(2, 12288), (12290, 3)]
    mats = [gauss(s, 700 + i) for i, s in enumerate(shapes)]
    ins = [torch.from_numpy(m).cuda() for m in mats]
    outs = [torch.empty(m.shape, dtype=torch.float32, device="cuda") for m in mats]
    sig = torch.zeros(len(mats), dtype=torch.float32, device="cuda")
    A.opnorm_normalize(cfg, ins, outs, sig, A.make_workspace(cfg, shapes))
    torch.cuda.synchronize()
    assert A.last_device_status() == A.MUON_OK
    tol = 1e-5 if mode == "fp32" else 1e-2
    for i, m in enumerate(mats):
        N, s = O.scale_to_unit_operator_norm(m.astype(np.float64), 5)
        assert abs(sig[i].item() - s) <= tol * s, (m.shape, sig[i].item(), s)
        assert rel_fro(f64(outs[i]), N) <= tol, m.shape


def test_opnorm_bf16_inputs_match_oracle_closely():
    """With bf16 inputs the staged matrix is exact and the fused pass runs in
    fp32, so sigma and the normalised matrix match the oracle on the same
    values to about 1e-5 (the fp32-input bf16-mode test above allows 1e-2 for
    the staging rounding).  Shapes cover team widths 1 to 16 warps per row,
    several items, odd row counts and both orientations."""
    cfg = A.Config(gemm_mode=A.MUON_GEMM_BF16)
    shapes = [(256, 768), (1536, 200), (100, 3072), (6144, 64), (37, 12288), (1664, 300), (33, 2048),
              (2048, 4096), (100, 1000)]
    mats = [gauss(s, 900 + i) for i, s in enumerate(shapes)]
    ins = [torch.from_numpy(m).cuda().to(torch.bfloat16) for m in mats]
    vals = [f64(t) for t in ins]
    outs = [torch.empty(m.shape, dtype=torch.float32, device="cuda") for m in mats]
    sig = torch.zeros(len(mats), dtype=torch.float32, device="cuda")
    A.opnorm_normalize(cfg, ins, outs, sig, A.make_workspace(cfg, shapes))
    torch.cuda.synchronize()
    assert A.last_device_status() == A.MUON_OK
    for i, x in enumerate(vals):
        N, s_or = O.scale_to_unit_operator_norm(x, 5)
        assert abs(sig[i].item() - s_or) <= 5e-5 * s_or, (shapes[i], sig[i].item(), s_or)
        assert rel_fro(f64(outs[i]), N) <= 5e-5, shapes[i]


# ------------------------------------------------------------------ u/w floor
def test_uw_floor_apply_matches_oracle():
    shapes = [(64, 32), (100, 300), (7, 9)]
    Ws = [gauss(s, 500 + i) for i, s in enumerate(shapes)]
    Vs = [gauss(s, 600 + i, 1e-2 if i != 1 else 10.0) for i, s in enumerate(shapes)]   # [1]: floor inactive
    cfg = A.Config(param_dtype=A.MUON_F32, target_uw=0.35)
    p = [torch.from_numpy(w).cuda() for w in Ws]
    u = [torch.from_numpy(v).cuda() for v in Vs]
    ws = A.make_workspace(cfg, shapes)
    A.uw_floor_apply(cfg, p, u, ws)
    torch.cuda.synchronize()
    for w, v, g in zip(Ws, Vs, u):
        want = O.uw_floor(v.astype(np.float64), w.astype(np.float64), 0.35)
        assert rel_fro(f64(g), want) <= 1e-6


# ------------------------------------------------------------------ full step
def run_steps(wl, gemm_mode, indices=None, steps=None, want_v=True, w_scale=1.0):
    """Run `steps` optimizer steps on the GPU and on the oracle; compare each step."""
    idx = list(range(wl.n)) if indices is None else list(indices)
    steps = wl.steps if steps is None else steps
    Ws, Gs, Ms = WL.generate(wl, idx)
    if w_scale != 1.0:
        Ws = [WL.store(WL.to_f64(w, wl.param_dtype).astype(np.float32) * np.float32(w_scale), wl.param_dtype)
              for w in Ws]
    cfg = A.Config.from_step_config(wl.cfg, gemm_mode=gemm_mode,
                                    param_dtype=1 if wl.param_dtype == WL.BF16 else 0,
                                    grad_dtype=1 if wl.grad_dtype == WL.BF16 else 0)
    shapes = [wl.shapes[i] for i in idx]
    p = [to_dev(w, wl.param_dtype) for w in Ws]
    m = [torch.from_numpy(x).cuda() for x in Ms]
    v = [torch.empty(s, dtype=torch.float32, device="cuda") for s in shapes] if want_v else None
    ws = A.make_workspace(cfg, shapes)
    oW = [WL.to_f64(w, wl.param_dtype) for w in Ws]
    oM = [x.astype(np.float64) for x in Ms]
    tol = TOL_V[gemm_mode]
    worst = {"V": 0.0, "M": 0.0}
    for st in range(steps):
        G = WL.grads(wl, st, idx) if st > 0 else Gs
        g = [to_dev(x, wl.grad_dtype) for x in G]
        W_before = [f64(t) for t in p]
        A.muon_step(cfg, p, g, m, v, ws)
        torch.cuda.synchronize()
        assert A.last_device_status() == A.MUON_OK
        for k in range(len(idx)):
            gk = WL.to_f64(G[k], wl.grad_dtype)
            W_new, M_new, V = O.step(oW[k], gk, oM[k], wl.cfg, wl.param_dtype)
            em = rel_fro(f64(m[k]), M_new)
            assert em <= TOL_M, ("momentum", st, shapes[k], em)
            if want_v:
                ev = rel_fro(f64(v[k]), V)
                assert ev <= tol, ("V", st, shapes[k], ev)
                worst["V"] = max(worst["V"], ev)
            worst["M"] = max(worst["M"], em)
            dW_gpu = f64(p[k]) - W_before[k]
            dW_or = -wl.cfg.lr * V
            budget = tol * np.linalg.norm(dW_or)
            budget += np.linalg.norm(bf16_half_ulp(W_new)) * 1.01 if wl.param_dtype == WL.BF16 \
                else 1e-6 * np.linalg.norm(W_new)
            err = np.linalg.norm(dW_gpu - dW_or)
            assert err <= budget, ("W", st, shapes[k], err, budget)
            # continue both trajectories from their own state
            oW[k], oM[k] = W_new, M_new
    return worst


@pytest.mark.parametrize("mode", list(MODES))
def test_step_single_fp32_256x128(mode):
    wl = WL.single_aurora_256x128()
    run_steps(wl, MODES[mode])


@pytest.mark.parametrize("mode", ["bf16", "fp32"])
def test_step_floor_active(mode):
    wl = WL.single_aurora_256x128()
    run_steps(wl, MODES[mode], w_scale=100.0)


@pytest.mark.parametrize("mode", list(MODES))
def test_step_mixed_ragged_shapes(mode):
    shapes = [(96, 40), (40, 96), (65, 65), (129, 257), (300, 7), (1, 17), (513, 130)]
    wl = WL.custom("ragged_mix", 9, shapes, WL.aurora_stack(), WL.BF16, WL.BF16, w_std=0.05, steps=2)
    run_steps(wl, MODES[mode])


@pytest.mark.parametrize("mode", ["bf16", "fp32"])
def test_step_plain_muon_no_nesterov(mode):
    shapes = [(200, 100), (100, 200), (150, 150)]
    wl = WL.custom("plain_no_nesterov", 5, shapes, WL.plain_muon(nesterov=False, lr=0.02, mu=0.9), WL.F32, WL.F32,
                   steps=3)
    run_steps(wl, MODES[mode])


@pytest.mark.parametrize("mode", ["bf16", "fp32"])
def test_step_gpt2_layer0_five_steps(mode):
    """GPT-2 124M set, plain Muon, mu 0.90, lr 0.04, bf16 params/grads: first layer's 6 matrices, 5 steps."""
    wl = WL.gpt2_124m_plain()
    run_steps(wl, MODES[mode], indices=range(6))


@pytest.mark.parametrize("mode", ["bf16", "fp32"])
def test_step_aurora_sweep_one_per_shape(mode):
    """Aurora sweep shapes (1024x4096, 4096x1024, 2048^2, 768x3072), full stack, fp32, one of each."""
    wl = WL.aurora_shape_sweep()
    run_steps(wl, MODES[mode], indices=[0, 32, 64, 96])


def test_step_is_deterministic():
    shapes = [(300, 700), (700, 300), (256, 256)]
    wl = WL.custom("det", 3, shapes, WL.aurora_stack(), WL.BF16, WL.BF16, w_std=0.05)
    Ws, Gs, Ms = WL.generate(wl)
    cfg = A.Config()
    outs = []
    for _ in range(2):
        p = [to_dev(w, WL.BF16) for w in Ws]
        g = [to_dev(x, WL.BF16) for x in Gs]
        m = [torch.from_numpy(x).cuda() for x in Ms]
        ws = A.make_workspace(cfg, shapes)
        A.muon_step(cfg, p, g, m, None, ws)
        torch.cuda.synchronize()
        outs.append([t.view(torch.int16).cpu().numpy().copy() for t in p])
    for a, b in zip(*outs):
        assert np.array_equal(a, b)


def test_grads_not_mutated():
    shapes = [(128, 64)]
    wl = WL.custom("g", 4, shapes, WL.aurora_stack(), WL.BF16, WL.BF16)
    Ws, Gs, Ms = WL.generate(wl)
    cfg = A.Config()
    p = [to_dev(Ws[0], WL.BF16)]
    g = [to_dev(Gs[0], WL.BF16)]
    g0 = g[0].clone()
    m = [torch.from_numpy(Ms[0]).cuda()]
    A.muon_step(cfg, p, g, m, None, A.make_workspace(cfg, shapes))
    torch.cuda.synchronize()
    assert torch.equal(g[0], g0)


@pytest.mark.parametrize("mode", ["bf16", "fp32"])
def test_step_more_shape_buckets_than_one_gemm_launch_holds(mode):
    """20 distinct shapes: more buckets than one grouped GEMM launch carries,
    so every Newton-Schulz GEMM is split over several launches."""
    shapes = [(16 + 8 * i, 24 + 4 * i) if i % 2 else (40 + 4 * i, 16 + 8 * i) for i in range(20)]
    wl = WL.custom("many_buckets", 11, shapes, WL.aurora_stack(), WL.BF16, WL.BF16, w_std=0.05)
    run_steps(wl, MODES[mode])
