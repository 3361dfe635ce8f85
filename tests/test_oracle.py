"""Pins of the float64 oracle against facts fixed outside it.

Each pin is chosen so that a plausible slip in the oracle fails it: a wrong
coefficient, sign or transpose in Newton-Schulz (spectral closed form), a
wrong D init or D update direction in Aurora (scale invariance, fixed point,
the pages' 2% claim), a wrong power-iteration side (spectral closed form),
a dropped restore or aspect factor (closed forms), a wrong floor branch.
"""
import json
import math
import os

import numpy as np
import pytest

import oracle.muon_oracle as O
import workloads as WL

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _orth(rng, n, k):
    q, r = np.linalg.qr(rng.standard_normal((n, k)))
    return q * np.sign(np.diag(r))


def _with_spectrum(rng, m, n, sig):
    k = min(m, n)
    Ql = _orth(rng, m, k)
    Qr = _orth(rng, n, k)
    return Ql @ np.diag(sig) @ Qr.T, Ql, Qr


def _poly_iter(x, steps, a, b, c):
    for _ in range(steps):
        x = a * x + b * x ** 3 + c * x ** 5
    return x


# --------------------------------------------------------------- Newton-Schulz
@pytest.mark.parametrize("shape", [(8, 4), (16, 16), (4, 12), (64, 32), (5, 9)])
def test_ns_matches_svd_polar_when_well_conditioned(shape):
    rng = np.random.default_rng(10)
    m, n = shape
    k = min(m, n)
    sig = np.linspace(1.0, 10.0, k)                   # condition number 10
    G, Ql, Qr = _with_spectrum(rng, m, n, sig)
    U = O.newton_schulz(G, 12, 2.0, -1.5, 0.5, 1e-7)
    polar = Ql @ Qr.T
    assert np.linalg.norm(U - polar) / np.linalg.norm(polar) <= 1e-3
    # 12 steps of the (2,-1.5,0.5) map converge far below the 1e-3 bound
    assert np.linalg.norm(U - polar) / np.linalg.norm(polar) <= 1e-9


@pytest.mark.parametrize("shape,coef,steps", [
    ((6, 10), (2.0, -1.5, 0.5), 12),
    ((10, 6), (2.0, -1.5, 0.5), 3),
    ((7, 7), (3.4445, -4.7750, 2.0315), 5),
    ((12, 5), (3.4445, -4.7750, 2.0315), 5),
    ((5, 12), (0.0, 1.0, 0.0), 1),
    ((5, 12), (1.0, 0.0, 0.0), 2),
    ((5, 12), (0.0, 0.0, 1.0), 1),
])
def test_ns_acts_on_singular_values_by_the_polynomial(shape, coef, steps):
    """NS(Q diag(s) P^T) = Q diag(p^k(s / (|s| + eps))) P^T for any spectrum."""
    rng = np.random.default_rng(11)
    m, n = shape
    k = min(m, n)
    sig = np.exp(rng.uniform(-6, 1, k))               # includes far-from-converged values
    G, Ql, Qr = _with_spectrum(rng, m, n, sig)
    a, b, c = coef
    eps = 1e-7
    x = _poly_iter(sig / (np.sqrt(np.sum(sig ** 2)) + eps), steps, a, b, c)
    want = Ql @ np.diag(x) @ Qr.T
    got = O.newton_schulz(G, steps, a, b, c, eps)
    assert got.shape == G.shape
    assert np.allclose(got, want, rtol=1e-10, atol=1e-12 * np.abs(want).max())


def test_ns_polynomial_fixed_point_properties():
    g = json.load(open(os.path.join(GOLD, "page_constants.json")))
    a, b, c = g["ns_a"]["value"], g["ns_b"]["value"], g["ns_c"]["value"]
    p = lambda x: a * x + b * x ** 3 + c * x ** 5
    assert p(1.0) == pytest.approx(1.0, abs=1e-15)                 # fixed point
    assert a + 3 * b + 5 * c == pytest.approx(0.0, abs=1e-15)      # p'(1) = 0
    xs = np.linspace(0, 1, 100001)
    assert p(xs).max() < 1.0025                                     # no blow-up on [0,1]
    qa, qb, qc = g["quintic_a"]["value"], g["quintic_b"]["value"], g["quintic_c"]["value"]
    assert qa + qb + qc == pytest.approx(0.701, abs=1e-12)         # quintic is not a polar


def test_ns_scale_invariant_and_zero_safe():
    rng = np.random.default_rng(12)
    G = rng.standard_normal((9, 20))
    U1 = O.newton_schulz(G)
    U2 = O.newton_schulz(1e3 * G)
    assert np.allclose(U1, U2, rtol=1e-6, atol=1e-9)
    Z = O.newton_schulz(np.zeros((4, 6)))
    assert np.all(Z == 0.0)


# --------------------------------------------------------------- Aurora
def test_aurora_square_is_plain_polar():
    rng = np.random.default_rng(13)
    G = rng.standard_normal((24, 24))
    assert np.array_equal(O.aurora_orthogonalize(G, 2, 0.5), O.newton_schulz(G))


def test_aurora_pp1_is_row_normalised_polar():
    """'pp_iterations=1 degenerates to the Muon-EQ baseline' (row L2 normalise, then polar)."""
    rng = np.random.default_rng(14)
    G = rng.standard_normal((40, 16))
    rn = G / np.linalg.norm(G, axis=1, keepdims=True)
    assert np.allclose(O.aurora_orthogonalize(G, 1, 0.5), O.newton_schulz(rn), atol=1e-12)
    Gw = rng.standard_normal((16, 40))
    cn = Gw / np.linalg.norm(Gw, axis=0, keepdims=True)
    assert np.allclose(O.aurora_orthogonalize(Gw, 1, 0.5), O.newton_schulz(cn), atol=1e-12)


def test_aurora_wide_is_transposed_tall():
    rng = np.random.default_rng(15)
    G = rng.standard_normal((48, 20))
    assert np.allclose(O.aurora_orthogonalize(G.T, 2, 0.5), O.aurora_orthogonalize(G, 2, 0.5).T,
                       atol=1e-13)


@pytest.mark.parametrize("pp", [1, 2, 3])
def test_aurora_invariant_to_row_scaling_on_tall(pp):
    rng = np.random.default_rng(16)
    G = rng.standard_normal((64, 24))
    r = np.exp(rng.standard_normal(64))
    a = O.aurora_orthogonalize(G, pp, 0.5)
    b = O.aurora_orthogonalize(r[:, None] * G, pp, 0.5)
    assert np.allclose(a, b, atol=1e-9)
    # plain polar is NOT invariant: the test would catch a dropped D
    assert np.linalg.norm(O.newton_schulz(G) - O.newton_schulz(r[:, None] * G)) > 1e-2


def test_aurora_row_norms_within_two_percent_rms():
    """The pages: with pp_iterations=2, pp_beta=0.5 the polar's row norms end within 2% of uniform.

    Read as the RMS relative deviation of the row norms from sqrt(min/max)."""
    g = json.load(open(os.path.join(GOLD, "page_constants.json")))
    rng = np.random.default_rng(0)
    G = rng.standard_normal((256, 128))
    U = O.aurora_orthogonalize(G, 2, 0.5)
    target = math.sqrt(128 / 256)
    dev = np.linalg.norm(U, axis=1) / target - 1.0
    assert np.sqrt(np.mean(dev ** 2)) <= g["row_norm_claim"]["value"]
    # and the equilibration is doing work: one polar alone is far from uniform
    dev1 = np.linalg.norm(O.newton_schulz(G), axis=1) / target - 1.0
    assert np.sqrt(np.mean(dev1 ** 2)) > 2 * np.sqrt(np.mean(dev ** 2))


def test_aurora_fixed_point_reached_with_many_iterations():
    """D <- D (target/row_sq)^beta drives the row norms to sqrt(n/m) (sign of the update)."""
    rng = np.random.default_rng(17)
    G = rng.standard_normal((60, 20)) * np.exp(rng.standard_normal(60))[:, None]
    U = O.aurora_orthogonalize(G, 40, 0.5)
    rn = np.linalg.norm(U, axis=1)
    assert np.max(np.abs(rn / math.sqrt(20 / 60) - 1.0)) < 1e-4
    assert np.allclose(U.T @ U, np.eye(20), atol=1e-6)   # still a polar factor


# --------------------------------------------------------------- power iteration
@pytest.mark.parametrize("shape,iters", [((30, 12), 5), ((12, 30), 5), ((20, 20), 1), ((50, 7), 9)])
def test_operator_norm_estimate_spectral_closed_form(shape, iters):
    rng = np.random.default_rng(18)
    m, n = shape
    k = min(m, n)
    s = np.sort(np.exp(rng.uniform(-1, 1, k)))[::-1]
    A, Ql, Qr = _with_spectrum(rng, m, n, s)
    c = Qr.T @ np.full(n, 1.0 / math.sqrt(n))          # start vector in the right singular basis
    wts = s ** (2 * iters) * c
    want = np.linalg.norm(s * wts) / np.linalg.norm(wts)
    got = O.operator_norm_estimate(A, iters)
    assert got == pytest.approx(want, rel=1e-10)
    assert got <= s[0] * (1 + 1e-12)


def test_operator_norm_estimate_converges_to_sigma_max():
    rng = np.random.default_rng(19)
    A = rng.standard_normal((40, 25))
    smax = np.linalg.svd(A, compute_uv=False)[0]
    assert O.operator_norm_estimate(A, 400) == pytest.approx(smax, rel=1e-8)
    assert O.operator_norm_estimate(A, 5) <= smax
    # rank one: exact after one iteration
    x, y = rng.standard_normal(9), rng.standard_normal(5)
    R = 3.0 * np.outer(x, y)
    assert O.operator_norm_estimate(R, 1) == pytest.approx(3.0 * np.linalg.norm(x) * np.linalg.norm(y),
                                                          rel=1e-12)


def test_unit_operator_norm_zero_input():
    N, s = O.scale_to_unit_operator_norm(np.zeros((5, 3)), 5)
    assert s == 0.0 and np.all(N == 0.0)


# --------------------------------------------------------------- contra / aspect / floor
def test_contra_restore_closed_form():
    U = np.eye(3)
    N = np.diag([1.0, 0.0, 0.0])
    V = O.contra_restore(U, N, 0.4)
    want = np.diag([0.8, 1.0, 1.0]) * math.sqrt(3.0) / math.sqrt(0.64 + 2.0)
    assert np.allclose(V, want, atol=1e-15)


def test_contra_restore_preserves_frobenius():
    rng = np.random.default_rng(20)
    U = rng.standard_normal((13, 7))
    N = rng.standard_normal((13, 7))
    for C in (0.0, 0.4, 1.5):
        assert np.linalg.norm(O.contra_restore(U, N, C)) == pytest.approx(np.linalg.norm(U), rel=1e-13)


def test_aspect_scale():
    V = np.ones((4, 2))
    assert np.allclose(O.aspect_scale(V, 4, 2), math.sqrt(2.0))
    assert np.allclose(O.aspect_scale(np.ones((2, 4)), 2, 4), 1.0)
    assert np.allclose(O.aspect_scale(np.ones((3, 3)), 3, 3), 1.0)


def test_uw_floor_active_and_inactive():
    rng = np.random.default_rng(21)
    W = rng.standard_normal((10, 6))
    V = 1e-3 * rng.standard_normal((10, 6))
    out = O.uw_floor(V, W, 0.35)
    assert np.linalg.norm(out) / np.linalg.norm(W) == pytest.approx(0.35, rel=1e-13)
    assert np.allclose(out / np.linalg.norm(out), V / np.linalg.norm(V))     # direction kept
    big = 10 * rng.standard_normal((10, 6))
    assert np.array_equal(O.uw_floor(big, W, 0.35), big)
    assert np.array_equal(O.uw_floor(V, W, 0.0), V)                          # disabled


# --------------------------------------------------------------- momentum
def test_momentum_closed_form_constant_grad():
    rng = np.random.default_rng(22)
    g = rng.standard_normal((5, 4))
    m = np.zeros_like(g)
    mu = 0.9
    for k in range(1, 8):
        u, m = O.momentum_nesterov(g, m, mu, True)
        assert np.allclose(m, (1 - mu ** k) * g, atol=1e-14)
        assert np.allclose(u, (1 - mu ** (k + 1)) * g, atol=1e-14)
    u2, m2 = O.momentum_nesterov(g, np.zeros_like(g), mu, False)
    assert np.allclose(u2, (1 - mu) * g) and np.array_equal(u2, m2)


def test_momentum_warmup_values():
    g = json.load(open(os.path.join(GOLD, "page_constants.json")))
    assert O.momentum_warmup(0) == pytest.approx(g["warmup_mu0"]["value"])
    assert O.momentum_warmup(250) == pytest.approx(0.90)
    assert O.momentum_warmup(10 ** 4) == pytest.approx(g["warmup_mu1"]["value"])


# --------------------------------------------------------------- storage rounding
def test_round_to_bf16_against_torch_and_ties():
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(23)
    x = (rng.standard_normal(20000) * np.exp(rng.uniform(-20, 20, 20000))).astype(np.float32)
    want = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(O.round_to_bf16(x.astype(np.float64)), want)
    one = 1.0
    assert O.round_to_bf16(np.array([one + 2.0 ** -8]))[0] == 1.0              # tie -> even
    assert O.round_to_bf16(np.array([one + 3 * 2.0 ** -8]))[0] == 1.0 + 2.0 ** -6
    assert O.round_to_bf16(np.array([one + 2.0 ** -8 + 2.0 ** -30]))[0] == 1.0 + 2.0 ** -7


def test_input_casts_roundtrip():
    rng = np.random.default_rng(24)
    x = rng.standard_normal(1000).astype(np.float32)
    b = WL.f32_to_bf16_bits(x)
    assert np.array_equal(WL.to_f64(b, "bf16"), O.round_to_bf16(x.astype(np.float64)))


# --------------------------------------------------------------- whole step
def test_plain_muon_step_converged_closed_form():
    """Plain Muon, converged polar: W_new = W - lr sqrt(max(1,m/n)) U V^T."""
    rng = np.random.default_rng(25)
    m, n = 32, 16
    G, Ql, Qr = _with_spectrum(rng, m, n, np.linspace(1, 5, n))
    W = 0.02 * rng.standard_normal((m, n))
    cfg = WL.plain_muon(lr=0.04, mu=0.9)
    W_new, m_new, V = O.step(W, G, np.zeros_like(G), cfg, "f32")
    assert np.allclose(m_new, (0.1 * G).astype(np.float32), atol=0)
    assert np.allclose(V, math.sqrt(2.0) * Ql @ Qr.T, atol=1e-9)
    assert np.allclose(W_new, (W - 0.04 * math.sqrt(2.0) * Ql @ Qr.T).astype(np.float32), atol=1e-7)


def test_full_stack_step_invariants():
    wl = WL.single_aurora_256x128()
    Ws, Gs, Ms = WL.generate(wl)
    W, G, M = (WL.to_f64(Ws[0], "f32"), WL.to_f64(Gs[0], "f32"), Ms[0].astype(np.float64))
    W_new, m_new, V, parts = O.step(W, G, M, wl.cfg, "f32", return_parts=True)
    U = parts["U"]
    # contra keeps |V|_F = |U|_F, then aspect sqrt(2) for 256 x 128
    assert np.linalg.norm(V) == pytest.approx(math.sqrt(2.0) * np.linalg.norm(U), rel=1e-12)
    assert np.linalg.norm(V) / np.linalg.norm(W) >= wl.cfg.target_uw
    assert np.allclose(W_new, (W - wl.cfg.lr * V).astype(np.float32), atol=0)
    assert parts["sigma"] <= np.linalg.svd(parts["u"], compute_uv=False)[0]


def test_floor_triggers_on_heavy_weights():
    wl = WL.single_aurora_256x128()
    Ws, Gs, Ms = WL.generate(wl)
    W = 100.0 * WL.to_f64(Ws[0], "f32")
    G = WL.to_f64(Gs[0], "f32")
    _, _, V = O.step(W, G, np.zeros_like(G), wl.cfg, "f32")
    assert np.linalg.norm(V) / np.linalg.norm(W) == pytest.approx(wl.cfg.target_uw, rel=1e-12)


def _hadamard(n):
    H = np.ones((1, 1))
    while H.shape[0] < n:
        H = np.block([[H, H], [H, -H]])
    return H


def _grad_for_blend(u_star, m0, mu):
    """The gradient whose Nesterov blend with momentum m0 is exactly u_star.

    With m' = m0 + (1 - mu)(g - m0) and u = g + mu (m' - g), u is
    (1 - mu^2) g + mu^2 m0, so g = (u_star - mu^2 m0) / (1 - mu^2)."""
    return (u_star - mu * mu * m0) / (1.0 - mu * mu)


def _power_closed_form(s, Qr, n, iters):
    """sigma-hat of the power iteration from v0 = ones(n)/sqrt(n), by its spectral form."""
    c = Qr.T @ np.full(n, 1.0 / math.sqrt(n))
    wts = s ** (2 * iters) * c
    return np.linalg.norm(s * wts) / np.linalg.norm(wts)


def _contra_closed_form(s, sigma, contra):
    """Singular values of restore(U - contra/2 * u/sigma) when U = Q P^T and u = Q diag(s) P^T."""
    d = 1.0 - 0.5 * contra * s / sigma
    return d * math.sqrt(len(s)) / np.linalg.norm(d)


def test_step_composition_with_momentum_plain_ns_closed_form():
    """Composition of the update ([T3] 组合优化栈 / Contra-Muon) with non-zero
    momentum, so that the Nesterov blend u is not a multiple of g.

    g is chosen so the blend is exactly u* = Q diag(s) P^T (condition 8).  The
    converged polar of u* is Q P^T, sigma-hat has its spectral closed form, so
    V = Q diag(d) P^T * aspect with d from the restore of 1 - (C/2) s / sigma.
    Fails if N is taken from U or from g, if g (not u) goes into the polar, or
    if the aspect factor is applied before the restore."""
    rng = np.random.default_rng(40)
    m, n = 24, 10
    s = np.linspace(1.0, 8.0, n)[rng.permutation(n)]
    u_star, Ql, Qr = _with_spectrum(rng, m, n, s)
    m0 = rng.standard_normal((m, n))
    cfg = WL.plain_muon(contra=0.4, power_iters=5, mu=0.9, ns_steps=12)
    g = _grad_for_blend(u_star, m0, cfg.mu)
    V, m_new, parts = O.muon_update(g, m0, cfg, return_parts=True)
    assert np.allclose(parts["u"], u_star, atol=1e-12)
    assert np.allclose(m_new, m0 + (1.0 - cfg.mu) * (g - m0), atol=1e-12)
    sigma = _power_closed_form(s, Qr, n, cfg.power_iters)
    assert parts["sigma"] == pytest.approx(sigma, rel=1e-10)
    want = math.sqrt(m / n) * Ql @ np.diag(_contra_closed_form(s, sigma, cfg.contra)) @ Qr.T
    assert np.allclose(V, want, atol=1e-8)
    # the blend is far from a multiple of g, so the slips above are visible
    cosine = np.sum(g * u_star) / (np.linalg.norm(g) * np.linalg.norm(u_star))
    assert cosine < 0.9


def test_step_composition_with_momentum_aurora_wide_closed_form():
    """The same composition with Aurora on a wide matrix.

    u* = Q diag(s) P^T with P = columns of a Hadamard matrix / sqrt(n): every
    column of u* has the same norm and every row of P has norm^2 m/n (the
    Aurora target), so D stays constant and Aurora(u*) = Q P^T ([T3] 要点解释:
    row norms already equal are a fixed point).  The all-ones column of H is
    one of P's columns, so the power iteration from ones/sqrt(n) sees only
    its singular value: sigma-hat = s[j0] exactly (not sigma_max).  Aurora of
    g instead of u*, N from U, or N from g all change V."""
    rng = np.random.default_rng(41)
    m, n = 6, 16
    H = _hadamard(n)
    cols = [3, 0, 9, 5, 12, 6]                 # H's all-ones column sits at position 1
    P = H[:, cols] / math.sqrt(n)
    Q = _orth(rng, m, m)
    s = np.array([2.0, 3.0, 5.0, 1.5, 4.0, 2.5])
    u_star = Q @ np.diag(s) @ P.T
    m0 = rng.standard_normal((m, n))
    cfg = WL.aurora_stack(mu=0.95, target_uw=0.0)
    g = _grad_for_blend(u_star, m0, cfg.mu)
    # the construction: equal column norms of u*, and Aurora(u*) is the plain polar
    assert np.allclose(np.linalg.norm(u_star, axis=0), np.linalg.norm(s) / math.sqrt(n), rtol=1e-12)
    V, _, parts = O.muon_update(g, m0, cfg, return_parts=True)
    assert np.allclose(parts["u"], u_star, atol=1e-12)
    assert parts["sigma"] == pytest.approx(s[1], rel=1e-12)
    assert np.allclose(parts["U"], Q @ P.T, atol=1e-8)
    want = Q @ np.diag(_contra_closed_form(s, s[1], cfg.contra)) @ P.T     # wide: aspect 1
    assert np.allclose(V, want, atol=1e-8)
    # Aurora of the raw gradient is a different matrix
    assert np.linalg.norm(O.aurora_orthogonalize(g) - Q @ P.T) > 0.1


@pytest.mark.parametrize("shape", [(256, 128), (96, 160), (64, 64)])
def test_zero_gradient_step_leaves_weights_unchanged(shape):
    """Degenerate input: g = 0 from zero momentum.  Every guard (the NS eps,
    the power-iteration and operator-norm floors, Aurora's pp_eps, the
    restore's 1e-10, the floor's 1e-8) must keep the step finite, so V = 0
    and W is returned as it was (a dropped or misplaced eps gives NaN)."""
    wl = WL.single_aurora_256x128()
    rng = np.random.default_rng(5)
    W = rng.standard_normal(shape) * 0.02
    g = np.zeros(shape)
    W_new, m_new, V = O.step(W, g, np.zeros(shape), wl.cfg, "f32")
    assert np.all(np.isfinite(V)) and np.all(V == 0.0)
    assert np.all(m_new == 0.0)
    assert np.array_equal(W_new, W.astype(np.float32).astype(np.float64))


def test_weight_decay_rejected():
    cfg = WL.aurora_stack(weight_decay=0.1)
    with pytest.raises(ValueError):
        O.step(np.zeros((2, 2)), np.ones((2, 2)), np.zeros((2, 2)), cfg)


def test_workload_constants_match_pages():
    g = json.load(open(os.path.join(GOLD, "page_constants.json")))
    c = WL.aurora_stack()
    for k in ("ns_steps", "ns_a", "ns_b", "ns_c", "ns_eps", "pp_iterations", "pp_beta",
              "pp_eps", "contra", "power_iters", "target_uw", "mu", "weight_decay"):
        assert getattr(c, k) == g[k]["value"], k
    assert c.lr == g["lr_aurora"]["value"]
    assert sum(m * n for m, n in WL.llama_3p8b_shapes()) == 2_818_572_288
    assert len(WL.gpt2_124m_shapes()) == 72


# --------------------------------------------------------------- auxiliary AdamW
def test_adamw_constant_gradient_closed_form():
    """Constant g from zero state: m_hat = g, v_hat = g^2, so each step moves lr g/(|g| + eps)."""
    rng = np.random.default_rng(30)
    g = rng.standard_normal(50) + 0.5
    p0 = rng.standard_normal(50)
    p, m, v = p0.copy(), np.zeros(50), np.zeros(50)
    lr, eps = 0.01, 1e-10
    for t in range(1, 8):
        p, m, v = O.adamw_step(p, g, m, v, lr, 0.8, 0.95, eps, 0.0, t)
        assert np.allclose(m, (1 - 0.8 ** t) * g, rtol=1e-13)
        assert np.allclose(v, (1 - 0.95 ** t) * g * g, rtol=1e-13)
        assert np.allclose(p, p0 - t * lr * g / (np.abs(g) + eps), rtol=1e-12, atol=1e-14)


def test_adamw_matches_torch_adamw_float64():
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(31)
    p0 = rng.standard_normal((7, 5))
    grads = [rng.standard_normal((7, 5)) for _ in range(4)]
    tp = torch.tensor(p0, dtype=torch.float64, requires_grad=True)
    opt = torch.optim.AdamW([tp], lr=0.3, betas=(0.8, 0.95), eps=1e-10, weight_decay=0.05)
    p, m, v = p0.copy(), np.zeros_like(p0), np.zeros_like(p0)
    for t, g in enumerate(grads, start=1):
        tp.grad = torch.tensor(g, dtype=torch.float64)
        opt.step()
        p, m, v = O.adamw_step(p, g, m, v, 0.3, 0.8, 0.95, 1e-10, 0.05, t)
        assert np.allclose(p, tp.detach().numpy(), rtol=1e-12, atol=1e-14)
