"""Pins of the fp64 CPU oracle to facts outside itself (no GPU needed).

Method: "MesaNet: Sequence Modeling by Locally Optimal Test-Time Training"
(gist.science, ja/ko/hi editions), Technical summary > Method > Mesa layer
(objective, CG solve of (H_t + Lambda)^-1 q_t, chunkwise parallelisation,
dynamic compute).

Each test checks the oracle against something it does not compute itself:
  * the objective of the Mesa layer minimised numerically (brute force);
  * the Galerkin characterisation of CG (x_k minimises the A-norm error over
    the Krylov space K_k(A, q)), built with an independent Arnoldi basis;
  * closed forms: finite termination (k = n gives the exact solve), one CG
    step, Sherman-Morrison for a rank-1 statistic, the gamma = beta = 1 sums,
    the large-Lambda (linear-attention) limit;
  * invariants: chunked = per-token for any chunk size, scale invariance of
    (beta, Lambda), linearity in v, causality, permutation of sequences,
    decode steps = forward, prefix state + suffix = whole.
"""
import numpy as np
import pytest
import scipy.optimize

import mesa_inputs as mi


def rand_inputs(rng, B, H, T, dk, dv, gamma_shift=3.0):
    q = rng.standard_normal((B, H, T, dk))
    q /= np.linalg.norm(q, axis=-1, keepdims=True)
    k = rng.standard_normal((B, H, T, dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((B, H, T, dv))
    gamma = 1.0 / (1.0 + np.exp(-(rng.standard_normal((B, H, T)) + gamma_shift)))
    beta = 1.0 / (1.0 + np.exp(-rng.standard_normal((B, H, T))))
    lam = np.log1p(np.exp(rng.standard_normal((H, dk)))) + 0.1
    return q, k, v, gamma, beta, lam


def spd(rng, n, lo=0.5, hi=5.0):
    Q, _ = np.linalg.qr(rng.standard_normal((n, n)))
    return Q @ np.diag(rng.uniform(lo, hi, n)) @ Q.T


def krylov_solution(A, b, kdim):
    """Galerkin solution on K_k(A, b) from an Arnoldi basis (twice-orthogonalised)."""
    n = b.shape[0]
    V = np.zeros((n, kdim))
    V[:, 0] = b / np.linalg.norm(b)
    for j in range(1, kdim):
        w = A @ V[:, j - 1]
        for _ in range(2):
            w -= V[:, :j] @ (V[:, :j].T @ w)
        V[:, j] = w / np.linalg.norm(w)
    Tm = V.T @ A @ V
    return V @ np.linalg.solve(Tm, V.T @ b)


def zeta_matrix(gamma, beta, t):
    """zeta_{t t'} for t' <= t from explicit products (no recurrence)."""
    z = np.zeros(t + 1)
    for tp in range(t + 1):
        z[tp] = beta[tp] * np.prod(gamma[tp + 1:t + 1])
    return z


def explicit_stats(k, v, gamma, beta, t):
    z = zeta_matrix(gamma, beta, t)
    Hm = sum(z[tp] * np.outer(k[tp], k[tp]) for tp in range(t + 1))
    Gm = sum(z[tp] * np.outer(v[tp], k[tp]) for tp in range(t + 1))
    return Hm, Gm


# --------------------------------------------------------------------------
# CG rule on dense systems
# --------------------------------------------------------------------------

@pytest.mark.parametrize("n", [4, 9, 16])
def test_cg_iterates_equal_krylov_galerkin(oracle_mod, n):
    rng = np.random.default_rng(n)
    A = spd(rng, n)
    b = rng.standard_normal(n)
    for kdim in range(1, n + 1):
        x, it = oracle_mod.cg_dense(A, b, kdim)
        assert it == kdim
        ref = krylov_solution(A, b, kdim)
        assert np.allclose(x, ref, rtol=1e-9, atol=1e-11), (kdim, np.abs(x - ref).max())


def test_cg_finite_termination_is_exact_solve(oracle_mod):
    rng = np.random.default_rng(1)
    for n in (3, 8, 16, 32):
        A = spd(rng, n)
        b = rng.standard_normal(n)
        x, _ = oracle_mod.cg_dense(A, b, n)
        assert np.allclose(x, np.linalg.solve(A, b), rtol=1e-9, atol=1e-12)


def test_cg_one_step_closed_form(oracle_mod):
    rng = np.random.default_rng(2)
    A = spd(rng, 12)
    b = rng.standard_normal(12)
    x, it = oracle_mod.cg_dense(A, b, 1)
    assert it == 1
    assert np.allclose(x, (b @ b) / (b @ A @ b) * b, rtol=1e-13)


def test_cg_tolerance_stop_is_first_small_true_residual(oracle_mod):
    rng = np.random.default_rng(3)
    A = spd(rng, 24, 0.2, 3.0)
    b = rng.standard_normal(24)
    bn = np.linalg.norm(b)
    for tol in (1e-1, 1e-2, 1e-3, 1e-5):
        x, it = oracle_mod.cg_dense(A, b, 24, tol)
        # first k whose Galerkin iterate has a true residual below tol*|b|
        kstop = next(kk for kk in range(0, 25)
                     if np.linalg.norm(b - A @ (krylov_solution(A, b, kk) if kk else np.zeros(24))) <= tol * bn)
        assert it == kstop, (tol, it, kstop)
        assert np.linalg.norm(b - A @ x) <= tol * bn * (1 + 1e-6)


def test_cg_breakdown_freezes(oracle_mod):
    x, it = oracle_mod.cg_dense(np.eye(5), np.zeros(5), 10)
    assert it == 0 and np.all(x == 0)
    x, it = oracle_mod.cg_dense(-np.eye(5), np.ones(5), 10)    # p.Ap < 0 at once
    assert it == 0 and np.all(x == 0)
    x, it = oracle_mod.cg_dense(np.eye(5), np.ones(5), 10)     # exact after 1 step, then r.r = 0
    assert it == 1 and np.allclose(x, 1.0)


# --------------------------------------------------------------------------
# The layer against its objective (brute force) and closed forms
# --------------------------------------------------------------------------

@pytest.mark.parametrize("dk,dv,T", [(3, 2, 6), (4, 4, 8), (2, 3, 5)])
def test_cholesky_minimises_the_mesa_objective(oracle_mod, dk, dv, T):
    """Phi_t = argmin 1/2 sum zeta |v - Phi k|^2 + 1/2 Tr(Phi Lambda Phi^T); o_t = Phi_t q_t."""
    rng = np.random.default_rng(10 + dk * dv + T)
    q, k, v, g, be, lam = rand_inputs(rng, 1, 1, T, dk, dv, gamma_shift=0.5)
    out, _, _ = oracle_mod.forward_cholesky(q, k, v, g, be, lam)
    L = np.diag(lam[0])
    for t in range(T):
        z = zeta_matrix(g[0, 0], be[0, 0], t)

        def f(phi):
            P = phi.reshape(dv, dk)
            res = v[0, 0, :t + 1] - k[0, 0, :t + 1] @ P.T
            val = 0.5 * np.sum(z[:, None] * res ** 2) + 0.5 * np.trace(P @ L @ P.T)
            grad = -(z[:, None] * res).T @ k[0, 0, :t + 1] + P @ L
            return val, grad.ravel()

        sol = scipy.optimize.minimize(f, np.zeros(dv * dk), jac=True, method="BFGS",
                                      options=dict(gtol=1e-13, maxiter=10000))
        o_bf = sol.x.reshape(dv, dk) @ q[0, 0, t]
        assert np.allclose(out[0, 0, t], o_bf, rtol=1e-6, atol=1e-8), (t, out[0, 0, t], o_bf)


def test_cg_full_steps_equals_cholesky_on_tiny_workload(oracle_mod):
    w = mi.WORKLOADS["tiny_fp32"]
    x = mi.batch(w)
    o_cg, it, Hf, Gf = oracle_mod.forward_cg(x["q"], x["k"], x["v"], x["gamma"], x["beta"], x["lam"], w.cg_steps)
    o_ch, Hc, Gc = oracle_mod.forward_cholesky(x["q"], x["k"], x["v"], x["gamma"], x["beta"], x["lam"])
    assert np.all(it == w.dk)
    assert np.abs(o_cg - o_ch).max() <= 1e-9 * np.abs(o_ch).max()
    assert np.array_equal(Hf, Hc) and np.array_equal(Gf, Gc)


def test_unconverged_cg_equals_galerkin_on_explicit_statistics(oracle_mod):
    """Fixed N < d: the iterate is the Galerkin solution on K_N(H_t + Lambda, q_t),
    with H_t, G_t rebuilt from explicit zeta products."""
    rng = np.random.default_rng(4)
    T, dk, dv, N = 12, 16, 8, 5
    q, k, v, g, be, lam = rand_inputs(rng, 1, 1, T, dk, dv)
    out, it, _, _ = oracle_mod.forward_cg(q, k, v, g, be, lam, N)
    assert np.all(it == N)
    for t in range(T):
        Hm, Gm = explicit_stats(k[0, 0], v[0, 0], g[0, 0], be[0, 0], t)
        xk = krylov_solution(Hm + np.diag(lam[0]), q[0, 0, t], N)
        assert np.allclose(out[0, 0, t], Gm @ xk, rtol=1e-9, atol=1e-12)


def test_gamma_beta_one_gives_plain_sums(oracle_mod):
    rng = np.random.default_rng(5)
    q, k, v, _, _, lam = rand_inputs(rng, 2, 2, 10, 6, 5)
    ones = np.ones((2, 2, 10))
    _, _, Hf, Gf = oracle_mod.forward_cg(q, k, v, ones, ones, lam, 3)
    assert np.allclose(Hf, np.einsum("bhti,bhtj->bhij", k, k), rtol=1e-13, atol=1e-14)
    assert np.allclose(Gf, np.einsum("bhti,bhtj->bhij", v, k), rtol=1e-13, atol=1e-14)


def sherman_morrison_out(q, k, v, beta, lam):
    """o = beta v (k^T L^-1 q) / (1 + beta k^T L^-1 k) for H = beta k k^T, G = beta v k^T."""
    kl = k / lam
    return beta * v * (kl @ q) / (1.0 + beta * (kl @ k))


def test_first_token_and_gamma_zero_match_sherman_morrison(oracle_mod):
    rng = np.random.default_rng(6)
    T, dk, dv = 7, 8, 5
    q, k, v, g, be, lam = rand_inputs(rng, 1, 1, T, dk, dv)
    g0 = np.zeros_like(g)                          # every step resets the state
    for gam in (g, g0):
        o_ch, _, _ = oracle_mod.forward_cholesky(q, k, v, gam, be, lam)
        o_cg, _, _, _ = oracle_mod.forward_cg(q, k, v, gam, be, lam, dk)
        ts = range(T) if gam is g0 else [0]
        for t in ts:
            ref = sherman_morrison_out(q[0, 0, t], k[0, 0, t], v[0, 0, t], be[0, 0, t], lam[0])
            assert np.allclose(o_ch[0, 0, t], ref, rtol=1e-12, atol=1e-15)
            assert np.allclose(o_cg[0, 0, t], ref, rtol=1e-9, atol=1e-12)


def test_one_cg_step_through_the_layer(oracle_mod):
    rng = np.random.default_rng(7)
    T, dk, dv = 9, 6, 4
    q, k, v, g, be, lam = rand_inputs(rng, 1, 1, T, dk, dv)
    out, it, _, _ = oracle_mod.forward_cg(q, k, v, g, be, lam, 1)
    assert np.all(it == 1)
    for t in range(T):
        Hm, Gm = explicit_stats(k[0, 0], v[0, 0], g[0, 0], be[0, 0], t)
        A = Hm + np.diag(lam[0])
        qt = q[0, 0, t]
        assert np.allclose(out[0, 0, t], Gm @ ((qt @ qt) / (qt @ A @ qt) * qt), rtol=1e-12)


def test_large_lambda_gives_linear_attention(oracle_mod):
    """Lambda = c I with c -> inf: c * o_t -> G_t q_t (gated linear attention)."""
    rng = np.random.default_rng(8)
    T, dk, dv = 16, 8, 8
    q, k, v, g, be, _ = rand_inputs(rng, 1, 1, T, dk, dv)
    c = 1e7
    lam = np.full((1, dk), c)
    out, _, _ = oracle_mod.forward_cholesky(q, k, v, g, be, lam)
    for t in range(T):
        _, Gm = explicit_stats(k[0, 0], v[0, 0], g[0, 0], be[0, 0], t)
        assert np.allclose(c * out[0, 0, t], Gm @ q[0, 0, t], rtol=1e-5, atol=1e-7)


# --------------------------------------------------------------------------
# Invariants
# --------------------------------------------------------------------------

@pytest.mark.parametrize("chunk", [1, 2, 3, 4, 8, 16, 37])
@pytest.mark.parametrize("tol", [0.0, 1e-3])
def test_chunked_equals_per_token(oracle_mod, chunk, tol):
    rng = np.random.default_rng(100 + chunk)
    B, H, T, dk, dv = 2, 2, 37, 8, 6
    q, k, v, g, be, lam = rand_inputs(rng, B, H, T, dk, dv, gamma_shift=1.0)
    N = 6 if tol == 0 else 30
    o1, i1, H1, G1 = oracle_mod.forward_cg(q, k, v, g, be, lam, N, tol)
    o2, i2, H2, G2 = oracle_mod.forward_chunked(q, k, v, g, be, lam, chunk, N, tol)
    assert np.allclose(o1, o2, rtol=1e-9, atol=1e-12)
    assert np.array_equal(i1, i2)
    assert np.allclose(H1, H2, rtol=1e-10, atol=1e-13) and np.allclose(G1, G2, rtol=1e-10, atol=1e-13)


def test_beta_lambda_scale_invariance(oracle_mod):
    rng = np.random.default_rng(11)
    q, k, v, g, be, lam = rand_inputs(rng, 1, 2, 20, 8, 8)
    o1, i1, _, _ = oracle_mod.forward_cg(q, k, v, g, be, lam, 5)
    for c in (0.25, 3.0, 1e3):
        o2, i2, _, _ = oracle_mod.forward_cg(q, k, v, g, c * be, c * lam, 5)
        assert np.allclose(o1, o2, rtol=1e-9, atol=1e-13)
        assert np.array_equal(i1, i2)


def test_linear_in_v(oracle_mod):
    rng = np.random.default_rng(12)
    q, k, v, g, be, lam = rand_inputs(rng, 1, 1, 15, 8, 8)
    v2 = rng.standard_normal(v.shape)
    oa, _, _, _ = oracle_mod.forward_cg(q, k, v, g, be, lam, 7)
    ob, _, _, _ = oracle_mod.forward_cg(q, k, v2, g, be, lam, 7)
    oc, _, _, _ = oracle_mod.forward_cg(q, k, v + 2.0 * v2, g, be, lam, 7)
    assert np.allclose(oc, oa + 2.0 * ob, rtol=1e-10, atol=1e-12)


def test_causal(oracle_mod):
    rng = np.random.default_rng(13)
    q, k, v, g, be, lam = rand_inputs(rng, 1, 1, 20, 8, 8)
    o1, _, _, _ = oracle_mod.forward_cg(q, k, v, g, be, lam, 7)
    t0 = 11
    q2, k2, v2, g2, be2 = (a.copy() for a in (q, k, v, g, be))
    for a in (q2, k2, v2):
        a[:, :, t0 + 1:] = rng.standard_normal(a[:, :, t0 + 1:].shape)
    g2[:, :, t0 + 1:] = 0.5
    be2[:, :, t0 + 1:] = 0.9
    o2, _, _, _ = oracle_mod.forward_cg(q2, k2, v2, g2, be2, lam, 7)
    assert np.array_equal(o1[:, :, :t0 + 1], o2[:, :, :t0 + 1])
    assert not np.allclose(o1[:, :, t0 + 1:], o2[:, :, t0 + 1:])


def test_sequence_permutation(oracle_mod):
    rng = np.random.default_rng(14)
    B, H = 3, 2
    q, k, v, g, be, lam = rand_inputs(rng, B, H, 9, 6, 6)
    o1, _, _, _ = oracle_mod.forward_cg(q, k, v, g, be, lam, 4)
    pb, ph = [2, 0, 1], [1, 0]
    perm = lambda a: a[pb][:, ph]
    o2, _, _, _ = oracle_mod.forward_cg(perm(q), perm(k), perm(v), perm(g), perm(be), lam[ph], 4)
    assert np.array_equal(o2, perm(o1))


@pytest.mark.parametrize("tol", [0.0, 1e-3])
def test_decode_steps_equal_forward(oracle_mod, tol):
    rng = np.random.default_rng(15)
    B, H, T, dk, dv = 2, 3, 12, 8, 5
    q, k, v, g, be, lam = rand_inputs(rng, B, H, T, dk, dv)
    o_f, i_f, Hf, Gf = oracle_mod.forward_cg(q, k, v, g, be, lam, 6, tol)
    Hs = np.zeros((B, H, dk, dk))
    Gs = np.zeros((B, H, dv, dk))
    for t in range(T):
        o_s, i_s, Hs, Gs = oracle_mod.step(q[:, :, t], k[:, :, t], v[:, :, t], g[:, :, t], be[:, :, t],
                                           lam, Hs, Gs, 6, tol)
        assert np.array_equal(o_s, o_f[:, :, t]) and np.array_equal(i_s, i_f[:, :, t])
    assert np.array_equal(Hs, Hf) and np.array_equal(Gs, Gf)


def test_prefix_state_then_suffix_equals_whole(oracle_mod):
    rng = np.random.default_rng(16)
    B, H, T, dk, dv, t0 = 1, 2, 30, 8, 8, 17
    q, k, v, g, be, lam = rand_inputs(rng, B, H, T, dk, dv)
    o_all, _, Ha, Ga = oracle_mod.forward_cg(q, k, v, g, be, lam, 6)
    sl1 = lambda a: a[:, :, :t0]
    sl2 = lambda a: a[:, :, t0:]
    _, _, H1, G1 = oracle_mod.forward_cg(*map(sl1, (q, k, v, g, be)), lam, 6)
    o2, _, H2, G2 = oracle_mod.forward_cg(*map(sl2, (q, k, v, g, be)), lam, 6, H0=H1, G0=G1)
    assert np.allclose(o2, o_all[:, :, t0:], rtol=1e-12, atol=1e-14)
    o3, _, _, _ = oracle_mod.forward_chunked(*map(sl2, (q, k, v, g, be)), lam, 5, 6, H0=H1, G0=G1)
    assert np.allclose(o3, o_all[:, :, t0:], rtol=1e-9, atol=1e-12)


def test_empty_sequence(oracle_mod):
    z = np.zeros((1, 1, 0, 4))
    out, it, Hf, Gf = oracle_mod.forward_cg(z, z, z, np.zeros((1, 1, 0)), np.zeros((1, 1, 0)),
                                            np.ones((1, 4)), 3)
    assert out.shape == (1, 1, 0, 4) and np.all(Hf == 0) and np.all(Gf == 0)


# ---------------------------------------------------------------------------
# Input preprocessing (MesaNet page, Architecture, "Preprocessing"): causal
# depthwise convolution over time, then L2 normalisation per token.
# ---------------------------------------------------------------------------

def test_preprocess_matches_numpy_convolution(oracle_mod):
    rng = np.random.default_rng(11)
    B, H, T, d, W = 2, 3, 19, 8, 4
    x = rng.standard_normal((B, H, T, d))
    conv = rng.standard_normal((H, W, d))
    y = oracle_mod.preprocess(x, conv)
    for b in range(B):
        for h in range(H):
            u = np.stack([np.convolve(x[b, h, :, i], conv[h, :, i])[:T] for i in range(d)], axis=1)
            ref = u / np.maximum(np.linalg.norm(u, axis=1, keepdims=True), 1e-6)
            assert np.allclose(y[b, h], ref, rtol=0, atol=1e-13)


def test_preprocess_window_one_is_normalisation(oracle_mod):
    rng = np.random.default_rng(12)
    x = rng.standard_normal((1, 2, 7, 16))
    y = oracle_mod.preprocess(x, np.ones((2, 1, 16)))
    assert np.allclose(np.linalg.norm(y, axis=-1), 1.0, atol=1e-14)
    cos = (y * x).sum(-1) / np.linalg.norm(x, axis=-1)
    assert np.allclose(cos, 1.0, atol=1e-14)


def test_preprocess_delta_filter_shifts(oracle_mod):
    rng = np.random.default_rng(13)
    T, d, s = 9, 8, 2
    x = rng.standard_normal((1, 1, T, d))
    conv = np.zeros((1, 4, d))
    conv[0, s] = 1.0
    y = oracle_mod.preprocess(x, conv)
    assert np.all(y[0, 0, :s] == 0.0)                          # nothing before the sequence start
    ref = x[0, 0, :T - s] / np.linalg.norm(x[0, 0, :T - s], axis=-1, keepdims=True)
    assert np.allclose(y[0, 0, s:], ref, atol=1e-14)


def test_preprocess_causal_and_scale_invariant(oracle_mod):
    rng = np.random.default_rng(14)
    x = rng.standard_normal((1, 2, 12, 8))
    conv = rng.standard_normal((2, 3, 8))
    y = oracle_mod.preprocess(x, conv)
    x2 = x.copy()
    x2[:, :, 7:] = rng.standard_normal(x2[:, :, 7:].shape)     # change the future
    assert np.array_equal(oracle_mod.preprocess(x2, conv)[:, :, :7], y[:, :, :7])
    assert np.allclose(oracle_mod.preprocess(3.5 * x, conv), y, atol=1e-14)
    assert np.allclose(oracle_mod.preprocess(-x, conv), -y, atol=1e-14)


# ---------------------------------------------------------------------------
# Warm-started CG (MesaNet page, Significance and claims: warm starts named as
# the way to cut the solver's cost). CG from x0 on A x = b is, in exact
# arithmetic, x0 plus CG from zero on the residual system A e = b - A x0.
# ---------------------------------------------------------------------------

def _spd(rng, n):
    M = rng.standard_normal((n, n))
    return M @ M.T / n + 0.5 * np.eye(n)


def test_warm_cg_equals_shifted_cold_cg(oracle_mod):
    rng = np.random.default_rng(21)
    n = 12
    A, b, x0 = _spd(rng, n), rng.standard_normal(n), rng.standard_normal(n)
    r0 = b - A @ x0
    for k in range(1, n + 1):
        xw, itw = oracle_mod.cg_dense(A, b, k, 0.0, x0=x0)
        xc, itc = oracle_mod.cg_dense(A, r0, k, 0.0)
        assert itw == itc == k
        assert np.allclose(xw, x0 + xc, rtol=0, atol=1e-10), k


def test_warm_cg_one_step_closed_form(oracle_mod):
    rng = np.random.default_rng(22)
    n = 7
    A, b, x0 = _spd(rng, n), rng.standard_normal(n), rng.standard_normal(n)
    r0 = b - A @ x0
    x1, it = oracle_mod.cg_dense(A, b, 1, 0.0, x0=x0)
    assert it == 1
    assert np.allclose(x1, x0 + (r0 @ r0) / (r0 @ A @ r0) * r0, rtol=0, atol=1e-13)


def test_warm_cg_from_the_solution_stops_at_once(oracle_mod):
    rng = np.random.default_rng(23)
    n = 9
    A, b = _spd(rng, n), rng.standard_normal(n)
    xs = np.linalg.solve(A, b)
    x, it = oracle_mod.cg_dense(A, b, 20, 1e-6, x0=xs)
    assert it == 0 and np.array_equal(x, xs)
    # the stopping test is relative to |b|, not to the first residual
    x, it = oracle_mod.cg_dense(A, b, 20, 1e-3, x0=xs + 1e-6 * rng.standard_normal(n))
    assert it == 0


def test_warm_step_from_zero_is_the_cold_step(oracle_mod):
    w = mi.Workload("t", 2, 3, 6, 8, 8, 2, "f32", 5, 0.0, False, 24)
    x = mi.batch(w)
    rng = np.random.default_rng(24)
    Hs = rng.standard_normal((2, 3, 8, 8)) * 0.1
    Hs = Hs @ np.swapaxes(Hs, -1, -2)
    Gs = rng.standard_normal((2, 3, 8, 8))
    args = (x["q"][:, :, 0], x["k"][:, :, 0], x["v"][:, :, 0], x["gamma"][:, :, 0], x["beta"][:, :, 0], x["lam"],
            Hs, Gs, 5)
    cold = oracle_mod.step(*args)
    warm = oracle_mod.step(*args, x_state=np.zeros((2, 3, 8)))
    for a, b_ in zip(cold, warm[:4]):
        assert np.array_equal(a, b_)
    # the returned x reproduces the output through the updated G
    assert np.allclose(np.einsum("bhij,bhj->bhi", warm[3], warm[4]), warm[0], atol=1e-12)


# Warm-started forward (the same reading applied to every token of a
# sequence): token t's CG starts from a caller-given x0_t.

def _explicit_systems(q, k, v, gamma, beta, lam):
    """(A_t, G_t) for every token from the gated recurrences written out in numpy."""
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    A = np.zeros((B, H, T, dk, dk))
    G = np.zeros((B, H, T, dv, dk))
    for b in range(B):
        for h in range(H):
            Hm = np.zeros((dk, dk))
            Gm = np.zeros((dv, dk))
            for t in range(T):
                Hm = gamma[b, h, t] * Hm + beta[b, h, t] * np.outer(k[b, h, t], k[b, h, t])
                Gm = gamma[b, h, t] * Gm + beta[b, h, t] * np.outer(v[b, h, t], k[b, h, t])
                A[b, h, t] = Hm + np.diag(lam[h])
                G[b, h, t] = Gm
    return A, G


def test_warm_forward_from_zero_is_the_cold_forward(oracle_mod):
    rng = np.random.default_rng(31)
    q, k, v, gamma, beta, lam = rand_inputs(rng, 2, 2, 9, 5, 4)
    cold, it_c, Hc, Gc = oracle_mod.forward_cg(q, k, v, gamma, beta, lam, 3, 1e-2)
    for x0 in (None, np.zeros((2, 2, 9, 5))):
        warm, it_w, x, Hw, Gw = oracle_mod.forward_cg_x0(q, k, v, gamma, beta, lam, 3, 1e-2, x0=x0)
        assert np.array_equal(warm, cold) and np.array_equal(it_w, it_c)
        assert np.array_equal(Hw, Hc) and np.array_equal(Gw, Gc)
        # the returned solutions reproduce the outputs through G_t
        _, G = _explicit_systems(q, k, v, gamma, beta, lam)
        assert np.allclose(np.einsum("bhtij,bhtj->bhti", G, x), warm, rtol=0, atol=1e-12)


def test_warm_forward_is_the_shifted_cold_solve_per_token(oracle_mod):
    """With a fixed step count, CG from x0_t on A_t x = q_t equals x0_t plus
    CG from zero on A_t e = q_t - A_t x0_t, token by token (dk != dv)."""
    rng = np.random.default_rng(32)
    q, k, v, gamma, beta, lam = rand_inputs(rng, 1, 2, 7, 6, 3)
    x0 = rng.standard_normal((1, 2, 7, 6))
    A, G = _explicit_systems(q, k, v, gamma, beta, lam)
    for N in (1, 2, 4):
        out, it, x, _, _ = oracle_mod.forward_cg_x0(q, k, v, gamma, beta, lam, N, 0.0, x0=x0)
        assert np.all(it == N)
        for h in range(2):
            for t in range(7):
                At = A[0, h, t]
                e, _ = oracle_mod.cg_dense(At, q[0, h, t] - At @ x0[0, h, t], N, 0.0)
                assert np.allclose(x[0, h, t], x0[0, h, t] + e, rtol=0, atol=1e-10), (N, h, t)
                assert np.allclose(out[0, h, t], G[0, h, t] @ x[0, h, t], rtol=0, atol=1e-10)


def test_warm_forward_from_the_exact_solutions(oracle_mod):
    """x0_t = A_t^-1 q_t: no token takes a step under a tolerance, and the
    outputs equal the exact (Cholesky) layer."""
    rng = np.random.default_rng(33)
    q, k, v, gamma, beta, lam = rand_inputs(rng, 2, 1, 8, 5, 5)
    A, _ = _explicit_systems(q, k, v, gamma, beta, lam)
    xs = np.linalg.solve(A, q[..., None])[..., 0]
    out, it, x, _, _ = oracle_mod.forward_cg_x0(q, k, v, gamma, beta, lam, 10, 1e-8, x0=xs)
    assert np.all(it == 0) and np.array_equal(x, xs)
    exact, _, _ = oracle_mod.forward_cholesky(q, k, v, gamma, beta, lam)
    assert np.allclose(out, exact, rtol=0, atol=1e-12)


# --------------------------------------------------------------------------
# Backward pass (implicit differentiation with an adjoint CG solve)
# --------------------------------------------------------------------------

def _bwd_inputs(seed, B=2, H=2, T=4, d=3):
    rng = np.random.default_rng(seed)
    q, k, v, _, _, _ = rand_inputs(rng, B, H, T, d, d)
    gamma = rng.uniform(0.5, 1.0, (B, H, T))
    beta = rng.uniform(0.2, 1.0, (B, H, T))
    lam = rng.uniform(0.3, 1.3, (H, d))
    dout = rng.standard_normal((B, H, T, d))
    return {"q": q, "k": k, "v": v, "gamma": gamma, "beta": beta, "lam": lam}, dout


def _exact_loss(oracle_mod, x, dout):
    o, _, _ = oracle_mod.forward_cholesky(x["q"], x["k"], x["v"], x["gamma"], x["beta"], x["lam"])
    return float(np.sum(o * dout))


def test_backward_matches_finite_differences_of_the_exact_layer(oracle_mod):
    """With CG run to convergence, the implicit gradient is the gradient of
    the exact layer: central differences of L = sum(dout * o), o from the
    Cholesky forward (code the backward does not use)."""
    x, dout = _bwd_inputs(0)
    d = x["q"].shape[-1]
    g = oracle_mod.backward(x["q"], x["k"], x["v"], x["gamma"], x["beta"], x["lam"], dout, 3 * d, 1e-13)
    h = 1e-6
    for name, key in (("q", "dq"), ("k", "dk"), ("v", "dv"), ("gamma", "dgamma"), ("beta", "dbeta"),
                      ("lam", "dlambda")):
        a = x[name]
        num = np.zeros_like(a)
        for idx in np.ndindex(a.shape):
            xp = dict(x)
            xp[name] = a.copy()
            xp[name][idx] += h
            lp = _exact_loss(oracle_mod, xp, dout)
            xp[name][idx] -= 2 * h
            lm = _exact_loss(oracle_mod, xp, dout)
            num[idx] = (lp - lm) / (2 * h)
        np.testing.assert_allclose(g[key], num, rtol=1e-6, atol=1e-8, err_msg=name)


def test_backward_adjoint_solves_converge_like_the_forward(oracle_mod):
    """The adjoint solves use the same CG rule: with tol > 0 every adjoint
    count stays within [1, cg_steps], and with a tiny step budget both solves
    take exactly that many updates."""
    x, dout = _bwd_inputs(1, B=1, H=1, T=6, d=4)
    g = oracle_mod.backward(x["q"], x["k"], x["v"], x["gamma"], x["beta"], x["lam"], dout, 12, 1e-10)
    assert g["iters_adj"].min() >= 1 and g["iters_adj"].max() <= 12
    g2 = oracle_mod.backward(x["q"], x["k"], x["v"], x["gamma"], x["beta"], x["lam"], dout, 2, 0.0)
    assert (g2["iters_fwd"] == 2).all() and (g2["iters_adj"] == 2).all()


def test_backward_one_step_closed_form(oracle_mod):
    """One CG step gives x = (q.q / q.Aq) q and u = (g.g / g.Ag) g with
    g = G^T do; on a single token (H = beta k k^T, G = beta v k^T) every
    gradient then follows from the definitions in closed form."""
    rng = np.random.default_rng(5)
    d = 4
    q = rng.standard_normal(d)
    k = rng.standard_normal(d)
    k /= np.linalg.norm(k)
    v = rng.standard_normal(d)
    do = rng.standard_normal(d)
    gam, bet = 0.8, 0.6
    lam = rng.uniform(0.3, 1.3, d)
    A = bet * np.outer(k, k) + np.diag(lam)
    G = bet * np.outer(v, k)
    x = (q @ q) / (q @ A @ q) * q
    gv = G.T @ do
    u = (gv @ gv) / (gv @ A @ gv) * gv
    Hbar = -np.outer(u, x)
    Gbar = np.outer(do, x)
    r = oracle_mod.backward(q[None, None, None], k[None, None, None], v[None, None, None],
                            np.array([[[gam]]]), np.array([[[bet]]]), lam[None], do[None, None, None], 1, 0.0)
    np.testing.assert_allclose(r["dq"][0, 0, 0], u, rtol=1e-12)
    np.testing.assert_allclose(r["dlambda"][0], -u * x, rtol=1e-12)
    np.testing.assert_allclose(r["dv"][0, 0, 0], bet * Gbar @ k, rtol=1e-12)
    np.testing.assert_allclose(r["dk"][0, 0, 0], bet * ((Hbar + Hbar.T) @ k + Gbar.T @ v), rtol=1e-12)
    np.testing.assert_allclose(r["dbeta"][0, 0, 0], k @ Hbar @ k + v @ Gbar @ k, rtol=1e-12)
    assert r["dgamma"][0, 0, 0] == 0.0              # the state before the first token is zero


def test_state_after_a_slice_is_affine_in_the_initial_state(oracle_mod):
    """The recurrence is affine in the state: the state after a slice from S
    equals prod(gamma) S plus the state after the slice from zero (the fact a
    sequence-sharded forward rests on)."""
    rng = np.random.default_rng(8)
    q, k, v, gamma, beta, lam = rand_inputs(rng, 1, 2, 11, 3, 4)
    S_H = rng.standard_normal((1, 2, 3, 3))
    S_H = S_H @ np.swapaxes(S_H, -1, -2)
    S_G = rng.standard_normal((1, 2, 4, 3))
    _, _, H1, G1 = oracle_mod.forward_cg(q, k, v, gamma, beta, lam, 3, H0=S_H, G0=S_G)
    _, _, H0, G0 = oracle_mod.forward_cg(q, k, v, gamma, beta, lam, 3)
    D = np.prod(gamma, axis=-1)[..., None, None]
    np.testing.assert_allclose(H1, D * S_H + H0, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(G1, D * S_G + G0, rtol=1e-12, atol=1e-14)


def test_backward_respects_the_beta_lambda_scale_invariance(oracle_mod):
    """(beta, Lambda) -> (c beta, c Lambda) leaves o unchanged (the objective
    is scaled as a whole), so the exact gradient has no component along that
    direction: per head, sum over its tokens of beta dbeta plus
    sum_i lambda_i dlambda_i is zero. Holds when the adjoint has converged."""
    x, dout = _bwd_inputs(4, B=2, H=2, T=5, d=3)
    g = oracle_mod.backward(x["q"], x["k"], x["v"], x["gamma"], x["beta"], x["lam"], dout, 9, 1e-14)
    for h in range(2):
        along = np.sum(x["beta"][:, h] * g["dbeta"][:, h]) + np.sum(x["lam"][h] * g["dlambda"][h])
        scale = np.sum(np.abs(x["beta"][:, h] * g["dbeta"][:, h])) + np.sum(np.abs(x["lam"][h] * g["dlambda"][h]))
        assert abs(along) <= 1e-10 * scale, (h, along, scale)
