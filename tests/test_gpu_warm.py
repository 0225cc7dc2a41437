"""mesa_forward_warm (every token's CG started from a caller-given guess)
against the fp64 oracle's warm-started forward, through the C ABI, on the
fp32 CUDA-core path and the tensor-core path.

Source of the method: the MesaNet page, Significance and claims (warm starts
are named as the way to cut the solver's cost). The guesses used here are
random (so that the start matters for the result), the exact solutions
(no step is taken), and the solutions of an earlier forward over the same
sequence with one token inserted at the front (the situation the entry point
serves: a context that has been edited since it was last solved).
"""
import numpy as np
import pytest
import torch

import mesa_inputs as mi
from helpers import TOL_BF16, TOL_F32, count_agreement, log_parity, rel_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def mesa():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from test_sequence_layer_b200 import build, mesa as m
    build.build()
    return m


def dev(x, dtype):
    dt = torch.bfloat16 if dtype == "bf16" else torch.float32
    d = {n: torch.from_numpy(np.ascontiguousarray(x[n])).cuda() for n in ("q", "k", "v", "gamma", "beta", "lam")}
    for n in ("q", "k", "v"):
        d[n] = d[n].to(dt)
    return d


SHAPES = [("f32", 64, 16, TOL_F32), ("f32", 32, 64, TOL_F32), ("bf16", 128, 64, TOL_BF16)]


@pytest.mark.parametrize("dtype,d,chunk,tol_err", SHAPES)
def test_warm_from_zero_or_none_is_the_cold_forward(mesa, dtype, d, chunk, tol_err):
    w = mi.Workload("w", 2, 2, 150, d, d, chunk, dtype, 8, 0.0, False, 71)
    g = dev(mi.batch(w), dtype)
    cold, it_c = mesa.forward(g["q"], g["k"], g["v"], g["gamma"], g["beta"], g["lam"], chunk=chunk, cg_steps=8,
                              return_iters=True)
    for x0 in (None, torch.zeros((2, 2, 150, d), device="cuda")):
        warm, x, it_w = mesa.forward_warm(g["q"], g["k"], g["v"], g["gamma"], g["beta"], g["lam"], x0, chunk=chunk,
                                          cg_steps=8, return_iters=True)
        torch.cuda.synchronize()
        assert mesa.get_error() == 0
        assert torch.equal(it_w, it_c)
        assert rel_err(warm.cpu().numpy(), cold.cpu().numpy()) <= (1e-6 if x0 is None else tol_err)


@pytest.mark.parametrize("dtype,d,chunk,tol_err", SHAPES)
@pytest.mark.parametrize("T", [1, 77, 300])
def test_warm_random_start_matches_oracle(mesa, oracle_mod, dtype, d, chunk, tol_err, T):
    N = 4                                        # few steps: the start shows in the result
    w = mi.Workload("w", 1, 3, T, d, d, chunk, dtype, N, 0.0, False, 72 + T)
    x = mi.batch(w)
    rng = np.random.default_rng(T)
    x0 = (0.5 * rng.standard_normal((1, 3, T, d))).astype(np.float32)
    ref, it_ref, xr, _, _ = oracle_mod.forward_cg_x0(x["q"], x["k"], x["v"], x["gamma"], x["beta"], x["lam"], N,
                                                     x0=x0)
    g = dev(x, dtype)
    out, xs, it = mesa.forward_warm(g["q"], g["k"], g["v"], g["gamma"], g["beta"], g["lam"],
                                    torch.from_numpy(x0).cuda(), chunk=chunk, cg_steps=N, return_iters=True)
    torch.cuda.synchronize()
    assert mesa.get_error() == 0
    rep = log_parity(f"warm:{dtype}_d{d}_T{T}", out.cpu().numpy(), ref)
    assert rep["rel"] <= tol_err, rep
    assert rel_err(xs.cpu().numpy(), xr) <= tol_err
    assert np.array_equal(it.cpu().numpy(), it_ref)


@pytest.mark.parametrize("dtype,d,chunk", [("f32", 64, 16), ("bf16", 128, 64)])
def test_warm_from_exact_solutions_takes_no_step(mesa, oracle_mod, dtype, d, chunk):
    w = mi.Workload("w", 1, 2, 200, d, d, chunk, dtype, 30, 1e-3, False, 73)
    x = mi.batch(w)
    # exact solutions from the oracle's converged CG (d steps, no tolerance)
    _, _, xs, _, _ = oracle_mod.forward_cg_x0(x["q"], x["k"], x["v"], x["gamma"], x["beta"], x["lam"], 4 * d)
    exact, _, _ = oracle_mod.forward_cholesky(x["q"], x["k"], x["v"], x["gamma"], x["beta"], x["lam"])
    g = dev(x, dtype)
    out, xo, it = mesa.forward_warm(g["q"], g["k"], g["v"], g["gamma"], g["beta"], g["lam"],
                                    torch.from_numpy(xs.astype(np.float32)).cuda(), chunk=chunk, cg_steps=30,
                                    tol=1e-3, return_iters=True)
    torch.cuda.synchronize()
    assert mesa.get_error() == 0
    it = it.cpu().numpy()
    # fp32: the start's residual is ~1e-7 |q|, far inside the tolerance; the
    # tensor-core path forms it with fp16 operands (~5e-4 |q|), so a token may
    # take one step
    assert (it <= (0 if dtype == "f32" else 1)).mean() >= 0.99, np.bincount(it.ravel())
    assert rel_err(out.cpu().numpy(), exact) <= (TOL_F32 * 10 if dtype == "f32" else TOL_BF16)


def insert_front(x, rng, bf16):
    """The same sequences with one new token inserted at the front (the last
    token drops out, so T is unchanged)."""
    y = {n: x[n].copy() for n in x}
    for n in ("q", "k", "v", "gamma", "beta"):
        y[n][:, :, 1:] = x[n][:, :, :-1]
    qk = rng.standard_normal(y["q"][:, :, 0].shape).astype(np.float32)
    y["q"][:, :, 0] = qk / np.linalg.norm(qk, axis=-1, keepdims=True)
    kk = rng.standard_normal(y["k"][:, :, 0].shape).astype(np.float32)
    y["k"][:, :, 0] = kk / np.linalg.norm(kk, axis=-1, keepdims=True)
    y["v"][:, :, 0] = rng.standard_normal(y["v"][:, :, 0].shape).astype(np.float32)
    y["gamma"][:, :, 0] = 0.9
    y["beta"][:, :, 0] = 0.5
    for n in ("q", "k", "v"):
        y[n] = mi.bf16_round(y[n]) if bf16 else y[n]
    return y


@pytest.mark.parametrize("dtype,d,chunk", [("f32", 64, 16), ("bf16", 128, 64)])
def test_warm_after_an_edit_saves_steps_and_matches_oracle(mesa, oracle_mod, dtype, d, chunk):
    """Solve a sequence, insert a token at the front, and re-solve from the
    shifted earlier solutions: fewer CG steps than a cold start, outputs as
    the oracle's warm-started forward from the same guesses (counts within
    one of the oracle's, as for any tolerance-stopped run)."""
    w = mi.Workload("w", 1, 3, 400, d, d, chunk, dtype, 30, 1e-3, True, 74)
    x = mi.batch(w)
    y = insert_front(x, np.random.default_rng(9), dtype == "bf16")
    g = dev(x, dtype)
    _, x_old = mesa.forward_warm(g["q"], g["k"], g["v"], g["gamma"], g["beta"], g["lam"], None, chunk=chunk,
                                 cg_steps=30, tol=1e-3)
    x0 = torch.zeros_like(x_old)
    x0[:, :, 1:] = x_old[:, :, :-1]
    gy = dev(y, dtype)
    cold, it_cold = mesa.forward(gy["q"], gy["k"], gy["v"], gy["gamma"], gy["beta"], gy["lam"], chunk=chunk,
                                 cg_steps=30, tol=1e-3, return_iters=True)
    warm, _, it_warm = mesa.forward_warm(gy["q"], gy["k"], gy["v"], gy["gamma"], gy["beta"], gy["lam"], x0,
                                         chunk=chunk, cg_steps=30, tol=1e-3, return_iters=True)
    torch.cuda.synchronize()
    assert mesa.get_error() == 0
    it_cold, it_warm = it_cold.cpu().numpy(), it_warm.cpu().numpy()
    assert it_warm.mean() < 0.8 * it_cold.mean(), (it_warm.mean(), it_cold.mean())
    ref, it_ref, _, _, _ = oracle_mod.forward_cg_x0(y["q"], y["k"], y["v"], y["gamma"], y["beta"], y["lam"], 30,
                                                    1e-3, x0=x0.cpu().numpy())
    rep = log_parity(f"warm_edit:{dtype}", warm.cpu().numpy(), ref, iters_cold=float(it_cold.mean()),
                     iters_warm=float(it_warm.mean()))
    assert rep["rel"] <= TOL_BF16, rep
    # a warm start puts most tokens' first residual near the threshold itself
    # (the tensor-core path forms it with fp16 operands, ~5e-4 |q| against
    # tol 1e-3), so a one-step disagreement is more frequent than from zero
    mx, frac = count_agreement(it_warm, it_ref)
    assert mx <= 1 and frac <= 0.05, (mx, frac)


def test_warm_in_place(mesa):
    """x_out may be x0 itself: the solutions replace the guesses."""
    w = mi.Workload("w", 2, 2, 260, 128, 128, 64, "bf16", 6, 0.0, False, 75)
    g = dev(mi.batch(w), "bf16")
    x0 = torch.randn((2, 2, 260, 128), device="cuda") * 0.3
    out1, x1 = mesa.forward_warm(g["q"], g["k"], g["v"], g["gamma"], g["beta"], g["lam"], x0.clone(), chunk=64,
                                 cg_steps=6)
    buf = x0.clone()
    out2, x2 = mesa.forward_warm(g["q"], g["k"], g["v"], g["gamma"], g["beta"], g["lam"], buf, chunk=64,
                                 cg_steps=6, x_out=buf)
    torch.cuda.synchronize()
    assert x2.data_ptr() == buf.data_ptr()
    assert torch.equal(out1, out2) and torch.equal(x1, buf)
