"""Tensor-core path (bf16 inputs, d = 128, C = 64) at input magnitudes the
ABI accepts beyond the synthetic workloads' distributions, against the fp64
CPU oracle element by element.

The Mesa objective (MesaNet page, Technical summary > Method > Mesa layer)
takes any symmetric positive definite Lambda and any cumulative forget
factors, and the ABI asks only 0 < gamma <= 1, beta >= 0, lambda > 0 and
finite values. Every fp16 operand image of the tensor-core path is divided by
a power of two taken from a bound on its entries, so these inputs must stay
finite and within the bf16-mode bound:
  * (beta, Lambda) -> (c beta, c Lambda), which leaves o unchanged in exact
    arithmetic, for c in {1e-3, 1e3, 1e4};
  * gamma = 1 over a span of several 128-token blocks;
  * beta = 0 on a whole first block and on a quarter of the later tokens;
  * |v| up to 1e5 in the first block;
  * keys of norm 1e-2 and 1e2 (the latter with beta scaled by 1e-4, which
    keeps beta k k^T, and so the conditioning of H + Lambda, as in the
    synthetic workload; the plain norm-1e2 case, whose conditioning makes
    the 15-step iterate unstable at any precision, is in its own test below);
  * queries of norm 1e3 and 1e-3.
"""
import numpy as np
import pytest
import torch

import mesa_inputs as mi
from helpers import TOL_BF16, log_parity, rel_err

pytestmark = pytest.mark.gpu

N_STEPS = 15


@pytest.fixture(scope="module")
def mesa():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from test_sequence_layer_b200 import build, mesa as m
    build.build()
    return m


def base(T=333, seed=101):
    w = mi.Workload("ranges", 2, 2, T, 128, 128, 64, "bf16", N_STEPS, 0.0, False, seed)
    return mi.batch(w)


def _scale_bf16(x, c):
    return mi.bf16_round(np.asarray(x, np.float32) * np.float32(c))


def case_inputs(name):
    if name.startswith("beta_lambda_x"):
        c = np.float32(float(name[len("beta_lambda_x"):]))
        x = base()
        x["beta"] = (x["beta"] * c).astype(np.float32)
        x["lam"] = (x["lam"] * c).astype(np.float32)
        return x
    if name == "gamma_one_span":
        x = base(T=600, seed=102)
        x["gamma"][:, :, 100:460] = 1.0
        return x
    if name == "beta_zero":
        x = base(seed=103)
        rng = np.random.default_rng(5)
        x["beta"][:, :, :128] = 0.0
        x["beta"][rng.random(x["beta"].shape) < 0.25] = 0.0
        return x
    if name == "v_1e5_first_block":
        x = base(seed=104)
        x["v"][:, :, :128] = _scale_bf16(x["v"][:, :, :128], 1e5 / 4.0)   # |v| up to ~1e5
        return x
    if name == "keys_norm_1e-2":
        x = base(seed=105)
        x["k"] = _scale_bf16(x["k"], 1e-2)
        return x
    if name == "keys_norm_1e2_beta_1e-4":
        x = base(seed=106)
        x["k"] = _scale_bf16(x["k"], 1e2)
        x["beta"] = (x["beta"] * np.float32(1e-4)).astype(np.float32)
        return x
    if name == "queries_norm_1e3":
        x = base(seed=107)
        x["q"] = _scale_bf16(x["q"], 1e3)
        return x
    if name == "queries_norm_1e-3":
        x = base(seed=108)
        x["q"] = _scale_bf16(x["q"], 1e-3)
        return x
    raise KeyError(name)


CASES = ["beta_lambda_x1e-3", "beta_lambda_x1e3", "beta_lambda_x1e4", "gamma_one_span", "beta_zero",
         "v_1e5_first_block", "keys_norm_1e-2", "keys_norm_1e2_beta_1e-4", "queries_norm_1e3",
         "queries_norm_1e-3"]


def run_tc(mesa, x, N=N_STEPS, tol=0.0):
    d = {n: torch.from_numpy(np.ascontiguousarray(x[n])).cuda() for n in ("q", "k", "v", "gamma", "beta", "lam")}
    for n in ("q", "k", "v"):
        d[n] = d[n].to(torch.bfloat16)
    out, it = mesa.forward(d["q"], d["k"], d["v"], d["gamma"], d["beta"], d["lam"], chunk=64, cg_steps=N, tol=tol,
                           return_iters=True)
    torch.cuda.synchronize()
    assert mesa.get_error() == 0
    return out.cpu().numpy(), it.cpu().numpy()


@pytest.mark.parametrize("name", CASES)
def test_range_case_matches_oracle(mesa, oracle_mod, name):
    x = case_inputs(name)
    ref, it_ref, _, _ = oracle_mod.forward_cg(x["q"], x["k"], x["v"], x["gamma"], x["beta"], x["lam"], N_STEPS)
    out, it = run_tc(mesa, x)
    assert np.isfinite(out).all()
    rep = log_parity(f"range:{name}", out, ref)
    assert rep["rel"] <= TOL_BF16, rep
    assert np.array_equal(it, it_ref)


def test_beta_lambda_scaling_leaves_output_unchanged(mesa):
    """The GPU outputs themselves are invariant under (beta, Lambda) ->
    (c beta, c Lambda) up to the bf16-mode bound (c a power of two leaves
    every fp16 image bit for bit the same, so the outputs agree closely)."""
    x = base(seed=109)
    o1, _ = run_tc(mesa, x)
    for c in (2.0 ** -12, 2.0 ** 12, 1e-3, 1e4):
        y = dict(x)
        y["beta"] = (x["beta"] * np.float32(c)).astype(np.float32)
        y["lam"] = (x["lam"] * np.float32(c)).astype(np.float32)
        o2, _ = run_tc(mesa, y)
        assert rel_err(o2, o1) <= TOL_BF16, c


def test_keys_norm_1e2_plain_beta(mesa, oracle_mod):
    """Keys of norm 1e2 with the workload's beta: H grows by 1e4 while Lambda
    does not, so the condition number of H + Lambda reaches ~1e5 and 15 CG
    steps are far from converged. There the truncated CG iterate is not a
    stable quantity: rounding at any precision below the oracle's fp64 moves
    it by O(1) (the fp32 CUDA-core path on the same values is ~7x off the
    oracle). What this checks is that the tensor-core path stays finite and
    is no further from the oracle than a correct single-precision run; both
    distances go to the parity log."""
    x = base(seed=110)
    x["k"] = _scale_bf16(x["k"], 1e2)
    ref, _, _, _ = oracle_mod.forward_cg(x["q"], x["k"], x["v"], x["gamma"], x["beta"], x["lam"], N_STEPS)
    out, _ = run_tc(mesa, x)
    assert np.isfinite(out).all()
    d = {n: torch.from_numpy(np.ascontiguousarray(x[n])).cuda() for n in ("q", "k", "v", "gamma", "beta", "lam")}
    o32 = mesa.forward(d["q"], d["k"], d["v"], d["gamma"], d["beta"], d["lam"], chunk=64, cg_steps=N_STEPS)
    torch.cuda.synchronize()
    rep32 = log_parity("range:keys_norm_1e2_plain_beta:fp32_path", o32.cpu().numpy(), ref)
    rep = log_parity("range:keys_norm_1e2_plain_beta", out, ref, fp32_path_rel=rep32["rel"])
    assert np.isfinite(o32.cpu().numpy()).all()
    assert rep["rel"] <= 2.0 * rep32["rel"] + TOL_BF16, rep
