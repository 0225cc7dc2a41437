"""GPU parity of mesa_backward against the fp64 CPU oracle (through the C ABI).

Every gradient (dq, dk, dv, dgamma, dbeta, dlambda) is compared on small
cases that span several chunks with a ragged tail; the full-size workload
compares sampled (b, h) sequences (dlambda, a sum over the batch, is covered
by the small cases). The backward computes in fp32 on the CUDA cores, so the
fp32 bound applies (the oracle reads the same bf16-rounded inputs), except
for bf16 inputs at d = 128, C = 64: there the forward solutions come from the
tensor-core solve (fp16 operands), and the bf16-mode bound applies.
"""
import numpy as np
import pytest
import torch

import mesa_inputs as mi
from helpers import TOL_BF16, TOL_F32, err_report, rel_err

pytestmark = pytest.mark.gpu

NAMES = ("dq", "dk", "dv", "dgamma", "dbeta", "dlambda")


def bound(dtype, d, chunk):
    return TOL_BF16 if (dtype, d, chunk) == ("bf16", 128, 64) else TOL_F32


@pytest.fixture(scope="module")
def mesa():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from test_sequence_layer_b200 import build, mesa as m
    build.build()
    return m


def to_dev(x, dtype):
    dt = torch.bfloat16 if dtype == "bf16" else torch.float32
    d = {n: torch.from_numpy(np.ascontiguousarray(x[n])).cuda() for n in ("q", "k", "v", "gamma", "beta", "lam")}
    for n in ("q", "k", "v"):
        d[n] = d[n].to(dt)
    return d


def gpu_backward(mesa, d, do, chunk, N, tol):
    g = mesa.backward(d["q"], d["k"], d["v"], d["gamma"], d["beta"], d["lam"], do, chunk=chunk, cg_steps=N, tol=tol)
    torch.cuda.synchronize()
    assert mesa.get_error() == 0
    return dict(zip(NAMES, (t.cpu().numpy() for t in g)))


CASES = [
    # dtype, d, chunk, T, B, H, cg_steps, tol
    ("f32", 16, 16, 37, 2, 2, 16, 0.0),
    ("f32", 32, 32, 70, 1, 2, 8, 0.0),
    ("f32", 64, 64, 130, 1, 2, 15, 0.0),
    ("f32", 128, 64, 150, 1, 2, 15, 0.0),
    ("f32", 128, 16, 40, 2, 1, 15, 0.0),
    ("bf16", 128, 64, 200, 2, 1, 15, 0.0),
    ("bf16", 64, 64, 150, 1, 2, 15, 0.0),
    ("f32", 64, 32, 64, 1, 1, 3, 0.0),
    # 96 sequences: the tensor-core scans carry both states in one CTA per sequence
    ("bf16", 128, 64, 100, 6, 16, 6, 0.0),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "-".join(map(str, c)))
def test_backward_matches_oracle(mesa, oracle_mod, case):
    dtype, d, chunk, T, B, H, N, tol = case
    w = mi.Workload("t", B, H, T, d, d, chunk, dtype, N, tol, False, 11)
    x = mi.batch(w)
    do = mi.dout(11, B, H, T, d)
    g = gpu_backward(mesa, to_dev(x, dtype), torch.from_numpy(do).cuda(), chunk, N, tol)
    ref = oracle_mod.backward(x["q"], x["k"], x["v"], x["gamma"], x["beta"], x["lam"], do, N, tol)
    for n in NAMES:
        assert rel_err(g[n], ref[n]) <= bound(dtype, d, chunk), (n, err_report(g[n], ref[n]))


def test_backward_tolerance_stopping(mesa, oracle_mod):
    """tol > 0: both solves stop per token; near the threshold a count may
    differ by one between fp32 and fp64, which moves x and u by at most
    ~tol relative (|x_k - x*| <= |r_k| / lambda_min), hence the 2e-2 bound."""
    w = mi.Workload("t", 1, 2, 100, 64, 64, 32, "f32", 30, 1e-3, True, 12)
    x = mi.batch(w)
    do = mi.dout(12, 1, 2, 100, 64)
    g = gpu_backward(mesa, to_dev(x, "f32"), torch.from_numpy(do).cuda(), 32, 30, 1e-3)
    ref = oracle_mod.backward(x["q"], x["k"], x["v"], x["gamma"], x["beta"], x["lam"], do, 30, 1e-3)
    for n in NAMES:
        assert rel_err(g[n], ref[n]) <= 2e-2, (n, err_report(g[n], ref[n]))


def test_backward_zero_upstream_gradient_gives_zeros(mesa):
    w = mi.Workload("t", 1, 2, 70, 32, 32, 16, "f32", 8, 0.0, False, 13)
    d = to_dev(mi.batch(w), "f32")
    g = gpu_backward(mesa, d, torch.zeros((1, 2, 70, 32), device="cuda"), 16, 8, 0.0)
    for n in NAMES:
        assert not np.any(g[n]), n


def test_backward_homogeneous_in_the_upstream_gradient(mesa):
    """CG with a fixed step count is homogeneous of degree one in its
    right-hand side (alpha and rho are ratios of quadratic forms), so scaling
    dL/do by 2 scales every gradient by exactly 2 (a power of two: no rounding
    changes). dv = beta Gbar k does not involve the adjoint solve and is
    additive as well; the other gradients are not (CG truncated at N steps is
    not linear in its right-hand side)."""
    w = mi.Workload("t", 1, 2, 90, 64, 64, 32, "f32", 10, 0.0, False, 14)
    d = to_dev(mi.batch(w), "f32")
    do1 = torch.from_numpy(mi.dout(14, 1, 2, 90, 64)).cuda()
    do2 = torch.from_numpy(mi.dout(15, 1, 2, 90, 64)).cuda()
    g1 = gpu_backward(mesa, d, do1, 32, 10, 0.0)
    g2 = gpu_backward(mesa, d, do2, 32, 10, 0.0)
    g12 = gpu_backward(mesa, d, 2.0 * do1, 32, 10, 0.0)
    g3 = gpu_backward(mesa, d, do1 + do2, 32, 10, 0.0)
    for n in NAMES:
        assert np.array_equal(g12[n], 2.0 * g1[n]), n
    assert rel_err(g3["dv"], g1["dv"] + g2["dv"]) <= 1e-5


def test_backward_full_size_sampled(mesa, oracle_mod):
    """B=8, H=16, T=8192, d=128 bf16, 15 steps (the benchmark's backward
    workload): two sampled sequences against the oracle."""
    w = mi.Workload("bwd", 8, 16, 8192, 128, 128, 64, "bf16", 15, 0.0, False, 2)
    pairs = [(3, 5), (7, 15)]
    dev = mi.device_batch(w, "cuda")
    host = mi.plant_sequences(dev, w, pairs)
    g = torch.Generator(device="cuda")
    g.manual_seed(99)
    do = torch.randn((8, 16, 8192, 128), generator=g, device="cuda")
    do_host = mi.dout(2, 8, 16, 8192, 128, seqs=pairs)
    for i, (b, h) in enumerate(pairs):
        do[b, h].copy_(torch.from_numpy(do_host[0, i]))
    res = mesa.backward(dev["q"], dev["k"], dev["v"], dev["gamma"], dev["beta"], dev["lam"], do, chunk=64,
                        cg_steps=15)
    torch.cuda.synchronize()
    assert mesa.get_error() == 0
    ref = oracle_mod.backward(host["q"], host["k"], host["v"], host["gamma"], host["beta"], host["lam"], do_host, 15)
    for n, t in zip(NAMES[:5], res[:5]):
        got = np.stack([t[b, h].cpu().numpy() for (b, h) in pairs])[None]
        assert rel_err(got, ref[n]) <= TOL_BF16, (n, err_report(got, ref[n]))


@pytest.mark.parametrize("dtype,d,chunk,T", [("f32", 16, 16, 1), ("bf16", 128, 64, 1), ("f32", 64, 64, 64),
                                              ("bf16", 128, 64, 128)])
def test_backward_edge_lengths(mesa, oracle_mod, dtype, d, chunk, T):
    """A single token (the state is one outer product) and sequences that end
    exactly on a chunk or block boundary."""
    w = mi.Workload("t", 1, 2, T, d, d, chunk, dtype, 15, 0.0, False, 31)
    x = mi.batch(w)
    do = mi.dout(31, 1, 2, T, d)
    g = gpu_backward(mesa, to_dev(x, dtype), torch.from_numpy(do).cuda(), chunk, 15, 0.0)
    ref = oracle_mod.backward(x["q"], x["k"], x["v"], x["gamma"], x["beta"], x["lam"], do, 15)
    for n in NAMES:
        assert rel_err(g[n], ref[n]) <= bound(dtype, d, chunk), (n, err_report(g[n], ref[n]))


def test_backward_empty_sequence(mesa):
    e = torch.empty((1, 2, 0, 16), device="cuda")
    g = torch.empty((1, 2, 0), device="cuda")
    lam = torch.ones((2, 16), device="cuda")
    res = mesa.backward(e, e, e, g, g, lam, e, chunk=16, cg_steps=4)
    torch.cuda.synchronize()
    assert mesa.get_error() == 0
    assert torch.equal(res[5], torch.zeros_like(lam))


def test_backward_tolerance_stopping_tensor_core_shape(mesa, oracle_mod):
    """bf16 inputs at d = 128, C = 64 with tol = 1e-3 and the gamma mixture:
    the forward solutions come from the tensor-core solve, whose counts may
    differ by one near the threshold (as in the forward)."""
    w = mi.Workload("t", 1, 2, 200, 128, 128, 64, "bf16", 30, 1e-3, True, 33)
    x = mi.batch(w)
    do = mi.dout(33, 1, 2, 200, 128)
    g = gpu_backward(mesa, to_dev(x, "bf16"), torch.from_numpy(do).cuda(), 64, 30, 1e-3)
    ref = oracle_mod.backward(x["q"], x["k"], x["v"], x["gamma"], x["beta"], x["lam"], do, 30, 1e-3)
    for n in NAMES:
        assert rel_err(g[n], ref[n]) <= TOL_BF16, (n, err_report(g[n], ref[n]))
