"""Input preprocessing on the GPU (mesa_preprocess) against the fp64 oracle:
causal depthwise convolution over time, then per-token L2 normalisation."""
import numpy as np
import pytest
import torch

import mesa_inputs as mi
from helpers import TOL_BF16, rel_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def mesa():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from test_sequence_layer_b200 import build, mesa as m
    build.build()
    return m


def raw_inputs(B, H, T, d, W, seed):
    rng = np.random.default_rng(seed)
    xq = rng.standard_normal((B, H, T, d)).astype(np.float32)
    xk = rng.standard_normal((B, H, T, d)).astype(np.float32)
    cq = (rng.standard_normal((H, W, d)) / np.sqrt(W)).astype(np.float32)
    ck = (rng.standard_normal((H, W, d)) / np.sqrt(W)).astype(np.float32)
    return xq, xk, cq, ck


def on_device(a, dtype):
    t = torch.from_numpy(np.ascontiguousarray(a)).cuda()
    return t.to(torch.bfloat16) if dtype == "bf16" else t


def check(got, ref, dtype):
    # bf16: one rounding of each output (relative 2^-9) plus fp32 arithmetic; fp32: arithmetic only
    rel, ab = (2.0 ** -8, 1e-5) if dtype == "bf16" else (1e-6, 1e-6)
    err = np.abs(got - ref) - (rel * np.abs(ref) + ab)
    assert err.max() <= 0, f"max excess {err.max():.3e} at {np.unravel_index(err.argmax(), err.shape)}"


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("d,W,T", [(128, 4, 130), (128, 1, 37), (64, 3, 5), (16, 4, 300), (32, 2, 129)])
def test_preprocess_matches_oracle(mesa, oracle_mod, dtype, d, W, T):
    B, H = 2, 3
    xq, xk, cq, ck = raw_inputs(B, H, T, d, W, seed=d + W + T)
    q_raw, k_raw = on_device(xq, dtype), on_device(xk, dtype)
    q, k = mesa.preprocess(q_raw, k_raw, torch.from_numpy(cq).cuda(), torch.from_numpy(ck).cuda())
    torch.cuda.synchronize()
    # the oracle sees the same (rounded) inputs the GPU read
    ref_q = oracle_mod.preprocess(q_raw.float().cpu().numpy(), cq)
    ref_k = oracle_mod.preprocess(k_raw.float().cpu().numpy(), ck)
    check(q.float().cpu().numpy(), ref_q, dtype)
    check(k.float().cpu().numpy(), ref_k, dtype)


def test_preprocess_zero_rows_stay_zero(mesa):
    B, H, T, d, W = 1, 2, 40, 128, 4
    xq, xk, cq, ck = raw_inputs(B, H, T, d, W, seed=3)
    xq[0, 1, 10:20] = 0.0                              # u_t = 0 for t in 13..19 (window 4)
    q, _ = mesa.preprocess(on_device(xq, "bf16"), on_device(xk, "bf16"), torch.from_numpy(cq).cuda(),
                           torch.from_numpy(ck).cuda())
    qn = q.float().cpu().numpy()
    assert np.all(qn[0, 1, 13:20] == 0.0)
    assert np.allclose(np.linalg.norm(qn[0, 1, 20:], axis=-1), 1.0, atol=1e-2)


def test_preprocess_then_forward(mesa, oracle_mod):
    """Raw projections -> mesa_preprocess -> mesa_forward (tensor-core path),
    against the oracle forward on the same preprocessed (bf16) q and k."""
    B, H, T, d, W = 1, 2, 200, 128, 4
    xq, xk, cq, ck = raw_inputs(B, H, T, d, W, seed=8)
    w = mi.Workload("t", B, H, T, d, d, 64, "bf16", 15, 0.0, False, 19)
    x = mi.batch(w)
    q, k = mesa.preprocess(on_device(xq, "bf16"), on_device(xk, "bf16"), torch.from_numpy(cq).cuda(),
                           torch.from_numpy(ck).cuda())
    v = on_device(x["v"], "bf16")
    g, b, lam = (torch.from_numpy(np.ascontiguousarray(x[n])).cuda() for n in ("gamma", "beta", "lam"))
    out = mesa.forward(q, k, v, g, b, lam, chunk=64, cg_steps=15)
    torch.cuda.synchronize()
    assert mesa.get_error() == 0
    ref, _, _, _ = oracle_mod.forward_cg(q.float().cpu().numpy(), k.float().cpu().numpy(), v.float().cpu().numpy(),
                                         x["gamma"], x["beta"], x["lam"], 15)
    assert rel_err(out.cpu().numpy(), ref) <= TOL_BF16


def test_preprocess_full_size_sampled(mesa, oracle_mod):
    B, H, T, d, W = 8, 16, 8192, 128, 4
    g = torch.Generator(device="cuda").manual_seed(4)
    q_raw = torch.randn((B, H, T, d), generator=g, device="cuda").to(torch.bfloat16)
    k_raw = torch.randn((B, H, T, d), generator=g, device="cuda").to(torch.bfloat16)
    cq = torch.randn((H, W, d), generator=g, device="cuda") / 2
    ck = torch.randn((H, W, d), generator=g, device="cuda") / 2
    q, k = mesa.preprocess(q_raw, k_raw, cq, ck)
    torch.cuda.synchronize()
    for b, h in [(0, 0), (7, 15), (3, 9)]:
        for got, raw, c in ((q, q_raw, cq), (k, k_raw, ck)):
            ref = oracle_mod.preprocess(raw[b:b + 1, h:h + 1].float().cpu().numpy(),
                                        c[h:h + 1].cpu().numpy())
            check(got[b:b + 1, h:h + 1].float().cpu().numpy(), ref, "bf16")


# ---------------------------------------------------------------------------
# mesa_forward_preprocessed: the preprocessing folded into the forward's own
# staged loads (tensor-core shape) must give exactly the bits of the two-step
# path, mesa_preprocess followed by mesa_forward.
# ---------------------------------------------------------------------------

def layer_inputs(B, H, T, d, seed, dtype):
    w = mi.Workload("pre", B, H, T, d, d, 64, dtype, 15, 0.0, False, seed)
    x = mi.batch(w)
    rng = np.random.default_rng(seed + 1)
    raw_q = rng.standard_normal((B, H, T, d)).astype(np.float32)
    raw_k = rng.standard_normal((B, H, T, d)).astype(np.float32)
    return x, raw_q, raw_k


@pytest.mark.parametrize("B,H,T,W,tol", [(2, 3, 1, 4, 0.0), (2, 3, 3, 4, 0.0), (2, 3, 64, 2, 0.0), (2, 3, 65, 4, 0.0),
                                         (2, 3, 130, 3, 0.0), (2, 3, 333, 4, 0.0), (2, 3, 700, 1, 0.0),
                                         (2, 3, 300, 4, 1e-3),
                                         # 96 sequences: the scan carries both states in one CTA per sequence
                                         (6, 16, 200, 4, 0.0), (6, 16, 150, 3, 1e-3)])
def test_fused_forward_equals_preprocess_then_forward(mesa, B, H, T, W, tol):
    d = 128
    x, rq, rk = layer_inputs(B, H, T, d, 90 + T, "bf16")
    rng = np.random.default_rng(T)
    cq = torch.from_numpy((rng.standard_normal((H, W, d)) / np.sqrt(W)).astype(np.float32)).cuda()
    ck = torch.from_numpy((rng.standard_normal((H, W, d)) / np.sqrt(W)).astype(np.float32)).cuda()
    q_raw, k_raw = on_device(rq, "bf16"), on_device(rk, "bf16")
    v = on_device(x["v"], "bf16")
    g, b = torch.from_numpy(x["gamma"]).cuda(), torch.from_numpy(x["beta"]).cuda()
    lam = torch.from_numpy(x["lam"]).cuda()
    q, k = mesa.preprocess(q_raw, k_raw, cq, ck)
    ref, it_ref, H_ref, G_ref = mesa.forward(q, k, v, g, b, lam, chunk=64, cg_steps=30 if tol else 15, tol=tol,
                                             return_iters=True, return_state=True)
    out, it, H_o, G_o = mesa.forward_preprocessed(q_raw, k_raw, v, g, b, lam, cq, ck, chunk=64,
                                                  cg_steps=30 if tol else 15, tol=tol, return_iters=True,
                                                  return_state=True)
    torch.cuda.synchronize()
    assert mesa.get_error() == 0
    assert torch.equal(out, ref) and torch.equal(it, it_ref)
    assert torch.equal(H_o, H_ref) and torch.equal(G_o, G_ref)


@pytest.mark.parametrize("dtype,d,chunk", [("bf16", 128, 64), ("f32", 64, 16), ("bf16", 32, 32)])
def test_fused_forward_matches_oracle(mesa, oracle_mod, dtype, d, chunk):
    """Against the oracle's preprocessing followed by its CG forward (the other
    shapes take the two-step path inside the same entry point)."""
    B, H, T, W = 1, 2, 200, 4
    x, rq, rk = layer_inputs(B, H, T, d, 97, dtype)
    rng = np.random.default_rng(5)
    cq = (rng.standard_normal((H, W, d)) / 2).astype(np.float32)
    ck = (rng.standard_normal((H, W, d)) / 2).astype(np.float32)
    q_raw, k_raw = on_device(rq, dtype), on_device(rk, dtype)
    v = on_device(x["v"], dtype)
    out = mesa.forward_preprocessed(q_raw, k_raw, v, torch.from_numpy(x["gamma"]).cuda(),
                                    torch.from_numpy(x["beta"]).cuda(), torch.from_numpy(x["lam"]).cuda(),
                                    torch.from_numpy(cq).cuda(), torch.from_numpy(ck).cuda(), chunk=chunk,
                                    cg_steps=15)
    torch.cuda.synchronize()
    assert mesa.get_error() == 0
    # the oracle preprocesses the same raw values; the GPU's q and k are rounded
    # to the input type after preprocessing, so the oracle sees that rounding too
    pq = oracle_mod.preprocess(q_raw.float().cpu().numpy(), cq)
    pk = oracle_mod.preprocess(k_raw.float().cpu().numpy(), ck)
    if dtype == "bf16":
        pq, pk = mi.bf16_round(pq.astype(np.float32)), mi.bf16_round(pk.astype(np.float32))
    ref, _, _, _ = oracle_mod.forward_cg(pq, pk, v.float().cpu().numpy(), x["gamma"], x["beta"], x["lam"], 15)
    tol = TOL_BF16 if dtype == "bf16" else 1e-4
    assert rel_err(out.cpu().numpy(), ref) <= tol
