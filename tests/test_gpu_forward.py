"""GPU parity of mesa_forward against the fp64 CPU oracle (through the C ABI).

Small cases compare every output; the full-size workloads run in the launch
configuration the benchmark times and compare sampled (b, h) sequences, whose
inputs come from their per-sequence host streams (the rest of the batch is
drawn on the device with the same distributions).
"""
import numpy as np
import pytest
import torch

import mesa_inputs as mi
from helpers import TOL_BF16, TOL_F32, count_agreement, err_report, log_parity, rel_err

pytestmark = pytest.mark.gpu


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


def run(mesa, d, chunk, N, tol, **kw):
    out, iters = mesa.forward(d["q"], d["k"], d["v"], d["gamma"], d["beta"], d["lam"], chunk=chunk,
                              cg_steps=N, tol=tol, return_iters=True, **kw)
    torch.cuda.synchronize()
    assert mesa.get_error() == 0
    return out.cpu().numpy(), iters.cpu().numpy()


def rand_workload(d, chunk, dtype, T, B=1, H=2, N=8, tol=0.0, mixture=False, seed=7):
    return mi.Workload("t", B, H, T, d, d, chunk, dtype, N, tol, mixture, seed)


def test_tiny_fp32_workload(mesa, oracle_mod):
    w = mi.WORKLOADS["tiny_fp32"]
    x = mi.batch(w)
    ref, it_ref, _, _ = oracle_mod.forward_cg(x["q"], x["k"], x["v"], x["gamma"], x["beta"], x["lam"], w.cg_steps)
    out, it = run(mesa, to_dev(x, w.dtype), w.chunk, w.cg_steps, w.tol)
    assert rel_err(out, ref) <= TOL_F32, err_report(out, ref)
    assert np.array_equal(it, it_ref)


@pytest.mark.parametrize("d", [16, 32, 64, 128])
@pytest.mark.parametrize("chunk", [16, 32, 64])
@pytest.mark.parametrize("T", [1, 50, 200])
def test_fp32_shapes(mesa, oracle_mod, d, chunk, T):
    w = rand_workload(d, chunk, "f32", T, N=8, seed=d * 1000 + chunk + T)
    x = mi.batch(w)
    ref, it_ref, _, _ = oracle_mod.forward_cg(x["q"], x["k"], x["v"], x["gamma"], x["beta"], x["lam"], w.cg_steps)
    out, it = run(mesa, to_dev(x, "f32"), chunk, w.cg_steps, 0.0)
    assert rel_err(out, ref) <= TOL_F32, err_report(out, ref)
    assert np.array_equal(it, it_ref)


@pytest.mark.parametrize("T", [1, 63, 64, 65, 130, 333])
def test_bf16_d128_chunk64(mesa, oracle_mod, T):
    w = rand_workload(128, 64, "bf16", T, B=2, H=2, N=15, seed=T)
    x = mi.batch(w)
    ref, _, _, _ = oracle_mod.forward_cg(x["q"], x["k"], x["v"], x["gamma"], x["beta"], x["lam"], w.cg_steps)
    out, it = run(mesa, to_dev(x, "bf16"), 64, w.cg_steps, 0.0)
    rep = log_parity(f"bf16_d128_T{T}", out, ref)
    assert rep["rel"] <= TOL_BF16, rep
    assert np.all(it == 15)


@pytest.mark.parametrize("dtype,d,chunk", [("f32", 64, 16), ("bf16", 128, 64)])
def test_tolerance_stopping(mesa, oracle_mod, dtype, d, chunk):
    w = rand_workload(d, chunk, dtype, 300, B=1, H=3, N=30, tol=1e-3, mixture=True, seed=11)
    x = mi.batch(w)
    ref, it_ref, _, _ = oracle_mod.forward_cg(x["q"], x["k"], x["v"], x["gamma"], x["beta"], x["lam"], 30, 1e-3)
    exact, _, _ = oracle_mod.forward_cholesky(x["q"], x["k"], x["v"], x["gamma"], x["beta"], x["lam"])
    out, it = run(mesa, to_dev(x, dtype), chunk, 30, 1e-3)
    assert rel_err(out, ref) <= TOL_BF16, err_report(out, ref)
    assert rel_err(out, exact) <= TOL_BF16, err_report(out, exact)
    mx, frac = count_agreement(it, it_ref)
    assert mx <= 1 and frac <= 0.01, (mx, frac)
    assert it.min() < it.max()        # the mixture makes the counts vary


@pytest.mark.parametrize("dtype,d,chunk", [("f32", 32, 16), ("bf16", 128, 64)])
def test_state_in_and_out(mesa, oracle_mod, dtype, d, chunk):
    w = rand_workload(d, chunk, dtype, 150, B=2, H=2, N=6, seed=3)
    x = mi.batch(w)
    t0 = 77
    pre = {n: x[n][:, :, :t0] for n in ("q", "k", "v", "gamma", "beta")}
    post = {n: x[n][:, :, t0:] for n in ("q", "k", "v", "gamma", "beta")}
    _, _, H1, G1 = oracle_mod.forward_cg(*(pre[n] for n in ("q", "k", "v", "gamma", "beta")), x["lam"], 6)
    ref, _, Hf, Gf = oracle_mod.forward_cg(*(post[n] for n in ("q", "k", "v", "gamma", "beta")), x["lam"], 6,
                                           H0=H1, G0=G1)
    dpre = to_dev(dict(pre, lam=x["lam"]), dtype)
    dpost = to_dev(dict(post, lam=x["lam"]), dtype)
    _, Hg, Gg = mesa.forward(dpre["q"], dpre["k"], dpre["v"], dpre["gamma"], dpre["beta"], dpre["lam"],
                             chunk=chunk, cg_steps=6, return_state=True)
    out, Hg2, Gg2 = mesa.forward(dpost["q"], dpost["k"], dpost["v"], dpost["gamma"], dpost["beta"], dpost["lam"],
                                 chunk=chunk, cg_steps=6, H_in=Hg, G_in=Gg, return_state=True)
    torch.cuda.synchronize()
    assert np.allclose(Hg.cpu().numpy(), H1, rtol=1e-5, atol=1e-5)
    assert np.allclose(Gg.cpu().numpy(), G1, rtol=1e-5, atol=1e-5)
    assert np.allclose(Hg2.cpu().numpy(), Hf, rtol=1e-5, atol=1e-5)
    assert np.allclose(Gg2.cpu().numpy(), Gf, rtol=1e-5, atol=1e-5)
    tol = TOL_F32 if dtype == "f32" else TOL_BF16
    assert rel_err(out.cpu().numpy(), ref) <= tol


def test_state_in_and_out_wide_batch(mesa, oracle_mod):
    """A batch of 96 sequences: more than half the SM count, so the tensor-core
    scan carries both states in one CTA per sequence (G transposed in tensor
    memory, in its images and in the reads of G_in and writes of G_out).
    The smaller batches above use one CTA per state."""
    w = rand_workload(128, 64, "bf16", 100, B=6, H=16, N=4, seed=11)
    x = mi.batch(w)
    t0 = 37
    pre = {n: x[n][:, :, :t0] for n in ("q", "k", "v", "gamma", "beta")}
    post = {n: x[n][:, :, t0:] for n in ("q", "k", "v", "gamma", "beta")}
    _, _, H1, G1 = oracle_mod.forward_cg(*(pre[n] for n in ("q", "k", "v", "gamma", "beta")), x["lam"], 4)
    ref, _, Hf, Gf = oracle_mod.forward_cg(*(post[n] for n in ("q", "k", "v", "gamma", "beta")), x["lam"], 4,
                                           H0=H1, G0=G1)
    dpre = to_dev(dict(pre, lam=x["lam"]), "bf16")
    dpost = to_dev(dict(post, lam=x["lam"]), "bf16")
    _, Hg, Gg = mesa.forward(dpre["q"], dpre["k"], dpre["v"], dpre["gamma"], dpre["beta"], dpre["lam"],
                             chunk=64, cg_steps=4, return_state=True)
    out, Hg2, Gg2 = mesa.forward(dpost["q"], dpost["k"], dpost["v"], dpost["gamma"], dpost["beta"], dpost["lam"],
                                 chunk=64, cg_steps=4, H_in=Hg, G_in=Gg, return_state=True)
    torch.cuda.synchronize()
    assert mesa.get_error() == 0
    assert np.allclose(Hg.cpu().numpy(), H1, rtol=1e-5, atol=1e-5)
    assert np.allclose(Gg.cpu().numpy(), G1, rtol=1e-5, atol=1e-5)
    assert np.allclose(Hg2.cpu().numpy(), Hf, rtol=1e-5, atol=1e-5)
    assert np.allclose(Gg2.cpu().numpy(), Gf, rtol=1e-5, atol=1e-5)
    got = out.cpu().numpy()
    assert rel_err(got, ref) <= TOL_BF16, err_report(got, ref)


def test_scan_forms_agree(mesa):
    """96 sequences in one call (the scan carries both states per CTA) and the
    same sequences in two calls of 48 (one CTA per state) give the same
    outputs, iteration counts and final states up to the products' rounding."""
    w = rand_workload(128, 64, "bf16", 333, B=6, H=16, N=15, tol=1e-3, mixture=True, seed=23)
    x = mi.batch(w)
    d = to_dev(x, "bf16")
    whole, it_w, Hw, Gw = mesa.forward(d["q"], d["k"], d["v"], d["gamma"], d["beta"], d["lam"], chunk=64,
                                       cg_steps=15, tol=1e-3, return_iters=True, return_state=True)
    parts = []
    for b0 in (0, 3):
        sl = slice(b0, b0 + 3)
        parts.append(mesa.forward(d["q"][sl].contiguous(), d["k"][sl].contiguous(), d["v"][sl].contiguous(),
                                  d["gamma"][sl].contiguous(), d["beta"][sl].contiguous(), d["lam"], chunk=64,
                                  cg_steps=15, tol=1e-3, return_iters=True, return_state=True))
    torch.cuda.synchronize()
    assert mesa.get_error() == 0
    split = [torch.cat([p[i] for p in parts], dim=0) for i in range(4)]
    assert np.allclose(split[2].cpu().numpy(), Hw.cpu().numpy(), rtol=1e-5, atol=1e-5)
    assert np.allclose(split[3].cpu().numpy(), Gw.cpu().numpy(), rtol=1e-5, atol=1e-5)
    # the solve sees the same state images up to the last bits of the fp32 states
    # (an fp16 rounding may land on the other side), so a token may stop one
    # step apart: outputs within the bf16 bound, iteration counts within one
    got, ref = split[0].cpu().numpy(), whole.cpu().numpy()
    assert rel_err(got, ref) <= TOL_BF16, err_report(got, ref)
    assert (split[1] - it_w).abs().max().item() <= 1


def test_empty_sequence_copies_state(mesa):
    B, H, d = 2, 3, 16
    z = torch.zeros((B, H, 0, d), device="cuda")
    zg = torch.zeros((B, H, 0), device="cuda")
    lam = torch.ones((H, d), device="cuda")
    Hi = torch.randn((B, H, d, d), device="cuda")
    Gi = torch.randn((B, H, d, d), device="cuda")
    out, Ho, Go = mesa.forward(z, z, z, zg, zg, lam, chunk=16, cg_steps=4, H_in=Hi, G_in=Gi, return_state=True)
    torch.cuda.synchronize()
    assert out.shape == (B, H, 0, d)
    assert torch.equal(Ho, Hi) and torch.equal(Go, Gi)
    _, Ho, Go = mesa.forward(z, z, z, zg, zg, lam, chunk=16, cg_steps=4, return_state=True)
    torch.cuda.synchronize()
    assert not Ho.any() and not Go.any()


def test_zero_steps_and_zero_query(mesa, oracle_mod):
    w = rand_workload(32, 16, "f32", 40, N=4, seed=5)
    x = mi.batch(w)
    x["q"][:, :, 7] = 0.0                      # q = 0: CG stops at once, x = 0, o = 0
    d = to_dev(x, "f32")
    out, it = run(mesa, d, 16, 0, 0.0)
    assert not out.any() and not it.any()
    out, it = run(mesa, d, 16, 4, 0.0)
    ref, it_ref, _, _ = oracle_mod.forward_cg(x["q"], x["k"], x["v"], x["gamma"], x["beta"], x["lam"], 4)
    assert np.array_equal(it, it_ref) and it[0, 0, 7] == 0 and not out[:, :, 7].any()
    assert rel_err(out, ref) <= TOL_F32


@pytest.mark.parametrize("dtype,d,chunk", [("f32", 64, 64), ("bf16", 128, 64)])
def test_nan_input_does_not_hang(mesa, dtype, d, chunk):
    """A NaN poisons the tokens of its chunk (on the tensor-core path: of its
    pair of chunks, which share every MMA) and all later tokens of the
    sequence, and nothing else; the call completes with no device error."""
    w = rand_workload(d, chunk, dtype, 300, B=1, H=2, N=15, seed=9)
    x = mi.batch(w)
    x["v"][0, 0, 150, 3] = np.nan
    x["k"][0, 0, 170, 1] = np.nan
    out, _ = run(mesa, to_dev(x, dtype), chunk, 15, 0.0)
    assert np.isfinite(out[0, 0, :128]).all()
    assert not np.isfinite(out[0, 0, 192:]).all()
    assert np.isfinite(out[0, 1]).all()


def test_host_buffer_variant(mesa, oracle_mod):
    w = rand_workload(128, 64, "bf16", 200, B=1, H=2, N=15, seed=21)
    x = mi.batch(w)
    ref, it_ref, Hf, _ = oracle_mod.forward_cg(x["q"], x["k"], x["v"], x["gamma"], x["beta"], x["lam"], 15)
    h = {n: torch.from_numpy(np.ascontiguousarray(x[n])) for n in ("q", "k", "v", "gamma", "beta", "lam")}
    for n in ("q", "k", "v"):
        h[n] = h[n].to(torch.bfloat16).pin_memory()
    out = torch.empty((1, 2, 200, 128)).pin_memory()
    iters = torch.empty((1, 2, 200), dtype=torch.int32)
    Hout = torch.empty((1, 2, 128, 128))
    Gout = torch.empty((1, 2, 128, 128))
    mesa.forward_host(h["q"], h["k"], h["v"], h["gamma"], h["beta"], h["lam"], chunk=64, cg_steps=15, out=out,
                      iters=iters, H_out=Hout, G_out=Gout)
    assert rel_err(out.numpy(), ref) <= TOL_BF16
    assert np.array_equal(iters.numpy(), it_ref)
    assert np.allclose(Hout.numpy(), Hf, rtol=1e-4, atol=1e-5)


@pytest.mark.parametrize("dtype,chunk,B,T", [("bf16", 64, 11, 1536), ("f32", 32, 3, 2100), ("bf16", 64, 17, 1024)])
def test_host_pipeline_matches_device(mesa, dtype, chunk, B, T):
    """Inputs above 16 MiB go through the sliced copy/compute pipeline: runs of
    heads inside a batch row (B = 11, B = 3), groups of whole rows (B = 17).
    Every sequence is independent, so the host-buffer
    call must reproduce the device-buffer call bit for bit, initial and final
    states included."""
    w = rand_workload(128, chunk, dtype, T, B=B, H=4, N=15, seed=33)
    dev = mi.device_batch(w, "cuda")
    g = torch.Generator(device="cuda").manual_seed(5)
    Hin = torch.randn((B, 4, 128, 128), generator=g, device="cuda") * 0.01
    Hin = Hin @ Hin.transpose(-1, -2)                  # symmetric positive semi-definite
    Gin = torch.randn((B, 4, 128, 128), generator=g, device="cuda") * 0.01
    out_d, it_d, Ho_d, Go_d = mesa.forward(dev["q"], dev["k"], dev["v"], dev["gamma"], dev["beta"], dev["lam"],
                                           chunk=chunk, cg_steps=15, return_iters=True, H_in=Hin, G_in=Gin,
                                           return_state=True)
    torch.cuda.synchronize()
    assert mesa.get_error() == 0
    h = {n: dev[n].cpu().pin_memory() for n in ("q", "k", "v", "gamma", "beta", "lam")}
    out = torch.empty((B, 4, T, 128)).pin_memory()
    iters = torch.empty((B, 4, T), dtype=torch.int32).pin_memory()
    Hout = torch.empty((B, 4, 128, 128)).pin_memory()
    Gout = torch.empty((B, 4, 128, 128)).pin_memory()
    mesa.forward_host(h["q"], h["k"], h["v"], h["gamma"], h["beta"], h["lam"], chunk=chunk, cg_steps=15, out=out,
                      iters=iters, H_in=Hin.cpu(), G_in=Gin.cpu(), H_out=Hout, G_out=Gout)
    assert mesa.get_error() == 0
    assert torch.equal(out, out_d.cpu())
    assert torch.equal(iters, it_d.cpu())
    assert torch.equal(Hout, Ho_d.cpu()) and torch.equal(Gout, Go_d.cpu())


FULL = ["bf16_T2048", "bf16_T8192", "bf16_T8192_tol"]


@pytest.mark.parametrize("name", FULL)
def test_full_size_sampled(mesa, oracle_mod, name):
    w = mi.WORKLOADS[name]
    dev = mi.device_batch(w, "cuda")
    pairs = [(0, 0), (w.B - 1, w.H - 1), (w.B // 2, 5)]
    host = mi.plant_sequences(dev, w, pairs)
    out, it = mesa.forward(dev["q"], dev["k"], dev["v"], dev["gamma"], dev["beta"], dev["lam"], chunk=w.chunk,
                           cg_steps=w.cg_steps, tol=w.tol, return_iters=True)
    torch.cuda.synchronize()
    assert mesa.get_error() == 0
    ref, it_ref, _, _ = oracle_mod.forward_cg(host["q"], host["k"], host["v"], host["gamma"], host["beta"],
                                              host["lam"], w.cg_steps, w.tol)
    got = np.stack([out[b, h].cpu().numpy() for b, h in pairs])[None]
    got_it = np.stack([it[b, h].cpu().numpy() for b, h in pairs])[None]
    rep = log_parity(f"full:{name}", got, ref)
    assert rep["rel"] <= TOL_BF16, rep
    if w.tol > 0:
        mx, frac = count_agreement(got_it, it_ref)
        assert mx <= 1 and frac <= 0.01, (mx, frac)
        exact, _, _ = oracle_mod.forward_cholesky(host["q"], host["k"], host["v"], host["gamma"], host["beta"],
                                                  host["lam"])
        assert rel_err(got, exact) <= TOL_BF16
    else:
        assert np.all(got_it == w.cg_steps)
    assert torch.isfinite(out).all()
