"""GPU parity of mesa_step (recurrent decode on explicit state) against the
fp64 oracle, and consistency of decode with the chunkwise forward."""
import numpy as np
import pytest
import torch

import mesa_inputs as mi
from helpers import TOL_F32, count_agreement, err_report, log_parity, rel_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def mesa():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from test_sequence_layer_b200 import build, mesa as m
    build.build()
    return m


def cuda(a, dt=torch.float32):
    return torch.from_numpy(np.ascontiguousarray(a)).to("cuda", dt)


@pytest.mark.parametrize("d", [16, 32, 64, 128])
@pytest.mark.parametrize("tol", [0.0, 1e-3])
def test_steps_match_oracle(mesa, oracle_mod, d, tol):
    w = mi.Workload("t", 2, 3, 40, d, d, 16, "f32", 15, tol, tol > 0, 31 + d)
    x = mi.batch(w)
    t0 = 25
    N = 30 if tol > 0 else 15
    # oracle: prefix via the per-token recurrence, then single steps
    _, _, Hs, Gs = oracle_mod.forward_cg(*(x[n][:, :, :t0] for n in ("q", "k", "v", "gamma", "beta")), x["lam"], N, tol)
    # GPU: same prefix through mesa_forward's final state, then mesa_step
    dq = {n: cuda(x[n]) for n in ("q", "k", "v", "gamma", "beta")}
    lam = cuda(x["lam"])
    _, Hg, Gg = mesa.forward(*(dq[n][:, :, :t0].contiguous() for n in ("q", "k", "v", "gamma", "beta")), lam,
                             chunk=16, cg_steps=N, tol=tol, return_state=True)
    iters = torch.empty((2, 3), dtype=torch.int32, device="cuda")
    for t in range(t0, w.T):
        ref, it_ref, Hs, Gs = oracle_mod.step(*(x[n][:, :, t] for n in ("q", "k", "v", "gamma", "beta")), x["lam"],
                                              Hs, Gs, N, tol)
        out = mesa.step(*(dq[n][:, :, t].contiguous() for n in ("q", "k", "v", "gamma", "beta")), lam, Hg, Gg,
                        cg_steps=N, tol=tol, iters=iters)
        torch.cuda.synchronize()
        o = out.cpu().numpy()
        if tol == 0:
            assert rel_err(o, ref) <= TOL_F32, (t, err_report(o, ref))
            assert np.all(iters.cpu().numpy() == N)
        else:
            assert rel_err(o, ref) <= 2e-2, (t, err_report(o, ref))
            mx, _ = count_agreement(iters.cpu().numpy(), it_ref)
            assert mx <= 1
    assert np.allclose(Hg.cpu().numpy(), Hs, rtol=1e-4, atol=1e-5)
    assert np.allclose(Gg.cpu().numpy(), Gs, rtol=1e-4, atol=1e-5)
    assert mesa.get_error() == 0


def test_every_head_of_a_wide_batch(mesa, oracle_mod):
    """More heads than the step kernel has CTAs (two per SM), and a count that
    is not a multiple of them: the CTAs walk the heads, so every head, the
    last ones included, is checked against the oracle over a few steps."""
    H = 17
    B = 2 * torch.cuda.get_device_properties(0).multi_processor_count // H + 2     # 323 heads on 148 SMs
    w = mi.Workload("walk", B, H, 12, 32, 32, 16, "f32", 15, 0.0, False, 77)
    x = mi.batch(w)
    t0 = 8
    _, _, Hs, Gs = oracle_mod.forward_cg(*(x[n][:, :, :t0] for n in ("q", "k", "v", "gamma", "beta")), x["lam"], 15)
    Hg, Gg = cuda(Hs), cuda(Gs)
    lam = cuda(x["lam"])
    for t in range(t0, w.T):
        ref, _, Hs, Gs = oracle_mod.step(*(x[n][:, :, t] for n in ("q", "k", "v", "gamma", "beta")), x["lam"],
                                         Hs, Gs, 15, 0.0)
        out = mesa.step(*(cuda(x[n][:, :, t]) for n in ("q", "k", "v", "gamma", "beta")), lam, Hg, Gg, cg_steps=15)
        torch.cuda.synchronize()
        o = out.cpu().numpy()
        for b in range(B):                             # every head on its own
            for h in range(H):
                assert rel_err(o[b, h], ref[b, h]) <= TOL_F32, (t, b, h)
    assert np.allclose(Hg.cpu().numpy(), Hs, rtol=1e-4, atol=1e-5)
    assert np.allclose(Gg.cpu().numpy(), Gs, rtol=1e-4, atol=1e-5)
    assert mesa.get_error() == 0


def test_decode_equals_forward_on_gpu(mesa):
    """T single steps from a zero state reproduce the chunkwise forward (fp32)."""
    w = mi.Workload("t", 1, 4, 48, 64, 64, 16, "f32", 12, 0.0, False, 5)
    x = mi.batch(w)
    d = {n: cuda(x[n]) for n in ("q", "k", "v", "gamma", "beta", "lam")}
    ref, Hf, Gf = mesa.forward(d["q"], d["k"], d["v"], d["gamma"], d["beta"], d["lam"], chunk=16, cg_steps=12,
                               return_state=True)
    Hs = torch.zeros((1, 4, 64, 64), device="cuda")
    Gs = torch.zeros((1, 4, 64, 64), device="cuda")
    outs = []
    for t in range(48):
        outs.append(mesa.step(*(d[n][:, :, t].contiguous() for n in ("q", "k", "v", "gamma", "beta")), d["lam"],
                              Hs, Gs, cg_steps=12).clone())
    got = torch.stack(outs, 2).cpu().numpy()
    assert rel_err(got, ref.cpu().numpy()) <= TOL_F32
    assert torch.allclose(Hs, Hf, rtol=1e-5, atol=1e-6) and torch.allclose(Gs, Gf, rtol=1e-5, atol=1e-6)


def test_full_size_decode_sampled(mesa, oracle_mod):
    """The decode workload: 256 x 16 heads, d = 128, 4096-token prefill, then
    its 1000 successive single-token steps; sampled heads against the oracle
    at every step (the fp32 state is updated 1000 times in place)."""
    w = mi.WORKLOADS["decode"]
    steps = w.decode_steps
    T = w.T + steps
    pairs = [(0, 0), (w.B - 1, w.H - 1), (100, 7)]
    Hs = torch.empty((w.B, w.H, w.dk, w.dk), device="cuda")
    Gs = torch.empty((w.B, w.H, w.dv, w.dk), device="cuda")
    dec = {}
    slab = 32
    for b0 in range(0, w.B, slab):
        dev = mi.device_batch(w, "cuda", T=T, B=slab, seed_offset=b0)
        local = [(b - b0, h) for (b, h) in pairs if b0 <= b < b0 + slab]
        if local:
            host = mi.batch(w, T=T, seqs=[(b + b0, h) for (b, h) in local])
            for i, (bl, h) in enumerate(local):
                for n in ("q", "k", "v"):
                    dev[n][bl, h].copy_(torch.from_numpy(host[n][0, i]).to(dev[n].dtype))
                dev["gamma"][bl, h].copy_(torch.from_numpy(host["gamma"][0, i]))
                dev["beta"][bl, h].copy_(torch.from_numpy(host["beta"][0, i]))
        pre = {n: dev[n][:, :, :w.T].contiguous() for n in ("q", "k", "v", "gamma", "beta")}
        _, Hp, Gp = mesa.forward(pre["q"], pre["k"], pre["v"], pre["gamma"], pre["beta"], dev["lam"], chunk=64,
                                 cg_steps=w.cg_steps, return_state=True)
        Hs[b0:b0 + slab].copy_(Hp)
        Gs[b0:b0 + slab].copy_(Gp)
        for n in ("q", "k", "v", "gamma", "beta"):
            dec.setdefault(n, []).append(dev[n][:, :, w.T:].float())
        del dev, pre, Hp, Gp
    dec = {n: torch.cat(v, 0) for n, v in dec.items()}
    lam = torch.from_numpy(mi.lambdas(w.seed, w.H, w.dk)).cuda()
    outs = []
    for s in range(steps):
        o = mesa.step(*(dec[n][:, :, s].contiguous() for n in ("q", "k", "v", "gamma", "beta")), lam, Hs, Gs,
                      cg_steps=w.cg_steps)
        outs.append(o[[b for b, _ in pairs], [h for _, h in pairs]].clone())
    torch.cuda.synchronize()
    assert mesa.get_error() == 0
    got = torch.stack(outs, 1).cpu().numpy()          # [pairs, steps, dv]
    host = mi.batch(w, T=T, seqs=pairs)
    _, _, Ho, Go = oracle_mod.forward_cg(*(host[n][:, :, :w.T] for n in ("q", "k", "v", "gamma", "beta")),
                                         host["lam"], w.cg_steps)
    refs = []
    for s in range(steps):
        r, _, Ho, Go = oracle_mod.step(*(host[n][:, :, w.T + s] for n in ("q", "k", "v", "gamma", "beta")),
                                       host["lam"], Ho, Go, w.cg_steps)
        refs.append(r[0])
    ref = np.stack(refs, 1)
    # the prefill runs in bf16-input mode; the steps themselves are fp32
    rep = log_parity("decode_1000_steps", got, ref)
    assert rep["rel"] <= 2e-3, rep
    # the last 100 steps alone: no drift of the state over the 1000 updates
    late = log_parity("decode_steps_900_999", got[:, -100:], ref[:, -100:])
    assert late["rel"] <= 2e-3, late


@pytest.mark.parametrize("d", [16, 64, 128])
@pytest.mark.parametrize("tol", [0.0, 1e-3])
def test_warm_steps_match_oracle(mesa, oracle_mod, d, tol):
    """mesa_step_warm carrying x between steps (each solve starts from the
    previous step's solution) against oracle_step_warm, step by step."""
    w = mi.Workload("t", 2, 3, 24, d, d, 16, "f32", 15, tol, tol > 0, 61 + d)
    x = mi.batch(w)
    t0 = 8
    N = 30 if tol > 0 else 4                     # few steps: the start matters for the result
    _, _, Hs, Gs = oracle_mod.forward_cg(*(x[n][:, :, :t0] for n in ("q", "k", "v", "gamma", "beta")), x["lam"], N, tol)
    Hg = torch.from_numpy(Hs).float().cuda()
    Gg = torch.from_numpy(Gs).float().cuda()
    xs_ref = np.zeros((2, 3, d))
    xs = torch.zeros((2, 3, d), device="cuda")
    lam = torch.from_numpy(x["lam"]).float().cuda()
    iters = torch.empty((2, 3), dtype=torch.int32, device="cuda")
    for t in range(t0, w.T):
        step_in = [x[n][:, :, t] for n in ("q", "k", "v", "gamma", "beta")]
        ref, it_ref, Hs, Gs, xs_ref = oracle_mod.step(*step_in, x["lam"], Hs, Gs, N, tol, x_state=xs_ref)
        o = mesa.step(*(torch.from_numpy(np.ascontiguousarray(a)).float().cuda() for a in step_in), lam, Hg, Gg,
                      cg_steps=N, tol=tol, iters=iters, x_state=xs)
        torch.cuda.synchronize()
        # with a tolerance an iteration count may differ by one, which moves the result by ~tol
        bound = TOL_F32 if tol == 0 else 2e-2
        assert rel_err(o.cpu().numpy(), ref) <= bound, (t, err_report(o.cpu().numpy(), ref))
        assert rel_err(xs.cpu().numpy(), xs_ref) <= bound, t
        if tol == 0:
            assert np.all(iters.cpu().numpy() == N)
        else:
            assert np.abs(iters.cpu().numpy() - it_ref).max() <= 1
    assert mesa.get_error() == 0


def test_warm_step_from_zero_equals_cold_step(mesa):
    """x_state = 0 gives exactly mesa_step, and x_state receives the solution."""
    B, H, d = 4, 16, 128
    g = torch.Generator(device="cuda").manual_seed(3)
    kr = torch.nn.functional.normalize(torch.randn((B, H, 32, d), generator=g, device="cuda"), dim=-1)
    Hs = kr.transpose(-1, -2) @ kr
    Gs = torch.randn((B, H, 32, d), generator=g, device="cuda").transpose(-1, -2) @ kr
    q = torch.nn.functional.normalize(torch.randn((B, H, d), generator=g, device="cuda"), dim=-1)
    k = torch.nn.functional.normalize(torch.randn((B, H, d), generator=g, device="cuda"), dim=-1)
    v = torch.randn((B, H, d), generator=g, device="cuda")
    gam = torch.full((B, H), 0.9, device="cuda")
    bet = torch.full((B, H), 0.5, device="cuda")
    lam = torch.full((H, d), 0.3, device="cuda")
    H1, G1, H2, G2 = Hs.clone(), Gs.clone(), Hs.clone(), Gs.clone()
    o1 = mesa.step(q, k, v, gam, bet, lam, H1, G1, cg_steps=15)
    xs = torch.zeros((B, H, d), device="cuda")
    o2 = mesa.step(q, k, v, gam, bet, lam, H2, G2, cg_steps=15, x_state=xs)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(H1, H2) and torch.equal(G1, G2)
    assert torch.allclose(torch.einsum("bhij,bhj->bhi", G2, xs), o2, rtol=1e-5, atol=1e-5)
