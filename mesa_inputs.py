"""Seeded synthetic inputs for the Mesa layer (shared by tests, bench, smoke).

This module holds none of the layer's arithmetic: it only draws random
tensors with the shapes and distributions of the workloads below, so the CUDA
path and the CPU oracle can be fed identical bits.

Recipe (every workload):
  * Each (b, h) sequence has its own numpy PCG64 stream, keyed by
    SeedSequence([seed, b, h]); Lambda has its own stream keyed by
    SeedSequence([seed, 0x4C414D42]). A sampled sequence can therefore be
    regenerated alone, bit for bit.
  * Draw order inside a sequence stream (all standard normal, float32):
    q [T, dk], k [T, dk], v [T, dv], gamma-logits [T], beta-logits [T], then
    (mixture workloads only) a uniform coin [T].
  * q and k are L2-normalised per token; v is used as drawn.
  * gamma = sigmoid(z + 3) (z the gamma-logit); mixture workloads use
    sigmoid(z + 5) where coin < 0.5, else sigmoid(z), so per-token decay (and
    therefore the CG iteration count) varies widely.
  * beta = sigmoid(z); lambda = softplus(z) + 0.1 per head and key channel.
  * bf16 workloads round q, k, v to bf16 (round to nearest even) after the
    normalisation; gamma, beta, lambda stay float32.

The shapes mirror language-model layers (the MesaNet pages give no head
dimension or head count; 16 heads of width 128 at 2k-8k context are used).
No dataset is read: the pages' SlimPajama training text is stood in for by
these seeded tensors.
"""
from __future__ import annotations

import dataclasses

import numpy as np

LAMBDA_STREAM = 0x4C414D42


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    T: int
    dk: int
    dv: int
    chunk: int
    dtype: str          # "f32" or "bf16": element type of q, k, v
    cg_steps: int
    tol: float
    mixture: bool
    seed: int
    decode_steps: int = 0   # >0: recurrent decode workload (T tokens of prefill first)

    @property
    def tokens(self) -> int:
        return self.B * self.H * self.T


WORKLOADS = {
    # tiny fp32 forward, CG run to d steps (exact in exact arithmetic)
    "tiny_fp32": Workload("tiny_fp32", 1, 1, 64, 16, 16, 16, "f32", 16, 0.0, False, 0),
    # bf16 forward, T=2048
    "bf16_T2048": Workload("bf16_T2048", 8, 16, 2048, 128, 128, 64, "bf16", 15, 0.0, False, 1),
    # long-context bf16 forward, T=8192 (the throughput workload)
    "bf16_T8192": Workload("bf16_T8192", 8, 16, 8192, 128, 128, 64, "bf16", 15, 0.0, False, 2),
    # tolerance-stopped bf16 forward with a 50/50 decay mixture
    "bf16_T8192_tol": Workload("bf16_T8192_tol", 4, 16, 8192, 128, 128, 64, "bf16", 30, 1e-3, True, 3),
    # recurrent decode: 4096-token prefill, then 1000 single-token steps
    "decode": Workload("decode", 256, 16, 4096, 128, 128, 64, "bf16", 15, 0.0, False, 4, decode_steps=1000),
}


def bf16_round(x: np.ndarray) -> np.ndarray:
    """Round float32 to the nearest bf16 (ties to even), returned as float32."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    b = x.view(np.uint32).astype(np.uint64)
    r = ((b + 0x7FFF + ((b >> 16) & 1)) >> 16) << 16
    out = r.astype(np.uint32).view(np.float32)
    # keep NaN as NaN (rounding could carry into the exponent of a NaN payload)
    return np.where(np.isnan(x), x, out)


def _sigmoid(z):
    return (1.0 / (1.0 + np.exp(-z.astype(np.float64)))).astype(np.float32)


def _softplus(z):
    return np.log1p(np.exp(z.astype(np.float64))).astype(np.float32)


def _l2n(x):
    n = np.sqrt((x.astype(np.float64) ** 2).sum(-1, keepdims=True))
    return (x / n).astype(np.float32)


def sequence(seed: int, b: int, h: int, T: int, dk: int, dv: int, mixture: bool, dtype: str):
    """One (b, h) sequence: dict of float32 arrays q[T,dk], k[T,dk], v[T,dv], gamma[T], beta[T]."""
    rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, b, h])))
    q = rng.standard_normal((T, dk), dtype=np.float32)
    k = rng.standard_normal((T, dk), dtype=np.float32)
    v = rng.standard_normal((T, dv), dtype=np.float32)
    zg = rng.standard_normal(T, dtype=np.float32)
    zb = rng.standard_normal(T, dtype=np.float32)
    if mixture:
        coin = rng.random(T, dtype=np.float32)
        gamma = np.where(coin < 0.5, _sigmoid(zg + 5.0), _sigmoid(zg))
    else:
        gamma = _sigmoid(zg + 3.0)
    beta = _sigmoid(zb)
    q, k = _l2n(q), _l2n(k)
    if dtype == "bf16":
        q, k, v = bf16_round(q), bf16_round(k), bf16_round(v)
    return dict(q=q, k=k, v=v, gamma=gamma.astype(np.float32), beta=beta)


def lambdas(seed: int, H: int, dk: int) -> np.ndarray:
    rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, LAMBDA_STREAM])))
    return (_softplus(rng.standard_normal((H, dk), dtype=np.float32)) + np.float32(0.1)).astype(np.float32)


def batch(w: Workload, T: int | None = None, B: int | None = None, H: int | None = None,
          seqs=None):
    """Stacked inputs as float32 numpy arrays [B,H,T,*] (values bf16-exact for bf16
    workloads). ``seqs`` optionally restricts to a list of (b, h) pairs, returned
    as B=1 with one pseudo-head per pair (H=len(seqs)) and the matching lambda
    rows."""
    T = w.T + w.decode_steps if T is None else T
    B = w.B if B is None else B
    H = w.H if H is None else H
    lam = lambdas(w.seed, w.H, w.dk)
    pairs = [(b, h) for b in range(B) for h in range(H)] if seqs is None else list(seqs)
    n = len(pairs)
    q = np.empty((n, T, w.dk), np.float32)
    k = np.empty((n, T, w.dk), np.float32)
    v = np.empty((n, T, w.dv), np.float32)
    g = np.empty((n, T), np.float32)
    be = np.empty((n, T), np.float32)
    for i, (b, h) in enumerate(pairs):
        s = sequence(w.seed, b, h, T, w.dk, w.dv, w.mixture, w.dtype)
        q[i], k[i], v[i], g[i], be[i] = s["q"], s["k"], s["v"], s["gamma"], s["beta"]
    if seqs is None:
        shp = (B, H, T)
        return dict(q=q.reshape(*shp, w.dk), k=k.reshape(*shp, w.dk), v=v.reshape(*shp, w.dv),
                    gamma=g.reshape(shp), beta=be.reshape(shp), lam=lam[:H].copy())
    # sampled sequences as one batch row with one pseudo-head per sequence,
    # each carrying the lambda row of its own head
    lam_rows = np.stack([lam[h] for (_, h) in pairs])
    return dict(q=q[None], k=k[None], v=v[None], gamma=g[None], beta=be[None], lam=lam_rows)


def device_batch(w: Workload, device, T: int | None = None, B: int | None = None,
                 H: int | None = None, seed_offset: int = 0):
    """The same distributions drawn on the device with a seeded torch generator
    (for full-size runs where drawing every sequence on the host is too slow).
    Returns torch tensors: q, k, v in the workload dtype, gamma, beta, lam float32."""
    import torch
    T = w.T + w.decode_steps if T is None else T
    B = w.B if B is None else B
    H = w.H if H is None else H
    g = torch.Generator(device=device)
    g.manual_seed(1_000_003 * w.seed + seed_offset)
    f32 = torch.float32
    q = torch.randn((B, H, T, w.dk), generator=g, device=device, dtype=f32)
    k = torch.randn((B, H, T, w.dk), generator=g, device=device, dtype=f32)
    v = torch.randn((B, H, T, w.dv), generator=g, device=device, dtype=f32)
    zg = torch.randn((B, H, T), generator=g, device=device, dtype=f32)
    zb = torch.randn((B, H, T), generator=g, device=device, dtype=f32)
    if w.mixture:
        coin = torch.rand((B, H, T), generator=g, device=device, dtype=f32)
        gamma = torch.where(coin < 0.5, torch.sigmoid(zg + 5.0), torch.sigmoid(zg))
    else:
        gamma = torch.sigmoid(zg + 3.0)
    beta = torch.sigmoid(zb)
    q = q / q.norm(dim=-1, keepdim=True)
    k = k / k.norm(dim=-1, keepdim=True)
    dt = torch.bfloat16 if w.dtype == "bf16" else f32
    lam = torch.from_numpy(lambdas(w.seed, w.H, w.dk)[:H].copy()).to(device)
    return dict(q=q.to(dt), k=k.to(dt), v=v.to(dt), gamma=gamma.contiguous(), beta=beta.contiguous(), lam=lam)


def plant_sequences(dev: dict, w: Workload, pairs, T: int | None = None):
    """Overwrites the (b, h) sequences listed in ``pairs`` of a device batch with
    their host per-sequence streams, so those sequences match ``batch(w, seqs=pairs)``."""
    import torch
    T = dev["q"].shape[2] if T is None else T
    host = batch(w, T=T, seqs=pairs)
    dt = dev["q"].dtype
    for i, (b, h) in enumerate(pairs):
        for name in ("q", "k", "v"):
            dev[name][b, h].copy_(torch.from_numpy(host[name][0, i]).to(dt))
        dev["gamma"][b, h].copy_(torch.from_numpy(host["gamma"][0, i]))
        dev["beta"][b, h].copy_(torch.from_numpy(host["beta"][0, i]))
    return host


DOUT_STREAM = 0x444F5554


def dout(seed: int, B: int, H: int, T: int, dv: int, seqs=None) -> np.ndarray:
    """Upstream gradient dL/do for backward runs: standard normal float32,
    one stream per (b, h) keyed by SeedSequence([seed, DOUT_STREAM, b, h]).
    Shape [B,H,T,dv], or [1,len(seqs),T,dv] for a list of (b, h) pairs."""
    pairs = [(b, h) for b in range(B) for h in range(H)] if seqs is None else list(seqs)
    out = np.empty((len(pairs), T, dv), np.float32)
    for i, (b, h) in enumerate(pairs):
        rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, DOUT_STREAM, b, h])))
        out[i] = rng.standard_normal((T, dv), dtype=np.float32)
    return out.reshape(B, H, T, dv) if seqs is None else out[None]
