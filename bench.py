#!/usr/bin/env python
"""Throughput benchmark of the Mesa layer forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

One "step" is one mesa_forward over the whole workload (all tokens of every
(b, h) sequence), with inputs resident in HBM. The default workload is the
long-context bf16 forward (B=8, H=16, T=8192, d=128, chunk 64, 15 CG steps).
Under torchrun every rank runs its own copy of the workload on its own GPU
(sequences are independent: weak scaling, no data-path collective); the
timed region is bracketed by a barrier and a device synchronisation, and the
slowest rank's time is reported. Rank 0 prints one JSON line.

--impl reference times the fp64 CPU oracle on the host cores instead (rank 0
only), each step on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import datetime
import json
import os
import statistics
import subprocess
import tempfile
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import mesa_inputs as mi  # noqa: E402

# fp32 FMA peak on CUDA cores: 148 SMs x 128 FMA/clk x 2 flop x 1.965 GHz.
SIMT_FP32_PEAK_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        d["_source"] = "measured"
        return d
    d = dict(FALLBACK_PEAKS)
    d["_source"] = "fallback"
    return d


# DRAM bytes moved per token (per head for the decode step) by each kernel, from
# one ncu capture of that kernel on a small case of its workload
# (dram__bytes_read.sum + dram__bytes_write.sum of one launch / units of that launch).
# Reported only while the kernel source still hashes to the captured version;
# otherwise the field is null.
MEASURED_TRAFFIC = {
    "tc_cg": {"src_sha16": "e4bafe8b775e8e79",
              "files": ("tc_forward.cu", "tc_layout.cuh", "tc_common.cuh", "preproc_row.cuh"),
              "bytes_per_token": (337.756672e6 + 109.066752e6) / 262144},
    "tc_scan": {"src_sha16": "7e35aa166da95c08",
                "files": ("tc_scan.cu", "tc_layout.cuh", "tc_common.cuh", "preproc_row.cuh"),
                "bytes_per_token": (136.395520e6 + 91.302400e6) / 262144},
    "preprocess": {"src_sha16": "49bdcb4b9d87fc99", "files": ("preprocess.cu", "preproc_row.cuh"),
                   "bytes_per_token": (536.979456e6 + 489.550848e6) / 1048576},
    "decode_step": {"src_sha16": "6e6713cd01e91c39", "files": ("decode.cu", "tc_common.cuh"),
                    "bytes_per_token": (543.233792e6 + 478.705664e6) / 4096},
}


def kernel_source_sha16(files):
    """Hash of the release kernel source: MESA_DEBUG blocks (compiled only into
    the debug library) are left out."""
    import hashlib
    import re
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, "test_sequence_layer_b200", "csrc", f)) as fh:
            src = re.sub(r"#ifdef MESA_DEBUG.*?#endif\n?", "", fh.read(), flags=re.S)
        h.update(src.encode())
    return h.hexdigest()[:16]


def measured_traffic(kernel, units):
    """Measured DRAM bytes of one launch processing `units` tokens (heads for
    the decode step), or None when the source changed since the capture."""
    rec = MEASURED_TRAFFIC.get(kernel)
    if rec is None or rec["src_sha16"] != kernel_source_sha16(rec["files"]):
        return None
    return rec["bytes_per_token"] * units


def flops_per_token_iter(d, C):
    """Useful causal flops of one CG matvec per token: inter-chunk 2d^2 plus
    the masked intra-chunk scores and their read-back, 2d(C+1)."""
    return 2 * d * d + 2 * d * (C + 1)


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms."""
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        # raw samples of the timed region, kept beside the JSON line's summary
        self.path = os.path.join(tempfile.gettempdir(), f"mesa_bench_clocks_rank{index}.csv")

    def start(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.QUERY}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
            return
        # the first sample lands before the timed region starts (the GPU is busy
        # with the warm-up), so that a region shorter than the sampling period
        # still has one
        t0 = time.perf_counter()
        while time.perf_counter() - t0 < 3.0 and self.proc.poll() is None:
            self.f.flush()
            if os.path.getsize(self.path) > 0:
                break
            time.sleep(0.02)

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.f.close()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for n, val in zip(names, parts[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


def max_over_ranks(value, world, device):
    """Slowest rank's value (the benchmark's clock for N > 1); identity for N = 1."""
    if world <= 1:
        return float(value)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_rank, world, ms):
    """Weak scaling: every rank processes `units_per_rank` in `ms` (slowest rank)."""
    return world * units_per_rank / (ms / 1e3)


def cpu_oracle_sample(w, n_seq, T_s):
    """Times the oracle on n_seq sequences x T_s tokens of workload w; returns tokens/s."""
    import oracle
    oracle.build()
    pairs = [(i // w.H, i % w.H) for i in range(n_seq)]
    x = mi.batch(w, T=T_s, seqs=pairs)
    t0 = time.perf_counter()
    oracle.forward_cg(x["q"], x["k"], x["v"], x["gamma"], x["beta"], x["lam"], w.cg_steps, w.tol)
    dt = time.perf_counter() - t0
    return n_seq * T_s / dt, dt


def host_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def run_reference(args, w, rank):
    if rank != 0:
        return
    cores = host_cores()
    os.environ.setdefault("OMP_NUM_THREADS", str(cores))
    n_seq, T_s = min(cores, w.B * w.H), 256
    rates = []
    for s in range(args.warmup + args.steps):
        rate, _ = cpu_oracle_sample(w, n_seq, T_s)
        if s >= args.warmup:
            rates.append(rate)
    value = statistics.median(rates)
    sample = f"{n_seq} sequences x first {T_s} tokens of {w.name} per step (OpenMP over sequences)"
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * n_seq * T_s / value,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "H": w.H, "T": w.T, "d": w.dk, "chunk": w.chunk,
                   "cg_steps": w.cg_steps, "tol": w.tol},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


METRIC = "Mesa-layer fwd tokens/s (B*H*T) at T=8192,d=128,15 CG steps; % tensor peak"
DECODE_METRIC = "Mesa decode tokens/s (sequences x heads per mesa_step), d=128, 15 CG steps; % HBM peak"
BWD_METRIC = "Mesa-layer bwd tokens/s (B*H*T): implicit-differentiation backward, d=128, 15 CG steps; % of the dominant kernel's peak"
PRE_METRIC = "Mesa input preprocessing tokens/s (q and k: causal depthwise conv, window 4, + L2 norm); % HBM peak"


def run_decode(args, w, world, rank, local):
    """Recurrent decode: a 4096-token prefill through mesa_forward's final
    state, then timed mesa_step calls (one new token for every head)."""
    import torch
    import torch.distributed as dist
    from test_sequence_layer_b200 import build as mbuild, mesa
    mbuild.build()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=dev)
    B, H, d = w.B, w.H, w.dk
    steps_total = args.warmup + args.steps
    Hs = torch.empty((B, H, d, d), device=dev)
    Gs = torch.empty((B, H, d, d), device=dev)
    dec = {n: [] for n in ("q", "k", "v", "gamma", "beta")}
    slab = 32
    if args.decode_state == "random":
        # Seeded stand-in for a prefilled state (rank-32 sums of the same gated
        # outer products), for profiling the step kernel without the 13 GB prefill.
        g = torch.Generator(device=dev).manual_seed(77 + rank)
        for b0 in range(0, B, slab):
            kr = torch.nn.functional.normalize(torch.randn((slab, H, 32, d), generator=g, device=dev), dim=-1)
            vr = torch.randn((slab, H, 32, d), generator=g, device=dev)
            br = torch.sigmoid(torch.randn((slab, H, 32, 1), generator=g, device=dev))
            Hs[b0:b0 + slab] = (kr * br).transpose(-1, -2) @ kr
            Gs[b0:b0 + slab] = (vr * br).transpose(-1, -2) @ kr
            x = mi.device_batch(w, dev, T=steps_total, B=slab, seed_offset=1000 * rank + b0)
            for n in dec:
                dec[n].append(x[n].float())
            del x
    for b0 in (range(0, B, slab) if args.decode_state == "prefill" else ()):
        x = mi.device_batch(w, dev, T=w.T + steps_total, B=slab, seed_offset=1000 * rank + b0)
        _, Hp, Gp = mesa.forward(*(x[n][:, :, :w.T].contiguous() for n in ("q", "k", "v", "gamma", "beta")),
                                 x["lam"], chunk=w.chunk, cg_steps=w.cg_steps, return_state=True)
        Hs[b0:b0 + slab].copy_(Hp)
        Gs[b0:b0 + slab].copy_(Gp)
        for n in dec:
            dec[n].append(x[n][:, :, w.T:].float())
        del x, Hp, Gp
    dec = {n: torch.cat(v, 0) for n, v in dec.items()}
    # one contiguous [steps, B, H, ...] block per input, resident before timing
    tok = {n: dec[n].movedim(2, 0).contiguous() for n in dec}
    del dec
    if args.query_walk > 0:
        # correlated query stream (stand-in for consecutive queries of a language model):
        # q_s = normalise(q_{s-1} + sigma * eps_s), eps seeded
        gq = torch.Generator(device=dev).manual_seed(91 + rank)
        qw = tok["q"]
        for s_ in range(1, qw.shape[0]):
            nxt = qw[s_ - 1] + args.query_walk * torch.randn(qw[s_].shape, generator=gq, device=dev)
            qw[s_] = nxt / nxt.norm(dim=-1, keepdim=True)
    tol = w.tol if args.tol is None else args.tol
    xs = torch.zeros((B, H, d), device=dev) if args.warm_start else None
    its = torch.zeros((steps_total, B, H), dtype=torch.int32, device=dev)
    lam = torch.from_numpy(mi.lambdas(w.seed, w.H, w.dk)).to(dev)
    out = torch.empty((B, H, d), device=dev)
    stream = torch.cuda.current_stream(dev)
    for s in range(args.warmup):
        mesa.step(tok["q"][s], tok["k"][s], tok["v"][s], tok["gamma"][s], tok["beta"][s], lam, Hs, Gs,
                  cg_steps=w.cg_steps, tol=tol, out=out, iters=its[s], x_state=xs, stream=stream)
    torch.cuda.synchronize()
    assert mesa.get_error(stream) == 0
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.4)
    mesa.timing_enable(True)
    mesa.timing_read()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    ev0.record(stream)
    for s in range(args.warmup, steps_total):
        mesa.step(tok["q"][s], tok["k"][s], tok["v"][s], tok["gamma"][s], tok["beta"][s], lam, Hs, Gs,
                  cg_steps=w.cg_steps, tol=tol, out=out, iters=its[s], x_state=xs, stream=stream)
    ev1.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    mesa.timing_enable(False)
    kernels = mesa.timing_read()
    clk = clocks.stop()
    ms = max_over_ranks(ev0.elapsed_time(ev1), world, dev)
    if world > 1:
        dist.destroy_process_group()
    assert mesa.get_error(stream) == 0
    if rank != 0:
        return
    heads = B * H
    launches, kms = kernels["decode_step"]
    avg_ms = kms / launches
    # state read + write (H and G, fp32) plus q, k, v, gamma, beta in and out per head
    bytes_per_launch = heads * (4 * d * d * 4 + (3 * d + 2) * 4 + d * 4)
    peaks = load_peaks()
    achieved = bytes_per_launch / (avg_ms / 1e3) / 1e9
    line = {
        "metric": DECODE_METRIC, "value": whole_job_rate(heads * args.steps, world, ms), "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": w.name, "sequences": B, "H": H, "d": d, "prefill_tokens": w.T,
                   "cg_steps": w.cg_steps, "tol": tol, "warm_start": bool(args.warm_start),
                   "query_walk": args.query_walk,
                   "mean_cg_iters": float(its[args.warmup:].float().mean().item()), "state": args.decode_state,
                   "l2": "state larger than L2 (%.2f GB)" % (2 * Hs.numel() * 4 / 1e9)},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": achieved / peaks["hbm_gbs"], "traffic": measured_traffic("decode_step", heads),
                     "kernel": "decode_step",
                     "avg_ms": avg_ms, "peak_kind": f"{peaks['_source']} HBM copy bandwidth"},
        "kernels": {k: {"launches": v[0], "total_ms": v[1]} for k, v in kernels.items()},
        "gpu_launches": sum(v[0] for v in kernels.values()),
        "clocks": clk, "e2e": None, "cpu_baseline": None,
    }
    print(json.dumps(line), flush=True)


def run_preprocess(args, w, world, rank, local):
    """mesa_preprocess alone on the workload's shape: causal depthwise
    convolution (window 4) and per-token L2 normalisation of q and k."""
    import torch
    import torch.distributed as dist
    from test_sequence_layer_b200 import build as mbuild, mesa
    mbuild.build()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    B, H, T, d, W = w.B, w.H, w.T, w.dk, 4
    g = torch.Generator(device=dev).manual_seed(5 + rank)
    dt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    q_raw = torch.randn((B, H, T, d), generator=g, device=dev).to(dt)
    k_raw = torch.randn((B, H, T, d), generator=g, device=dev).to(dt)
    cq = torch.randn((H, W, d), generator=g, device=dev) / 2
    ck = torch.randn((H, W, d), generator=g, device=dev) / 2
    q_out, k_out = torch.empty_like(q_raw), torch.empty_like(k_raw)
    stream = torch.cuda.current_stream(dev)

    def step():
        mesa.preprocess(q_raw, k_raw, cq, ck, q_out=q_out, k_out=k_out, stream=stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.4)
    mesa.timing_enable(True)
    mesa.timing_read()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    ev0.record(stream)
    for _ in range(args.steps):
        step()
    ev1.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    mesa.timing_enable(False)
    kernels = mesa.timing_read()
    clk = clocks.stop()
    ms = max_over_ranks(ev0.elapsed_time(ev1), world, dev)
    if world > 1:
        dist.destroy_process_group()
    if rank != 0:
        return
    tokens = B * H * T
    launches, kms = kernels["preprocess"]
    avg_ms = kms / launches
    bytes_per_launch = 2 * 2 * tokens * d * q_raw.element_size()      # q and k, read and written
    peaks = load_peaks()
    achieved = bytes_per_launch / (avg_ms / 1e3) / 1e9
    line = {
        "metric": PRE_METRIC, "value": whole_job_rate(tokens, world, ms / args.steps), "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16-in/f32/bf16-out" if w.dtype == "bf16" else "f32", "data": "synthetic",
        "config": {"workload": w.name + "+preprocess", "B": B, "H": H, "T": T, "d": d, "window": W,
                   "l2": "inputs larger than L2 (%.2f GB per step)" % (2 * q_raw.numel() * q_raw.element_size() / 1e9)},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": achieved / peaks["hbm_gbs"], "traffic": measured_traffic("preprocess", tokens),
                     "kernel": "preprocess", "avg_ms": avg_ms,
                     "peak_kind": f"{peaks['_source']} HBM copy bandwidth"},
        "kernels": {k: {"launches": v[0], "total_ms": v[1]} for k, v in kernels.items()},
        "gpu_launches": sum(v[0] for v in kernels.values()),
        "clocks": clk, "e2e": None, "cpu_baseline": None,
    }
    print(json.dumps(line), flush=True)


def run_fused_preprocess(args, w, world, rank, local):
    """The forward with the q/k preprocessing folded into its staged loads
    (mesa_forward_preprocessed) on the workload, from raw q and k (window 4).
    Also times, on the same inputs, the plain forward of already-preprocessed
    q and k, and the two-step path (mesa_preprocess, then mesa_forward), so the
    cost of the preprocessing inside the forward reads off directly."""
    import torch
    import torch.distributed as dist
    from test_sequence_layer_b200 import build as mbuild, mesa
    mbuild.build()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    x = mi.device_batch(w, dev, seed_offset=rank)
    B, H, T, d, C, W = w.B, w.H, w.T, w.dk, w.chunk, 4
    g = torch.Generator(device=dev).manual_seed(5 + rank)
    q_raw = torch.randn((B, H, T, d), generator=g, device=dev).to(x["q"].dtype)
    k_raw = torch.randn((B, H, T, d), generator=g, device=dev).to(x["q"].dtype)
    cq = torch.randn((H, W, d), generator=g, device=dev) / 2
    ck = torch.randn((H, W, d), generator=g, device=dev) / 2
    q_pre, k_pre = torch.empty_like(q_raw), torch.empty_like(k_raw)
    out = torch.empty((B, H, T, d), device=dev)
    ws = torch.empty(max(mesa.workspace_size(B, H, T, d, d, C, x["q"].dtype), 1), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    kw = dict(chunk=C, cg_steps=w.cg_steps, tol=w.tol, out=out, workspace=ws, stream=stream)

    def fused():
        mesa.forward_preprocessed(q_raw, k_raw, x["v"], x["gamma"], x["beta"], x["lam"], cq, ck, **kw)

    def plain():
        mesa.forward(q_pre, k_pre, x["v"], x["gamma"], x["beta"], x["lam"], **kw)

    def two_step():
        mesa.preprocess(q_raw, k_raw, cq, ck, q_out=q_pre, k_out=k_pre, stream=stream)
        plain()

    def timed(fn):
        for _ in range(args.warmup):
            fn()
        torch.cuda.synchronize()
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        ev0.record(stream)
        for _ in range(args.steps):
            fn()
        ev1.record(stream)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        return max_over_ranks(ev0.elapsed_time(ev1), world, dev) / args.steps

    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.4)
    mesa.timing_enable(True)
    mesa.timing_read()
    ms_two = timed(two_step)            # also leaves q_pre, k_pre for the plain forward
    k_two = mesa.timing_read()
    ms_plain = timed(plain)
    k_plain = mesa.timing_read()
    ms_fused = timed(fused)
    kernels = mesa.timing_read()
    mesa.timing_enable(False)
    clk = clocks.stop()
    assert mesa.get_error(stream) == 0
    if world > 1:
        dist.destroy_process_group()
    if rank != 0:
        return
    tokens = B * H * T
    per = lambda ks: {k: {"launches": v[0], "total_ms": v[1]} for k, v in ks.items()}    # noqa: E731
    line = {
        "metric": "Mesa-layer fwd tokens/s (B*H*T) from raw q, k with the input preprocessing folded into the "
                  "forward's loads",
        "value": whole_job_rate(tokens, world, ms_fused), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_fused, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16-in/f16-mma/f32-acc" if w.dtype == "bf16" else "f32", "data": "synthetic",
        "config": {"workload": w.name + "+fused-preprocess", "B": B, "H": H, "T": T, "d": d, "chunk": C,
                   "cg_steps": w.cg_steps, "window": W, "l2": "inputs larger than L2"},
        "fused": {"ms_per_step": ms_fused, "kernels": per(kernels)},
        "plain_forward": {"ms_per_step": ms_plain, "kernels": per(k_plain)},
        "preprocess_then_forward": {"ms_per_step": ms_two, "kernels": per(k_two)},
        "roofline": None, "gpu_launches": sum(v[0] for v in kernels.values()),
        "clocks": clk, "e2e": None, "cpu_baseline": None,
    }
    print(json.dumps(line), flush=True)


# Useful flops per token of each backward kernel (d, chunk C, N CG steps):
# a CG matvec or a read-out-shaped product counts 2d^2 + 2d(C+1) (the causal
# intra-chunk terms j <= t only), a chunk-state update 2 d^2 per matrix.
def bwd_flops_per_token(d, C, N, tc):
    mv = 2 * d * d + 2 * d * (C + 1)
    fl = {"simt_scan": 4 * d * d, "simt_cg": N * mv, "bwd_adjoint": (N + 2) * mv,
          "bwd_rscan": 4 * d * d, "bwd_grad": 8 * d * d + 8 * d * (C + 1)}
    if tc:    # tensor-core shape: the forward solve with its read-out, the right-hand sides, adjoint CG + H x
        fl.update({"tc_scan": 4 * d * d, "tc_cg": (N + 1) * mv, "bwd_rhs": mv, "bwd_adjoint": (N + 1) * mv})
        del fl["simt_scan"], fl["simt_cg"]
    return fl


BWD_TENSOR_KERNELS = ("tc_scan", "tc_cg", "bwd_rhs", "bwd_adjoint")


def fp32_fma_peak_tflops(sm_mhz):
    """148 SMs x 128 fp32 lanes x 2 flops per FMA x clock."""
    return 148 * 128 * 2 * sm_mhz * 1e6 / 1e12


def run_backward(args, w, world, rank, local):
    """mesa_backward on the workload's shape with device-resident inputs and a
    seeded upstream gradient: forward solve, adjoint solve, reverse scan and
    gradient kernels. On the tensor-core shape the forward solve, the adjoint
    right-hand sides and the adjoint solve run on tcgen05; the reverse scans
    and gradient kernels are fp32 on the CUDA cores."""
    import torch
    import torch.distributed as dist
    from test_sequence_layer_b200 import build as mbuild, mesa
    mbuild.build()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    x = mi.device_batch(w, dev, seed_offset=rank)
    g = torch.Generator(device=dev).manual_seed(17 + rank)
    do = torch.randn((w.B, w.H, w.T, w.dv), generator=g, device=dev)
    ws = torch.empty(int(mesa._load().mesa_backward_workspace_size(w.B, w.H, w.T, w.dk, w.dv, w.chunk,
                                                                    1 if w.dtype == "bf16" else 0)),
                     dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    N = w.cg_steps

    def step():
        mesa.backward(x["q"], x["k"], x["v"], x["gamma"], x["beta"], x["lam"], do, chunk=w.chunk, cg_steps=N,
                      tol=w.tol, workspace=ws, stream=stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.4)
    mesa.timing_enable(True)
    mesa.timing_read()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    ev0.record(stream)
    for _ in range(args.steps):
        step()
    ev1.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    mesa.timing_enable(False)
    kernels = mesa.timing_read()
    clk = clocks.stop()
    assert mesa.get_error() == 0
    ms = max_over_ranks(ev0.elapsed_time(ev1), world, dev)
    if world > 1:
        dist.destroy_process_group()
    if rank != 0:
        return
    tokens = w.B * w.H * w.T
    tc = w.dtype == "bf16" and w.dk == 128 and w.dv == 128 and w.chunk == 64
    fl = bwd_flops_per_token(w.dk, w.chunk, N, tc)
    top = max((k for k in kernels if k in fl), key=lambda k: kernels[k][1])
    launches, kms = kernels[top]
    avg_ms = kms / launches
    achieved = fl[top] * tokens / (avg_ms / 1e3) / 1e12
    on_tensor = tc and top in BWD_TENSOR_KERNELS
    peaks = load_peaks()
    peak = peaks["bf16_tflops"] if on_tensor else fp32_fma_peak_tflops(1965.0)
    line = {
        "metric": BWD_METRIC, "value": whole_job_rate(tokens, world, ms / args.steps), "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": ("bf16-in/" if w.dtype == "bf16" else "") + "f32", "data": "synthetic",
        "config": {"workload": w.name + "+backward", "B": w.B, "H": w.H, "T": w.T, "d": w.dk, "chunk": w.chunk,
                   "cg_steps": N, "tol": w.tol, "flops_per_token": sum(fl.values()),
                   "l2": "inputs larger than L2 (%.2f GB per step)" % (
                       (3 * x["q"].numel() * x["q"].element_size() + do.numel() * 4) / 1e9)},
        "roofline": {"bound": "tensor" if on_tensor else "alu", "achieved": achieved, "peak": peak,
                     "unit": "TFLOP/s", "frac": achieved / peak, "traffic": None, "kernel": top, "avg_ms": avg_ms,
                     "peak_kind": (f"{peaks['_source']} bf16 dense burst (fp16 operands run at the bf16 rate)"
                                   if on_tensor else
                                   "derived fp32 FMA peak: 148 SMs x 128 lanes x 2 flop x 1965 MHz")},
        "kernels": {k: {"launches": v[0], "total_ms": v[1]} for k, v in kernels.items()},
        "gpu_launches": sum(v[0] for v in kernels.values()),
        "clocks": clk, "e2e": None, "cpu_baseline": None,
    }
    print(json.dumps(line), flush=True)


SHARD_METRIC = "Mesa-layer fwd tokens/s (B*H*T), sequence-sharded over ranks (each rank one slice of T); d=128, 15 CG steps"


def run_seq_sharded(args, w, world, rank, local):
    """Sequence-sharded forward: rank r holds tokens [r T/N, (r+1) T/N) of
    every sequence; per step one scan of the slice (mesa_chunk_state), one
    all-gather of the slice summaries, the prefix (mesa_state_prefix) and the
    slice's forward from that state. Total work is fixed as N grows."""
    import torch
    import torch.distributed as dist
    from test_sequence_layer_b200 import build as mbuild, mesa, sharded
    mbuild.build()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    Tr = w.T // world
    x = mi.device_batch(w, dev, T=Tr, seed_offset=rank)
    stream = torch.cuda.current_stream(dev)
    ws = torch.empty(mesa.workspace_size(w.B, w.H, Tr, w.dk, w.dv, w.chunk,
                                         torch.bfloat16 if w.dtype == "bf16" else torch.float32),
                     dtype=torch.uint8, device=dev)

    def step():
        sharded.forward_sequence_sharded(x["q"], x["k"], x["v"], x["gamma"], x["beta"], x["lam"], chunk=w.chunk,
                                         cg_steps=w.cg_steps, tol=w.tol, workspace=ws, stream=stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.4)
    mesa.timing_enable(True)
    mesa.timing_read()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    ev0.record(stream)
    for _ in range(args.steps):
        step()
    ev1.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    mesa.timing_enable(False)
    kernels = mesa.timing_read()
    clk = clocks.stop()
    assert mesa.get_error() == 0
    ms = max_over_ranks(ev0.elapsed_time(ev1), world, dev)
    if world > 1:
        dist.destroy_process_group()
    if rank != 0:
        return
    tokens = w.B * w.H * Tr * world
    line = {
        "metric": SHARD_METRIC, "value": tokens / (ms / args.steps / 1e3), "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms / args.steps,
        "higher_is_better": True, "scaling": "strong", "vs_baseline": None,
        "dtype": "bf16-in/f16-mma/f32-acc" if w.dtype == "bf16" else "f32", "data": "synthetic",
        "config": {"workload": w.name + "+seq-sharded", "B": w.B, "H": w.H, "T": Tr * world, "T_per_rank": Tr,
                   "d": w.dk, "chunk": w.chunk, "cg_steps": w.cg_steps, "tol": w.tol,
                   "exchange": "one all-gather of (H, G, decay) per step: %d bytes per rank" % (
                       w.B * w.H * (w.dk * w.dk + w.dv * w.dk + 1) * 4)},
        "roofline": None,
        "kernels": {k: {"launches": v[0], "total_ms": v[1]} for k, v in kernels.items()},
        "gpu_launches": sum(v[0] for v in kernels.values()),
        "clocks": clk, "e2e": None, "cpu_baseline": None,
    }
    print(json.dumps(line), flush=True)


def run_forward_warm(args, w, world, rank, local):
    """Forward warm start on a forward workload: the sequences are solved
    once, then one token is inserted at the front of each (the last drops out,
    T is unchanged: a context edited since it was solved), and the edited
    batch is solved again, cold (mesa_forward) and from the shifted earlier
    solutions (mesa_forward_warm). Both are timed over the same steps; the
    line's value is the warm re-solve's rate, with the cold one beside it."""
    import torch
    import torch.distributed as dist
    from test_sequence_layer_b200 import build as mbuild, mesa
    mbuild.build()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    tol = w.tol if args.tol is None else args.tol
    x = mi.device_batch(w, dev, seed_offset=rank)
    B, H, T, d, C = w.B, w.H, w.T, w.dk, w.chunk
    tokens = B * H * T
    stream = torch.cuda.current_stream(dev)
    ws = torch.empty(max(mesa.workspace_size(B, H, T, d, d, C, x["q"].dtype), 1), dtype=torch.uint8, device=dev)
    _, x_old = mesa.forward_warm(x["q"], x["k"], x["v"], x["gamma"], x["beta"], x["lam"], None, chunk=C,
                                 cg_steps=w.cg_steps, tol=tol, workspace=ws, stream=stream)
    g = torch.Generator(device=dev)
    g.manual_seed(777 + rank)
    y = {}
    for n in ("q", "k", "v", "gamma", "beta"):
        y[n] = torch.roll(x[n], 1, dims=2).contiguous()
    for n in ("q", "k"):
        e = torch.randn((B, H, d), generator=g, device=dev)
        y[n][:, :, 0] = (e / e.norm(dim=-1, keepdim=True)).to(y[n].dtype)
    y["v"][:, :, 0] = torch.randn((B, H, d), generator=g, device=dev).to(y["v"].dtype)
    y["gamma"][:, :, 0] = 0.9
    y["beta"][:, :, 0] = 0.5
    x0 = torch.roll(x_old, 1, dims=2).contiguous()
    x0[:, :, 0] = 0.0
    del x_old, x
    out = torch.empty((B, H, T, d), device=dev)
    xs = torch.empty((B, H, T, d), device=dev)
    it_c = torch.empty((B, H, T), dtype=torch.int32, device=dev)
    it_w = torch.empty((B, H, T), dtype=torch.int32, device=dev)

    def cold():
        mesa.forward(y["q"], y["k"], y["v"], y["gamma"], y["beta"], x_lam, chunk=C, cg_steps=w.cg_steps, tol=tol,
                     out=out, iters=it_c, return_iters=True, workspace=ws, stream=stream)

    def warm():
        mesa.forward_warm(y["q"], y["k"], y["v"], y["gamma"], y["beta"], x_lam, x0, chunk=C, cg_steps=w.cg_steps,
                          tol=tol, out=out, x_out=xs, iters=it_w, return_iters=True, workspace=ws, stream=stream)

    x_lam = torch.from_numpy(mi.lambdas(w.seed, w.H, w.dk)).to(dev)

    def timed(fn):
        for _ in range(args.warmup):
            fn()
        torch.cuda.synchronize()
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        ev0.record(stream)
        for _ in range(args.steps):
            fn()
        ev1.record(stream)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        return max_over_ranks(ev0.elapsed_time(ev1), world, dev) / args.steps

    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.4)
    mesa.timing_enable(True)
    mesa.timing_read()
    ms_cold = timed(cold)
    kernels_cold = mesa.timing_read()
    ms_warm = timed(warm)
    kernels = mesa.timing_read()
    mesa.timing_enable(False)
    clk = clocks.stop()
    assert mesa.get_error(stream) == 0
    if world > 1:
        dist.destroy_process_group()
    if rank != 0:
        return
    line = {
        "metric": "Mesa-layer fwd tokens/s (B*H*T), re-solve of an edited context (one token inserted at the "
                  "front) warm-started from the earlier solutions",
        "value": whole_job_rate(tokens, world, ms_warm), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_warm, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16-in/f16-mma/f32-acc" if w.dtype == "bf16" else "f32", "data": "synthetic",
        "config": {"workload": w.name + "+edit-warm-start", "B": B, "H": H, "T": T, "d": d, "chunk": C,
                   "cg_steps": w.cg_steps, "tol": tol, "l2": "inputs larger than L2"},
        "warm": {"ms_per_step": ms_warm, "mean_iters": float(it_w.double().mean().item()),
                 "kernels": {k: {"launches": v[0], "total_ms": v[1]} for k, v in kernels.items()}},
        "cold": {"ms_per_step": ms_cold, "mean_iters": float(it_c.double().mean().item()),
                 "value": whole_job_rate(tokens, world, ms_cold),
                 "kernels": {k: {"launches": v[0], "total_ms": v[1]} for k, v in kernels_cold.items()}},
        "roofline": None, "gpu_launches": sum(v[0] for v in kernels.values()),
        "clocks": clk, "e2e": None, "cpu_baseline": None,
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="bf16_T8192", choices=list(mi.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--preprocess", action="store_true",
                    help="time mesa_preprocess (q/k convolution + normalisation) on the workload's shape")
    ap.add_argument("--backward", action="store_true",
                    help="time mesa_backward (implicit-differentiation gradients) on the workload's shape")
    ap.add_argument("--fused-preprocess", action="store_true",
                    help="time mesa_forward_preprocessed (raw q, k) against the plain and the two-step forward")
    ap.add_argument("--seq-sharded", action="store_true",
                    help="sequence-sharded forward: each rank one slice of T, one all-gather of slice states")
    ap.add_argument("--warm-start", action="store_true",
                    help="decode: start each step's CG from the previous step's solution (mesa_step_warm); "
                         "forward workloads: re-solve an edited context from its earlier solutions "
                         "(mesa_forward_warm) against a cold re-solve")
    ap.add_argument("--tol", type=float, default=None, help="override the workload's CG tolerance")
    ap.add_argument("--query-walk", type=float, default=0.0,
                    help="decode: queries as a random walk on the sphere with this step size (correlated stream)")
    ap.add_argument("--decode-state", default="prefill", choices=["prefill", "random"],
                    help="decode: state from a mesa_forward prefill (default) or a seeded random stand-in")
    args = ap.parse_args()
    assert args.warmup >= 3 or args.impl == "reference" or os.environ.get("MESA_BENCH_ALLOW_SHORT"), \
        "at least 3 warm-up steps"

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    w = mi.WORKLOADS[args.workload]

    if args.impl == "reference":
        run_reference(args, w, rank)
        return
    if args.preprocess:
        run_preprocess(args, w, world, rank, local)
        return
    if args.backward:
        run_backward(args, w, world, rank, local)
        return
    if args.fused_preprocess:
        run_fused_preprocess(args, w, world, rank, local)
        return
    if args.seq_sharded:
        run_seq_sharded(args, w, world, rank, local)
        return
    if w.decode_steps > 0:
        run_decode(args, w, world, rank, local)
        return
    if args.warm_start:
        run_forward_warm(args, w, world, rank, local)
        return

    import torch
    import torch.distributed as dist

    from test_sequence_layer_b200 import build as mbuild, mesa
    mbuild.build()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    def barrier():
        if world > 1:
            dist.barrier()

    x = mi.device_batch(w, dev, seed_offset=rank)
    B, H, T, d, C = w.B, w.H, w.T, w.dk, w.chunk
    tokens = B * H * T
    out = torch.empty((B, H, T, d), device=dev)
    iters = torch.empty((B, H, T), dtype=torch.int32, device=dev)
    ws = torch.empty(max(mesa.workspace_size(B, H, T, d, d, C, x["q"].dtype), 1), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        mesa.forward(x["q"], x["k"], x["v"], x["gamma"], x["beta"], x["lam"], chunk=C, cg_steps=w.cg_steps,
                     tol=w.tol, out=out, iters=iters, return_iters=True, workspace=ws, stream=stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    assert mesa.get_error(stream) == 0

    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.4)
    mesa.timing_enable(True)
    mesa.timing_read()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    ev0.record(stream)
    for _ in range(args.steps):
        step()
    ev1.record(stream)
    torch.cuda.synchronize()
    barrier()
    mesa.timing_enable(False)
    kernels = mesa.timing_read()
    clk = clocks.stop()
    ms = max_over_ranks(ev0.elapsed_time(ev1), world, dev)
    assert mesa.get_error(stream) == 0
    ms_per_step = ms / args.steps
    value = whole_job_rate(tokens, world, ms_per_step)
    total_iters = int(iters.sum().item())

    # dominant kernel and its roofline
    name, (launches, kms) = max(kernels.items(), key=lambda kv: kv[1][1])
    gpu_launches = sum(v[0] for v in kernels.values())
    avg_ms = kms / max(launches, 1)
    peaks = load_peaks()
    fti = flops_per_token_iter(d, C)
    if name in ("tc_cg", "simt_cg"):
        # CG matvecs actually needed (sum of per-token iteration counts) + one read-out per token
        flops = (total_iters + tokens) * fti
    else:
        flops = tokens * 2 * (d * d + d * d)
    achieved = flops / (avg_ms / 1e3) / 1e12
    if name.startswith("tc_"):
        roof = {"bound": "tensor", "achieved": achieved, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                "peak_kind": f"{peaks['_source']} bf16 dense burst (fp16 operands run at the bf16 rate)"}
    else:
        roof = {"bound": "alu", "achieved": achieved, "peak": SIMT_FP32_PEAK_TFLOPS, "unit": "TFLOP/s",
                "peak_kind": "fp32 FMA: 148 SM x 128 FMA/clk x 2 x 1.965 GHz"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["traffic"] = measured_traffic(name, tokens)
    roof["kernel"] = name
    roof["avg_ms"] = avg_ms

    # end to end through the host-buffer C-ABI call (copies inside the timed region)
    e2e = None
    if not args.no_e2e:
        hx = {n: x[n].cpu().pin_memory() for n in ("q", "k", "v", "gamma", "beta", "lam")}
        hout = torch.empty((B, H, T, d)).pin_memory()
        hws = torch.empty(mesa.host_workspace_size(B, H, T, d, d, C, x["q"].dtype), dtype=torch.uint8, device=dev)
        del ws
        e_steps = max(3, args.steps // 4)

        def hstep():
            mesa.forward_host(hx["q"], hx["k"], hx["v"], hx["gamma"], hx["beta"], hx["lam"], chunk=C,
                              cg_steps=w.cg_steps, tol=w.tol, out=hout, workspace=hws, device=dev,
                              stream=stream)
        hstep()
        barrier()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(e_steps):
            hstep()
        e1.record(stream)
        torch.cuda.synchronize()
        ems = max_over_ranks(e0.elapsed_time(e1), world, dev)
        h2d = sum(hx[n].numel() * hx[n].element_size() for n in ("q", "k", "v", "gamma", "beta", "lam"))
        e2e = {"value": whole_job_rate(tokens, world, ems / e_steps), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": hout.numel() * hout.element_size(), "steps": e_steps}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cores = host_cores()
        n_seq = min(w.B * w.H, 8 * max(cores, 1))
        T_s = min(w.T, 4096)
        rate, dt = cpu_oracle_sample(w, n_seq, T_s)
        cpu = {"value": rate, "unit": "tokens/s", "cores": cores, "kind": "oracle",
               "sample": f"{n_seq} sequences x first {T_s} tokens of {w.name} ({dt:.1f} s, OpenMP over sequences)"}

    if world > 1:
        dist.destroy_process_group()
    if rank != 0:
        return
    path = "tensor-core (tcgen05)" if name.startswith("tc_") else "fp32 CUDA-core"
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16-in/f16-mma/f32-acc" if name.startswith("tc_") else "bf16-in/f32",
        "data": "synthetic",
        "config": {"workload": w.name, "B": B, "H": H, "T": T, "d": d, "chunk": C, "cg_steps": w.cg_steps,
                   "tol": w.tol, "path": path, "per_gpu_tokens": tokens,
                   "l2": "inputs larger than L2 (%.2f GB per step)" % ((x["q"].numel() * 3 * x["q"].element_size()
                                                                       + out.numel() * 4) / 1e9),
                   "cg_iters_total": total_iters},
        "roofline": roof,
        "kernels": {k: {"launches": v[0], "total_ms": v[1]} for k, v in kernels.items()},
        "gpu_launches": gpu_launches,
        "clocks": clk,
        "e2e": e2e,
        "cpu_baseline": cpu,
    }
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
