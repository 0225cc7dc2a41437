"""mesa_forward_noalloc: the forward for callers that cannot allocate device
memory (it takes its scratch from a fixed library-owned device array instead
of a caller workspace). Called through the C ABI and checked against
mesa_forward on the same inputs, on two calls in a row (the second call finds
the previous call's data in the shared array), and on a smaller shape after a
larger one (stale bytes beyond the smaller call's layout must go unread).

The file name sorts after every other test file, so pytest collects it last:
a run that stops at the first failure has then already run every other test
before this one. The tests pass alone in a fresh process as well."""
import ctypes

import numpy as np
import pytest
import torch

import mesa_inputs as mi
from helpers import TOL_BF16, TOL_F32, rel_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from test_sequence_layer_b200 import build, mesa
    build.build()
    lib = mesa._load()
    P, I, F = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
    lib.mesa_forward_noalloc.argtypes = [P, P, P, P, P, P, I, I, I, I, I, I, I, I, F, P, P, P, P, P, P, P]
    lib.mesa_forward_noalloc.restype = I
    return lib


def ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def call_noalloc(lib, d, w, out, iters, Ho, Go):
    B, H, T, dk = d["q"].shape
    code = 1 if d["q"].dtype == torch.bfloat16 else 0
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return lib.mesa_forward_noalloc(ptr(d["q"]), ptr(d["k"]), ptr(d["v"]), ptr(d["gamma"]), ptr(d["beta"]),
                                    ptr(d["lam"]), B, H, T, dk, dk, w.chunk, code, w.cg_steps, w.tol, ptr(out),
                                    ptr(iters), None, None, ptr(Ho), ptr(Go), stream)


@pytest.mark.parametrize("dtype,d,chunk", [("bf16", 128, 64), ("f32", 64, 32)])
def test_noalloc_matches_forward_twice(lib, dtype, d, chunk):
    from test_sequence_layer_b200 import mesa
    tol = TOL_BF16 if dtype == "bf16" else TOL_F32
    for call, seed in enumerate((41, 42)):     # second call: different data, stale scratch
        w = mi.Workload("na", 2, 4, 300, d, d, chunk, dtype, 15, 0.0, False, seed)
        x = mi.batch(w)
        dt = torch.bfloat16 if dtype == "bf16" else torch.float32
        dev = {n: torch.from_numpy(np.ascontiguousarray(x[n])).cuda() for n in ("q", "k", "v", "gamma", "beta", "lam")}
        for n in ("q", "k", "v"):
            dev[n] = dev[n].to(dt)
        ref, ref_it, rH, rG = mesa.forward(dev["q"], dev["k"], dev["v"], dev["gamma"], dev["beta"], dev["lam"],
                                           chunk=chunk, cg_steps=15, return_iters=True, return_state=True)
        out = torch.full_like(ref, float("nan"))
        iters = torch.full_like(ref_it, -1)
        Ho, Go = torch.empty_like(rH), torch.empty_like(rG)
        assert call_noalloc(lib, dev, w, out, iters, Ho, Go) == 0
        torch.cuda.synchronize()
        assert mesa.get_error() == 0
        assert rel_err(out.cpu().numpy(), ref.cpu().numpy()) <= tol, call
        assert torch.equal(iters, ref_it)
        assert torch.allclose(Ho, rH, rtol=1e-5, atol=1e-6) and torch.allclose(Go, rG, rtol=1e-5, atol=1e-6)


def test_noalloc_refuses_sizes_beyond_its_scratch(lib):
    from test_sequence_layer_b200 import mesa
    # 8 x 16 sequences of 8192 tokens need far more than the fixed scratch
    need = mesa.workspace_size(8, 16, 8192, 128, 128, 64)
    assert need > (32 << 20)
    dummy = torch.empty(16, device="cuda")
    w = mi.Workload("big", 8, 16, 8192, 128, 128, 64, "bf16", 15, 0.0, False, 0)
    d = {n: dummy for n in ("q", "k", "v", "gamma", "beta", "lam")}
    B, H, T = 8, 16, 8192
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = lib.mesa_forward_noalloc(ptr(dummy), ptr(dummy), ptr(dummy), ptr(dummy), ptr(dummy), ptr(dummy), B, H, T,
                                  128, 128, 64, 1, 15, 0.0, ptr(dummy), None, None, None, None, None, stream)
    assert rc == 3    # MESA_ERR_WORKSPACE, refused before any device work


@pytest.mark.parametrize("dtype,d,chunk", [("bf16", 128, 64), ("f32", 32, 16)])
def test_noalloc_smaller_call_after_larger(lib, dtype, d, chunk):
    """A large call fills more of the shared array than the small call that
    follows it; the small call must match mesa_forward all the same."""
    from test_sequence_layer_b200 import mesa
    tol = TOL_BF16 if dtype == "bf16" else TOL_F32
    dt = torch.bfloat16 if dtype == "bf16" else torch.float32
    for B, H, T, seed in ((4, 4, 700, 51), (1, 2, 130, 52)):
        w = mi.Workload("na", B, H, T, d, d, chunk, dtype, 15, 0.0, False, seed)
        x = mi.batch(w)
        dev = {n: torch.from_numpy(np.ascontiguousarray(x[n])).cuda() for n in ("q", "k", "v", "gamma", "beta", "lam")}
        for n in ("q", "k", "v"):
            dev[n] = dev[n].to(dt)
        ref, ref_it, rH, rG = mesa.forward(dev["q"], dev["k"], dev["v"], dev["gamma"], dev["beta"], dev["lam"],
                                           chunk=chunk, cg_steps=15, return_iters=True, return_state=True)
        out = torch.full_like(ref, float("nan"))
        iters = torch.full_like(ref_it, -1)
        Ho, Go = torch.empty_like(rH), torch.empty_like(rG)
        assert call_noalloc(lib, dev, w, out, iters, Ho, Go) == 0
        torch.cuda.synchronize()
        assert mesa.get_error() == 0
        assert rel_err(out.cpu().numpy(), ref.cpu().numpy()) <= tol, (B, H, T)
        assert torch.equal(iters, ref_it)
        assert torch.allclose(Ho, rH, rtol=1e-5, atol=1e-6) and torch.allclose(Go, rG, rtol=1e-5, atol=1e-6)
