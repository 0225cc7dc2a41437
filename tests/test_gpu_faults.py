"""Failure detection on the GPU, made on the host side (no GPU fault, trap or hang).

The MESA_DEBUG build of the library can leave out one MMA completion signal in
the tensor-core solve kernel. Every thread's bounded wait on that signal
(about one second of clock cycles) runs out; the kernel records a timeout in
the device error word, drains what it issued, frees its tensor memory and
returns. The host must see MESA_ERR_DEVICE_TIMEOUT from mesa_get_error, and
the same context must then run the next forward correctly.
"""
import ctypes

import numpy as np
import pytest
import torch

import mesa_inputs as mi
from helpers import TOL_BF16, rel_err

pytestmark = pytest.mark.gpu

MESA_BF16 = 1
MESA_OK = 0
MESA_ERR_DEVICE_TIMEOUT = 5


@pytest.fixture(scope="module")
def dlib():
    from test_sequence_layer_b200 import build as b
    lib = ctypes.CDLL(b.build(debug=True))
    vp, i, f = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
    lib.mesa_forward_workspace_size.restype = ctypes.c_size_t
    lib.mesa_forward_workspace_size.argtypes = [i, i, i, i, i, i, i]
    lib.mesa_forward.argtypes = [vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, i, i, f, vp, vp, vp, vp, vp, vp,
                                 vp, ctypes.c_size_t, vp]
    lib.mesa_get_error.argtypes = [vp]
    lib.mesa_debug_skip_commit.argtypes = [i]
    return lib


def forward(lib, x, T, ws, out):
    p = lambda t: ctypes.c_void_p(t.data_ptr())   # noqa: E731
    return lib.mesa_forward(p(x["q"]), p(x["k"]), p(x["v"]), p(x["gamma"]), p(x["beta"]), p(x["lam"]),
                            1, 1, T, 128, 128, 64, MESA_BF16, 15, 0.0, p(out), None, None, None, None, None,
                            p(ws), ws.numel(), None)


def test_bounded_wait_timeout_is_reported_and_context_survives(dlib, oracle_mod):
    T = 128                                         # one CTA of the solve kernel
    w = mi.Workload("t", 1, 1, T, 128, 128, 64, "bf16", 15, 0.0, False, 51)
    xh = mi.batch(w)
    x = {n: torch.from_numpy(np.ascontiguousarray(xh[n])).cuda() for n in ("q", "k", "v", "gamma", "beta", "lam")}
    for n in ("q", "k", "v"):
        x[n] = x[n].to(torch.bfloat16)
    ws = torch.empty(dlib.mesa_forward_workspace_size(1, 1, T, 128, 128, 64, MESA_BF16), dtype=torch.uint8,
                     device="cuda")
    out = torch.zeros((1, 1, T, 128), device="cuda")
    assert dlib.mesa_get_error(None) == MESA_OK

    assert dlib.mesa_debug_skip_commit(1) == MESA_OK
    assert forward(dlib, x, T, ws, out) == MESA_OK          # the launch itself succeeds
    assert dlib.mesa_get_error(None) == MESA_ERR_DEVICE_TIMEOUT
    assert dlib.mesa_get_error(None) == MESA_OK             # read and cleared

    out.zero_()
    assert forward(dlib, x, T, ws, out) == MESA_OK          # next launch: no injection
    assert dlib.mesa_get_error(None) == MESA_OK
    ref, _, _, _ = oracle_mod.forward_cg(xh["q"], xh["k"], xh["v"], xh["gamma"], xh["beta"], xh["lam"], 15)
    assert rel_err(out.cpu().numpy(), ref) <= TOL_BF16
