"""fp64 CPU oracle of the Mesa layer (test infrastructure).

Only the test suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package. The product library
(``test_sequence_layer_b200``) never imports it, and this package imports
nothing from the product.

The arithmetic lives in ``mesa_oracle.c`` (plain C, fp64). This module only
compiles it with gcc and marshals numpy arrays through ctypes. Every array is
converted to contiguous float64 (bf16 and fp32 inputs convert exactly).

Method: "MesaNet: Sequence Modeling by Locally Optimal Test-Time Training"
(gist.science, ja/ko/hi editions), Technical summary > Method > Mesa layer.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "mesa_oracle.c")
_BUILD = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD, "libmesa_oracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (-O2, OpenMP over independent sequences)."""
    os.makedirs(_BUILD, exist_ok=True)
    hdr = os.path.join(_HERE, "mesa_oracle.h")
    stale = (not os.path.exists(_LIB_PATH)
             or os.path.getmtime(_LIB_PATH) < max(os.path.getmtime(_SRC), os.path.getmtime(hdr)))
    if force or stale:
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        # -ffp-contract=off: no fused multiply-adds, so each line rounds as written.
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
               "-Wall", "-Wextra", "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _configure(lib):
    """Declares the C signatures on a loaded oracle library."""
    D = ctypes.POINTER(ctypes.c_double)
    I32 = ctypes.POINTER(ctypes.c_int32)
    i, d = ctypes.c_int, ctypes.c_double
    lib.oracle_forward_cg.argtypes = [D, D, D, D, D, D, i, i, i, i, i, i, d, D, D, D, I32, D, D]
    lib.oracle_forward_cg_x0.argtypes = [D, D, D, D, D, D, i, i, i, i, i, i, d, D, D, D, D, I32, D, D, D]
    lib.oracle_forward_cholesky.argtypes = [D, D, D, D, D, D, i, i, i, i, i, D, D, D, D, D]
    lib.oracle_forward_chunked.argtypes = [D, D, D, D, D, D, i, i, i, i, i, i, i, d, D, D, D, I32, D, D]
    lib.oracle_step.argtypes = [D, D, D, D, D, D, i, i, i, i, D, D, i, d, D, I32]
    lib.oracle_step_warm.argtypes = [D, D, D, D, D, D, i, i, i, i, D, D, D, i, d, D, I32]
    lib.oracle_cg_dense.argtypes = [i, D, D, D, i, d, D, I32]
    lib.oracle_preprocess.argtypes = [D, D, i, i, i, i, i, D]
    lib.oracle_backward.argtypes = [D, D, D, D, D, D, i, i, i, i, i, i, d, D, D, D, D, D, D, D, I32, I32]
    for f in (lib.oracle_forward_cg, lib.oracle_forward_cg_x0, lib.oracle_forward_cholesky, lib.oracle_forward_chunked,
              lib.oracle_step, lib.oracle_step_warm, lib.oracle_cg_dense, lib.oracle_preprocess,
              lib.oracle_backward):
        f.restype = ctypes.c_int
    return lib


def _load():
    global _lib
    if _lib is None:
        build()
        _lib = _configure(ctypes.CDLL(_LIB_PATH))
    return _lib


def _f64(a):
    if a is None:
        return None
    if hasattr(a, "detach"):  # torch tensor -> numpy (exact widening to fp64)
        a = a.detach().to("cpu").double().numpy()
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a):
    if a is None:
        return None
    if a.dtype == np.int32:
        return a.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _check(rc, name):
    if rc != 0:
        raise RuntimeError(f"{name} failed with code {rc}")


def _shapes(q, v):
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    return B, H, T, dk, dv


def forward_cg(q, k, v, gamma, beta, lam, cg_steps, tol=0.0, H0=None, G0=None):
    """Per-token recurrence + CG. Returns (out, iters, H_final, G_final)."""
    q, k, v, gamma, beta, lam = map(_f64, (q, k, v, gamma, beta, lam))
    H0, G0 = _f64(H0), _f64(G0)
    B, H, T, dk, dv = _shapes(q, v)
    out = np.zeros((B, H, T, dv))
    iters = np.zeros((B, H, T), dtype=np.int32)
    Hf = np.zeros((B, H, dk, dk))
    Gf = np.zeros((B, H, dv, dk))
    rc = _load().oracle_forward_cg(_ptr(q), _ptr(k), _ptr(v), _ptr(gamma), _ptr(beta), _ptr(lam),
                                   B, H, T, dk, dv, int(cg_steps), float(tol), _ptr(H0), _ptr(G0),
                                   _ptr(out), _ptr(iters), _ptr(Hf), _ptr(Gf))
    _check(rc, "oracle_forward_cg")
    return out, iters, Hf, Gf


def forward_cg_x0(q, k, v, gamma, beta, lam, cg_steps, tol=0.0, x0=None, H0=None, G0=None):
    """Per-token recurrence + CG started from x0 [B,H,T,dk] (None: zero).
    Returns (out, iters, x, H_final, G_final)."""
    q, k, v, gamma, beta, lam = map(_f64, (q, k, v, gamma, beta, lam))
    x0, H0, G0 = _f64(x0), _f64(H0), _f64(G0)
    B, H, T, dk, dv = _shapes(q, v)
    out = np.zeros((B, H, T, dv))
    iters = np.zeros((B, H, T), dtype=np.int32)
    x = np.zeros((B, H, T, dk))
    Hf = np.zeros((B, H, dk, dk))
    Gf = np.zeros((B, H, dv, dk))
    rc = _load().oracle_forward_cg_x0(_ptr(q), _ptr(k), _ptr(v), _ptr(gamma), _ptr(beta), _ptr(lam),
                                      B, H, T, dk, dv, int(cg_steps), float(tol), _ptr(x0), _ptr(H0), _ptr(G0),
                                      _ptr(out), _ptr(iters), _ptr(x), _ptr(Hf), _ptr(Gf))
    _check(rc, "oracle_forward_cg_x0")
    return out, iters, x, Hf, Gf


def forward_cholesky(q, k, v, gamma, beta, lam, H0=None, G0=None):
    """Per-token recurrence + exact solve. Returns (out, H_final, G_final)."""
    q, k, v, gamma, beta, lam = map(_f64, (q, k, v, gamma, beta, lam))
    H0, G0 = _f64(H0), _f64(G0)
    B, H, T, dk, dv = _shapes(q, v)
    out = np.zeros((B, H, T, dv))
    Hf = np.zeros((B, H, dk, dk))
    Gf = np.zeros((B, H, dv, dk))
    rc = _load().oracle_forward_cholesky(_ptr(q), _ptr(k), _ptr(v), _ptr(gamma), _ptr(beta), _ptr(lam),
                                         B, H, T, dk, dv, _ptr(H0), _ptr(G0), _ptr(out), _ptr(Hf), _ptr(Gf))
    _check(rc, "oracle_forward_cholesky")
    return out, Hf, Gf


def forward_chunked(q, k, v, gamma, beta, lam, chunk, cg_steps, tol=0.0, H0=None, G0=None):
    """Chunked form with the same CG rule. Returns (out, iters, H_final, G_final)."""
    q, k, v, gamma, beta, lam = map(_f64, (q, k, v, gamma, beta, lam))
    H0, G0 = _f64(H0), _f64(G0)
    B, H, T, dk, dv = _shapes(q, v)
    out = np.zeros((B, H, T, dv))
    iters = np.zeros((B, H, T), dtype=np.int32)
    Hf = np.zeros((B, H, dk, dk))
    Gf = np.zeros((B, H, dv, dk))
    rc = _load().oracle_forward_chunked(_ptr(q), _ptr(k), _ptr(v), _ptr(gamma), _ptr(beta), _ptr(lam),
                                        B, H, T, dk, dv, int(chunk), int(cg_steps), float(tol),
                                        _ptr(H0), _ptr(G0), _ptr(out), _ptr(iters), _ptr(Hf), _ptr(Gf))
    _check(rc, "oracle_forward_chunked")
    return out, iters, Hf, Gf


def step(q, k, v, gamma, beta, lam, Hstate, Gstate, cg_steps, tol=0.0, x_state=None):
    """One decode step. q,k,v: [B,H,d]; gamma,beta: [B,H]. States are copied
    (not modified). x_state [B,H,dk] (optional): CG starts from it (warm start).
    Returns (out, iters, H_new, G_new), plus x_new when x_state is given."""
    q, k, v, gamma, beta, lam = map(_f64, (q, k, v, gamma, beta, lam))
    Hs = _f64(Hstate).copy()
    Gs = _f64(Gstate).copy()
    xs = None if x_state is None else _f64(x_state).copy()
    B, H, dk = q.shape
    dv = v.shape[-1]
    out = np.zeros((B, H, dv))
    iters = np.zeros((B, H), dtype=np.int32)
    rc = _load().oracle_step_warm(_ptr(q), _ptr(k), _ptr(v), _ptr(gamma), _ptr(beta), _ptr(lam),
                                  B, H, dk, dv, _ptr(Hs), _ptr(Gs), _ptr(xs), int(cg_steps), float(tol),
                                  _ptr(out), _ptr(iters))
    _check(rc, "oracle_step_warm")
    return (out, iters, Hs, Gs) if xs is None else (out, iters, Hs, Gs, xs)


def cg_dense(A, b, cg_steps, tol=0.0, x0=None):
    """CG on one dense SPD system, from x0 (default zero). Returns (x, iters)."""
    A, b, x0 = _f64(A), _f64(b), _f64(x0)
    n = b.shape[0]
    x = np.zeros(n)
    it = np.zeros(1, dtype=np.int32)
    rc = _load().oracle_cg_dense(n, _ptr(A), _ptr(b), _ptr(x0), int(cg_steps), float(tol), _ptr(x), _ptr(it))
    _check(rc, "oracle_cg_dense")
    return x, int(it[0])


def preprocess(x, conv):
    """Causal depthwise convolution over time, then per-token L2 normalisation.
    x: [B,H,T,d]; conv: [H,W,d] (w = lag). Returns y [B,H,T,d]."""
    x, conv = _f64(x), _f64(conv)
    B, H, T, dd = x.shape
    W = conv.shape[1]
    y = np.zeros((B, H, T, dd))
    rc = _load().oracle_preprocess(_ptr(x), _ptr(conv), B, H, T, dd, W, _ptr(y))
    _check(rc, "oracle_preprocess")
    return y


def backward(q, k, v, gamma, beta, lam, dout, cg_steps, tol=0.0):
    """Gradients of L = sum(dout * o) through the layer (zero initial states),
    by implicit differentiation with an adjoint CG solve under the same rule.
    Returns a dict with dq, dk, dv, dgamma, dbeta, dlambda, iters_fwd, iters_adj."""
    q, k, v, gamma, beta, lam, dout = map(_f64, (q, k, v, gamma, beta, lam, dout))
    B, H, T, dk, dv = _shapes(q, v)
    r = {"dq": np.zeros((B, H, T, dk)), "dk": np.zeros((B, H, T, dk)), "dv": np.zeros((B, H, T, dv)),
         "dgamma": np.zeros((B, H, T)), "dbeta": np.zeros((B, H, T)), "dlambda": np.zeros((H, dk)),
         "iters_fwd": np.zeros((B, H, T), dtype=np.int32), "iters_adj": np.zeros((B, H, T), dtype=np.int32)}
    rc = _load().oracle_backward(_ptr(q), _ptr(k), _ptr(v), _ptr(gamma), _ptr(beta), _ptr(lam),
                                 B, H, T, dk, dv, int(cg_steps), float(tol), _ptr(dout),
                                 _ptr(r["dq"]), _ptr(r["dk"]), _ptr(r["dv"]), _ptr(r["dgamma"]), _ptr(r["dbeta"]),
                                 _ptr(r["dlambda"]), _ptr(r["iters_fwd"]), _ptr(r["iters_adj"]))
    _check(rc, "oracle_backward")
    return r
