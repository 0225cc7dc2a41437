"""ctypes binding of libmesa_b200.so (argument marshalling only).

Every step of the layer runs in the library's CUDA kernels; this module only
turns torch tensors into the pointers, sizes and stream the C ABI takes
(include/mesa.h) and turns status codes into exceptions. There is no
fallback: if the library cannot be loaded, every call raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libmesa_b200.so")
_lib = None

MESA_F32, MESA_BF16 = 0, 1
_STATUS = {0: "MESA_OK", 1: "MESA_ERR_INVALID_ARG", 2: "MESA_ERR_UNSUPPORTED", 3: "MESA_ERR_WORKSPACE",
           4: "MESA_ERR_CUDA", 5: "MESA_ERR_DEVICE_TIMEOUT"}


class MesaError(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"{where}: {_STATUS.get(status, status)}")
        self.status = status


def library_path() -> str:
    return _LIB_PATH


def _load():
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(_LIB_PATH):
        raise ImportError(f"{_LIB_PATH} is missing; build it with `python -m test_sequence_layer_b200.build`")
    lib = ctypes.CDLL(_LIB_PATH)
    P, I, F, Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    fwd = [P, P, P, P, P, P, I, I, I, I, I, I, I, I, F, P, P, P, P, P, P, P, Z, P]
    lib.mesa_forward.argtypes = fwd
    lib.mesa_forward.restype = I
    lib.mesa_forward_host.argtypes = fwd
    lib.mesa_forward_warm.argtypes = [P, P, P, P, P, P, I, I, I, I, I, I, I, I, F, P, P, P, P, P, P, P, P, P, Z, P]
    lib.mesa_forward_warm.restype = I
    lib.mesa_forward_host.restype = I
    lib.mesa_forward_workspace_size.argtypes = [I, I, I, I, I, I, I]
    lib.mesa_forward_workspace_size.restype = Z
    lib.mesa_forward_host_workspace_size.argtypes = [I, I, I, I, I, I, I]
    lib.mesa_forward_host_workspace_size.restype = Z
    lib.mesa_step.argtypes = [P, P, P, P, P, P, I, I, I, I, P, P, I, F, P, P, P]
    lib.mesa_step.restype = I
    lib.mesa_step_warm.argtypes = [P, P, P, P, P, P, I, I, I, I, P, P, P, I, F, P, P, P]
    lib.mesa_step_warm.restype = I
    lib.mesa_get_error.argtypes = [P]
    lib.mesa_get_error.restype = I
    lib.mesa_status_string.argtypes = [I]
    lib.mesa_status_string.restype = ctypes.c_char_p
    lib.mesa_version.argtypes = []
    lib.mesa_version.restype = I
    lib.mesa_timing_enable.argtypes = [I]
    lib.mesa_timing_enable.restype = I
    lib.mesa_timing_read.argtypes = [ctypes.POINTER(ctypes.c_char_p), ctypes.POINTER(I),
                                     ctypes.POINTER(ctypes.c_double), I]
    lib.mesa_timing_read.restype = I
    lib.mesa_preprocess.argtypes = [P, P, P, P, I, I, I, I, I, I, P, P, P]
    lib.mesa_preprocess.restype = I
    lib.mesa_forward_preprocessed.argtypes = [P, P, P, P, P, P, P, P, I, I, I, I, I, I, I, I, I, F, P, P, P, P,
                                              P, P, P, Z, P]
    lib.mesa_forward_preprocessed.restype = I
    lib.mesa_forward_preprocessed_workspace_size.argtypes = [I, I, I, I, I, I, I]
    lib.mesa_forward_preprocessed_workspace_size.restype = Z
    lib.mesa_chunk_state_workspace_size.argtypes = [I, I, I, I, I, I, I]
    lib.mesa_chunk_state_workspace_size.restype = Z
    lib.mesa_chunk_state.argtypes = [P, P, P, P, I, I, I, I, I, I, I, P, P, P, P, P, P, Z, P]
    lib.mesa_chunk_state.restype = I
    lib.mesa_state_prefix.argtypes = [P, P, P, I, I, I, I, I, I, P, P, P]
    lib.mesa_state_prefix.restype = I
    lib.mesa_backward_workspace_size.argtypes = [I, I, I, I, I, I, I]
    lib.mesa_backward_workspace_size.restype = Z
    lib.mesa_backward.argtypes = [P, P, P, P, P, P, I, I, I, I, I, I, I, I, F, P, P, P, P, P, P, P, P, Z, P]
    lib.mesa_backward.restype = I
    _lib = lib
    return lib


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return MESA_F32
    if t.dtype == torch.bfloat16:
        return MESA_BF16
    raise TypeError(f"q/k/v must be float32 or bfloat16, got {t.dtype}")


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream, device):
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return ctypes.c_void_p(stream.cuda_stream)


def _check(rc: int, where: str):
    if rc != 0:
        raise MesaError(rc, where)


def workspace_size(B, H, T, dk, dv, chunk, dtype=torch.bfloat16) -> int:
    code = MESA_BF16 if dtype == torch.bfloat16 else MESA_F32
    return int(_load().mesa_forward_workspace_size(B, H, T, dk, dv, chunk, code))


def host_workspace_size(B, H, T, dk, dv, chunk, dtype=torch.bfloat16) -> int:
    code = MESA_BF16 if dtype == torch.bfloat16 else MESA_F32
    return int(_load().mesa_forward_host_workspace_size(B, H, T, dk, dv, chunk, code))


def forward(q, k, v, gamma, beta, lam, *, chunk=64, cg_steps=15, tol=0.0, out=None,
            return_iters=False, iters=None, H_in=None, G_in=None, return_state=False, workspace=None,
            stream=None):
    """Chunkwise-parallel Mesa forward on CUDA tensors.

    q, k: [B,H,T,dk]; v: [B,H,T,dv] (float32 or bfloat16, same dtype);
    gamma, beta: [B,H,T] float32; lam: [H,dk] float32.
    Returns out [B,H,T,dv] float32, plus iters [B,H,T] int32 if return_iters
    (written into `iters` when given), plus (H_out, G_out) if return_state.
    """
    lib = _load()
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    code = _dtype_code(q)
    dev = q.device
    if out is None:
        out = torch.empty((B, H, T, dv), dtype=torch.float32, device=dev)
    if return_iters and iters is None:
        iters = torch.empty((B, H, T), dtype=torch.int32, device=dev)
    H_out = torch.empty((B, H, dk, dk), dtype=torch.float32, device=dev) if return_state else None
    G_out = torch.empty((B, H, dv, dk), dtype=torch.float32, device=dev) if return_state else None
    need = int(lib.mesa_forward_workspace_size(B, H, T, dk, dv, chunk, code))
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    rc = lib.mesa_forward(_ptr(q), _ptr(k), _ptr(v), _ptr(gamma), _ptr(beta), _ptr(lam),
                          B, H, T, dk, dv, chunk, code, int(cg_steps), float(tol),
                          _ptr(out), _ptr(iters), _ptr(H_in), _ptr(G_in), _ptr(H_out), _ptr(G_out),
                          _ptr(workspace), ws_bytes, _stream(stream, dev))
    _check(rc, "mesa_forward")
    res = (out,)
    if return_iters:
        res += (iters,)
    if return_state:
        res += (H_out, G_out)
    return res[0] if len(res) == 1 else res


def forward_warm(q, k, v, gamma, beta, lam, x0, *, chunk=64, cg_steps=15, tol=0.0, out=None, x_out=None,
                 return_iters=False, iters=None, H_in=None, G_in=None, return_state=False, workspace=None,
                 stream=None):
    """forward() with every token's CG started from x0 [B,H,T,dk] float32
    (None: from zero). Returns (out, x) where x [B,H,T,dk] float32 holds the
    solutions (written into `x_out` when given; x_out may be x0 itself), plus
    iters if return_iters, plus (H_out, G_out) if return_state."""
    lib = _load()
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    code = _dtype_code(q)
    dev = q.device
    if out is None:
        out = torch.empty((B, H, T, dv), dtype=torch.float32, device=dev)
    if x_out is None:
        x_out = torch.empty((B, H, T, dk), dtype=torch.float32, device=dev)
    if return_iters and iters is None:
        iters = torch.empty((B, H, T), dtype=torch.int32, device=dev)
    H_out = torch.empty((B, H, dk, dk), dtype=torch.float32, device=dev) if return_state else None
    G_out = torch.empty((B, H, dv, dk), dtype=torch.float32, device=dev) if return_state else None
    need = int(lib.mesa_forward_workspace_size(B, H, T, dk, dv, chunk, code))
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    rc = lib.mesa_forward_warm(_ptr(q), _ptr(k), _ptr(v), _ptr(gamma), _ptr(beta), _ptr(lam),
                               B, H, T, dk, dv, chunk, code, int(cg_steps), float(tol), _ptr(x0), _ptr(x_out),
                               _ptr(out), _ptr(iters), _ptr(H_in), _ptr(G_in), _ptr(H_out), _ptr(G_out),
                               _ptr(workspace), ws_bytes, _stream(stream, dev))
    _check(rc, "mesa_forward_warm")
    res = (out, x_out)
    if return_iters:
        res += (iters,)
    if return_state:
        res += (H_out, G_out)
    return res


def backward(q, k, v, gamma, beta, lam, dout, *, chunk=64, cg_steps=15, tol=0.0, workspace=None, stream=None):
    """Gradients of L given dout = dL/do for the inputs of forward() with zero
    initial states (implicit differentiation, adjoint CG under the same rule).

    dout: [B,H,T,dv] float32. Returns (dq, dk, dv, dgamma, dbeta, dlambda),
    all float32 with the shapes of q, k, v, gamma, beta, lam.
    """
    lib = _load()
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    code = _dtype_code(q)
    dev = q.device
    f32 = dict(dtype=torch.float32, device=dev)
    dq = torch.empty((B, H, T, dk), **f32)
    dk_ = torch.empty((B, H, T, dk), **f32)
    dv_ = torch.empty((B, H, T, dv), **f32)
    dgamma = torch.empty((B, H, T), **f32)
    dbeta = torch.empty((B, H, T), **f32)
    dlam = torch.empty((H, dk), **f32)
    need = int(lib.mesa_backward_workspace_size(B, H, T, dk, dv, chunk, code))
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    rc = lib.mesa_backward(_ptr(q), _ptr(k), _ptr(v), _ptr(gamma), _ptr(beta), _ptr(lam),
                           B, H, T, dk, dv, chunk, code, int(cg_steps), float(tol), _ptr(dout),
                           _ptr(dq), _ptr(dk_), _ptr(dv_), _ptr(dgamma), _ptr(dbeta), _ptr(dlam),
                           _ptr(workspace), ws_bytes, _stream(stream, dev))
    _check(rc, "mesa_backward")
    return dq, dk_, dv_, dgamma, dbeta, dlam


def chunk_state(k, v, gamma, beta, *, chunk=64, H_in=None, G_in=None, workspace=None, stream=None):
    """The scan of forward() without the solve: (H_out, G_out, decay) with the
    states after the T tokens (from H_in, G_in or zero) and decay [B,H] =
    prod_t gamma_t. The summary a slice of a sequence-sharded forward exchanges."""
    lib = _load()
    B, H, T, dk = k.shape
    dv = v.shape[-1]
    code = _dtype_code(k)
    dev = k.device
    H_out = torch.empty((B, H, dk, dk), dtype=torch.float32, device=dev)
    G_out = torch.empty((B, H, dv, dk), dtype=torch.float32, device=dev)
    decay = torch.empty((B, H), dtype=torch.float32, device=dev)
    need = int(lib.mesa_chunk_state_workspace_size(B, H, T, dk, dv, chunk, code))
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    rc = lib.mesa_chunk_state(_ptr(k), _ptr(v), _ptr(gamma), _ptr(beta), B, H, T, dk, dv, chunk, code,
                              _ptr(H_in), _ptr(G_in), _ptr(H_out), _ptr(G_out), _ptr(decay),
                              _ptr(workspace), ws_bytes, _stream(stream, dev))
    _check(rc, "mesa_chunk_state")
    return H_out, G_out, decay


def state_prefix(H_slices, G_slices, decay_slices, r, *, stream=None):
    """State entering slice r from the stacked summaries [n, B, H, ...] of the
    slices before it (in sequence order). Returns (H_in, G_in)."""
    lib = _load()
    n, B, H, dk, _ = H_slices.shape
    dv = G_slices.shape[3]
    dev = H_slices.device
    H_in = torch.empty((B, H, dk, dk), dtype=torch.float32, device=dev)
    G_in = torch.empty((B, H, dv, dk), dtype=torch.float32, device=dev)
    rc = lib.mesa_state_prefix(_ptr(H_slices), _ptr(G_slices), _ptr(decay_slices), n, int(r), B, H, dk, dv,
                               _ptr(H_in), _ptr(G_in), _stream(stream, dev))
    _check(rc, "mesa_state_prefix")
    return H_in, G_in


def forward_host(q, k, v, gamma, beta, lam, *, chunk=64, cg_steps=15, tol=0.0, out=None,
                 iters=None, H_in=None, G_in=None, H_out=None, G_out=None, workspace=None,
                 device=None, stream=None):
    """Forward with HOST (CPU, ideally pinned) tensors; the library copies them to the
    device, runs the forward and copies results back before returning."""
    lib = _load()
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    code = _dtype_code(q)
    device = torch.device("cuda", torch.cuda.current_device()) if device is None else device
    if out is None:
        out = torch.empty((B, H, T, dv), dtype=torch.float32)
    need = int(lib.mesa_forward_host_workspace_size(B, H, T, dk, dv, chunk, code))
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=device)
    ws_bytes = workspace.numel() * workspace.element_size()
    rc = lib.mesa_forward_host(_ptr(q), _ptr(k), _ptr(v), _ptr(gamma), _ptr(beta), _ptr(lam),
                               B, H, T, dk, dv, chunk, code, int(cg_steps), float(tol),
                               _ptr(out), _ptr(iters), _ptr(H_in), _ptr(G_in), _ptr(H_out), _ptr(G_out),
                               _ptr(workspace), ws_bytes, _stream(stream, device))
    _check(rc, "mesa_forward_host")
    return out


def preprocess(q_raw, k_raw, conv_q, conv_k, *, q_out=None, k_out=None, stream=None):
    """mesa_preprocess: causal depthwise convolution over time (conv [H,W,d],
    w = lag), then per-token L2 normalisation, for q and k. q_raw, k_raw:
    [B,H,T,d] float32 or bfloat16 CUDA tensors. Returns (q, k) in the same
    dtype, ready for forward()."""
    lib = _load()
    B, H, T, d = q_raw.shape
    W = conv_q.shape[1]
    assert k_raw.shape == q_raw.shape and k_raw.dtype == q_raw.dtype
    assert conv_q.shape == (H, W, d) and conv_k.shape == (H, W, d)
    assert conv_q.dtype == torch.float32 and conv_k.dtype == torch.float32
    for t in (q_raw, k_raw, conv_q, conv_k):
        assert t.is_cuda and t.is_contiguous()
    q_out = torch.empty_like(q_raw) if q_out is None else q_out
    k_out = torch.empty_like(k_raw) if k_out is None else k_out
    rc = lib.mesa_preprocess(_ptr(q_raw), _ptr(k_raw), _ptr(conv_q), _ptr(conv_k), B, H, T, d, W,
                             _dtype_code(q_raw), _ptr(q_out), _ptr(k_out), _stream(stream, q_raw.device))
    _check(rc, "mesa_preprocess")
    return q_out, k_out


def forward_preprocessed(q_raw, k_raw, v, gamma, beta, lam, conv_q, conv_k, *, chunk=64, cg_steps=15, tol=0.0,
                         out=None, return_iters=False, iters=None, H_in=None, G_in=None, return_state=False,
                         workspace=None, stream=None):
    """forward() of preprocess(q_raw, k_raw, conv_q, conv_k) in one call
    (mesa_forward_preprocessed): on the tensor-core shape the scan and the
    solve convolve and normalise the raw rows as they stage them. Same
    returns as forward()."""
    lib = _load()
    B, H, T, dk = q_raw.shape
    dv = v.shape[-1]
    W = conv_q.shape[1]
    assert conv_q.shape == (H, W, dk) and conv_k.shape == (H, W, dk)
    code = _dtype_code(q_raw)
    dev = q_raw.device
    if out is None:
        out = torch.empty((B, H, T, dv), dtype=torch.float32, device=dev)
    if return_iters and iters is None:
        iters = torch.empty((B, H, T), dtype=torch.int32, device=dev)
    H_out = torch.empty((B, H, dk, dk), dtype=torch.float32, device=dev) if return_state else None
    G_out = torch.empty((B, H, dv, dk), dtype=torch.float32, device=dev) if return_state else None
    need = int(lib.mesa_forward_preprocessed_workspace_size(B, H, T, dk, dv, chunk, code))
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    rc = lib.mesa_forward_preprocessed(_ptr(q_raw), _ptr(k_raw), _ptr(v), _ptr(gamma), _ptr(beta), _ptr(lam),
                                       _ptr(conv_q), _ptr(conv_k), W, B, H, T, dk, dv, chunk, code, int(cg_steps),
                                       float(tol), _ptr(out), _ptr(iters), _ptr(H_in), _ptr(G_in), _ptr(H_out),
                                       _ptr(G_out), _ptr(workspace), ws_bytes, _stream(stream, dev))
    _check(rc, "mesa_forward_preprocessed")
    res = (out,)
    if return_iters:
        res += (iters,)
    if return_state:
        res += (H_out, G_out)
    return res[0] if len(res) == 1 else res


def step(q, k, v, gamma, beta, lam, Hstate, Gstate, *, cg_steps=15, tol=0.0, out=None,
         iters=None, x_state=None, stream=None):
    """One decode step; Hstate [B,H,dk,dk] and Gstate [B,H,dv,dk] (float32) are
    updated in place. q, k: [B,H,dk]; v: [B,H,dv]; gamma, beta: [B,H].
    x_state [B,H,dk] float32 (optional, in/out): the CG starts from it and it
    receives the solution (mesa_step_warm)."""
    lib = _load()
    B, H, dk = q.shape
    dv = v.shape[-1]
    if out is None:
        out = torch.empty((B, H, dv), dtype=torch.float32, device=q.device)
    rc = lib.mesa_step_warm(_ptr(q), _ptr(k), _ptr(v), _ptr(gamma), _ptr(beta), _ptr(lam), B, H, dk, dv,
                            _ptr(Hstate), _ptr(Gstate), _ptr(x_state), int(cg_steps), float(tol), _ptr(out),
                            _ptr(iters), _stream(stream, q.device))
    _check(rc, "mesa_step_warm")
    return out


def get_error(stream=None) -> int:
    """Synchronises the stream and reads/clears the device error word (0 = none)."""
    lib = _load()
    s = ctypes.c_void_p(None) if stream is None else ctypes.c_void_p(stream.cuda_stream)
    return int(lib.mesa_get_error(s))


def timing_enable(on: bool = True):
    """Bracket every library kernel launch with CUDA events on its stream."""
    _load().mesa_timing_enable(1 if on else 0)


def timing_read() -> dict:
    """{kernel kind: (launches, total device ms)} since the last read (synchronises)."""
    lib = _load()
    n = 16
    names = (ctypes.c_char_p * n)()
    launches = (ctypes.c_int * n)()
    ms = (ctypes.c_double * n)()
    k = lib.mesa_timing_read(names, launches, ms, n)
    if k < 0:
        raise MesaError(4, "mesa_timing_read")
    return {names[i].decode(): (int(launches[i]), float(ms[i])) for i in range(k)}


def forward_noalloc(q, k, v, gamma, beta, lam, *, chunk=64, cg_steps=15, tol=0.0, out=None, iters=None,
                    H_in=None, G_in=None, H_out=None, G_out=None, stream=None):
    """mesa_forward_noalloc: the forward for callers that cannot allocate device
    memory; its scratch is a fixed library-owned device array (sizes beyond it
    raise MesaError MESA_ERR_WORKSPACE)."""
    lib = _load()
    if not getattr(lib, "_noalloc_typed", False):
        P, I, F = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
        lib.mesa_forward_noalloc.argtypes = [P, P, P, P, P, P, I, I, I, I, I, I, I, I, F, P, P, P, P, P, P, P]
        lib.mesa_forward_noalloc.restype = I
        lib._noalloc_typed = True
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    if out is None:
        out = torch.empty((B, H, T, dv), dtype=torch.float32, device=q.device)
    rc = lib.mesa_forward_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(gamma), _ptr(beta), _ptr(lam), B, H, T, dk, dv,
                                  chunk, _dtype_code(q), int(cg_steps), float(tol), _ptr(out), _ptr(iters),
                                  _ptr(H_in), _ptr(G_in), _ptr(H_out), _ptr(G_out), _stream(stream, q.device))
    _check(rc, "mesa_forward_noalloc")
    return out
