"""The C ABI on a machine without a GPU: the library loads, exports every
symbol include/mesa.h declares, and rejects bad arguments on the host before
any launch (no compute call is made here)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from test_sequence_layer_b200 import build, mesa
    build.build()
    return mesa._load()


def declared_functions(debug=False):
    """Entry points declared in include/*.h; the MESA_DEBUG blocks only for
    the debug build."""
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            if not debug:
                src = re.sub(r"#ifdef MESA_DEBUG.*?#endif", "", src, flags=re.S)
            names |= set(re.findall(r"\b(mesa_\w+)\s*\(", src))
    return sorted(names)


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert {"mesa_forward", "mesa_step", "mesa_forward_workspace_size", "mesa_get_error",
            "mesa_status_string", "mesa_forward_host"} <= set(names)
    assert "mesa_debug_skip_commit" not in names
    for n in names:
        assert hasattr(lib, n), n
    assert not hasattr(lib, "mesa_debug_skip_commit")          # fault injection lives in the debug build only


def test_debug_build_exports_the_injection_entry():
    from test_sequence_layer_b200 import build as b
    dlib = ctypes.CDLL(b.build(debug=True))
    names = declared_functions(debug=True)
    assert "mesa_debug_skip_commit" in names
    for n in names:
        assert hasattr(dlib, n), n
    dlib.mesa_debug_skip_commit.argtypes = [ctypes.c_int]
    assert dlib.mesa_debug_skip_commit(-1) == 1                 # MESA_ERR_INVALID_ARG, no device call


def test_status_strings(lib):
    for code, name in enumerate(["MESA_OK", "MESA_ERR_INVALID_ARG", "MESA_ERR_UNSUPPORTED",
                                 "MESA_ERR_WORKSPACE", "MESA_ERR_CUDA", "MESA_ERR_DEVICE_TIMEOUT"]):
        assert lib.mesa_status_string(code).decode() == name
    assert lib.mesa_status_string(99).decode() == "MESA_ERR_UNKNOWN"


def test_workspace_size(lib):
    f = lib.mesa_forward_workspace_size
    assert f(1, 1, 64, 16, 16, 16, 0) == 4 * (16 * 16 * 2) * 4            # 4 chunks x (H + G) fp32
    assert f(1, 1, 65, 16, 16, 16, 0) == 5 * (16 * 16 * 2) * 4            # ragged tail adds a chunk
    assert f(8, 16, 8192, 128, 128, 64, 1) > 0
    assert f(0, 1, 64, 16, 16, 16, 0) == 0                                # invalid
    assert f(1, 1, 64, 48, 48, 16, 0) == 0                                # unsupported width
    assert f(1, 1, 64, 16, 32, 16, 0) == 0                                # dk != dv
    assert f(1, 1, 64, 16, 16, 24, 0) == 0                                # unsupported chunk
    assert lib.mesa_forward_host_workspace_size(1, 1, 64, 16, 16, 16, 0) > f(1, 1, 64, 16, 16, 16, 0)


FAKE = 1 << 20   # aligned, never dereferenced: every call below is rejected first


def fwd(lib, **kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, gamma=FAKE, beta=FAKE, lam=FAKE, B=1, H=1, T=64, dk=16, dv=16,
             chunk=16, dtype=0, N=8, tol=0.0, out=FAKE, iters=None, Hi=None, Gi=None, Ho=None, Go=None,
             ws=FAKE, wsb=1 << 30)
    a.update(kw)
    return lib.mesa_forward(a["q"], a["k"], a["v"], a["gamma"], a["beta"], a["lam"], a["B"], a["H"], a["T"],
                            a["dk"], a["dv"], a["chunk"], a["dtype"], a["N"], ctypes.c_float(a["tol"]),
                            a["out"], a["iters"], a["Hi"], a["Gi"], a["Ho"], a["Go"], a["ws"], a["wsb"], None)


@pytest.mark.parametrize("kw,code", [
    (dict(q=None), 1), (dict(k=None), 1), (dict(v=None), 1), (dict(gamma=None), 1), (dict(beta=None), 1),
    (dict(lam=None), 1), (dict(out=None), 1),
    (dict(B=0), 1), (dict(H=-1), 1), (dict(T=-5), 1), (dict(dtype=7), 1),
    (dict(N=-1), 1), (dict(N=5000), 1), (dict(tol=float("nan")), 1),
    (dict(dk=48, dv=48), 2), (dict(dk=16, dv=32), 2), (dict(chunk=24), 2), (dict(B=300, H=300), 2),
    (dict(q=FAKE + 8), 1), (dict(out=FAKE + 4), 1), (dict(gamma=FAKE + 2), 1), (dict(iters=FAKE + 2), 1),
    (dict(Hi=FAKE + 4), 1), (dict(Ho=FAKE, Hi=FAKE), 1),
    (dict(ws=None), 3), (dict(wsb=100), 3), (dict(ws=FAKE + 16), 1),
])
def test_forward_rejects_bad_arguments(lib, kw, code):
    assert fwd(lib, **kw) == code


def step(lib, **kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, gamma=FAKE, beta=FAKE, lam=FAKE, B=2, H=2, dk=16, dv=16,
             Hs=FAKE, Gs=FAKE + 4096, N=8, tol=0.0, out=FAKE, iters=None)
    a.update(kw)
    return lib.mesa_step(a["q"], a["k"], a["v"], a["gamma"], a["beta"], a["lam"], a["B"], a["H"], a["dk"],
                         a["dv"], a["Hs"], a["Gs"], a["N"], ctypes.c_float(a["tol"]), a["out"], a["iters"], None)


@pytest.mark.parametrize("kw,code", [
    (dict(q=None), 1), (dict(Hs=None), 1), (dict(Gs=None), 1), (dict(out=None), 1), (dict(lam=None), 1),
    (dict(B=0), 1), (dict(N=-2), 1), (dict(tol=float("nan")), 1),
    (dict(dk=24, dv=24), 2), (dict(dk=16, dv=64), 2),
    (dict(q=FAKE + 4), 1), (dict(Hs=FAKE + 8), 1), (dict(Gs=FAKE), 1),
])
def test_step_rejects_bad_arguments(lib, kw, code):
    assert step(lib, **kw) == code


def test_host_variant_rejects_bad_arguments(lib):
    f = lib.mesa_forward_host
    args = [FAKE] * 6 + [1, 1, 64, 16, 16, 16, 0, 8, ctypes.c_float(0.0), FAKE, None, None, None, None, None]
    assert f(*args, None, 0, None) == 3                               # no workspace
    bad = list(args)
    bad[8] = -1
    assert f(*bad, FAKE, 1 << 30, None) == 1
    assert f(*args, FAKE + 64, 1 << 30, None) == 1                    # misaligned workspace


def test_product_does_not_import_oracle():
    pkg = os.path.join(ROOT, "test_sequence_layer_b200")
    for dirpath, _, files in os.walk(pkg):
        for fn in files:
            if fn.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                src = open(os.path.join(dirpath, fn)).read()
                assert "oracle" not in src.lower().replace("oracles", ""), fn


def test_preprocess_argument_errors(lib):
    P, I = ctypes.c_void_p, ctypes.c_int
    lib.mesa_preprocess.argtypes = [P, P, P, P, I, I, I, I, I, I, P, P, P]
    a, b_, c, o1, o2 = (ctypes.c_void_p(0x10000 * i) for i in (1, 3, 5, 7, 9))
    call = lambda W=4, d=128, T=8, dt=1, q=a, o=o1: lib.mesa_preprocess(q, b_, c, c, 1, 1, T, d, W, dt, o, o2, None)  # noqa: E731
    assert call(W=0) == 1 and call(W=5) == 1                    # window out of range
    assert call(d=48) == 2                                      # unsupported width
    assert call(dt=7) == 1                                      # bad dtype
    assert call(T=0, q=None) == 0                               # nothing to do, no pointer needed
    assert call(q=None) == 1                                    # null input
    assert call(q=ctypes.c_void_p(0x10008)) == 1                # misaligned
    assert call(o=a) == 1                                       # output overlaps input


def test_backward_argument_errors(lib):
    """Host-side checks of mesa_backward (fake, aligned device addresses; every
    case is rejected before any launch)."""
    B, H, T, d = 1, 2, 8, 16
    tok = B * H * T
    addr = iter(range(1 << 20, 1 << 40, 1 << 20))       # disjoint 1 MiB spans, 256-byte aligned
    bufs = {n: next(addr) for n in ("q", "k", "v", "g", "b", "lam", "do", "dq", "dk", "dv", "dg", "db", "dl", "ws")}
    need = lib.mesa_backward_workspace_size(B, H, T, d, d, 16, 0)
    assert need > tok * d * 4

    def call(ws_bytes=None, dk=d, **over):
        p = dict(bufs, **over)
        return lib.mesa_backward(p["q"], p["k"], p["v"], p["g"], p["b"], p["lam"], B, H, T, dk, dk, 16, 0, 15, 0.0,
                                 p["do"], p["dq"], p["dk"], p["dv"], p["dg"], p["db"], p["dl"], p["ws"],
                                 need if ws_bytes is None else ws_bytes, None)
    assert call(dk=24) == 2                               # unsupported width
    assert call(q=None) == 1
    assert call(do=bufs["do"] + 4) == 1                   # misaligned
    assert call(dq=bufs["q"]) == 1                        # output overlaps an input
    assert call(dv=bufs["dk"] + 64) == 1                  # outputs overlap each other
    assert call(ws_bytes=need - 1) == 3                   # workspace too small
    assert call(ws=bufs["ws"] + 16) == 1                  # workspace misaligned
    assert lib.mesa_backward_workspace_size(B, H, T, 24, 24, 16, 0) == 0


def test_sharding_argument_errors(lib):
    """mesa_chunk_state and mesa_state_prefix reject bad arguments on the host."""
    B, H, T, d = 1, 2, 8, 16
    a = 1 << 24
    need = lib.mesa_chunk_state_workspace_size(B, H, T, d, d, 16, 0)
    assert need > 0
    cs = lambda k=a, Ho=a + (1 << 20), Go=a + (2 << 20), dec=a + (3 << 20), ws=a + (4 << 20), wsb=need, dk=d: \
        lib.mesa_chunk_state(k, a, a, a, B, H, T, dk, dk, 16, 0, None, None, Ho, Go, dec, ws, wsb, None)  # noqa: E731
    assert cs(dk=24) == 2
    assert cs(k=None) == 1
    assert cs(Ho=None) == 1
    assert cs(Ho=a + (1 << 20) + 8) == 1                     # misaligned
    assert cs(wsb=need - 1) == 3
    sp = lambda n=2, r=1, Hi=a + (8 << 20), Gi=a + (9 << 20), dk=d: \
        lib.mesa_state_prefix(a, a + (1 << 20), a + (2 << 20), n, r, B, H, dk, dk, Hi, Gi, None)  # noqa: E731
    assert sp(r=3) == 1                                      # r > n_slices
    assert sp(r=-1) == 1
    assert sp(dk=24) == 2
    assert sp(Hi=a) == 1                                     # output overlaps the stacked inputs
    assert sp(Gi=a + (8 << 20)) == 1                         # outputs overlap each other
