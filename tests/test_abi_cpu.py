"""The C-ABI library builds, loads without a GPU, exports every entry point its header declares,
and rejects bad arguments with status codes before touching the device."""
import ctypes as C
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "gradsolve_b200.h")


@pytest.fixture(scope="module")
def G():
    from differentiable_adaptive_ode_b200 import build, gradsolve
    build.build()
    gradsolve.lib()
    return gradsolve


def declared():
    src = open(HEADER).read()
    return set(re.findall(r"^\s*(?:gs_status|void|const char\s*\*)\s*(gs_\w+)\s*\(", src, re.M))


def test_header_declares_the_boundary():
    names = declared()
    for must in ("gs_solve_forward", "gs_solve_record", "gs_replay_grad", "gs_replay_forward",
                 "gs_record_info", "gs_record_export", "gs_record_import", "gs_record_destroy",
                 "gs_last_error"):
        assert must in names


def test_library_exports_every_declared_symbol(G):
    L = G.lib()
    for name in declared():
        assert hasattr(L, name), name
    assert set(G.EXPORTS) == declared()


def test_argument_errors_without_device(G):
    L = G.lib()
    s = G.system("lorenz63")
    o = G.options()
    args = lambda sys_, N, rtol=1e-6: (C.byref(sys_), C.byref(o), N, None, None, 0.0, 1.0, rtol,
                                       1e-9, None, None, None, None, None)
    bad = G.system("lorenz63")
    bad.d = 4
    assert L.gs_solve_forward(*args(bad, 10)) == G.GS_ERR_INVALID_ARG
    assert "d=3" in G.last_error()
    unk = G.system("lorenz63")
    unk.field = 42
    assert L.gs_solve_forward(*args(unk, 10)) == G.GS_ERR_INVALID_ARG
    assert L.gs_solve_forward(*args(s, -1)) == G.GS_ERR_INVALID_ARG
    assert L.gs_solve_forward(*args(s, 10)) == G.GS_ERR_INVALID_ARG       # NULL arrays
    assert L.gs_solve_forward(*args(s, 0, rtol=0.0)) == G.GS_ERR_INVALID_ARG
    wrong = G.system("lorenz63", method="ros34pw2")
    assert L.gs_solve_forward(*args(wrong, 10)) == G.GS_ERR_UNSUPPORTED
    # forward sensitivities: Tsit5 fields other than the MLP only; S1 required
    sargs = lambda sys_, N, S1=None: (C.byref(sys_), C.byref(o), N, C.c_void_p(8), C.c_void_p(8),
                                      None, 0.0, 1.0, 1e-6, 1e-9, C.c_void_p(8), S1, None, None,
                                      None, None)
    rob = G.system("robertson")
    assert L.gs_solve_forward_sens(*sargs(rob, 10, C.c_void_p(8))) == G.GS_ERR_UNSUPPORTED
    mlp = G.system("mlp", dtype="f32", theta_shared=True)
    assert L.gs_solve_forward_sens(*sargs(mlp, 10, C.c_void_p(8))) == G.GS_ERR_UNSUPPORTED
    assert L.gs_solve_forward_sens(*sargs(G.system("log_halo", theta_shared=True), 10)) \
        == G.GS_ERR_INVALID_ARG
    assert L.gs_replay_grad(None, None, None, None, None, None) == G.GS_ERR_INVALID_ARG
    assert L.gs_record_info(None, None) == G.GS_ERR_INVALID_ARG
    L.gs_record_destroy(None)


def test_binding_refuses_without_library(monkeypatch):
    from differentiable_adaptive_ode_b200 import gradsolve
    monkeypatch.setattr(gradsolve, "_lib", None)
    monkeypatch.setattr(gradsolve, "LIB_PATH", "/nonexistent/libgradsolve_b200.so")
    with pytest.raises(RuntimeError):
        gradsolve.lib()


def test_normal_build_has_no_violation_counter(G):
    import ctypes as C
    v = C.c_int64(0)
    assert G.lib().gs_checked_violations(C.byref(v)) == G.GS_ERR_UNSUPPORTED


def test_checked_build_compiles_and_exports():
    import ctypes as C
    from differentiable_adaptive_ode_b200 import build
    path = build.build(checked=True)
    L = C.CDLL(path)
    for name in declared():
        assert hasattr(L, name), name


def test_binding_refuses_host_tensors(G):
    # a host tensor's address is not readable by the kernels: the binding refuses it before the
    # library is called (the library itself also asks the runtime, on a GPU machine)
    torch = pytest.importorskip("torch")
    s = G.system("lorenz63")
    th = torch.zeros((4, 3), dtype=torch.float64)
    y0 = torch.zeros((4, 3), dtype=torch.float64)
    y1 = torch.empty_like(y0)
    with pytest.raises(ValueError, match="CUDA device"):
        G.gs_solve_forward(s, 4, th, y0, 0.0, 1.0, 1e-6, 1e-9, y1)
    with pytest.raises(ValueError, match="CUDA device"):
        G.options(start_order=torch.arange(4, dtype=torch.int32))
