"""Python face of the CPU oracle (TEST INFRASTRUCTURE ONLY).

Only the test suite, the smoke check and the benchmark's CPU-baseline leg may import this
module.  It loads oracle/liboracle.so (building it with g++ when missing or stale) and passes
numpy arrays to the C entry points of gs_oracle.cpp.  Nothing here touches the CUDA library.

Records here are padded rectangles [N, Smax] with counts S[N] -- the layout the pages describe
for their replay ("gradsolve: fast exact gradients for ODE ensembles on GPUs", §3: each record
padded to the longest one).
"""
import ctypes as C
import os

import numpy as np

from . import build_oracle

FIELDS = {"lotka_volterra": 0, "lorenz63": 1, "mlp": 2, "robertson": 3, "nfw_mn": 4,
          "linear1": 5, "linear2": 6, "linear3": 7, "log_halo": 8, "hires": 9}
METHODS = {"tsit5": 0, "ros34pw2": 1, "vern7": 2, "rosenbrock23": 3}

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = build_oracle.build()
        L = C.CDLL(path)
        vp, i, ll, d = C.c_void_p, C.c_int, C.c_longlong, C.c_double
        L.orc_field_dims.argtypes = [i, C.POINTER(C.c_int), C.POINTER(C.c_int)]
        L.orc_solve.argtypes = [i, i, i, ll, i, vp, vp, d, d, d, d, ll, vp, vp, vp, vp, vp, i, i,
                                vp, vp, vp, i]
        L.orc_replay.argtypes = [i, i, i, ll, i, vp, vp, vp, vp, i, vp, i]
        L.orc_replay_grad.argtypes = [i, i, i, ll, i, vp, vp, vp, vp, i, vp, vp, vp, i]
        L.orc_replay_outputs.argtypes = [i, i, i, ll, i, vp, vp, vp, vp, vp, i, d, i, vp, vp, i]
        L.orc_replay_outputs_grad.argtypes = [i, i, i, ll, i, vp, vp, vp, vp, vp, i, d, i, vp, vp,
                                              vp, vp, i]
        L.orc_replay_jvp.argtypes = [i, i, i, ll, i, vp, vp, vp, vp, vp, vp, i, vp, vp, i]
        L.orc_solve_sens.argtypes = [i, i, ll, i, vp, vp, vp, d, d, d, d, ll, vp, vp, vp, vp, vp,
                                     i]
        L.orc_rhs.argtypes = [i, ll, i, vp, vp, vp]
        L.orc_jac.argtypes = [i, ll, i, vp, vp, vp]
        L.orc_trial.argtypes = [i, i, vp, vp, d, vp, vp]
        L.orc_count_ops.argtypes = [i, i, vp, vp, d, vp]
        L.orc_tsit5_tableau.argtypes = [vp, vp, vp, vp]
        L.orc_ros34pw2_tableau.argtypes = [vp, vp, vp, vp, vp]
        L.orc_vern7_tableau.argtypes = [vp, vp, vp]
        _lib = L
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data_as(C.c_void_p)


def _dt(dtype):
    return {np.float64: 0, np.float32: 1}[np.dtype(dtype).type]


def dims(field):
    D, M = C.c_int(), C.c_int()
    rc = lib().orc_field_dims(FIELDS[field], C.byref(D), C.byref(M))
    assert rc == 0
    return D.value, M.value


def _prep(field, theta, y0, dtype, theta_shared):
    D, M = dims(field)
    y0 = np.ascontiguousarray(y0, dtype=dtype).reshape(-1, D)
    N = y0.shape[0]
    theta = np.ascontiguousarray(theta, dtype=dtype)
    if theta_shared:
        theta = theta.reshape(M)
    else:
        theta = theta.reshape(N, M)
    return D, M, N, theta, y0


def solve(field, method, theta, y0, t0, t1, rtol, atol, dtype=np.float64, theta_shared=False,
          max_attempts=100000, keep_record=False, Smax=0, nthreads=1):
    """Adaptive solve of every trajectory; with keep_record, the accepted (t_n, h_n, y_n)."""
    D, M, N, theta, y0 = _prep(field, theta, y0, dtype, theta_shared)
    y1 = np.zeros((N, D), dtype)
    S = np.zeros(N, np.int32)
    rej = np.zeros(N, np.int32)
    status = np.zeros(N, np.int32)
    att = np.zeros(N, np.int64)
    T = H = Y = None
    if keep_record:
        if Smax <= 0:
            r = solve(field, method, theta, y0, t0, t1, rtol, atol, dtype, theta_shared,
                      max_attempts, False, 0, nthreads)
            Smax = max(1, int(r["S"].max()))
        T = np.zeros((N, Smax), dtype)
        H = np.zeros((N, Smax), dtype)
        Y = np.zeros((N, Smax, D), dtype)
    rc = lib().orc_solve(FIELDS[field], METHODS[method], _dt(dtype), N, int(theta_shared),
                         _p(theta), _p(y0), t0, t1, rtol, atol, max_attempts, _p(y1), _p(S),
                         _p(rej), _p(status), _p(att), int(keep_record), Smax, _p(T), _p(H),
                         _p(Y), nthreads)
    if rc < 0:
        raise ValueError("orc_solve rejected its arguments (%d)" % rc)
    if rc == 1:
        raise ValueError("a record exceeded Smax=%d" % Smax)
    out = dict(y1=y1, S=S, rejected=rej, status=status, attempts=att)
    if keep_record:
        out.update(T=T, H=H, Y=Y)
    return out


def replay(field, method, theta, y0, H, S, dtype=np.float64, theta_shared=False, nthreads=1):
    """y_S of the fixed-step chain over the padded mesh H[N, Smax] (first S[k] entries used)."""
    D, M, N, theta, y0 = _prep(field, theta, y0, dtype, theta_shared)
    H = np.ascontiguousarray(H, dtype=dtype).reshape(N, -1)
    S = np.ascontiguousarray(S, dtype=np.int32)
    out = np.zeros((N, D), dtype)
    rc = lib().orc_replay(FIELDS[field], METHODS[method], _dt(dtype), N, int(theta_shared),
                          _p(theta), _p(y0), _p(H), _p(S), H.shape[1], _p(out), nthreads)
    assert rc == 0, rc
    return out


def replay_grad(field, method, theta, y0, H, S, lam, dtype=np.float64, theta_shared=False,
                nthreads=1):
    """(dL/dy0 [N, D], dL/dtheta [N, M] per trajectory) of the replay with the mesh held fixed."""
    D, M, N, theta, y0 = _prep(field, theta, y0, dtype, theta_shared)
    H = np.ascontiguousarray(H, dtype=dtype).reshape(N, -1)
    S = np.ascontiguousarray(S, dtype=np.int32)
    lam = np.ascontiguousarray(lam, dtype=dtype).reshape(N, D)
    gy = np.zeros((N, D), dtype)
    gt = np.zeros((N, M), dtype)
    rc = lib().orc_replay_grad(FIELDS[field], METHODS[method], _dt(dtype), N, int(theta_shared),
                               _p(theta), _p(y0), _p(H), _p(S), H.shape[1], _p(lam), _p(gy),
                               _p(gt), nthreads)
    assert rc == 0, rc
    return gy, gt


def replay_outputs(field, method, theta, y0, T, H, S, t1, tau, dtype=np.float64,
                   theta_shared=False, nthreads=1):
    """States at requested times tau (ascending, in [t0, t1]): one extra step from the preceding
    recorded mesh point to each tau ([GS] §3.4).  Returns [N, J, D]."""
    D, M, N, theta, y0 = _prep(field, theta, y0, dtype, theta_shared)
    T = np.ascontiguousarray(T, dtype=dtype).reshape(N, -1)
    H = np.ascontiguousarray(H, dtype=dtype).reshape(N, -1)
    S = np.ascontiguousarray(S, dtype=np.int32)
    tau = np.ascontiguousarray(tau, dtype=dtype)
    out = np.zeros((N, len(tau), D), dtype)
    rc = lib().orc_replay_outputs(FIELDS[field], METHODS[method], _dt(dtype), N,
                                  int(theta_shared), _p(theta), _p(y0), _p(T), _p(H), _p(S),
                                  H.shape[1], t1, len(tau), _p(tau), _p(out), nthreads)
    assert rc == 0, rc
    return out


def replay_outputs_grad(field, method, theta, y0, T, H, S, t1, tau, lam, dtype=np.float64,
                        theta_shared=False, nthreads=1):
    """(dL/dy0 [N, D], dL/dtheta [N, M]) of L = sum_k sum_j lam[k, j] . y_k(tau_j)."""
    D, M, N, theta, y0 = _prep(field, theta, y0, dtype, theta_shared)
    T = np.ascontiguousarray(T, dtype=dtype).reshape(N, -1)
    H = np.ascontiguousarray(H, dtype=dtype).reshape(N, -1)
    S = np.ascontiguousarray(S, dtype=np.int32)
    tau = np.ascontiguousarray(tau, dtype=dtype)
    lam = np.ascontiguousarray(lam, dtype=dtype).reshape(N, len(tau), D)
    gy = np.zeros((N, D), dtype)
    gt = np.zeros((N, M), dtype)
    rc = lib().orc_replay_outputs_grad(FIELDS[field], METHODS[method], _dt(dtype), N,
                                       int(theta_shared), _p(theta), _p(y0), _p(T), _p(H),
                                       _p(S), H.shape[1], t1, len(tau), _p(tau), _p(lam), _p(gy),
                                       _p(gt), nthreads)
    assert rc == 0, rc
    return gy, gt


def replay_jvp(field, method, theta, y0, thdot, ydot0, H, S, dtype=np.float64, theta_shared=False,
               nthreads=1):
    """(y_S, tangent of y_S along (ydot0, thdot)) over the padded mesh H (forward mode)."""
    D, M, N, theta, y0 = _prep(field, theta, y0, dtype, theta_shared)
    thdot = np.ascontiguousarray(thdot, dtype=dtype).reshape(theta.shape)
    ydot0 = np.ascontiguousarray(ydot0, dtype=dtype).reshape(N, D)
    H = np.ascontiguousarray(H, dtype=dtype).reshape(N, -1)
    S = np.ascontiguousarray(S, dtype=np.int32)
    y1 = np.zeros((N, D), dtype)
    yd1 = np.zeros((N, D), dtype)
    rc = lib().orc_replay_jvp(FIELDS[field], METHODS[method], _dt(dtype), N, int(theta_shared),
                              _p(theta), _p(y0), _p(thdot), _p(ydot0), _p(H), _p(S), H.shape[1],
                              _p(y1), _p(yd1), nthreads)
    assert rc == 0, rc
    return y1, yd1


def solve_sens(field, theta, y0, t0, t1, rtol, atol, S0=None, dtype=np.float64,
               theta_shared=False, max_attempts=100000, nthreads=1):
    """Tsit5 solve of the orbit together with S = dy/dtheta [N, D, M], step control on y alone."""
    D, M, N, theta, y0 = _prep(field, theta, y0, dtype, theta_shared)
    if S0 is not None:
        S0 = np.ascontiguousarray(S0, dtype=dtype).reshape(N, D, M)
    y1 = np.zeros((N, D), dtype)
    S1 = np.zeros((N, D, M), dtype)
    S = np.zeros(N, np.int32)
    rej = np.zeros(N, np.int32)
    status = np.zeros(N, np.int32)
    rc = lib().orc_solve_sens(FIELDS[field], _dt(dtype), N, int(theta_shared), _p(theta), _p(y0),
                              _p(S0), t0, t1, rtol, atol, max_attempts, _p(y1), _p(S1), _p(S),
                              _p(rej), _p(status), nthreads)
    assert rc == 0, rc
    return {"y1": y1, "sens": S1, "S": S, "rejected": rej, "status": status}


def rhs(field, theta, y, theta_shared=False):
    D, M, N, theta, y = _prep(field, theta, y, np.float64, theta_shared)
    out = np.zeros((N, D))
    assert lib().orc_rhs(FIELDS[field], N, int(theta_shared), _p(theta), _p(y), _p(out)) == 0
    return out


def jac(field, theta, y, theta_shared=False):
    D, M, N, theta, y = _prep(field, theta, y, np.float64, theta_shared)
    out = np.zeros((N, D, D))
    assert lib().orc_jac(FIELDS[field], N, int(theta_shared), _p(theta), _p(y), _p(out)) == 0
    return out


def trial(field, method, theta, y, h):
    D, M = dims(field)
    theta = np.ascontiguousarray(theta, np.float64).reshape(M)
    y = np.ascontiguousarray(y, np.float64).reshape(D)
    ynew, e = np.zeros(D), np.zeros(D)
    assert lib().orc_trial(FIELDS[field], METHODS[method], _p(theta), _p(y), h, _p(ynew),
                           _p(e)) == 0
    return ynew, e


OP_NAMES = ("add", "mul", "div", "sqrt", "log1p", "tanh")


def count_ops(field, what, theta, y, h=0.1):
    """Tally of one f evaluation (what='f'), Tsit5 trial ('tsit5'), ROS34PW2 trial ('ros') or f
    with one tangent direction by the forward-mode rules ('f_dual'), or the plain reverse sweep
    of f's vector-Jacobian product with respect to (y, theta) ('vjp_reverse')."""
    D, M = dims(field)
    theta = np.ascontiguousarray(theta, np.float64).reshape(M)
    y = np.ascontiguousarray(y, np.float64).reshape(D)
    counts = np.zeros(6, np.int64)
    rc = lib().orc_count_ops(FIELDS[field], {"f": 0, "tsit5": 1, "ros": 2, "f_dual": 3, "vjp_reverse": 4}[what], _p(theta),
                             _p(y), h, _p(counts))
    assert rc == 0, rc
    return dict(zip(OP_NAMES, counts.tolist()))


def tsit5_tableau():
    c, A, b, bt = np.zeros(7), np.zeros((7, 7)), np.zeros(7), np.zeros(7)
    lib().orc_tsit5_tableau(_p(c), _p(A), _p(b), _p(bt))
    return c, A, b, bt


def vern7_tableau():
    A, b, bh = np.zeros((10, 10)), np.zeros(10), np.zeros(10)
    lib().orc_vern7_tableau(_p(A), _p(b), _p(bh))
    return A, b, bh


def ros34pw2_tableau():
    g = np.zeros(1)
    al, ga, b, bh = np.zeros((4, 4)), np.zeros((4, 4)), np.zeros(4), np.zeros(4)
    lib().orc_ros34pw2_tableau(_p(g), _p(al), _p(ga), _p(b), _p(bh))
    return float(g[0]), al, ga, b, bh


def host_threads():
    return len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count()
