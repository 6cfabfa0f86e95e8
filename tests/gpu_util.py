"""Helpers shared by the GPU parity tests: run the CUDA library through its C ABI (via the thin
binding) on seeded workloads, and bring results back as numpy arrays shaped like the oracle's."""
import numpy as np

from differentiable_adaptive_ode_b200 import gradsolve as G
from differentiable_adaptive_ode_b200 import workloads as W


def torch():
    import torch as _t
    return _t


def dev(a, dtype):
    t = torch()
    return t.as_tensor(np.ascontiguousarray(a), dtype=dtype, device="cuda")


def tdtype(w):
    t = torch()
    return t.float64 if w.dtype == np.float64 else t.float32


def gsys(w, method=None):
    field = "linear3" if w.field.startswith("linear") else w.field
    return G.system(field, method or w.method, "f64" if w.dtype == np.float64 else "f32",
                    w.theta_shared)


def forward(w, max_attempts=0):
    t = torch()
    dt = tdtype(w)
    th, y0 = dev(w.theta, dt), dev(w.y0, dt)
    y1 = t.empty((w.N, w.d), dtype=dt, device="cuda")
    S = t.empty(w.N, dtype=t.int32, device="cuda")
    rej = t.empty(w.N, dtype=t.int32, device="cuda")
    st = t.empty(w.N, dtype=t.int32, device="cuda")
    G.gs_solve_forward(gsys(w), w.N, th, y0, w.t0, w.t1, w.rtol, w.atol, y1, S, rej, st,
                       opts=G.options(max_attempts))
    t.cuda.synchronize()
    return dict(y1=y1.cpu().numpy(), S=S.cpu().numpy(), rejected=rej.cpu().numpy(),
                status=st.cpu().numpy())


def record(w, rec=None, capacity=0, allow_failed=False, max_attempts=0):
    t = torch()
    dt = tdtype(w)
    th, y0 = dev(w.theta, dt), dev(w.y0, dt)
    y1 = t.empty((w.N, w.d), dtype=dt, device="cuda")
    st = t.empty(w.N, dtype=t.int32, device="cuda")
    rec = G.gs_solve_record(gsys(w), w.N, th, y0, w.t0, w.t1, w.rtol, w.atol, y1, st, rec=rec,
                            opts=G.options(max_attempts, capacity), allow_failed=allow_failed)
    t.cuda.synchronize()
    return rec, dict(y1=y1.cpu().numpy(), status=st.cpu().numpy())


def export_padded(w, rec):
    """The record as the oracle's padded rectangle: S[N], T/H [N, Smax], Y [N, Smax, d]."""
    t = torch()
    dt = tdtype(w)
    info = rec.info()
    tot = int(info.total_steps)
    T = t.empty(max(tot, 1), dtype=dt, device="cuda")
    H = t.empty(max(tot, 1), dtype=dt, device="cuda")
    Y = t.empty((max(tot, 1), w.d), dtype=dt, device="cuda")
    off = t.empty(w.N + 1, dtype=t.int64, device="cuda")
    G.gs_record_export(rec, T, H, Y, off)
    t.cuda.synchronize()
    off = off.cpu().numpy()
    S = np.diff(off).astype(np.int32)
    Smax = max(1, int(S.max()) if w.N else 1)
    Tn, Hn, Yn = T.cpu().numpy(), H.cpu().numpy(), Y.cpu().numpy()
    Tp = np.zeros((w.N, Smax), w.dtype)
    Hp = np.zeros((w.N, Smax), w.dtype)
    Yp = np.zeros((w.N, Smax, w.d), w.dtype)
    for k in range(w.N):
        a, b = off[k], off[k + 1]
        Tp[k, :b - a] = Tn[a:b]
        Hp[k, :b - a] = Hn[a:b]
        Yp[k, :b - a] = Yn[a:b]
    return dict(S=S, T=Tp, H=Hp, Y=Yp, offsets=off, info=info)


def replay_grad(w, rec, lam, theta=None, want_theta=True, want_y0=True):
    t = torch()
    dt = tdtype(w)
    th = dev(w.theta if theta is None else theta, dt)
    lam_t = dev(lam, dt)
    gy = t.empty((w.N, w.d), dtype=dt, device="cuda") if want_y0 else None
    if want_theta:
        gt = t.empty((w.m,) if w.theta_shared else (w.N, w.m), dtype=dt, device="cuda")
    else:
        gt = None
    G.gs_replay_grad(rec, th, lam_t, gt, gy)
    t.cuda.synchronize()
    return (None if gy is None else gy.cpu().numpy(), None if gt is None else gt.cpu().numpy())


def import_record(w, S, T, H, Y):
    """Record from padded oracle arrays (ragged-packed here, then imported on the device)."""
    t = torch()
    dt = tdtype(w)
    S = np.asarray(S, np.int32)
    Tr = np.concatenate([T[k, :S[k]] for k in range(w.N)]) if S.sum() else np.zeros(1)
    Hr = np.concatenate([H[k, :S[k]] for k in range(w.N)]) if S.sum() else np.zeros(1)
    Yr = np.concatenate([Y[k, :S[k]] for k in range(w.N)]) if S.sum() else np.zeros((1, w.d))
    return G.gs_record_import(gsys(w), w.N, dev(S, t.int32), dev(Tr, dt), dev(Hr, dt),
                              dev(Yr, dt))


def rel_rows(a, b, floor):
    """Per-row relative max-norm difference ||a - b||_inf / max(||b||_inf, floor)."""
    a = np.asarray(a, np.float64).reshape(len(a), -1)
    b = np.asarray(b, np.float64).reshape(len(b), -1)
    return np.max(np.abs(a - b), axis=1) / np.maximum(np.max(np.abs(b), axis=1), floor)


def small(name, N):
    return W.by_name(name, N=N)


def forward_sens(w, S0=None, max_attempts=0):
    """gs_solve_forward_sens on the workload: y1, S (= dy/dtheta [N, d, m]), counts, status."""
    t = torch()
    dt = tdtype(w)
    th, y0 = dev(w.theta, dt), dev(w.y0, dt)
    y1 = t.empty((w.N, w.d), dtype=dt, device="cuda")
    S1 = t.empty((w.N, w.d, w.m), dtype=dt, device="cuda")
    S = t.empty(w.N, dtype=t.int32, device="cuda")
    rej = t.empty(w.N, dtype=t.int32, device="cuda")
    st = t.empty(w.N, dtype=t.int32, device="cuda")
    G.gs_solve_forward_sens(gsys(w), w.N, th, y0, w.t0, w.t1, w.rtol, w.atol, y1, S1,
                            None if S0 is None else dev(S0, dt), S, rej, st,
                            opts=G.options(max_attempts))
    t.cuda.synchronize()
    return dict(y1=y1.cpu().numpy(), sens=S1.cpu().numpy(), S=S.cpu().numpy(),
                rejected=rej.cpu().numpy(), status=st.cpu().numpy())
