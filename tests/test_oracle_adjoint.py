"""Pins of the oracle's replay gradient (the stop-gradient-mesh discrete adjoint).

"gradsolve: fast exact gradients for ODE ensembles on GPUs", §3: the returned quantity is the
derivative of the replay chain Psi(theta; sg[h]) with the recorded step sizes held fixed; the
correctness checks there perturb the same inputs inside the same recorded replay (central finite
differences), and the linear family has a closed-form sensitivity (§4.7).  Each check below
pins the oracle against something other than itself: a closed form for linear fields, central
differences of the replay for nonlinear ones.
"""
import numpy as np
import pytest

from differentiable_adaptive_ode_b200 import workloads as W


def _tsit5_Rmat(Z, A, b):
    d = Z.shape[0]
    R = np.eye(d)
    P = np.eye(d)
    v = np.ones(len(b))
    for q in range(1, len(b) + 1):
        P = P @ Z
        R = R + (b @ v) * P
        v = A @ v
    return R


def _ros_Rmat(Z, g, al, ga, b):
    d = Z.shape[0]
    I = np.eye(d, dtype=Z.dtype)
    beta = al + ga
    Minv = np.linalg.inv(I - g * Z)
    K = []
    for i in range(4):
        acc = I.copy()
        for j in range(i):
            acc = acc + beta[i, j] * K[j]
        K.append(Minv @ Z @ acc)
    return I + sum(b[i] * K[i] for i in range(4))


@pytest.mark.parametrize("method", ["tsit5", "ros34pw2"])
def test_linear_closed_form_y0_gradient(orc, method):
    rng = np.random.default_rng(7)
    A = rng.normal(size=(3, 3)) * 0.7 - 1.2 * np.eye(3)
    y0 = rng.normal(size=3)
    r = orc.solve("linear3", method, A.ravel(), y0, 0.0, 4.0, 1e-7, 1e-9, keep_record=True)
    S = int(r["S"][0])
    lam = rng.normal(size=3)
    gy, gA = orc.replay_grad("linear3", method, A.ravel(), y0, r["H"], r["S"], lam)
    if method == "tsit5":
        c, At, b, bt = orc.tsit5_tableau()
        Rm = lambda h: _tsit5_Rmat(h * A, At, b)
    else:
        g, al, ga, b, bh = orc.ros34pw2_tableau()
        Rm = lambda h: _ros_Rmat(h * A, g, al, ga, b)
    # y_S = R_{S-1} ... R_0 y0  =>  dL/dy0 = R_0^T ... R_{S-1}^T lam
    v = lam.copy()
    for n in range(S - 1, -1, -1):
        v = Rm(r["H"][0, n]).T @ v
    assert np.max(np.abs(gy[0] - v)) <= 1e-12 * np.max(np.abs(v))
    # dL/dA by perturbing A inside the closed form (complex step: exact to rounding)
    eps = 1e-30
    for (i, j) in [(0, 0), (1, 2), (2, 0)]:
        E = np.zeros((3, 3))
        E[i, j] = 1.0
        Ac = A + 1j * eps * E
        yv = y0.astype(complex)
        for n in range(S):
            h = r["H"][0, n]
            if method == "tsit5":
                yv = _tsit5_Rmat(h * Ac, At, b) @ yv
            else:
                yv = _ros_Rmat(h * Ac, g, al, ga, b) @ yv
        ref = (lam @ yv).imag / eps
        assert abs(gA[0, 3 * i + j] - ref) <= 1e-11 * max(1.0, abs(ref)), (i, j)


def test_scalar_theta_gradient_closed_form(orc):
    # y' = theta y: y_S = prod_n R(h_n theta) y0, so
    # dy_S/dtheta = y0 sum_n h_n R'(h_n theta) prod_{m != n} R(h_m theta)
    c, A, b, bt = orc.tsit5_tableau()
    coef = [1.0]
    v = np.ones(7)
    for q in range(1, 8):
        coef.append(b @ v)
        v = A @ v
    R = lambda z: sum(cq * z ** q for q, cq in enumerate(coef))
    dR = lambda z: sum(q * cq * z ** (q - 1) for q, cq in enumerate(coef) if q > 0)
    th, y0 = -1.3, 0.8
    r = orc.solve("linear1", "tsit5", [th], [y0], 0.0, 3.0, 1e-8, 1e-10, keep_record=True)
    S = int(r["S"][0])
    hs = r["H"][0, :S]
    Rs = np.array([R(h * th) for h in hs])
    dy = y0 * sum(hs[n] * dR(hs[n] * th) * np.prod(np.delete(Rs, n)) for n in range(S))
    gy, gt = orc.replay_grad("linear1", "tsit5", [th], [y0], r["H"], r["S"], [1.0])
    assert abs(gt[0, 0] - dy) <= 1e-12 * abs(dy)
    assert abs(gy[0, 0] - np.prod(Rs)) <= 1e-13 * abs(np.prod(Rs))


def _fd_check(orc, w, r, lam, idx_y, idx_t, rel_eps=1e-6, tol=1e-6):
    gy, gt = orc.replay_grad(w.field, w.method, w.theta, w.y0, r["H"], r["S"], lam,
                             theta_shared=w.theta_shared)
    L = lambda th, y0: np.sum(lam * orc.replay(w.field, w.method, th, y0, r["H"], r["S"],
                                                theta_shared=w.theta_shared))
    for (k, c) in idx_y:
        e = rel_eps * max(1.0, abs(w.y0[k, c]))
        yp, ym = w.y0.copy(), w.y0.copy()
        yp[k, c] += e
        ym[k, c] -= e
        fd = (L(w.theta, yp) - L(w.theta, ym)) / (2 * e)
        assert abs(fd - gy[k, c]) <= tol * max(1.0, abs(fd)), ("y0", k, c, fd, gy[k, c])
    for (k, j) in idx_t:
        th = w.theta
        e = rel_eps * max(1e-3, abs(th[j] if w.theta_shared else th[k, j]))
        tp, tm = th.copy(), th.copy()
        if w.theta_shared:
            tp[j] += e
            tm[j] -= e
            ref = gt[:, j].sum()
        else:
            tp[k, j] += e
            tm[k, j] -= e
            ref = gt[k, j]
        fd = (L(tp, w.y0) - L(tm, w.y0)) / (2 * e)
        assert abs(fd - ref) <= tol * max(1.0, abs(fd)), ("theta", k, j, fd, ref)


@pytest.mark.parametrize("name", ["lotka_volterra", "lorenz63", "nfw_mn", "robertson"])
def test_central_differences_in_the_recorded_replay(orc, name):
    w = W.by_name(name, N=4)
    r = orc.solve(w.field, w.method, w.theta, w.y0, w.t0, w.t1, w.rtol, w.atol,
                  keep_record=True, theta_shared=w.theta_shared)
    assert np.all(r["status"] == 0)
    lam = np.random.default_rng(3).normal(size=(w.N, w.d))
    idx_y = [(k, c) for k in range(2) for c in range(w.d)]
    idx_t = [(k, j) for k in range(2) for j in range(w.m)]
    if name == "robertson":
        # the rates span 10 decades; relative perturbations of each keep the FD well posed
        _fd_check(orc, w, r, lam, idx_y, idx_t, rel_eps=1e-6, tol=2e-5)
    else:
        _fd_check(orc, w, r, lam, idx_y, idx_t)


def test_central_differences_shared_mlp(orc):
    w = W.mlp(N=3)
    w.theta = w.theta.copy()
    w.theta[128:160] = 0.05                     # nonzero biases so every block is exercised
    w.theta[1344:1348] = [0.1, -0.1, 0.05, 0.0]
    r = orc.solve("mlp", "tsit5", w.theta, w.y0, 0.0, 1.0, 1e-7, 1e-9, keep_record=True,
                  theta_shared=True)
    lam = np.random.default_rng(4).normal(size=(3, 4))
    idx_t = [(0, j) for j in (0, 5, 130, 170, 1000, 1190, 1220, 1345)]
    _fd_check(orc, w, r, lam, [(0, 0), (1, 3), (2, 1)], idx_t, rel_eps=1e-5, tol=1e-6)


def test_fp32_gradient_tracks_fp64(orc):
    w = W.nfw_mn(N=8)
    r = orc.solve("nfw_mn", "tsit5", w.theta, w.y0, 0.0, 20.0, 1e-5, 1e-6, keep_record=True,
                  dtype=np.float32)
    lam = W.loss_cotangent(w, r["y1"], w.target)
    g64 = orc.replay_grad("nfw_mn", "tsit5", w.theta, w.y0, r["H"].astype(np.float64), r["S"],
                          lam)
    g32 = orc.replay_grad("nfw_mn", "tsit5", w.theta, w.y0, r["H"], r["S"], lam,
                          dtype=np.float32)
    for a, b in zip(g32, g64):
        rel = np.max(np.abs(a - b), axis=1) / np.max(np.abs(b), axis=1)
        assert np.median(rel) < 1e-4, rel
