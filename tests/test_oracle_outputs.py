"""Pins of the oracle's outputs at requested times and their gradient.

"gradsolve: fast exact gradients for ODE ensembles on GPUs", §3.4: the replay takes one extra
solver step from the preceding mesh point exactly to each requested time, so the returned state is
integrated, not interpolated.  Pinned here by: a requested time on a mesh point returns the
recorded state bit for bit; t1 returns the final state; the linear family's closed form
(R(h' A) times the product of the step matrices) for the outputs and their gradient; central
differences for a nonlinear field; and agreement with a tight solve to the tolerance's order.
"""
import numpy as np
import pytest

from differentiable_adaptive_ode_b200 import workloads as W


def _rec(orc, w):
    r = orc.solve(w.field, w.method, w.theta, w.y0, w.t0, w.t1, w.rtol, w.atol, keep_record=True,
                  theta_shared=w.theta_shared)
    assert np.all(r["status"] == 0)
    return r


def test_outputs_on_mesh_points_and_end(orc):
    w = W.lorenz63(N=3)
    r = _rec(orc, w)
    for k in range(3):
        S = int(r["S"][k])
        picks = [0, S // 3, S // 2, S - 1]
        tau = np.array([r["T"][k, n] for n in picks] + [w.t1])
        out = orc.replay_outputs(w.field, w.method, w.theta[k:k + 1], w.y0[k:k + 1],
                                 r["T"][k:k + 1], r["H"][k:k + 1], r["S"][k:k + 1], w.t1, tau)
        for j, n in enumerate(picks):
            assert np.array_equal(out[0, j], r["Y"][k, n])
        assert np.array_equal(out[0, -1], r["y1"][k])


def _tsit5_Rmat(Z, A, b):
    d = Z.shape[0]
    R = np.eye(d, dtype=Z.dtype)
    P = np.eye(d, dtype=Z.dtype)
    v = np.ones(len(b))
    for q in range(1, len(b) + 1):
        P = P @ Z
        R = R + (b @ v) * P
        v = A @ v
    return R


def test_outputs_and_gradient_linear_closed_form(orc):
    c, At, b, bt = orc.tsit5_tableau()
    rng = np.random.default_rng(3)
    Amat = rng.normal(size=(3, 3)) * 0.6 - 1.0 * np.eye(3)
    y0 = rng.normal(size=3)
    r = orc.solve("linear3", "tsit5", Amat.ravel(), y0, 0.0, 3.0, 1e-7, 1e-9, keep_record=True)
    S = int(r["S"][0])
    T, H = r["T"][0, :S], r["H"][0, :S]
    tau = np.sort(np.concatenate([rng.uniform(0, 3, size=5), [T[2], 3.0]]))
    out = orc.replay_outputs("linear3", "tsit5", Amat.ravel(), y0, r["T"], r["H"], r["S"], 3.0, tau)
    lam = rng.normal(size=(len(tau), 3))
    gy, gA = orc.replay_outputs_grad("linear3", "tsit5", Amat.ravel(), y0, r["T"], r["H"], r["S"],
                                     3.0, tau, lam)

    def closed(Amat_c):
        Ms, outs = [], []
        for tj in tau:
            if tj >= 3.0:
                n, hp = S, 0.0
            else:
                n = int(np.searchsorted(T, tj, side="right") - 1)
                hp = tj - T[n]
            M = np.eye(3, dtype=Amat_c.dtype)
            for m in range(n):
                M = _tsit5_Rmat(H[m] * Amat_c, At, b) @ M
            M = _tsit5_Rmat(hp * Amat_c, At, b) @ M
            Ms.append(M)
            outs.append(M @ y0)
        return Ms, outs

    Ms, outs = closed(Amat)
    for j in range(len(tau)):
        assert np.max(np.abs(out[0, j] - outs[j])) <= 1e-12 * (1 + np.max(np.abs(outs[j])))
    want_y0 = sum(Ms[j].T @ lam[j] for j in range(len(tau)))
    assert np.max(np.abs(gy[0] - want_y0)) <= 1e-12 * np.max(np.abs(want_y0))
    eps = 1e-30
    for (i, jj) in [(0, 1), (2, 2)]:
        E = np.zeros((3, 3))
        E[i, jj] = 1.0
        _, oc = closed(Amat + 1j * eps * E)
        ref = sum(lam[j] @ oc[j] for j in range(len(tau))).imag / eps
        assert abs(gA[0, 3 * i + jj] - ref) <= 1e-11 * max(1.0, abs(ref))


@pytest.mark.parametrize("name", ["lorenz63", "robertson", "nfw_mn"])
def test_outputs_gradient_central_differences(orc, name):
    w = W.by_name(name, N=2)
    r = _rec(orc, w)
    tau = np.linspace(w.t0, w.t1, 7)[1:]
    rng = np.random.default_rng(4)
    lam = rng.normal(size=(w.N, len(tau), w.d))
    gy, gt = orc.replay_outputs_grad(w.field, w.method, w.theta, w.y0, r["T"], r["H"], r["S"],
                                     w.t1, tau, lam)
    L = lambda th, y0: np.sum(lam * orc.replay_outputs(w.field, w.method, th, y0, r["T"], r["H"],
                                                       r["S"], w.t1, tau))
    tol = 2e-5 if name == "robertson" else 1e-6
    for c in range(w.d):
        e = 1e-6 * max(1.0, abs(w.y0[0, c]))
        yp, ym = w.y0.copy(), w.y0.copy()
        yp[0, c] += e
        ym[0, c] -= e
        fd = (L(w.theta, yp) - L(w.theta, ym)) / (2 * e)
        assert abs(fd - gy[0, c]) <= tol * max(1.0, abs(fd)), (c, fd, gy[0, c])
    for j in range(w.m):
        e = 1e-6 * abs(w.theta[0, j])
        tp, tm = w.theta.copy(), w.theta.copy()
        tp[0, j] += e
        tm[0, j] -= e
        fd = (L(tp, w.y0) - L(tm, w.y0)) / (2 * e)
        assert abs(fd - gt[0, j]) <= tol * max(1.0, abs(fd)), (j, fd, gt[0, j])


def test_outputs_are_integrated_to_tolerance(orc):
    w = W.lorenz63(N=4, seed=9)
    r = _rec(orc, w)
    tau = np.array([0.13, 0.41, 0.77])
    out = orc.replay_outputs(w.field, w.method, w.theta, w.y0, r["T"], r["H"], r["S"], w.t1, tau)
    for j, tj in enumerate(tau):
        ref = orc.solve(w.field, w.method, w.theta, w.y0, 0.0, tj, 1e-13, 1e-15)["y1"]
        err = np.max(np.abs(out[:, j] - ref) / (1 + np.abs(ref)))
        assert err < 1e-6, (tj, err)
