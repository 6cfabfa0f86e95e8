"""Pins of the oracle's forward-mode tangent of the replay (forward sensitivities along one
direction: "gradsolve: fast exact gradients for ODE ensembles on GPUs" §4.4; "Differentiable
astrophysics at scale" §2).  Pinned by the linear closed form, central differences, and the
transpose identity with the (separately pinned) reverse-mode gradient:
lam . (J v) = (J^T lam) . v."""
import numpy as np
import pytest

from differentiable_adaptive_ode_b200 import workloads as W


def test_jvp_linear_closed_form(orc):
    c, At, b, bt = orc.tsit5_tableau()
    rng = np.random.default_rng(8)
    A = rng.normal(size=(3, 3)) * 0.5 - np.eye(3)
    y0 = rng.normal(size=3)
    r = orc.solve("linear3", "tsit5", A.ravel(), y0, 0.0, 2.0, 1e-8, 1e-10, keep_record=True)
    S = int(r["S"][0])
    yd0 = rng.normal(size=3)
    y1, yd1 = orc.replay_jvp("linear3", "tsit5", A.ravel(), y0, np.zeros(9), yd0, r["H"], r["S"])
    M = np.eye(3)
    for n in range(S):
        Z = r["H"][0, n] * A
        R = np.eye(3)
        P = np.eye(3)
        v = np.ones(7)
        for q in range(1, 8):
            P = P @ Z
            R = R + (b @ v) * P
            v = At @ v
        M = R @ M
    assert np.max(np.abs(yd1[0] - M @ yd0)) <= 1e-12 * np.max(np.abs(M @ yd0))
    assert np.max(np.abs(y1[0] - M @ y0)) <= 1e-12 * np.max(np.abs(M @ y0))


@pytest.mark.parametrize("name", ["lotka_volterra", "lorenz63", "nfw_mn"])
def test_jvp_transpose_identity_and_differences(orc, name):
    w = W.by_name(name, N=3)
    r = orc.solve(w.field, w.method, w.theta, w.y0, w.t0, w.t1, w.rtol, w.atol, keep_record=True)
    rng = np.random.default_rng(9)
    thd = rng.normal(size=w.theta.shape) * w.theta * 1e-2
    yd0 = rng.normal(size=w.y0.shape)
    lam = rng.normal(size=(w.N, w.d))
    y1, yd1 = orc.replay_jvp(w.field, w.method, w.theta, w.y0, thd, yd0, r["H"], r["S"])
    assert np.array_equal(y1, orc.replay(w.field, w.method, w.theta, w.y0, r["H"], r["S"]))
    gy, gt = orc.replay_grad(w.field, w.method, w.theta, w.y0, r["H"], r["S"], lam)
    lhs = np.sum(lam * yd1, axis=1)
    rhs = np.sum(gy * yd0, axis=1) + np.sum(gt * thd, axis=1)
    assert np.max(np.abs(lhs - rhs) / (1 + np.abs(rhs))) <= 1e-11
    eps = 1e-6
    yp = orc.replay(w.field, w.method, w.theta + eps * thd, w.y0 + eps * yd0, r["H"], r["S"])
    ym = orc.replay(w.field, w.method, w.theta - eps * thd, w.y0 - eps * yd0, r["H"], r["S"])
    fd = (yp - ym) / (2 * eps)
    assert np.max(np.abs(fd - yd1) / (1 + np.abs(yd1))) <= 1e-6
