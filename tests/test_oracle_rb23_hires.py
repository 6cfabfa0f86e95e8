"""Pins of the oracle's Rosenbrock23 step and HIRES field ("gradsolve: fast exact gradients for
ODE ensembles on GPUs" §3.1: the second-order linearly implicit Rosenbrock23 method of the fused
stiff kernels; §4.5-4.6: the HIRES system, differentiated with respect to its initial state).

Rosenbrock23 is pinned by its stability function on y' = lambda y being a second-order
approximation of exp (R(z) - e^z = O(z^3)), L-stable (R(-inf) = 0) and A-stable; by the error
estimate scaling as h^3; by a global convergence slope of 2; by Robertson's linear invariant
(sum y = 1, kept exactly by a linearly implicit method with the exact Jacobian); and by its replay
gradient against central differences and the forward tangent.  HIRES is pinned by the published
reference solution at t = 321.8122 (Test Set for IVP Solvers, Hairer & Wanner II §IV.10), its
Jacobian against differences of f and its linear invariant y7 + y8."""
import numpy as np
import pytest

from differentiable_adaptive_ode_b200 import workloads as W

K_HIRES = np.array([1.71, 0.43, 8.32, 0.0007, 8.75, 10.03, 0.035, 1.12, 1.745, 280.0, 0.69, 1.81])
Y0_HIRES = np.array([1.0, 0, 0, 0, 0, 0, 0, 0.0057])
# published reference solution at t = 321.8122
Y_REF_HIRES = np.array([0.7371312573325668e-3, 0.1442485726316185e-3, 0.5888729740967575e-4,
                        0.1175651343283149e-2, 0.2386356198831331e-2, 0.6238968252742796e-2,
                        0.2849998395185769e-2, 0.2850001604814231e-2])


def _R(orc, z):
    """One Rosenbrock23 step of y' = lam y from y = 1 with h = 1, lam = z (real)."""
    return orc.replay("linear1", "rosenbrock23", [[z]], [[1.0]], [[1.0]], [1])[0, 0]


def test_rb23_stability_function(orc):
    # second order: (R(z) - e^z) / z^3 tends to a constant as z -> 0
    ratios = [(_R(orc, z) - np.exp(z)) / z ** 3 for z in (1e-2, 5e-3, 2.5e-3)]
    assert abs(ratios[0] - ratios[2]) < 0.02 * abs(ratios[2]) and abs(ratios[2]) > 1e-3
    # L-stable: the step annihilates infinitely stiff components; A-stable on the negative axis
    assert abs(_R(orc, -1e12)) < 1e-9
    for z in (-0.5, -3.0, -40.0, -1e3, -1e6):
        assert abs(_R(orc, z)) <= 1.0


def test_rb23_error_estimate_is_third_order(orc):
    es = []
    for h in (0.02, 0.01, 0.005):
        _, e = orc.trial("linear1", "rosenbrock23", [-1.3], [1.0], h)
        es.append(abs(e[0]))
    assert 7.0 < es[0] / es[1] < 9.0 and 7.0 < es[1] / es[2] < 9.0


def test_rb23_convergence_slope_two(orc):
    # a mildly stiff linear problem with a non-normal matrix
    A = np.array([[-2.0, 1.0, 0.3], [0.5, -3.0, 1.0], [0.0, 0.4, -1.5]])
    ref = orc.replay("linear3", "rosenbrock23", A.ravel(), [[1.0, -1.0, 0.5]],
                     np.full((1, 20000), 1.0 / 20000), [20000])
    ns = [50, 100, 200, 400]
    errs = [np.max(np.abs(orc.replay("linear3", "rosenbrock23", A.ravel(), [[1.0, -1.0, 0.5]],
                                     np.full((1, n), 1.0 / n), [n]) - ref)) for n in ns]
    slope = -np.polyfit(np.log(ns), np.log(errs), 1)[0]
    assert 1.9 <= slope <= 2.15, (slope, errs)


def test_rb23_robertson_mass_and_solve(orc):
    w = W.robertson(N=4)
    r = orc.solve("robertson", "rosenbrock23", w.theta, w.y0, 0.0, 1e4, 1e-6, 1e-10,
                  keep_record=True)
    assert np.all(r["status"] == 0)
    assert np.max(np.abs(r["y1"].sum(1) - 1.0)) < 1e-13
    tight = orc.solve("robertson", "ros34pw2", w.theta, w.y0, 0.0, 1e4, 1e-11, 1e-15)
    assert np.max(np.abs(r["y1"] - tight["y1"])) < 1e-4
    assert np.array_equal(orc.replay("robertson", "rosenbrock23", w.theta, w.y0, r["H"], r["S"]),
                          r["y1"])


def test_hires_reference_solution(orc):
    for method, tol, bar in (("ros34pw2", 1e-12, 1e-9), ("rosenbrock23", 1e-9, 2e-5)):
        r = orc.solve("hires", method, K_HIRES, Y0_HIRES[None, :], 0.0, 321.8122, tol,
                      tol * 1e-4)
        assert r["status"][0] == 0
        rel = np.max(np.abs(r["y1"][0] - Y_REF_HIRES) / Y_REF_HIRES)
        assert rel < bar, (method, rel)


def test_hires_jacobian_and_invariant(orc):
    rng = np.random.default_rng(51)
    for _ in range(3):
        y = rng.uniform(0, 1, size=8)
        th = K_HIRES * rng.uniform(0.8, 1.2, size=12)
        J = orc.jac("hires", th[None, :], y[None, :])[0]
        e = 1e-7
        Jfd = np.zeros((8, 8))
        for c in range(8):
            yp, ym = y.copy(), y.copy()
            yp[c] += e
            ym[c] -= e
            Jfd[:, c] = (orc.rhs("hires", th[None, :], yp[None, :])[0]
                         - orc.rhs("hires", th[None, :], ym[None, :])[0]) / (2 * e)
        assert np.max(np.abs(J - Jfd)) < 1e-6 * np.max(np.abs(J))
        f = orc.rhs("hires", th[None, :], y[None, :])[0]
        assert abs(f[6] + f[7]) < 1e-13 * (1 + abs(f[6]))


@pytest.mark.parametrize("field,method", [("hires", "rosenbrock23"), ("robertson", "rosenbrock23"),
                                          ("hires", "ros34pw2")])
def test_stiff_replay_gradient(orc, field, method):
    w = W.by_name(field, N=2)
    r = orc.solve(w.field, method, w.theta, w.y0, w.t0, w.t1, w.rtol, w.atol, keep_record=True,
                  theta_shared=w.theta_shared)
    assert np.all(r["status"] == 0)
    rng = np.random.default_rng(52)
    lam = rng.normal(size=(2, w.d))
    gy, gt = orc.replay_grad(w.field, method, w.theta, w.y0, r["H"], r["S"], lam,
                             theta_shared=w.theta_shared)
    L = lambda y0: np.sum(lam * orc.replay(w.field, method, w.theta, y0, r["H"], r["S"],
                                            theta_shared=w.theta_shared))
    for c in range(w.d):
        e = 1e-6 * max(1e-3, abs(w.y0[0, c]))
        yp, ym = w.y0.copy(), w.y0.copy()
        yp[0, c] += e
        ym[0, c] -= e
        fd = (L(yp) - L(ym)) / (2 * e)
        assert abs(fd - gy[0, c]) <= 1e-5 * max(1.0, abs(fd)), (c, fd, gy[0, c])
    # transpose identity with the forward tangent along a random direction
    th = np.ascontiguousarray(np.broadcast_to(w.theta, (2, w.m)) if w.theta_shared else w.theta)
    thd = rng.normal(size=th.shape) * th * 1e-2
    yd = rng.normal(size=w.y0.shape)
    _, tan = orc.replay_jvp(w.field, method, th, w.y0, thd, yd, r["H"], r["S"])
    gy2, gt2 = orc.replay_grad(w.field, method, th, w.y0, r["H"], r["S"], lam)
    lhs = np.sum(lam * tan, 1)
    rhs = np.sum(gy2 * yd, 1) + np.sum(gt2 * thd, 1)
    assert np.max(np.abs(lhs - rhs) / (1 + np.abs(rhs))) < 1e-9
