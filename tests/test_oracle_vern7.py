"""Pins of the oracle's Verner 7(6) pair ("gradsolve: fast exact gradients for ODE ensembles on
GPUs" §3.1: the seventh-order Verner pair offered next to Tsit5; §4.6: the Verner engine on the
Lorenz gradient).  The pages print no coefficients; the table is pinned by Butcher's order
conditions (all 85 rooted trees up to order 7 for b, up to order 6 for b_hat, and b is not of
order 8), by the one-step map on y' = lambda y equalling the stability polynomial built from the
table, by the error estimate equalling the difference of the two polynomials, by the global
convergence slope 7, and by the replay gradient against the linear closed form and central
differences."""
import numpy as np
import pytest

from test_oracle_tableaux import density, order, trees_up_to, weight_vector
from differentiable_adaptive_ode_b200 import workloads as W


def test_vern7_order_conditions(orc):
    A, b, bh = orc.vern7_tableau()
    assert np.all(np.triu(A) == 0)
    assert b[1] == 0 and b[2] == 0 and b[9] == 0
    worst_b, worst_bh6, worst_bh7, worst_b8 = 0.0, 0.0, 0.0, 0.0
    for t in trees_up_to(8):
        w = weight_vector(t, A)
        rb = abs(b @ w - 1.0 / density(t))
        rh = abs(bh @ w - 1.0 / density(t))
        if order(t) <= 7:
            worst_b = max(worst_b, rb)
        else:
            worst_b8 = max(worst_b8, rb)
        if order(t) <= 6:
            worst_bh6 = max(worst_bh6, rh)
        elif order(t) == 7:
            worst_bh7 = max(worst_bh7, rh)
    assert worst_b < 1e-13 and worst_bh6 < 1e-13
    assert worst_bh7 > 1e-6 and worst_b8 > 1e-6      # exactly orders 7 and 6


def _R(z, A, b):
    s = 1.0 + 0j
    v = np.ones(len(b))
    for q in range(1, len(b) + 1):
        s += z ** q * (b @ v)
        v = A @ v
    return s


def test_vern7_one_step_and_error_are_polynomials(orc):
    A, b, bh = orc.vern7_tableau()
    for lam in (-1.0, -3.7, 0.8, -12.0):
        for h in (0.01, 0.2, 0.5):
            y = orc.replay("linear1", "vern7", [[lam]], [[1.0]], [[h]], [1])
            R = _R(h * lam, A, b).real
            assert abs(y[0, 0] - R) <= 1e-13 * max(1.0, abs(R)), (lam, h)
            ynew, e = orc.trial("linear1", "vern7", [lam], [1.0], h)
            E = (_R(h * lam, A, b) - _R(h * lam, A, bh)).real
            # the stage weights reach |a_ij| ~ 190: rounding of the sums scales with |E|
            assert abs(e[0] - E) <= 1e-13 * max(1.0, abs(R), abs(E)), (lam, h, e, E)


def test_vern7_convergence_slope(orc):
    w = W.lorenz63(N=1)
    w.t1 = 0.5
    ref = orc.replay("lorenz63", "vern7", w.theta, w.y0, np.full((1, 4000), 0.5 / 4000), [4000])
    errs = []
    ns = [40, 56, 80, 112]
    for n in ns:
        y = orc.replay("lorenz63", "vern7", w.theta, w.y0, np.full((1, n), 0.5 / n), [n])
        errs.append(np.max(np.abs(y - ref)))
    slope = -np.polyfit(np.log(ns), np.log(errs), 1)[0]
    assert 6.6 <= slope <= 7.5, (slope, errs)


def test_vern7_adaptive_solve_meets_tolerance(orc):
    w = W.lorenz63(N=4, seed=3)
    r = orc.solve("lorenz63", "vern7", w.theta, w.y0, 0.0, 1.0, 1e-9, 1e-11, keep_record=True)
    assert np.all(r["status"] == 0)
    tight = orc.solve("lorenz63", "tsit5", w.theta, w.y0, 0.0, 1.0, 1e-13, 1e-15)
    err = np.max(np.abs(r["y1"] - tight["y1"]) / (1 + np.abs(tight["y1"])))
    assert err < 1e-7
    # fewer steps than Tsit5 at the same tight tolerance (the point of a higher-order pair)
    t5 = orc.solve("lorenz63", "tsit5", w.theta, w.y0, 0.0, 1.0, 1e-9, 1e-11)
    assert np.all(r["S"] < t5["S"])
    # replaying the record reproduces the solve bitwise
    y = orc.replay("lorenz63", "vern7", w.theta, w.y0, r["H"], r["S"])
    assert np.array_equal(y, r["y1"])


def test_vern7_gradient_linear_closed_form_and_differences(orc):
    A, b, bh = orc.vern7_tableau()
    rng = np.random.default_rng(41)
    M = rng.normal(size=(3, 3)) * 0.5 - 0.7 * np.eye(3)
    y0 = rng.normal(size=3)
    r = orc.solve("linear3", "vern7", M.ravel(), y0, 0.0, 2.0, 1e-9, 1e-11, keep_record=True)
    S = int(r["S"][0])
    lam = rng.normal(size=(1, 3))
    gy, gM = orc.replay_grad("linear3", "vern7", M.ravel(), y0, r["H"], r["S"], lam)

    def Rmat(Z):
        R = np.eye(3, dtype=Z.dtype)
        P = np.eye(3, dtype=Z.dtype)
        v = np.ones(10)
        for q in range(1, 11):
            P = P @ Z
            R = R + (b @ v) * P
            v = A @ v
        return R

    def prod(Mc):
        P = np.eye(3, dtype=Mc.dtype)
        for h in r["H"][0, :S]:
            P = Rmat(h * Mc) @ P
        return P

    P = prod(M)
    assert np.max(np.abs(gy[0] - P.T @ lam[0])) <= 1e-12 * np.max(np.abs(P.T @ lam[0]))
    eps = 1e-30
    for (i, j) in [(0, 0), (1, 2), (2, 1)]:
        E = np.zeros((3, 3))
        E[i, j] = 1.0
        want = (lam[0] @ (prod(M + 1j * eps * E) @ y0)).imag / eps
        assert abs(gM[0, 3 * i + j] - want) <= 1e-11 * max(1.0, abs(want))
    # nonlinear: central differences inside the recorded replay
    w = W.nfw_mn(N=2)
    rr = orc.solve(w.field, "vern7", w.theta, w.y0, w.t0, w.t1, w.rtol, w.atol, keep_record=True)
    lam = rng.normal(size=(2, 6))
    gy, gt = orc.replay_grad(w.field, "vern7", w.theta, w.y0, rr["H"], rr["S"], lam)
    for j in range(5):
        e = 1e-6 * abs(w.theta[0, j])
        tp, tm = w.theta.copy(), w.theta.copy()
        tp[0, j] += e
        tm[0, j] -= e
        L = lambda th: np.sum(lam * orc.replay(w.field, "vern7", th, w.y0, rr["H"], rr["S"]))
        fd = (L(tp) - L(tm)) / (2 * e)
        assert abs(fd - gt[0, j]) <= 1e-6 * max(1.0, abs(fd)), (j, fd, gt[0, j])
