"""Pins of the oracle's adaptive solve, record and replay.

Sources: "gradsolve: fast exact gradients for ODE ensembles on GPUs", §2.1 (trial steps, the
RMS error test, reject-and-retry), §3 (the record keeps the accepted step sizes; rejected trials
leave no trace; the replay over the recorded mesh reproduces the accepted trajectory; zero
padding steps change nothing); "Differentiable astrophysics at scale", §3 (orbit energy and
angular momentum as conservation checks).
"""
import numpy as np
import pytest

from differentiable_adaptive_ode_b200 import workloads as W


def _tsit5_R(z, A, b):
    s, v = 1.0, np.ones(len(b))
    for q in range(1, len(b) + 1):
        s += z ** q * (b @ v)
        v = A @ v
    return s


def test_convergence_order_tsit5_scalar(orc):
    # fixed-step replay of y' = -4 y on [0, 1]: global error ~ C h^5 (+ a z^7 term whose share
    # shrinks with h, so the observed slope falls toward 5 from above)
    errs = []
    hs = [1 / 16, 1 / 32, 1 / 64, 1 / 128, 1 / 256]
    for h in hs:
        n = int(round(1 / h))
        y = orc.replay("linear1", "tsit5", [[-4.0]], [[1.0]], [[h] * n], [n])
        errs.append(abs(y[0, 0] - np.exp(-4.0)))
    slopes = np.diff(np.log(errs)) / np.diff(np.log(hs))
    assert np.all(np.diff(slopes) < 0) and abs(slopes[-1] - 5.0) < 0.2, slopes


def test_convergence_order_tsit5_nonlinear(orc):
    # a nonlinear field exercises every order condition: an orbit in the halo + disk potential
    # over t in [0, 3]; the fixed-step error against a 16384-step replay falls as h^5
    th = [[1.0, 1.0, 0.1, 0.3, 0.03]]
    y0 = [[0.7, 0.2, 0.1, 0.1, 0.5, 0.05]]
    T = 3.0
    ref = orc.replay("nfw_mn", "tsit5", th, y0, [[T / 16384] * 16384], [16384])
    errs, hs = [], [T / 32, T / 64, T / 128]
    for h in hs:
        n = int(round(T / h))
        y = orc.replay("nfw_mn", "tsit5", th, y0, [[h] * n], [n])
        errs.append(np.max(np.abs(y - ref)))
    slopes = np.diff(np.log(errs)) / np.diff(np.log(hs))
    assert np.all(np.abs(slopes - 5.0) < 0.25), slopes


def test_convergence_order_ros34pw2(orc):
    # order 3 on a mildly stiff linear system at fixed steps (against the matrix exponential)
    A = np.array([[-2.0, 1.0, 0.0], [1.0, -3.0, 0.5], [0.0, 0.2, -50.0]])
    y0 = np.array([1.0, 0.5, -0.3])
    w, V = np.linalg.eig(A)
    exact = (V @ np.diag(np.exp(w * 1.0)) @ np.linalg.inv(V) @ y0).real
    errs, hs = [], [1 / 8, 1 / 16, 1 / 32, 1 / 64]
    for h in hs:
        n = int(round(1 / h))
        y = orc.replay("linear3", "ros34pw2", [A.ravel()], [y0], [[h] * n], [n])
        errs.append(np.max(np.abs(y[0] - exact)))
    slopes = np.diff(np.log(errs)) / np.diff(np.log(hs))
    assert np.all(np.abs(slopes - 3.0) < 0.35), slopes


def test_accepted_steps_pass_the_error_test(orc):
    # y' = lambda y: the error estimate of a step from y with step h is |E(h lambda)| |y|, with
    # E = R - R_hat from the two polynomials; every recorded step must satisfy err <= 1.
    c, A, b, bt = orc.tsit5_tableau()
    lam, rtol, atol = -2.3, 1e-6, 1e-9
    r = orc.solve("linear1", "tsit5", [[lam]], [[1.0]], 0.0, 5.0, rtol, atol, keep_record=True)
    S = int(r["S"][0])
    assert r["status"][0] == 0 and S > 5
    Eb = bt
    for n in range(S):
        h, y = r["H"][0, n], r["Y"][0, n, 0]
        z = h * lam
        R = _tsit5_R(z, A, b)
        E = _tsit5_R(z, A, Eb) - 1.0
        err = abs(E * y) / (atol + rtol * max(abs(y), abs(R * y)))
        assert err <= 1.0 + 1e-9
    # the record's times chain: t_{n+1} = t_n + h_n, and the last step lands on t1
    T, H = r["T"][0, :S], r["H"][0, :S]
    assert T[0] == 0.0
    assert np.allclose(T[1:], T[:-1] + H[:-1], rtol=0, atol=1e-14)
    assert abs(T[-1] + H[-1] - 5.0) < 1e-14


def test_rejected_trials_leave_no_trace(orc):
    # Lorenz at its chaotic parameters rejects some trials; the record holds only accepted
    # steps, and replaying the recorded mesh reproduces the final state bitwise.
    w = W.lorenz63(N=16, seed=11)
    r = orc.solve("lorenz63", "tsit5", w.theta, w.y0, 0.0, 1.0, 1e-6, 1e-9, keep_record=True)
    assert np.all(r["status"] == 0)
    assert r["rejected"].sum() > 0
    assert np.array_equal(r["attempts"], r["S"] + r["rejected"])
    y = orc.replay("lorenz63", "tsit5", w.theta, w.y0, r["H"], r["S"])
    assert np.array_equal(y, r["y1"])
    # every recorded state is the replay of the prefix before it
    for k in range(3):
        for n in (1, int(r["S"][k]) // 2, int(r["S"][k]) - 1):
            yk = orc.replay("lorenz63", "tsit5", w.theta[k:k + 1], w.y0[k:k + 1],
                            r["H"][k:k + 1, :n], [n])
            assert np.array_equal(yk[0], r["Y"][k, n])


def test_replay_reproduces_record_all_fields(orc):
    cases = [("lotka_volterra", W.lotka_volterra(N=8)), ("nfw_mn", W.nfw_mn(N=8)),
             ("robertson", W.robertson(N=4))]
    for name, w in cases:
        r = orc.solve(w.field, w.method, w.theta, w.y0, w.t0, w.t1, w.rtol, w.atol,
                      keep_record=True, theta_shared=w.theta_shared)
        assert np.all(r["status"] == 0), name
        y = orc.replay(w.field, w.method, w.theta, w.y0, r["H"], r["S"],
                       theta_shared=w.theta_shared)
        assert np.array_equal(y, r["y1"]), name


def test_zero_padding_is_identity(orc):
    w = W.lorenz63(N=4, seed=3)
    r = orc.solve("lorenz63", "tsit5", w.theta, w.y0, 0.0, 1.0, 1e-8, 1e-10, keep_record=True)
    Hp = np.concatenate([r["H"], np.zeros((4, 7))], axis=1)
    Sp = r["S"] + 7
    # pad every record with seven h = 0 steps at its end (ragged: place them after S_k)
    Hr = np.zeros_like(Hp)
    for k in range(4):
        Hr[k, :r["S"][k]] = r["H"][k, :r["S"][k]]
    y = orc.replay("lorenz63", "tsit5", w.theta, w.y0, Hr, Sp)
    assert np.array_equal(y, r["y1"])
    lam = np.random.default_rng(0).normal(size=(4, 3))
    g0 = orc.replay_grad("lorenz63", "tsit5", w.theta, w.y0, r["H"], r["S"], lam)
    g1 = orc.replay_grad("lorenz63", "tsit5", w.theta, w.y0, Hr, Sp, lam)
    assert np.array_equal(g0[0], g1[0]) and np.array_equal(g0[1], g1[1])
    # the same for the Rosenbrock map
    rr = orc.solve("robertson", "ros34pw2", [[0.04, 3e7, 1e4]], [[1.0, 0, 0]], 0.0, 10.0, 1e-6,
                   1e-10, keep_record=True)
    S = int(rr["S"][0])
    H2 = np.zeros((1, S + 3))
    H2[0, :S] = rr["H"][0, :S]
    y2 = orc.replay("robertson", "ros34pw2", [[0.04, 3e7, 1e4]], [[1.0, 0, 0]], H2, [S + 3])
    assert np.array_equal(y2, rr["y1"])


def test_robertson_mass_conserved_along_solve(orc):
    w = W.robertson(N=4)
    r = orc.solve("robertson", "ros34pw2", w.theta, w.y0, 0.0, 1e4, 1e-6, 1e-10,
                  keep_record=True)
    assert np.all(r["status"] == 0)
    for k in range(4):
        S = int(r["S"][k])
        assert np.max(np.abs(r["Y"][k, :S].sum(1) - 1.0)) < 1e-13
        assert abs(r["y1"][k].sum() - 1.0) < 1e-13
    assert 200 < r["S"].mean() < 600


def test_lotka_volterra_first_integral(orc):
    w = W.lotka_volterra(N=8)
    r = orc.solve("lotka_volterra", "tsit5", w.theta, w.y0, 0.0, 10.0, 1e-6, 1e-8)
    a, b, g, d = w.theta.T
    V = lambda y: d * y[:, 0] - g * np.log(y[:, 0]) + b * y[:, 1] - a * np.log(y[:, 1])
    assert np.max(np.abs(V(r["y1"]) - V(w.y0))) < 1e-4
    r2 = orc.solve("lotka_volterra", "tsit5", w.theta, w.y0, 0.0, 10.0, 1e-10, 1e-12)
    assert np.max(np.abs(V(r2["y1"]) - V(w.y0))) < 1e-8


def test_nfw_mn_energy_and_lz(orc):
    w = W.nfw_mn(N=16)
    r = orc.solve("nfw_mn", "tsit5", w.theta, w.y0, 0.0, 20.0, w.rtol, w.atol)
    assert np.all(r["status"] == 0)

    def E(y, th):
        Mh, rs, Md, a, b = th.T
        x, yy, z = y[:, 0], y[:, 1], y[:, 2]
        rr = np.sqrt(x * x + yy * yy + z * z)
        phi = (-Mh * np.log1p(rr / rs) / rr
               - Md / np.sqrt(x * x + yy * yy + (a + np.sqrt(z * z + b * b)) ** 2))
        return 0.5 * (y[:, 3:] ** 2).sum(1) + phi

    Lz = lambda y: y[:, 0] * y[:, 4] - y[:, 1] * y[:, 3]
    assert np.max(np.abs(E(r["y1"], w.theta) - E(w.y0, w.theta))) < 1e-6
    assert np.max(np.abs(Lz(r["y1"]) - Lz(w.y0))) < 1e-6
    assert 40 < r["S"].mean() < 400


def test_mlp_zero_weights_is_constant_drift(orc):
    th = np.zeros(1348)
    th[1344:1348] = [0.5, -0.25, 1.0, 0.0]
    y0 = np.random.default_rng(1).normal(size=(3, 4))
    r = orc.solve("mlp", "tsit5", th, y0, 0.0, 1.0, 1e-5, 1e-6, theta_shared=True)
    assert np.max(np.abs(r["y1"] - (y0 + th[1344:1348]))) < 1e-14


def test_global_error_consistent_with_tolerance(orc):
    w = W.lorenz63(N=8, seed=5)
    tight = orc.solve("lorenz63", "tsit5", w.theta, w.y0, 0.0, 1.0, 1e-13, 1e-15)
    for rtol in (1e-5, 1e-8):
        r = orc.solve("lorenz63", "tsit5", w.theta, w.y0, 0.0, 1.0, rtol, rtol * 1e-2)
        err = np.max(np.abs(r["y1"] - tight["y1"]) / (1 + np.abs(tight["y1"])))
        assert 1e-4 * rtol < err < 1e3 * rtol, (rtol, err)


def test_status_codes(orc):
    th = np.array([[10.0, 28.0, 8 / 3], [np.nan, 28.0, 8 / 3]])
    y0 = np.ones((2, 3))
    r = orc.solve("lorenz63", "tsit5", th, y0, 0.0, 1.0, 1e-8, 1e-10)
    assert list(r["status"]) == [0, 3]                       # non-finite f(y0)
    r = orc.solve("lorenz63", "tsit5", th[:1], y0[:1], 0.0, 1.0, 1e-8, 1e-10, max_attempts=10)
    assert r["status"][0] == 1 and r["attempts"][0] == 10    # attempt cap
    r = orc.solve("lorenz63", "tsit5", th[:1], y0[:1], 0.0, 1.0, 1e-300, 1e-300)
    assert r["status"][0] == 2 and r["S"][0] == 0            # step size underflow
    r = orc.solve("lorenz63", "tsit5", th[:1], y0[:1], 1.0, 1.0, 1e-8, 1e-10)
    assert r["status"][0] == 0 and r["S"][0] == 0 and np.array_equal(r["y1"], y0[:1])


def test_fp32_solve_tracks_fp64(orc):
    w = W.nfw_mn(N=16, dtype=np.float32)
    r32 = orc.solve("nfw_mn", "tsit5", w.theta, w.y0, 0.0, 20.0, 1e-5, 1e-6, dtype=np.float32)
    r64 = orc.solve("nfw_mn", "tsit5", w.theta, w.y0, 0.0, 20.0, 1e-9, 1e-11)
    assert np.all(r32["status"] == 0)
    err = np.max(np.abs(r32["y1"] - r64["y1"]), axis=1) / np.max(np.abs(r64["y1"]), axis=1)
    assert np.median(err) < 1e-3


def _rk_poly(z, A, v):
    """1 + sum_q z^q v^T A^(q-1) 1: what the weights v of an explicit RK method give on y' = z y
    over one step (z = h lambda); with v = b - b_hat, 1 + the error estimate's factor."""
    s, u = 1.0, np.ones(A.shape[0])
    for q in range(1, A.shape[0] + 1):
        s += z ** q * (v @ u)
        u = A @ u
    return s


def _scalar_step(method, orc):
    """(R, E)(h, lam): step factor and error-estimate factor of one step on y' = lam y, y = 1."""
    if method == "tsit5":
        c, A, b, bt = orc.tsit5_tableau()
        return lambda h, lam: (_rk_poly(h * lam, A, b), _rk_poly(h * lam, A, bt) - 1.0)
    if method == "vern7":
        A, b, bh = orc.vern7_tableau()
        return lambda h, lam: (_rk_poly(h * lam, A, b), _rk_poly(h * lam, A, b - bh) - 1.0)
    if method == "ros34pw2":
        g, al, ga, b, bh = orc.ros34pw2_tableau()
        beta = al + ga

        def ros(h, lam):
            z, K = h * lam, []
            for i in range(4):                  # (1 - g z) K_i = z (1 + sum_j beta_ij K_j)
                K.append(z / (1 - g * z) * (1 + sum(beta[i, j] * K[j] for j in range(i))))
            return 1 + sum(b[i] * K[i] for i in range(4)), sum((b[i] - bh[i]) * K[i] for i in range(4))
        return ros
    # Rosenbrock23 (Shampine & Reichelt): W = 1 - d h lam, slopes k1, k2, k3, e = h (k1 - 2k2 + k3)/6
    d, e32 = 1 / (2 + np.sqrt(2)), 6 + np.sqrt(2)

    def rb23(h, lam):
        W = 1 - d * h * lam
        F0 = lam
        k1 = F0 / W
        F1 = lam * (1 + h * k1 / 2)
        k2 = (F1 - k1) / W + k1
        y1 = 1 + h * k2
        k3 = (lam * y1 - e32 * (k2 - F1) - 2 * (k1 - F0)) / W
        return y1, h * (k1 - 2 * k2 + k3) / 6
    return rb23


@pytest.mark.parametrize("method,q", [("tsit5", 5), ("vern7", 7), ("ros34pw2", 3),
                                      ("rosenbrock23", 3)])
def test_controller_settles_at_its_fixed_point(orc, method, q):
    # On y' = lam y with a pure relative tolerance the scaled error of a step depends on h alone:
    # err(h) = |E(h lam)| / (rtol max(1, |R(h lam)|)).  The I-controller h <- 0.9 err^(-1/q) h
    # therefore settles where 0.9 err^(-1/q) = 1, i.e. err(h*) = 0.9^q; h* is found here by
    # bisection on the closed-form factors, independently of the solver's loop.  A wrong safety
    # factor, exponent or error norm moves the recorded steps off h*.
    lam, rtol = -1.0, 1e-6 if method != "vern7" else 1e-8
    step = _scalar_step(method, orc)
    r = orc.solve("linear1", method, [[lam]], [[1.0]], 0.0, 40.0, rtol, 1e-300, keep_record=True)
    S = int(r["S"][0])
    H = r["H"][0, :S]
    assert r["status"][0] == 0 and r["rejected"][0] == 0 and S > 100

    def err(h):
        R, E = step(h, lam)
        return abs(E) / (rtol * max(1.0, abs(R)))
    lo, hi = 1e-9, 4 * H.max()
    assert err(lo) < 0.9 ** q < err(hi)
    for _ in range(200):
        mid = 0.5 * (lo + hi)
        lo, hi = (mid, hi) if err(mid) < 0.9 ** q else (lo, mid)
    h_star = 0.5 * (lo + hi)
    settled = H[S // 2:S - 1]               # past the start-up, before the step clipped to t1
    assert np.max(np.abs(settled - h_star)) <= 1e-7 * h_star, (h_star, settled[:3])
    # and the start-up grows the step by at most the factor cap of 10 per accepted step
    assert np.all(H[1:S - 1] <= 10 * H[:S - 2] * (1 + 1e-12))
    if method == "rosenbrock23":            # a tiny first step: the cap itself is reached
        assert abs(H[1] / H[0] - 10.0) < 1e-12
