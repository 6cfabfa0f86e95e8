"""Pins of the oracle's forward sensitivities ("Differentiable astrophysics at scale" §2-§3: the
sensitivity equations S' = J_y S + J_theta integrated in the same solve as the orbit, the step
size controlled on the orbit alone) and of the flattened logarithmic halo field of §3
(Phi = v_c^2/2 ln(R_c^2 + x^2 + y^2 + z^2/q^2)).

Pinned by: the accepted mesh and final state equal those of the plain solve bit for bit (control
on the orbit alone); on that mesh the sensitivities equal the tangent of the replay chain (the
forward-mode replay, itself pinned by its closed form and by the transpose identity with the
reverse-mode gradient); the linear family's closed form; central differences of tight adaptive
solves (the continuous sensitivity, to the tolerance's order); a seeded S0 propagates as the
replay's tangent; and the halo force against central differences of the printed potential, with
its energy and angular-momentum invariants."""
import numpy as np
import pytest

from differentiable_adaptive_ode_b200 import workloads as W


@pytest.mark.parametrize("name", ["log_halo", "lorenz63", "nfw_mn", "lotka_volterra"])
def test_sens_mesh_is_the_plain_mesh_and_matches_replay_tangent(orc, name):
    w = W.by_name(name, N=5)
    r = orc.solve_sens(w.field, w.theta, w.y0, w.t0, w.t1, w.rtol, w.atol,
                       theta_shared=w.theta_shared)
    p = orc.solve(w.field, w.method, w.theta, w.y0, w.t0, w.t1, w.rtol, w.atol, keep_record=True,
                  theta_shared=w.theta_shared)
    assert np.all(r["status"] == 0)
    assert np.array_equal(r["S"], p["S"]) and np.array_equal(r["rejected"], p["rejected"])
    assert np.array_equal(r["y1"], p["y1"])
    th = np.broadcast_to(w.theta, (w.N, w.m)) if w.theta_shared else w.theta
    for j in range(w.m):
        thd = np.zeros((w.N, w.m))
        thd[:, j] = 1.0
        _, col = orc.replay_jvp(w.field, w.method, np.ascontiguousarray(th), w.y0, thd,
                                np.zeros_like(w.y0), p["H"], p["S"])
        scale = np.max(np.abs(r["sens"][:, :, j]), axis=1, keepdims=True) + 1e-300
        assert np.max(np.abs(col - r["sens"][:, :, j]) / scale) <= 1e-12, (name, j)


def _tsit5_R(Z, A, b):
    R = np.eye(Z.shape[0], dtype=Z.dtype)
    P = np.eye(Z.shape[0], dtype=Z.dtype)
    v = np.ones(len(b))
    for q in range(1, len(b) + 1):
        P = P @ Z
        R = R + (b @ v) * P
        v = A @ v
    return R


def test_sens_linear_closed_form(orc):
    c, At, b, bt = orc.tsit5_tableau()
    rng = np.random.default_rng(21)
    A = rng.normal(size=(3, 3)) * 0.5 - 0.8 * np.eye(3)
    y0 = rng.normal(size=3)
    r = orc.solve_sens("linear3", A.ravel(), y0, 0.0, 2.5, 1e-7, 1e-9)
    p = orc.solve("linear3", "tsit5", A.ravel(), y0, 0.0, 2.5, 1e-7, 1e-9, keep_record=True)
    H = p["H"][0, :int(p["S"][0])]
    eps = 1e-30
    for i in range(3):
        for j in range(3):
            E = np.zeros((3, 3))
            E[i, j] = 1.0
            Ac = A + 1j * eps * E
            y = y0.astype(complex)
            for h in H:
                y = _tsit5_R(h * Ac, At, b) @ y
            want = y.imag / eps
            got = r["sens"][0, :, 3 * i + j]
            assert np.max(np.abs(got - want)) <= 1e-12 * (1 + np.max(np.abs(want)))


def test_sens_seeded_start_propagates_as_replay_tangent(orc):
    w = W.log_halo(N=4)
    rng = np.random.default_rng(22)
    S0 = rng.normal(size=(4, 6, 2)) * 0.1
    r = orc.solve_sens(w.field, w.theta, w.y0, w.t0, w.t1, w.rtol, w.atol, S0=S0,
                       theta_shared=True)
    p = orc.solve(w.field, w.method, w.theta, w.y0, w.t0, w.t1, w.rtol, w.atol, keep_record=True,
                  theta_shared=True)
    th = np.ascontiguousarray(np.broadcast_to(w.theta, (4, 2)))
    for j in range(2):
        thd = np.zeros((4, 2))
        thd[:, j] = 1.0
        _, col = orc.replay_jvp(w.field, w.method, th, w.y0, thd, S0[:, :, j], p["H"], p["S"])
        assert np.max(np.abs(col - r["sens"][:, :, j])) <= 1e-12 * np.max(np.abs(col))


def test_sens_is_the_continuous_sensitivity_to_tolerance(orc):
    w = W.log_halo(N=3, seed=11)
    w.t1 = 8.0
    tight = dict(rtol=1e-12, atol=1e-12)
    r = orc.solve_sens(w.field, w.theta, w.y0, w.t0, w.t1, theta_shared=True, **tight)
    for j, e in enumerate([1e-5, 1e-5]):
        tp, tm = w.theta.copy(), w.theta.copy()
        tp[j] += e
        tm[j] -= e
        yp = orc.solve(w.field, w.method, tp, w.y0, w.t0, w.t1, theta_shared=True, **tight)["y1"]
        ym = orc.solve(w.field, w.method, tm, w.y0, w.t0, w.t1, theta_shared=True, **tight)["y1"]
        fd = (yp - ym) / (2 * e)
        err = np.max(np.abs(fd - r["sens"][:, :, j])) / np.max(np.abs(fd))
        assert err <= 1e-5, (j, err)


def _log_halo_phi(x, vc=1.0, q=0.7, Rc=0.2):
    return 0.5 * vc * vc * np.log(Rc * Rc + x[0] ** 2 + x[1] ** 2 + x[2] ** 2 / (q * q))


def test_log_halo_force_is_minus_grad_of_the_printed_potential(orc):
    rng = np.random.default_rng(23)
    for vc, q in [(1.0, 0.7), (1.3, 0.9), (0.8, 1.2)]:
        for _ in range(5):
            x = rng.normal(size=3)
            y = np.concatenate([x, rng.normal(size=3)])
            f = orc.rhs("log_halo", np.array([[vc, q]]), y[None, :])[0]
            e = 1e-6
            g = np.array([(_log_halo_phi(x + e * np.eye(3)[i], vc, q)
                           - _log_halo_phi(x - e * np.eye(3)[i], vc, q)) / (2 * e)
                          for i in range(3)])
            assert np.allclose(f[:3], y[3:], rtol=0, atol=0)
            assert np.max(np.abs(f[3:] + g)) <= 1e-8 * (1 + np.max(np.abs(g)))


def test_log_halo_orbits_conserve_energy_and_lz(orc):
    w = W.log_halo(N=16, seed=12)
    r = orc.solve(w.field, w.method, w.theta, w.y0, w.t0, w.t1, 1e-10, 1e-10, theta_shared=True)
    assert np.all(r["status"] == 0)
    for k in range(16):
        E0 = 0.5 * np.sum(w.y0[k, 3:] ** 2) + _log_halo_phi(w.y0[k, :3])
        E1 = 0.5 * np.sum(r["y1"][k, 3:] ** 2) + _log_halo_phi(r["y1"][k, :3])
        L0 = w.y0[k, 0] * w.y0[k, 4] - w.y0[k, 1] * w.y0[k, 3]
        L1 = r["y1"][k, 0] * r["y1"][k, 4] - r["y1"][k, 1] * r["y1"][k, 3]
        assert abs(E1 - E0) <= 1e-7 * (1 + abs(E0))
        assert abs(L1 - L0) <= 1e-7 * (1 + abs(L0))


def test_log_halo_workload_recipe():
    w = W.log_halo(N=4096)
    r = np.linalg.norm(w.y0[:, :3], axis=1)
    assert r.min() >= 0.5 - 1e-12 and r.max() <= 2.0 + 1e-12
    # velocity: eta in [0.05, 1] of v_circ perpendicular to r_hat, xi in [-0.2, 0.2] along it
    rh = w.y0[:, :3] / r[:, None]
    vr = np.sum(w.y0[:, 3:] * rh, axis=1) / W.log_halo_vcirc(r)
    vt = np.linalg.norm(w.y0[:, 3:] - (vr * W.log_halo_vcirc(r))[:, None] * rh, axis=1)
    vt /= W.log_halo_vcirc(r)
    assert np.all(np.abs(vr) <= 0.2 + 1e-12) and vt.min() >= 0.05 - 1e-12
    assert vt.max() <= 1.0 + 1e-12
    assert abs(w.t1 - 37.385) < 1e-3 and w.rtol == w.atol == 3.16e-7
