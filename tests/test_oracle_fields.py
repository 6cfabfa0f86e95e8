"""Pins of the oracle's right-hand sides against properties the mathematics fixes.

None of these retypes a field formula: each field is checked through a property that a wrong
term, sign or index would break (fixed points, divergence, conservation laws, a potential whose
negative gradient the force must be, a library MLP).
"""
import numpy as np
import pytest


def _fd_jac(orc, field, theta, y, eps=1e-6):
    D = len(y)
    J = np.zeros((D, D))
    for c in range(D):
        yp, ym = y.copy(), y.copy()
        yp[c] += eps
        ym[c] -= eps
        J[:, c] = (orc.rhs(field, theta, yp)[0] - orc.rhs(field, theta, ym)[0]) / (2 * eps)
    return J


def test_lorenz_fixed_points_and_divergence(orc):
    s, r, b = 10.0, 28.0, 8.0 / 3.0
    th = np.array([s, r, b])
    q = np.sqrt(b * (r - 1))
    for p in ([0, 0, 0], [q, q, r - 1], [-q, -q, r - 1]):
        assert np.max(np.abs(orc.rhs("lorenz63", th, np.array(p, float)))) < 1e-12
    rng = np.random.default_rng(0)
    for _ in range(5):
        y = rng.normal(size=3) * 5
        J = _fd_jac(orc, "lorenz63", th, y)
        assert abs(np.trace(J) + (s + 1 + b)) < 1e-6        # div f = -(sigma + 1 + beta)
        # the only nonlinear terms are x z and x y: J entries linear in the state
        assert abs(J[0, 0] + s) < 1e-6 and abs(J[0, 1] - s) < 1e-6


def test_lotka_volterra_fixed_point_and_first_integral(orc):
    a, b, g, d = 1.3, 0.9, 2.7, 1.1
    th = np.array([a, b, g, d])
    fp = np.array([g / d, a / b])
    assert np.max(np.abs(orc.rhs("lotka_volterra", th, fp))) < 1e-14
    # V = d x - g ln x + b y - a ln y is constant along solutions: grad V . f = 0
    rng = np.random.default_rng(1)
    for _ in range(5):
        x, y = rng.uniform(0.2, 3.0, size=2)
        f = orc.rhs("lotka_volterra", th, np.array([x, y]))[0]
        gradV = np.array([d - g / x, b - a / y])
        assert abs(gradV @ f) < 1e-13 * (1 + np.abs(f).sum())


def test_robertson_mass_and_jacobian(orc):
    rng = np.random.default_rng(2)
    th = np.array([0.04, 3e7, 1e4])
    for _ in range(5):
        y = rng.uniform(0, 1, size=3) * np.array([1, 1e-4, 1])
        f = orc.rhs("robertson", th, y)[0]
        assert abs(f.sum()) <= 1e-12 * np.abs(f).sum()      # total mass is conserved
        J = orc.jac("robertson", th, y)[0]
        Jfd = _fd_jac(orc, "robertson", th, y, eps=1e-7)
        assert np.max(np.abs(J - Jfd)) <= 1e-5 * np.max(np.abs(J))
        assert np.max(np.abs(J.sum(0))) <= 1e-9 * np.max(np.abs(J))   # column sums vanish


def _phi_nfw_mn(p, th):
    Mh, rs, Md, a, b = th
    x, y, z = p
    r = np.sqrt(x * x + y * y + z * z)
    return -Mh * np.log1p(r / rs) / r - Md / np.sqrt(x * x + y * y + (a + np.sqrt(z * z + b * b)) ** 2)


def test_nfw_mn_force_is_minus_grad_potential(orc):
    rng = np.random.default_rng(3)
    th = np.array([1.0, 1.0, 0.1, 0.3, 0.03]) * rng.uniform(0.9, 1.1, 5)
    for _ in range(10):
        p = rng.normal(size=3)
        v = rng.normal(size=3)
        f = orc.rhs("nfw_mn", th, np.concatenate([p, v]))[0]
        assert np.array_equal(f[:3], v)                      # x' = v
        g = np.zeros(3)
        for c in range(3):
            e = np.zeros(3)
            e[c] = 1e-5
            g[c] = (_phi_nfw_mn(p + e, th) - _phi_nfw_mn(p - e, th)) / 2e-5
        assert np.max(np.abs(f[3:] + g)) <= 1e-8 * max(1.0, np.max(np.abs(g)))


def test_mlp_matches_torch_layers(orc):
    torch = pytest.importorskip("torch")
    from differentiable_adaptive_ode_b200 import workloads as W
    th = W.glorot_mlp(7, 1)
    th[128:160] = np.linspace(-0.3, 0.3, 32)        # exercise every bias block
    th[1184:1216] = np.linspace(0.2, -0.2, 32)
    th[1344:1348] = [0.1, -0.2, 0.3, -0.4]
    net = torch.nn.Sequential(torch.nn.Linear(4, 32), torch.nn.Tanh(), torch.nn.Linear(32, 32),
                              torch.nn.Tanh(), torch.nn.Linear(32, 4)).double()
    with torch.no_grad():
        off = 0
        for layer in (net[0], net[2], net[4]):
            nW = layer.weight.numel()
            layer.weight.copy_(torch.from_numpy(th[off:off + nW]).view_as(layer.weight))
            off += nW
            nb = layer.bias.numel()
            layer.bias.copy_(torch.from_numpy(th[off:off + nb]))
            off += nb
        assert off == 1348
        y = np.random.default_rng(4).normal(size=(6, 4))
        ref = net(torch.from_numpy(y)).numpy()
    got = orc.rhs("mlp", th, y, theta_shared=True)
    assert np.max(np.abs(got - ref)) < 1e-14


def test_linear_field_and_jacobian(orc):
    rng = np.random.default_rng(5)
    A = rng.normal(size=(3, 3))
    y = rng.normal(size=3)
    assert np.max(np.abs(orc.rhs("linear3", A.ravel(), y)[0] - A @ y)) < 1e-15
    assert np.array_equal(orc.jac("linear3", A.ravel(), y)[0], A)
