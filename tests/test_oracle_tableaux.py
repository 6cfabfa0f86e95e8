"""Pins of the oracle's method tables against the mathematics that fixes them.

The pages name the methods ("gradsolve: fast exact gradients for ODE ensembles on GPUs", §2.1
and §3.1: the Tsit5 pair, a Rosenbrock-Wanner step) but print no coefficients, so the tables are
pinned by the order conditions of the published methods, computed here from rooted trees
(Butcher) and from the Rosenbrock conditions (Hairer & Wanner, Solving ODEs II, §IV.7), and by
the stability functions the one-step maps must realise on y' = lambda y.
"""
import numpy as np
import pytest


# ----------------------------------------------------------------------------- rooted trees
def _canon(children):
    return tuple(sorted(children))


def _graft(tree):
    """All trees obtained by attaching one new leaf to some node of `tree`."""
    out = {_canon(tree + ((),))}
    for i, ch in enumerate(tree):
        for g in _graft(ch):
            out.add(_canon(tree[:i] + (g,) + tree[i + 1:]))
    return out


def trees_up_to(p):
    level = {()}
    allt = [()]
    for _ in range(p - 1):
        nxt = set()
        for t in level:
            nxt |= _graft(t)
        level = nxt
        allt += sorted(level)
    return allt


def order(t):
    return 1 + sum(order(c) for c in t)


def density(t):
    g = order(t)
    for c in t:
        g *= density(c)
    return g


def weight_vector(t, A):
    v = np.ones(A.shape[0])
    for c in t:
        v = v * (A @ weight_vector(c, A))
    return v


def test_tree_counts():
    counts = [0] * 6
    for t in trees_up_to(5):
        counts[order(t)] += 1
    assert counts[1:] == [1, 1, 2, 4, 9]          # 17 trees up to order 5


def test_tsit5_order_conditions(orc):
    c, A, b, bt = orc.tsit5_tableau()
    bhat = b - bt
    # row sums define the nodes
    assert np.max(np.abs(A.sum(1) - c)) < 1e-14
    # strictly lower triangular (explicit method)
    assert np.all(np.triu(A) == 0)
    # first-same-as-last: the last row is b and b7 = 0
    assert np.max(np.abs(A[6] - b)) == 0.0 and b[6] == 0.0
    assert abs(bt.sum()) < 1e-15
    worst_b, worst_bhat5 = 0.0, 0.0
    for t in trees_up_to(5):
        phi_b = b @ weight_vector(t, A)
        phi_h = bhat @ weight_vector(t, A)
        res_b = abs(phi_b - 1.0 / density(t))
        worst_b = max(worst_b, res_b)
        if order(t) <= 4:
            assert abs(phi_h - 1.0 / density(t)) < 1e-13, t
        else:
            worst_bhat5 = max(worst_bhat5, abs(phi_h - 1.0 / density(t)))
    assert worst_b < 5e-14          # decimals of size ~13 carry ~1e-15 relative rounding
    # the embedded weights are genuinely of order 4 (they miss some order-5 condition)
    assert worst_bhat5 > 1e-6


def test_tsit5_not_order_six(orc):
    c, A, b, bt = orc.tsit5_tableau()
    worst = max(abs(b @ weight_vector(t, A) - 1.0 / density(t))
                for t in trees_up_to(6) if order(t) == 6)
    assert worst > 1e-6


def test_ros34pw2_conditions(orc):
    g, al, ga, b, bh = orc.ros34pw2_tableau()
    beta = al + ga                     # beta_ij = alpha_ij + gamma_ij (j < i)
    alpha_i = al.sum(1)
    betap = beta.sum(1)                # beta'_i
    # order 1..3 for b (Hairer-Wanner II, Table IV.7.1 in the beta' form)
    assert abs(b.sum() - 1) < 1e-15
    assert abs(b @ betap - (0.5 - g)) < 1e-15
    assert abs(b @ alpha_i ** 2 - 1.0 / 3.0) < 1e-15
    assert abs(b @ (beta @ betap) - (1.0 / 6.0 - g + g * g)) < 1e-15
    # order 1..2 for b_hat, and it is not order 3
    assert abs(bh.sum() - 1) < 1e-15
    assert abs(bh @ betap - (0.5 - g)) < 1e-15
    assert abs(bh @ alpha_i ** 2 - 1.0 / 3.0) > 1e-3
    # gamma is the root of 6 g^3 - 18 g^2 + 9 g - 1 that makes the method L-stable
    assert abs(6 * g ** 3 - 18 * g ** 2 + 9 * g - 1) < 1e-14
    # stiffly accurate: b_i = alpha_4i + gamma_4i with gamma_44 = gamma
    last = al[3] + ga[3]
    last[3] = g
    assert np.max(np.abs(b - last)) < 1e-15


def _tsit5_R(z, A, b, const=1.0):
    """Stability polynomial R(z) = 1 + sum_q z^q b^T A^(q-1) 1 of an explicit RK method
    (with const=0, the same sum without the leading 1)."""
    s = const + 0j
    v = np.ones(len(b))
    for q in range(1, len(b) + 1):
        s += z ** q * (b @ v)
        v = A @ v
    return s


def test_tsit5_one_step_is_stability_polynomial(orc):
    c, A, b, bt = orc.tsit5_tableau()
    for lam in (-1.0, -3.7, 0.8, -25.0):
        for h in (0.01, 0.2, 0.5):
            y = orc.replay("linear1", "tsit5", [[lam]], [[1.0]], [[h]], [1])
            R = _tsit5_R(h * lam, A, b).real
            assert abs(y[0, 0] - R) <= 1e-13 * max(1.0, abs(R)), (lam, h)


def test_tsit5_error_estimate_is_polynomial_difference(orc):
    c, A, b, bt = orc.tsit5_tableau()
    bhat = b - bt
    for lam, h in ((-1.0, 0.3), (-4.0, 0.1), (2.0, 0.05)):
        ynew, e = orc.trial("linear1", "tsit5", [lam], [1.7], h)
        z = h * lam
        R = _tsit5_R(z, A, b).real
        E = _tsit5_R(z, A, bt, const=0.0).real        # R - R_hat without cancellation
        assert abs(ynew[0] - 1.7 * R) <= 1e-14 * abs(1.7 * R)
        assert abs(e[0] - 1.7 * E) <= 1e-6 * abs(1.7 * E) + 1e-15   # rounding of the cancelling sum
        # and the embedded weights give a genuinely different polynomial
        Rh = _tsit5_R(z, A, bhat).real
        assert abs((R - Rh) - E) <= 1e-15 * 8


def _ros_matrices(Z, g, al, ga, b, bh):
    """For y' = A y, k_i = K_i y_n with (I - g Z) K_i = Z (I + sum_j beta_ij K_j), Z = h A."""
    d = Z.shape[0]
    I = np.eye(d)
    beta = al + ga
    K = []
    Minv = np.linalg.inv(I - g * Z)
    for i in range(4):
        acc = I.copy()
        for j in range(i):
            acc = acc + beta[i, j] * K[j]
        K.append(Minv @ Z @ acc)
    R = I + sum(b[i] * K[i] for i in range(4))
    E = sum((b[i] - bh[i]) * K[i] for i in range(4))
    return R, E


def test_ros34pw2_one_step_linear(orc):
    g, al, ga, b, bh = orc.ros34pw2_tableau()
    rng = np.random.default_rng(5)
    for h in (0.01, 0.3, 5.0):
        Amat = rng.normal(size=(3, 3)) - 2 * np.eye(3)
        y = rng.normal(size=3)
        ynew, e = orc.trial("linear3", "ros34pw2", Amat.ravel(), y, h)
        R, E = _ros_matrices(h * Amat, g, al, ga, b, bh)
        assert np.max(np.abs(ynew - R @ y)) <= 1e-13 * max(1, np.max(np.abs(R @ y)))
        assert np.max(np.abs(e - E @ y)) <= 1e-13 * max(1, np.max(np.abs(y)))


def test_ros34pw2_L_stable(orc):
    # R(z) -> 0 as z -> -inf (stiffly accurate + A-stable); one huge step of y' = -1e8 y
    y = orc.replay("linear1", "ros34pw2", [[-1e8]], [[1.0]], [[10.0]], [1], )
    assert abs(y[0, 0]) < 1e-6
