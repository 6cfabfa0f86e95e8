"""Closed-form pins of the oracle's starting step and of its step controller's accept/reject law.

Sources: "gradsolve: fast exact gradients for ODE ensembles on GPUs", §2.1 -- a trial step is
accepted when RMS(e / (atol + rtol max(|y|, |y_new|))) <= 1; a controller proposes the next step
size; a rejected trial is retried from the same (t, y) with a smaller step.  The pages print
neither the controller nor the starting-step rule; the readings pinned here are the textbook ones:
the I-controller h <- h clamp(0.9 err^(-1/q), 0.2, facmax) with facmax = 10, except 1 for the
proposal right after a reject, and Hairer, Norsett & Wanner's starting step (Solving ODEs I,
§II.4) with the same RMS norm and scales atol + rtol |y0|.

On a diagonal linear system y' = diag(lam) y every quantity the loop looks at is a closed-form
function of h: one step multiplies component i by R(h lam_i) and its error estimate is
E(h lam_i) y_i, with R and E the method's stability and error-estimate functions built from its
table (for Rosenbrock methods the rational functions of the linearly implicit stages).  So the
whole sequence of attempts -- which are accepted, which rejected, and every step size -- is
predicted here from those functions and the written law, without the oracle's stage code or loop,
and the oracle's record must reproduce it.
"""
import numpy as np
import pytest

from test_oracle_solve import _scalar_step

# (order p of the starting-step rule, controller exponent q)
ORDERS = {"tsit5": (5, 5), "vern7": (7, 7), "ros34pw2": (3, 3), "rosenbrock23": (2, 3)}


def _rms(v):
    v = np.asarray(v, dtype=np.float64)
    return float(np.sqrt(np.mean(v * v)))


def starting_step(lam, y0, t0, t1, rtol, atol, p):
    """HNW I §II.4 for y' = diag(lam) y: f(y0) = lam y0 and (f(y0 + h0 f0) - f0)/h0 = lam^2 y0."""
    lam, y0 = np.atleast_1d(np.asarray(lam, float)), np.atleast_1d(np.asarray(y0, float))
    sc = atol + rtol * np.abs(y0)
    d0 = _rms(y0 / sc)
    d1 = _rms(lam * y0 / sc)
    h0 = 1e-6 if (d0 < 1e-5 or d1 < 1e-5) else 0.01 * d0 / d1
    d2 = _rms(lam * lam * y0 / sc)
    dm = max(d1, d2)
    h1 = max(1e-6, 1e-3 * h0) if dm <= 1e-15 else (0.01 / dm) ** (1.0 / p)
    return min(100.0 * h0, h1, t1 - t0), h0, h1


def predict(orc, method, lam, y0, t0, t1, rtol, atol):
    """Every attempt of the adaptive loop on y' = diag(lam) y, from the closed-form factors."""
    p, q = ORDERS[method]
    step = _scalar_step(method, orc)
    lam, y = np.atleast_1d(np.asarray(lam, float)), np.atleast_1d(np.asarray(y0, float)).copy()
    h = starting_step(lam, y, t0, t1, rtol, atol, p)[0]
    t, last_rejected, attempts = t0, False, []
    while t < t1:
        clipped = t + h > t1
        if clipped:
            h = t1 - t
        RE = [step(h, l) for l in lam]
        ynew = np.array([r * yi for (r, _), yi in zip(RE, y)])
        e = np.array([er * yi for (_, er), yi in zip(RE, y)])
        err = _rms(e / (atol + rtol * np.maximum(np.abs(y), np.abs(ynew))))
        if err <= 1.0:
            facmax = 1.0 if last_rejected else 10.0
            raw = facmax if err == 0 else 0.9 * err ** (-1.0 / q)
            attempts.append(dict(ok=True, t=t, h=h, err=err, raw=raw, after_reject=last_rejected))
            t = t1 if (clipped or t + h >= t1) else t + h
            y = ynew
            h = h * min(facmax, max(0.2, raw))
            last_rejected = False
        else:
            raw = 0.9 * err ** (-1.0 / q)
            attempts.append(dict(ok=False, t=t, h=h, err=err, raw=raw, after_reject=last_rejected))
            h = h * min(10.0, max(0.2, raw))
            last_rejected = True
        assert len(attempts) < 20000
    return attempts


def _amplification(orc, method):
    """sum_j |b_j - b^_j| (1 + max_i sum_l |a_il|): rounding of the stages carried into e."""
    if method == "tsit5":
        _, A, _, bt = orc.tsit5_tableau()
        return np.abs(bt).sum() * (1 + np.abs(A).sum(1).max())
    if method == "vern7":
        A, b, bh = orc.vern7_tableau()
        return np.abs(b - bh).sum() * (1 + np.abs(A).sum(1).max())
    if method == "ros34pw2":
        _, al, ga, b, bh = orc.ros34pw2_tableau()
        return np.abs(b - bh).sum() * (1 + (np.abs(al) + np.abs(ga)).sum(1).max())
    # Rosenbrock23: e = h (k1 - 2 k2 + k3)/6, k3 built with the weights 6 + sqrt(2) and 2
    return (4.0 / 6.0) * (1 + 6 + np.sqrt(2) + 2)


def _field(lam):
    """The oracle's linear family y' = A y (theta = A row-major) with A = diag(lam)."""
    return "linear%d" % len(lam), [np.diag(np.asarray(lam, float)).ravel()]


def _run(orc, method, lam, y0, t1, rtol, atol):
    field, theta = _field(lam)
    y0 = np.atleast_1d(np.asarray(y0, float))
    r = orc.solve(field, method, theta, [y0], 0.0, t1, rtol, atol, keep_record=True)
    att = predict(orc, method, lam, y0, 0.0, t1, rtol, atol)
    # the predicted sequence must not hinge on a near-tie of the test err <= 1 (both sides round)
    assert min(abs(a["err"] - 1.0) for a in att) > 1e-6
    acc = [a for a in att if a["ok"]]
    S = int(r["S"][0])
    assert r["status"][0] == 0
    assert S == len(acc)
    assert int(r["rejected"][0]) == len(att) - len(acc)
    # The oracle forms e = h sum_j (b_j - b^_j) k_j from the stages: a difference of O(|y|) terms
    # that leaves |e| ~ err rtol |y|, so its relative rounding is ~ amp eps / rtol, with amp the
    # table's bound on how much stage rounding reaches e; a step size (h err^(-1/q)) inherits it.
    # The closed forms above carry no such cancellation.  The bar stays orders of magnitude below
    # what any change of the law (a safety factor, a cap, an exponent, the starting rule) moves.
    bar = 1e-12 + 16 * _amplification(orc, method) * np.finfo(float).eps / rtol
    H, T = r["H"][0, :S], r["T"][0, :S]
    np.testing.assert_allclose(H, [a["h"] for a in acc], rtol=bar, atol=0)
    np.testing.assert_allclose(T, [a["t"] for a in acc], rtol=bar, atol=1e-300)
    return r, att


def test_tsit5_reject_and_retry_sequence(orc):
    # lam = -100, rtol 1e-3: the step hovers at the edge of Tsit5's stability region, so the run
    # rejects repeatedly.  Every reject's factor is inside (0.2, 10) (the safety factor and the
    # exponent decide it), and every step accepted right after a reject would grow (0.9
    # err^(-1/5) > 1) but is held at the factor 1.
    r, att = _run(orc, "tsit5", [-100.0], 1.0, 1.0, 1e-3, 1e-6)
    rej = [a for a in att if not a["ok"]]
    assert len(rej) >= 3
    assert all(0.2 < a["raw"] < 10 for a in rej)
    held = [a for a in att if a["ok"] and a["after_reject"] and a["raw"] > 1.0]
    assert len(held) >= 3
    # retry from the same (t, y): every rejected attempt shares its t with the next attempt
    for i, a in enumerate(att[:-1]):
        if not a["ok"]:
            assert att[i + 1]["t"] == a["t"]
    # the starting step is 100 h0 here (h0 = 0.01 d0/d1 = 0.01/|lam|), and it is accepted
    h, h0, h1 = starting_step([-100.0], [1.0], 0.0, 1.0, 1e-3, 1e-6, 5)
    assert h == 100.0 * h0 < h1 and att[0]["ok"]
    assert abs(r["H"][0, 0] - 1.0 / 100.0) <= 1e-15


def test_tsit5_first_trial_rejected(orc):
    # rtol 1e-4: the starting step (100 h0 = 1/|lam|) fails the error test; the retry and the
    # rest of the sequence follow from the controller law
    r, att = _run(orc, "tsit5", [-100.0], 1.0, 1.0, 1e-4, 1e-8)
    assert not att[0]["ok"] and att[1]["t"] == 0.0
    h = starting_step([-100.0], [1.0], 0.0, 1.0, 1e-4, 1e-8, 5)[0]
    assert att[0]["h"] == h
    fac = min(10.0, max(0.2, 0.9 * att[0]["err"] ** (-0.2)))
    assert abs(r["H"][0, 0] - h * fac) <= 1e-12 * h


@pytest.mark.parametrize("method", ["tsit5", "vern7", "ros34pw2", "rosenbrock23"])
def test_starting_step_three_components(orc, method):
    # a diagonal system whose components have different scales and rates: the three norms d0,
    # d1, d2 of the rule differ (d2 != d1^2/d0), and the first step is the rule's
    lam, y0 = [-0.5, -3.0, 2.0], [1.0, -0.25, 0.04]
    rtol, atol = 1e-6, 1e-9
    r, att = _run(orc, method, lam, y0, 2.0, rtol, atol)
    p = ORDERS[method][0]
    h, h0, h1 = starting_step(lam, y0, 0.0, 2.0, rtol, atol, p)
    assert att[0]["h"] == h
    if att[0]["ok"]:
        assert abs(r["H"][0, 0] - h) <= 1e-13 * h


def test_starting_step_at_zero_state_and_growth_cap(orc):
    # y0 = 0: d0 = d1 = 0 gives h0 = 1e-6 and, with d2 = 0, h1 = max(1e-6, 1e-3 h0) = 1e-6.  Every
    # error estimate is then exactly zero, the controller takes its cap (10) on every step, and the
    # record is 1e-6, 1e-5, ... until the last step is clipped to reach t1.
    r, att = _run(orc, "tsit5", [-2.0], 0.0, 1.0, 1e-6, 1e-9)
    H = r["H"][0, :int(r["S"][0])]
    assert all(a["ok"] and a["err"] == 0.0 for a in att)
    np.testing.assert_allclose(H[:-1], 1e-6 * 10.0 ** np.arange(len(H) - 1), rtol=1e-12)
    assert abs(r["T"][0, len(H) - 1] + H[-1] - 1.0) < 1e-15


@pytest.mark.parametrize("method", ["vern7", "ros34pw2", "rosenbrock23"])
def test_other_methods_follow_the_law(orc, method):
    # the same law with each method's exponent on a mildly stiff diagonal system
    _run(orc, method, [-1.0, -40.0], [1.0, 0.5], 3.0, 1e-5, 1e-8)
