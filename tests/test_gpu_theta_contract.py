"""The replay calls differentiate the replay at the theta they are given, whatever theta the stored
states were made at ("gradsolve: fast exact gradients for ODE ensembles on GPUs", §3: the mesh
h = R(theta0) is held fixed as data and the replay Psi(theta; sg[h]) is differentiated; §4.8: one
recorded mesh serves the gradients of a whole fit).

The record keeps the theta of its stored states; a call at another theta replays the mesh forward
at that theta first.  Each case records at theta0 and calls at theta1 with no gs_replay_forward in
between; the result must match the oracle's replay gradient (or outputs) at theta1 on the GPU's
mesh, and a later call back at theta0 must match the oracle at theta0 again.
"""
import numpy as np
import pytest

import gpu_util as U
from differentiable_adaptive_ode_b200 import gradsolve as G
from differentiable_adaptive_ode_b200 import workloads as W

pytestmark = pytest.mark.gpu

STATE_TOL, GRAD_TOL = 1e-9, 1e-8   # the fp64 bars of the parity tests


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    G.lib()


def _oracle_grad(orc, w, theta, ex, lam):
    gy, gt = orc.replay_grad(w.field, w.method, theta, w.y0, ex["H"], ex["S"], lam,
                             theta_shared=w.theta_shared, nthreads=8)
    if w.theta_shared:
        gt = gt.sum(axis=0)
    return gy, gt


def _check(got, ref):
    gy, gt = got
    ry, rt = ref
    assert U.rel_rows(gy, ry, 1e-300).max() <= GRAD_TOL
    if rt.ndim == 1:
        assert np.max(np.abs(gt - rt)) / np.max(np.abs(rt)) <= GRAD_TOL
    else:
        assert U.rel_rows(gt, rt, 1e-300).max() <= GRAD_TOL


def _shared(w):
    w.theta_shared = True
    w.theta = w.theta[0].copy()
    return w


@pytest.mark.parametrize("name,N,shared", [("lorenz63", 300, False), ("nfw_mn", 300, False),
                                           ("nfw_mn", 300, True), ("robertson", 200, False),
                                           ("lorenz63_vern7", 200, False),
                                           ("robertson_rb23", 200, False)])
def test_gradient_at_a_new_theta_without_replay_forward(orc, name, N, shared):
    w = U.small(name, N)
    if shared:
        _shared(w)
    rec, _ = U.record(w)
    ex = U.export_padded(w, rec)
    lam = np.random.default_rng(5).normal(size=(w.N, w.d))
    th0 = w.theta.copy()
    th1 = th0 * 1.01
    got0 = U.replay_grad(w, rec, lam, theta=th0)
    got1 = U.replay_grad(w, rec, lam, theta=th1)          # no gs_replay_forward in between
    _check(got1, _oracle_grad(orc, w, th1, ex, lam))
    back = U.replay_grad(w, rec, lam, theta=th0)          # and back to the recorded theta
    _check(back, _oracle_grad(orc, w, th0, ex, lam))
    # the states replayed at theta0 equal the recorded ones to rounding (the replay step and the
    # solve's trial form y_{n+1} in a different order), so the gradients agree far inside the bar
    for a, b in zip(back, got0):
        assert U.rel_rows(np.atleast_2d(a), np.atleast_2d(b), 1e-300).max() <= 1e-10
    # the mesh itself is untouched
    ex2 = U.export_padded(w, rec)
    assert np.array_equal(ex2["H"], ex["H"]) and np.array_equal(ex2["T"], ex["T"])


def test_one_changed_trajectory_is_seen(orc):
    # a change in a single trajectory's theta (one component, one ulp) is enough to refresh
    w = U.small("lorenz63", 257)
    rec, _ = U.record(w)
    ex = U.export_padded(w, rec)
    lam = np.random.default_rng(6).normal(size=(w.N, w.d))
    th1 = w.theta.copy()
    th1[200, 1] = np.nextafter(th1[200, 1], np.inf) * 1.001
    got = U.replay_grad(w, rec, lam, theta=th1)
    _check(got, _oracle_grad(orc, w, th1, ex, lam))


def test_imported_states_are_replayed_on_first_use(orc):
    # an imported record carries states whose theta the library cannot know: here they are the
    # oracle's states at theta0, and the first call asks for theta1
    w = U.small("nfw_mn", 200)
    r = orc.solve(w.field, w.method, w.theta, w.y0, w.t0, w.t1, w.rtol, w.atol, keep_record=True,
                  nthreads=8)
    rec = U.import_record(w, r["S"], r["T"], r["H"], r["Y"])
    ex = dict(H=r["H"], S=r["S"])
    lam = np.random.default_rng(7).normal(size=(w.N, w.d))
    th1 = w.theta * 0.995
    _check(U.replay_grad(w, rec, lam, theta=th1), _oracle_grad(orc, w, th1, ex, lam))


def test_outputs_at_a_new_theta(orc):
    w = U.small("lorenz63", 200)
    rec, _ = U.record(w)
    ex = U.export_padded(w, rec)
    th1 = w.theta * 1.02
    tau = np.array([0.0, 0.25, 0.5, 0.75, 1.0])
    torch = U.torch()
    out = torch.empty((w.N, len(tau), w.d), dtype=torch.float64, device="cuda")
    G.gs_replay_outputs(rec, U.dev(th1, torch.float64), U.dev(w.y0, torch.float64), tau, out)
    torch.cuda.synchronize()
    ref = orc.replay_outputs(w.field, w.method, th1, w.y0, ex["T"], ex["H"], ex["S"], w.t1, tau,
                             nthreads=8)
    err = U.rel_rows(out.cpu().numpy().reshape(w.N, -1), ref.reshape(w.N, -1), w.atol)
    assert err.max() <= STATE_TOL, err.max()


def test_mlp_at_new_weights_equals_explicit_replay():
    # the neural field: a call at new weights equals gs_replay_forward(new weights) followed by
    # the call, bit for bit (the same kernels run either way).  Both run on one record: its
    # visiting order fixes how the weight cotangent's partial sums are grouped.
    w = W.mlp(N=256)
    rec, _ = U.record(w)
    lam = np.random.default_rng(8).normal(size=(w.N, w.d)).astype(np.float32)
    th1 = (w.theta * np.float32(1.01)).astype(np.float32)
    direct = U.replay_grad(w, rec, lam, theta=th1)
    torch = U.torch()
    y0 = U.dev(w.y0, torch.float32)
    G.gs_replay_forward(rec, U.dev(w.theta, torch.float32), y0)   # back to the recorded weights
    G.gs_replay_forward(rec, U.dev(th1, torch.float32), y0)       # and explicitly to th1
    explicit = U.replay_grad(w, rec, lam, theta=th1)
    for a, b in zip(direct, explicit):
        assert np.array_equal(a, b)
