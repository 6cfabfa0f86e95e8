"""GPU parity of the stiff methods against the oracle: Rosenbrock23 ("gradsolve: fast exact
gradients for ODE ensembles on GPUs" §3.1, the linearly implicit method of the fused stiff
kernels) on Robertson and HIRES, and ROS34PW2 on HIRES (§4.5-4.6: HIRES differentiated with
respect to its initial state).  Record counts and states, forward kernel = record kernel,
replay gradient on the GPU's mesh and on an imported oracle mesh."""
import numpy as np
import pytest

import gpu_util as U
from differentiable_adaptive_ode_b200 import gradsolve as G
from differentiable_adaptive_ode_b200 import workloads as W

pytestmark = pytest.mark.gpu

CASES = [("robertson_rb23", 200), ("hires", 150), ("hires_ros34pw2", 150)]


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    G.lib()


def _solve(orc, w, keep_record=False):
    return orc.solve(w.field, w.method, w.theta, w.y0, w.t0, w.t1, w.rtol, w.atol, dtype=w.dtype,
                     theta_shared=w.theta_shared, keep_record=keep_record, nthreads=8)


@pytest.mark.parametrize("name,N", CASES)
def test_stiff_record_forward_and_gradient(orc, name, N):
    w = U.small(name, N)
    rec, out = U.record(w)
    ex = U.export_padded(w, rec)
    ref = _solve(orc, w, keep_record=True)
    assert np.all(out["status"] == 0) and np.all(ref["status"] == 0)
    same = ex["S"] == ref["S"]
    assert same.mean() >= 0.999, same.mean()
    assert U.rel_rows(out["y1"][same], ref["y1"][same], w.atol).max() <= 1e-9
    fw = U.forward(w)
    assert np.array_equal(fw["S"], ex["S"]) and np.array_equal(fw["y1"], out["y1"])
    lam = np.random.default_rng(8).normal(size=(w.N, w.d))
    gy, gt = U.replay_grad(w, rec, lam)
    ry, rt = orc.replay_grad(w.field, w.method, w.theta, w.y0, ex["H"], ex["S"], lam,
                             theta_shared=w.theta_shared, nthreads=8)
    if w.theta_shared:
        rt, gt = rt.sum(0, keepdims=True), gt[None, :]
    assert U.rel_rows(gy, ry, 1e-300).max() <= 1e-8
    assert U.rel_rows(gt, rt, 1e-300).max() <= 1e-8


@pytest.mark.parametrize("name", ["robertson_rb23", "hires"])
def test_stiff_gradient_on_imported_oracle_mesh(orc, name):
    w = U.small(name, 64)
    ref = _solve(orc, w, keep_record=True)
    rec = U.import_record(w, ref["S"], ref["T"], ref["H"], ref["Y"])
    lam = np.random.default_rng(9).normal(size=(w.N, w.d))
    gy, gt = U.replay_grad(w, rec, lam)
    ry, rt = orc.replay_grad(w.field, w.method, w.theta, w.y0, ref["H"], ref["S"], lam,
                             theta_shared=w.theta_shared, nthreads=8)
    if w.theta_shared:
        rt, gt = rt.sum(0, keepdims=True), gt[None, :]
    assert U.rel_rows(gy, ry, 1e-300).max() <= 1e-8
    assert U.rel_rows(gt, rt, 1e-300).max() <= 1e-8


def test_hires_reference_solution_on_gpu():
    # the published reference solution of HIRES at t = 321.8122 (Test Set for IVP Solvers)
    ref = np.array([0.7371312573325668e-3, 0.1442485726316185e-3, 0.5888729740967575e-4,
                    0.1175651343283149e-2, 0.2386356198831331e-2, 0.6238968252742796e-2,
                    0.2849998395185769e-2, 0.2850001604814231e-2])
    w = W.hires(N=2)
    w.y0 = np.tile(np.array([1.0, 0, 0, 0, 0, 0, 0, 0.0057]), (2, 1))
    w.method, w.rtol, w.atol = "ros34pw2", 1e-11, 1e-15
    fw = U.forward(w)
    assert np.all(fw["status"] == 0)
    assert np.max(np.abs(fw["y1"][0] - ref) / ref) < 1e-8


@pytest.mark.parametrize("name,rtol,atol,t1", [("robertson_rb23", 1e-4, 1e-8, 1.0),
                                               ("lorenz63_vern7", 1e-5, 1e-6, None)])
def test_fp32_methods_on_their_own_mesh(orc, name, rtol, atol, t1):
    # fp32 reading: states against the fp32 oracle replay of the GPU's own mesh, gradients against
    # the exact (fp64) derivative of the replay over that mesh.  (Robertson over [0, 1e4] is out
    # of reach in fp32: the step-size floor 16 eps |t1 - t0| = 0.02 is above the initial
    # transient's steps, so every trajectory ends with status 2; the test takes [0, 1].)
    w = U.small(name, 300)
    w.dtype, w.rtol, w.atol = np.float32, rtol, atol
    if t1 is not None:
        w.t1 = t1
    rec, out = U.record(w)
    assert np.all(out["status"] == 0)
    ex = U.export_padded(w, rec)
    yrep = orc.replay(w.field, w.method, w.theta, w.y0, ex["H"], ex["S"], dtype=np.float32,
                      theta_shared=w.theta_shared)
    err = U.rel_rows(out["y1"], yrep, atol)
    assert np.quantile(err, 0.99) <= 1e-4 and err.max() <= 1e-3, err.max()
    lam = np.random.default_rng(12).normal(size=(w.N, w.d))
    gy, gt = U.replay_grad(w, rec, lam)
    ry, rt = orc.replay_grad(w.field, w.method, w.theta.astype(np.float32).astype(np.float64),
                             w.y0.astype(np.float32).astype(np.float64),
                             ex["H"].astype(np.float64), ex["S"], lam, nthreads=8)
    for got, want in ((gy, ry), (gt, rt)):
        rel = U.rel_rows(got, want, 1e-300)
        assert np.quantile(rel, 0.99) <= 1e-3 and rel.max() <= 1e-2, rel.max()


@pytest.mark.parametrize("name", ["robertson_rb23", "hires"])
def test_stiff_outputs_at_requested_times(orc, name):
    import torch
    w = U.small(name, 64)
    rec, out = U.record(w)
    ex = U.export_padded(w, rec)
    tau = np.array([w.t0 + (w.t1 - w.t0) * f for f in (0.001, 0.1, 0.5, 1.0)])
    dt = torch.float64
    yo = torch.empty((w.N, len(tau), w.d), dtype=dt, device="cuda")
    G.gs_replay_outputs(rec, U.dev(w.theta, dt), U.dev(w.y0, dt), tau, yo)
    lo = np.random.default_rng(13).normal(size=(w.N, len(tau), w.d))
    gy = torch.empty((w.N, w.d), dtype=dt, device="cuda")
    gt = torch.empty((w.m,) if w.theta_shared else (w.N, w.m), dtype=dt, device="cuda")
    G.gs_replay_grad_outputs(rec, U.dev(w.theta, dt), tau, U.dev(lo, dt), None, gt, gy)
    torch.cuda.synchronize()
    want = orc.replay_outputs(w.field, w.method, w.theta, w.y0, ex["T"], ex["H"], ex["S"], w.t1,
                              tau, theta_shared=w.theta_shared, nthreads=8)
    assert U.rel_rows(yo.cpu().numpy().reshape(w.N, -1), want.reshape(w.N, -1),
                      w.atol).max() <= 1e-9
    ry, rt = orc.replay_outputs_grad(w.field, w.method, w.theta, w.y0, ex["T"], ex["H"], ex["S"],
                                     w.t1, tau, lo, theta_shared=w.theta_shared, nthreads=8)
    assert U.rel_rows(gy.cpu().numpy(), ry, 1e-300).max() <= 1e-8
    got_t = gt.cpu().numpy()
    if w.theta_shared:
        got_t, rt = got_t[None, :], rt.sum(0, keepdims=True)
    assert U.rel_rows(got_t, rt, 1e-300).max() <= 1e-8
