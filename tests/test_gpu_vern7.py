"""GPU parity of the Verner 7(6) pair ("gradsolve: fast exact gradients for ODE ensembles on
GPUs" §3.1: the seventh-order Verner pair next to Tsit5; §4.6: the Verner engine on the Lorenz
gradient) against the oracle: record (counts, states, step sizes), forward-only kernel, replay
gradient on the GPU's own mesh and on an imported oracle mesh, and outputs at requested times."""
import numpy as np
import pytest

import gpu_util as U
from differentiable_adaptive_ode_b200 import gradsolve as G
from differentiable_adaptive_ode_b200 import workloads as W

pytestmark = pytest.mark.gpu

CASES = [("lorenz63_vern7", 400), ("lotka_volterra_vern7", 300), ("nfw_mn_vern7", 300),
         ("log_halo_vern7", 300)]


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
def test_vern7_record_forward_and_gradient(orc, name, N):
    w = U.small(name, N)
    rec, out = U.record(w)
    ex = U.export_padded(w, rec)
    ref = _solve(orc, w, keep_record=True)
    assert np.all(out["status"] == 0) and np.all(ref["status"] == 0)
    assert np.array_equal(ex["S"], ref["S"])
    assert U.rel_rows(out["y1"], ref["y1"], w.atol).max() <= 1e-9
    # step sizes: the Verner controller's step sequence sits on a wider rounding floor than
    # Tsit5's (its error estimate cancels terms of size |a_ij| ~ 190): the bar is the oracle's own
    # spread under a one-ulp change of y0 (same counts, measured 2e-3 on the stellar ensemble)
    yp = w.y0 * (1 + np.finfo(np.float64).eps)
    ref2 = orc.solve(w.field, w.method, w.theta, yp, w.t0, w.t1, w.rtol, w.atol,
                     theta_shared=w.theta_shared, keep_record=True, nthreads=8)

    def dh(Ha, Hb, S):
        return np.max(np.abs(Ha[:S] - Hb[:S])) / np.max(np.abs(Hb[:S]))

    same = np.flatnonzero(ref2["S"] == ref["S"])
    spread = max([dh(ref2["H"][k], ref["H"][k], ref["S"][k]) for k in same] + [1e-7])
    gpu = max(dh(ex["H"][k], ref["H"][k], ex["S"][k]) for k in range(N))
    print("vern7 step sizes: gpu %.3g, oracle 1-ulp spread %.3g" % (gpu, spread))
    assert gpu <= max(1e-6, 3 * spread)
    fw = U.forward(w)
    assert np.array_equal(fw["S"], ex["S"]) and np.array_equal(fw["y1"], out["y1"])
    assert np.array_equal(fw["rejected"], ref["rejected"])
    lam = np.random.default_rng(5).normal(size=(w.N, w.d))
    gy, gt = U.replay_grad(w, rec, lam)
    ry, rt = orc.replay_grad(w.field, w.method, w.theta, w.y0, ex["H"], ex["S"], lam,
                             theta_shared=w.theta_shared, nthreads=8)
    if w.theta_shared:
        rt, gt = rt.sum(0, keepdims=True), gt[None, :]
    assert U.rel_rows(gy, ry, 1e-300).max() <= 1e-8
    assert U.rel_rows(gt, rt, 1e-300).max() <= 1e-8


def test_vern7_imported_mesh_and_outputs(orc):
    w = U.small("lorenz63_vern7", 200)
    ref = _solve(orc, w, keep_record=True)
    rec = U.import_record(w, ref["S"], ref["T"], ref["H"], ref["Y"])
    lam = np.random.default_rng(6).normal(size=(w.N, w.d))
    gy, gt = U.replay_grad(w, rec, lam)
    ry, rt = orc.replay_grad(w.field, w.method, w.theta, w.y0, ref["H"], ref["S"], lam, nthreads=8)
    assert U.rel_rows(gy, ry, 1e-300).max() <= 1e-8 and U.rel_rows(gt, rt, 1e-300).max() <= 1e-8
    # outputs at requested times and their gradient
    import torch
    tau = np.array([0.05, 0.3, 0.55, 0.8, 1.0])
    rec2, out = U.record(w)
    ex = U.export_padded(w, rec2)
    yo = torch.empty((w.N, len(tau), w.d), dtype=torch.float64, device="cuda")
    G.gs_replay_outputs(rec2, U.dev(w.theta, torch.float64), U.dev(w.y0, torch.float64), tau, yo)
    torch.cuda.synchronize()
    want = orc.replay_outputs(w.field, w.method, w.theta, w.y0, ex["T"], ex["H"], ex["S"], w.t1,
                              tau, nthreads=8)
    assert U.rel_rows(yo.cpu().numpy().reshape(w.N, -1), want.reshape(w.N, -1), w.atol).max() \
        <= 1e-9
    lo = np.random.default_rng(7).normal(size=(w.N, len(tau), w.d))
    gy = torch.empty((w.N, w.d), dtype=torch.float64, device="cuda")
    gt = torch.empty((w.N, w.m), dtype=torch.float64, device="cuda")
    G.gs_replay_grad_outputs(rec2, U.dev(w.theta, torch.float64), tau, U.dev(lo, torch.float64),
                             None, gt, gy)
    torch.cuda.synchronize()
    ry, rt = orc.replay_outputs_grad(w.field, w.method, w.theta, w.y0, ex["T"], ex["H"], ex["S"],
                                     w.t1, tau, lo, nthreads=8)
    assert U.rel_rows(gy.cpu().numpy(), ry, 1e-300).max() <= 1e-8
    assert U.rel_rows(gt.cpu().numpy(), rt, 1e-300).max() <= 1e-8


def test_vern7_fp32_fixed_mesh_and_unsupported():
    import torch
    w = U.small("lorenz63_vern7", 300)
    w.dtype = np.float32
    w.rtol, w.atol = 1e-5, 1e-6
    rec, out = U.record(w)
    assert np.all(out["status"] == 0)
    m = W.mlp(N=4)
    sys_ = G.system("mlp", "vern7", "f32", True)
    y = torch.empty((4, 4), dtype=torch.float32, device="cuda")
    with pytest.raises(G.GradsolveError) as e:
        G.gs_solve_forward(sys_, 4, U.dev(m.theta, torch.float32), U.dev(m.y0, torch.float32),
                           0.0, 1.0, 1e-5, 1e-6, y)
    assert e.value.code == G.GS_ERR_UNSUPPORTED


def test_vern7_full_size_sampled(orc):
    import torch
    w = W.by_name("lorenz63_vern7")
    rec, out = U.record(w)
    info = rec.info()
    rng = np.random.default_rng(0)
    idx = np.unique(np.concatenate([[0, w.N - 1], rng.choice(w.N, size=24, replace=False)]))
    sub = W.subset(w, idx)
    ref = _solve(orc, sub, keep_record=True)
    off = torch.empty(w.N + 1, dtype=torch.int64, device="cuda")
    G.gs_record_export(rec, None, None, None, off)
    torch.cuda.synchronize()
    S = np.diff(off.cpu().numpy())
    assert np.array_equal(S[idx], ref["S"]) and int(info.total_steps) == int(S.sum())
    assert U.rel_rows(out["y1"][idx], ref["y1"], w.atol).max() <= 1e-9
