"""GPU parity of the outputs at requested times and of their gradient against the oracle, on the
GPU's own recorded mesh ("gradsolve: fast exact gradients for ODE ensembles on GPUs", §3.4:
one extra solver step from the preceding mesh point exactly to each requested time)."""
import numpy as np
import pytest

import gpu_util as U
from differentiable_adaptive_ode_b200 import gradsolve as G
from differentiable_adaptive_ode_b200 import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    G.lib()


def _times(w, ex):
    # t0, interior times, one exact mesh time of trajectory 0, t1 and a time past t1
    mesh = ex["T"][0, min(3, ex["S"][0] - 1)]
    tau = np.concatenate([[w.t0], np.linspace(w.t0, w.t1, 6)[1:-1], [mesh, w.t1, w.t1 * 1.5]])
    return np.sort(tau).astype(w.dtype).astype(np.float64)


def _gpu_outputs(w, rec, tau):
    torch = U.torch()
    dt = U.tdtype(w)
    out = torch.empty((w.N, len(tau), w.d), dtype=dt, device="cuda")
    G.gs_replay_outputs(rec, U.dev(w.theta, dt), U.dev(w.y0, dt), tau, out)
    torch.cuda.synchronize()
    return out.cpu().numpy()


def _gpu_grad(w, rec, tau, lam_out, lam1):
    torch = U.torch()
    dt = U.tdtype(w)
    gy = torch.empty((w.N, w.d), dtype=dt, device="cuda")
    gt = torch.empty((w.m,) if w.theta_shared else (w.N, w.m), dtype=dt, device="cuda")
    G.gs_replay_grad_outputs(rec, U.dev(w.theta, dt), tau, U.dev(lam_out, dt),
                             None if lam1 is None else U.dev(lam1, dt), gt, gy)
    torch.cuda.synchronize()
    return gy.cpu().numpy(), gt.cpu().numpy()


@pytest.mark.parametrize("name,N", [("lotka_volterra", 200), ("lorenz63", 300),
                                    ("robertson", 150), ("nfw_mn", 300)])
def test_outputs_and_gradient_match_oracle(orc, name, N):
    w = U.small(name, N)
    rec, out = U.record(w)
    ex = U.export_padded(w, rec)
    tau = _times(w, ex)
    got = _gpu_outputs(w, rec, tau)
    ref = orc.replay_outputs(w.field, w.method, w.theta, w.y0, ex["T"], ex["H"], ex["S"], w.t1, tau,
                             nthreads=8)
    err = U.rel_rows(got.reshape(N, -1), ref.reshape(N, -1), w.atol)
    assert err.max() <= 1e-9, err.max()
    # the last two times are t1 and beyond: the final state
    assert U.rel_rows(got[:, -1], out["y1"], w.atol).max() <= 1e-12
    rng = np.random.default_rng(6)
    lam_out = rng.normal(size=(N, len(tau), w.d))
    lam1 = rng.normal(size=(N, w.d))
    gy, gt = _gpu_grad(w, rec, tau, lam_out, lam1)
    ry, rt = orc.replay_outputs_grad(w.field, w.method, w.theta, w.y0, ex["T"], ex["H"], ex["S"],
                                     w.t1, tau, lam_out, nthreads=8)
    ry1, rt1 = orc.replay_grad(w.field, w.method, w.theta, w.y0, ex["H"], ex["S"], lam1, nthreads=8)
    assert U.rel_rows(gy, ry + ry1, 1e-300).max() <= 1e-8
    assert U.rel_rows(gt, rt + rt1, 1e-300).max() <= 1e-8


def test_outputs_shared_theta_and_fp32(orc):
    w = U.small("nfw_mn", 500)
    w.theta_shared = True
    w.theta = w.theta[0].copy()
    rec, out = U.record(w)
    ex = U.export_padded(w, rec)
    tau = _times(w, ex)
    lam_out = np.random.default_rng(7).normal(size=(w.N, len(tau), w.d))
    gy, gt = _gpu_grad(w, rec, tau, lam_out, None)
    ry, rt = orc.replay_outputs_grad(w.field, w.method, w.theta, w.y0, ex["T"], ex["H"], ex["S"],
                                     w.t1, tau, lam_out, theta_shared=True, nthreads=8)
    assert np.max(np.abs(gt - rt.sum(0))) <= 1e-8 * np.max(np.abs(rt.sum(0)))
    assert U.rel_rows(gy, ry, 1e-300).max() <= 1e-8
    # fp32: outputs against the fp32 oracle on the same mesh (fixed mesh, no accept decisions)
    w32 = U.small("nfw_mn_f32", 300)
    rec32, out32 = U.record(w32)
    ex32 = U.export_padded(w32, rec32)
    tau32 = _times(w32, ex32)
    got = _gpu_outputs(w32, rec32, tau32)
    ref = orc.replay_outputs(w32.field, w32.method, w32.theta, w32.y0, ex32["T"], ex32["H"],
                             ex32["S"], w32.t1, tau32, dtype=np.float32, nthreads=8)
    err = U.rel_rows(got.reshape(300, -1), ref.reshape(300, -1), w32.atol)
    assert np.quantile(err, 0.99) <= 1e-4 and err.max() <= 1e-3
    # fp32 gradient of a loss on the outputs against the exact (fp64) derivative over the GPU's
    # fp32 mesh.  Cotangents of random sign enter at nine times and partly cancel, so fp32
    # rounding alone moves a few trajectories' dL/dtheta by more than 1e-3: the oracle's own fp32
    # derivative on this mesh does (p99 1.2e-3).  Bars: the ensemble within 1e-3; 99 % of the
    # trajectories within 1e-3 or twice the fp32 oracle's 99th percentile, whichever is larger;
    # the worst within 1e-2.
    lo32 = np.random.default_rng(9).normal(size=(300, len(tau32), w32.d))
    gy, gt = _gpu_grad(w32, rec32, tau32, lo32, None)
    T64, H64 = ex32["T"].astype(np.float64), ex32["H"].astype(np.float64)
    ry, rt = orc.replay_outputs_grad(w32.field, w32.method, w32.theta, w32.y0, T64, H64,
                                     ex32["S"], w32.t1, tau32, lo32, nthreads=8)
    qy, qt = orc.replay_outputs_grad(w32.field, w32.method, w32.theta, w32.y0, ex32["T"],
                                     ex32["H"], ex32["S"], w32.t1, tau32, lo32, dtype=np.float32,
                                     nthreads=8)
    for got_, want, own in ((gy, ry, qy), (gt, rt, qt)):
        rel = U.rel_rows(got_, want, 1e-300)
        spread = np.quantile(U.rel_rows(own, want, 1e-300), 0.99)
        ens = np.linalg.norm(got_ - want) / np.linalg.norm(want)
        assert ens <= 1e-3, ens
        assert np.quantile(rel, 0.99) <= max(1e-3, 2 * spread), (np.quantile(rel, 0.99), spread)
        assert rel.max() <= 1e-2, rel.max()


def test_outputs_argument_checks():
    w = U.small("lorenz63", 8)
    rec, _ = U.record(w)
    torch = U.torch()
    out = torch.empty((8, 3, 3), dtype=torch.float64, device="cuda")
    th = U.dev(w.theta, torch.float64)
    with pytest.raises(G.GradsolveError) as e:
        G.gs_replay_outputs(rec, th, U.dev(w.y0, torch.float64), [0.5, 0.2, 0.9], out)
    assert e.value.code == G.GS_ERR_INVALID_ARG
    with pytest.raises(G.GradsolveError) as e:
        G.gs_replay_outputs(rec, th, U.dev(w.y0, torch.float64), [], out)
    assert e.value.code == G.GS_ERR_INVALID_ARG


@pytest.mark.parametrize("dtype", [np.float64, np.float32])
def test_mlp_outputs_and_gradient(orc, dtype):
    """The neural field (weights shared by the ensemble, one warp per trajectory): outputs at
    requested times and the gradient of a loss on them against the oracle on the GPU's own mesh;
    fp32 against the fp64 oracle on the fp32 mesh with the fp32 gradient bar of the replay
    gradient's test."""
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
    tau = _times(w, ex)
    T, H = ex["T"].astype(np.float64), ex["H"].astype(np.float64)
    got = _gpu_outputs(w, rec, tau)
    ref = orc.replay_outputs("mlp", "tsit5", w.theta, w.y0.astype(dtype).astype(np.float64), T, H,
                             ex["S"], w.t1, tau, theta_shared=True, nthreads=8)
    err = U.rel_rows(got.reshape(w.N, -1), ref.reshape(w.N, -1), w.atol)
    if dtype == np.float64:
        assert err.max() <= 1e-9, err.max()
        assert U.rel_rows(got[:, -1], out["y1"], w.atol).max() <= 1e-12
    else:
        assert np.quantile(err, 0.99) <= 1e-4 and err.max() <= 1e-3, err.max()
    rng = np.random.default_rng(8)
    lam_out = rng.normal(size=(w.N, len(tau), w.d))
    lam1 = rng.normal(size=(w.N, w.d))
    gy, gt = _gpu_grad(w, rec, tau, lam_out, lam1)
    ry, rt = orc.replay_outputs_grad("mlp", "tsit5", w.theta, w.y0, T, H, ex["S"], w.t1, tau,
                                     lam_out, theta_shared=True, nthreads=8)
    ry1, rt1 = orc.replay_grad("mlp", "tsit5", w.theta, w.y0, H, ex["S"], lam1, theta_shared=True,
                               nthreads=8)
    tol = 1e-8 if dtype == np.float64 else 1e-3
    rs = (rt + rt1).sum(0)
    assert gt.shape == (1348,)
    assert np.max(np.abs(gt - rs)) <= tol * np.max(np.abs(rs)), np.max(np.abs(gt - rs))
    assert np.quantile(U.rel_rows(gy, ry + ry1, 1e-300), 0.99) <= tol
    # the ensemble sum is reproducible bit for bit; every time at or after t1 (no first pass)
    gy2, gt2 = _gpu_grad(w, rec, tau, lam_out, lam1)
    assert np.array_equal(gt, gt2) and np.array_equal(gy, gy2)
    tau2 = np.array([w.t1, w.t1 * 1.25])
    lam2 = rng.normal(size=(w.N, 2, w.d))
    gy3, gt3 = _gpu_grad(w, rec, tau2, lam2, None)
    gy4, gt4 = U.replay_grad(w, rec, lam2.sum(1))
    # (the two kernels may run different grids, so the warp partials are summed in another
    # grouping; in fp32 the summed cotangent is also rounded once here and twice there)
    tight = 1e-12 if dtype == np.float64 else 1e-5
    assert np.max(np.abs(gt3 - gt4)) <= tight * np.max(np.abs(gt4))
    assert np.max(np.abs(gy3 - gy4)) <= tight * np.max(np.abs(gy4))


def test_outputs_gradient_windows_and_edges(orc):
    """The gradient's corner cases: many times with repeats, so that one step's window holds
    several outputs and some outputs fall on mesh points; a time before t0 (integrated backwards
    from y0, so in step 0's window); one of the two gradients asked for at a time; every time at
    or after t1 (the walk alone with the final state's cotangent); an ensemble that leaves the
    last 128-lane block partly empty."""
    torch = U.torch()
    w = U.small("lorenz63", 257)
    rec, _ = U.record(w)
    ex = U.export_padded(w, rec)
    rng = np.random.default_rng(11)
    T0 = ex["T"][0, :ex["S"][0]]
    tau = np.concatenate([[w.t0 - 0.05 * (w.t1 - w.t0)], rng.uniform(w.t0, w.t1, 40), T0[1:6],
                          T0[2:4], [w.t1, w.t1]])
    tau = np.sort(tau)
    lam_out = rng.normal(size=(w.N, len(tau), w.d))
    ry, rt = orc.replay_outputs_grad(w.field, w.method, w.theta, w.y0, ex["T"], ex["H"], ex["S"],
                                     w.t1, tau, lam_out, nthreads=8)
    gy, gt = _gpu_grad(w, rec, tau, lam_out, None)
    assert U.rel_rows(gy, ry, 1e-300).max() <= 1e-8
    assert U.rel_rows(gt, rt, 1e-300).max() <= 1e-8
    # one gradient at a time
    th, lo = U.dev(w.theta, torch.float64), U.dev(lam_out, torch.float64)
    gt1 = torch.empty((w.N, w.m), dtype=torch.float64, device="cuda")
    G.gs_replay_grad_outputs(rec, th, tau, lo, None, gt1, None)
    gy1 = torch.empty((w.N, w.d), dtype=torch.float64, device="cuda")
    G.gs_replay_grad_outputs(rec, th, tau, lo, None, None, gy1)
    torch.cuda.synchronize()
    assert U.rel_rows(gt1.cpu().numpy(), rt, 1e-300).max() <= 1e-8
    assert U.rel_rows(gy1.cpu().numpy(), ry, 1e-300).max() <= 1e-8
    # every time at or after t1: the gradient of the final state against the summed cotangent
    tau2 = np.array([w.t1, w.t1 * 1.25])
    lam2 = rng.normal(size=(w.N, 2, w.d))
    gy2, gt2 = _gpu_grad(w, rec, tau2, lam2, None)
    ry2, rt2 = orc.replay_grad(w.field, w.method, w.theta, w.y0, ex["H"], ex["S"], lam2.sum(1),
                               nthreads=8)
    assert U.rel_rows(gy2, ry2, 1e-300).max() <= 1e-8
    assert U.rel_rows(gt2, rt2, 1e-300).max() <= 1e-8


def test_full_size_outputs_gradient_sampled(orc):
    """The stellar ensemble at its benchmark size (2^20 orbits) with the 8 times the benchmark
    asks for (the last one t1): the outputs and the gradient of a loss on them for sampled orbits
    against the oracle on their own recorded meshes, through the same launches as the benchmark."""
    torch = U.torch()
    w = W.by_name("nfw_mn")
    rec, _ = U.record(w)
    tau = [w.t0 + (w.t1 - w.t0) * (j + 1) / 8.0 for j in range(8)]
    yout = _gpu_outputs(w, rec, tau)
    lam_out = np.random.default_rng(12).normal(size=(w.N, len(tau), w.d))
    gy, gt = _gpu_grad(w, rec, tau, lam_out, None)
    tot = int(rec.info().total_steps)
    T = torch.empty(tot, dtype=torch.float64, device="cuda")
    H = torch.empty(tot, dtype=torch.float64, device="cuda")
    off = torch.empty(w.N + 1, dtype=torch.int64, device="cuda")
    G.gs_record_export(rec, T, H, None, off)
    torch.cuda.synchronize()
    off = off.cpu().numpy()
    rng = np.random.default_rng(13)
    idx = np.unique(np.concatenate([[0, w.N - 1], rng.choice(w.N, size=24, replace=False)]))
    S = (off[idx + 1] - off[idx]).astype(np.int32)
    Ts, Hs = np.zeros((len(idx), S.max())), np.zeros((len(idx), S.max()))
    for r_, k in enumerate(idx):
        Ts[r_, :S[r_]] = T[off[k]:off[k + 1]].cpu().numpy()
        Hs[r_, :S[r_]] = H[off[k]:off[k + 1]].cpu().numpy()
    sub = W.subset(w, idx)
    ro = orc.replay_outputs(sub.field, sub.method, sub.theta, sub.y0, Ts, Hs, S, w.t1,
                            np.array(tau), nthreads=8)
    err = U.rel_rows(yout[idx].reshape(len(idx), -1), ro.reshape(len(idx), -1), w.atol)
    assert err.max() <= 1e-9, err.max()
    ry, rt = orc.replay_outputs_grad(sub.field, sub.method, sub.theta, sub.y0, Ts, Hs, S, w.t1,
                                     np.array(tau), lam_out[idx], nthreads=8)
    assert U.rel_rows(gy[idx], ry, 1e-300).max() <= 1e-8
    assert U.rel_rows(gt[idx], rt, 1e-300).max() <= 1e-8
