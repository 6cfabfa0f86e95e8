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
    m = W.mlp(N=4)
    recm, _ = U.record(m)
    with pytest.raises(G.GradsolveError) as e:
        G.gs_replay_outputs(recm, U.dev(m.theta, torch.float32), U.dev(m.y0, torch.float32),
                            [0.5], torch.empty((4, 1, 4), dtype=torch.float32, device="cuda"))
    assert e.value.code == G.GS_ERR_UNSUPPORTED
