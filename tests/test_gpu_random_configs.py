"""GPU parity on randomly drawn configurations (seeded): field, method, tolerances, interval and
ensemble size vary together, and every draw must meet the fp64 bars against the oracle — counts
identical on at least 99.9 % of trajectories, replay gradients on the GPU's
own mesh 1e-8 ("gradsolve: fast exact gradients for ODE ensembles on GPUs" §3: the derivative of
the recorded fixed-mesh chain), the final state against the oracle's replay of the GPU's mesh
1e-10, and against the oracle's own adaptive solve 1e-9 or ten times the oracle's spread under a
one-ulp change of y0, whichever is wider."""
import numpy as np
import pytest

import gpu_util as U
from differentiable_adaptive_ode_b200 import gradsolve as G
from differentiable_adaptive_ode_b200 import workloads as W

pytestmark = pytest.mark.gpu

# (workload, methods it takes, tolerance range, interval scale range)
SPACE = [("lotka_volterra", ("tsit5", "vern7"), (1e-9, 1e-5), (0.3, 1.5)),
         ("lorenz63", ("tsit5", "vern7"), (1e-10, 1e-6), (0.3, 2.0)),
         ("nfw_mn", ("tsit5", "vern7"), (1e-10, 1e-6), (0.2, 1.0)),
         ("log_halo", ("tsit5", "vern7"), (1e-9, 1e-6), (0.1, 0.6)),
         ("robertson", ("ros34pw2", "rosenbrock23"), (1e-7, 1e-4), (1e-3, 1.0))]


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    G.lib()


@pytest.mark.parametrize("draw", range(10))
def test_random_configuration(orc, draw):
    rng = np.random.default_rng(1000 + draw)
    name, methods, (tlo, thi), (slo, shi) = SPACE[draw % len(SPACE)]
    N = int(rng.integers(50, 400))
    w = W.by_name(name, N=N, seed=int(rng.integers(0, 1 << 20)))
    w.method = methods[(draw // len(SPACE)) % len(methods)]   # every field with each method
    w.rtol = float(np.exp(rng.uniform(np.log(tlo), np.log(thi))))
    w.atol = w.rtol * float(np.exp(rng.uniform(np.log(1e-3), 0.0)))
    w.t1 = w.t0 + (w.t1 - w.t0) * float(rng.uniform(slo, shi))
    rec, out = U.record(w)
    ex = U.export_padded(w, rec)
    ref = orc.solve(w.field, w.method, w.theta, w.y0, w.t0, w.t1, w.rtol, w.atol,
                    theta_shared=w.theta_shared, nthreads=8)
    assert np.all(out["status"] == 0) and np.all(ref["status"] == 0)
    same = ex["S"] == ref["S"]
    assert same.mean() >= 0.999, (name, w.method, same.mean())
    # on the GPU's own mesh the oracle's replay reproduces the GPU's final state to rounding
    yrep = orc.replay(w.field, w.method, w.theta, w.y0, ex["H"], ex["S"],
                      theta_shared=w.theta_shared, nthreads=8)
    assert U.rel_rows(out["y1"], yrep, w.atol).max() <= 1e-10
    # adaptive against adaptive: 1e-9, or ten times the oracle's own spread under a one-ulp change
    # of y0 where that is wider (the Verner controller at loose tolerances moves step sizes by up
    # to 1e-3 on the same count, measured; the final state moves with them)
    spread_ref = orc.solve(w.field, w.method, w.theta, w.y0 * (1 + np.finfo(float).eps), w.t0,
                           w.t1, w.rtol, w.atol, theta_shared=w.theta_shared, nthreads=8)
    both = same & (spread_ref["S"] == ref["S"])
    spread = U.rel_rows(spread_ref["y1"][both], ref["y1"][both], w.atol).max()
    err = U.rel_rows(out["y1"][same], ref["y1"][same], w.atol).max()
    assert err <= max(1e-9, 10 * spread), (err, spread)
    lam = rng.normal(size=(w.N, w.d))
    gy, gt = U.replay_grad(w, rec, lam)
    ry, rt = orc.replay_grad(w.field, w.method, w.theta, w.y0, ex["H"], ex["S"], lam,
                             theta_shared=w.theta_shared, nthreads=8)
    if w.theta_shared:
        rt, gt = rt.sum(0, keepdims=True), gt[None, :]
    assert U.rel_rows(gy, ry, 1e-300).max() <= 1e-8
    assert U.rel_rows(gt, rt, 1e-300).max() <= 1e-8
