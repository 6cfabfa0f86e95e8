"""GPU parity of the forward sensitivities against the oracle ("Differentiable astrophysics at
scale" §2-§3: S = dy/dtheta integrated with the orbit in the same kernel, the step size
controlled on the orbit alone).  The GPU's mesh, y1 and counts must be those of its own forward
solve (same trial, test and controller); S must match the oracle's sensitivity solve."""
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


def _oracle(orc, w, S0=None):
    return orc.solve_sens(w.field, w.theta, w.y0, w.t0, w.t1, w.rtol, w.atol, S0=S0,
                          dtype=w.dtype, theta_shared=w.theta_shared, nthreads=8)


@pytest.mark.parametrize("name,N", [("log_halo", 700), ("lorenz63", 500), ("nfw_mn", 300),
                                    ("lotka_volterra", 400)])
def test_sens_matches_oracle_and_forward_solve(orc, name, N):
    w = U.small(name, N)
    g = U.forward_sens(w)
    f = U.forward(w)
    # control on the orbit alone: the same mesh and state as the plain forward solve, bit for bit
    assert np.array_equal(g["S"], f["S"]) and np.array_equal(g["rejected"], f["rejected"])
    assert np.array_equal(g["y1"], f["y1"]) and np.all(g["status"] == 0)
    r = _oracle(orc, w)
    assert np.array_equal(g["S"], r["S"])
    assert U.rel_rows(g["y1"], r["y1"], w.atol).max() <= 1e-9
    err = U.rel_rows(g["sens"], r["sens"], 1e-300)
    assert err.max() <= 1e-8, err.max()


def test_sens_linear_per_trajectory_and_seeded_start(orc):
    rng = np.random.default_rng(31)
    N = 200
    A = rng.normal(size=(N, 3, 3)) * 0.4 - 0.7 * np.eye(3)[None]
    y0 = rng.normal(size=(N, 3))
    w = W.Workload("linear3", "linear3", "tsit5", np.float64, N, 3, 9, False, A.reshape(N, 9), y0,
                   0.0, 2.0, 1e-8, 1e-10, 0)
    S0 = rng.normal(size=(N, 3, 9)) * 0.2
    g = U.forward_sens(w, S0=S0)
    r = _oracle(orc, w, S0=S0)
    assert np.array_equal(g["S"], r["S"])
    assert U.rel_rows(g["sens"], r["sens"], 1e-300).max() <= 1e-9


def _fp32_sens_error(orc, w, sens32, ex):
    """Relative error of fp32 sensitivities against the exact (fp64) tangent of the replay over
    the fp32 mesh that produced them."""
    th = np.ascontiguousarray(np.broadcast_to(w.theta, (w.N, w.m)) if w.theta_shared else w.theta,
                              dtype=np.float64)
    y0 = w.y0.astype(np.float32).astype(np.float64)
    th = th.astype(np.float32).astype(np.float64)
    ref = np.zeros((w.N, w.d, w.m))
    for j in range(w.m):
        thd = np.zeros((w.N, w.m))
        thd[:, j] = 1.0
        _, ref[:, :, j] = orc.replay_jvp(w.field, w.method, th, y0, thd, np.zeros_like(y0),
                                         ex["H"].astype(np.float64), ex["S"], nthreads=8)
    return U.rel_rows(sens32, ref, 1e-30)


def test_sens_fp32_stellar(orc):
    # fp32 reading (as for the fp32 gradients): the reference is the exact fp64 derivative of the
    # replay over the mesh the fp32 solve took; the GPU's fp32 error against it must be of the
    # size of the oracle's own fp32 error against the same kind of reference
    w = U.small("nfw_mn_f32", 400)
    g = U.forward_sens(w)
    rec, out = U.record(w)
    ex = U.export_padded(w, rec)
    assert np.array_equal(ex["S"], g["S"])          # same mesh as the record kernel's
    e_gpu = _fp32_sens_error(orc, w, g["sens"], ex)
    r = _oracle(orc, w)
    ro = orc.solve(w.field, w.method, w.theta, w.y0, w.t0, w.t1, w.rtol, w.atol, dtype=np.float32,
                   keep_record=True, nthreads=8)
    e_orc = _fp32_sens_error(orc, w, r["sens"], dict(H=ro["H"], S=ro["S"]))
    for q in (0.5, 0.9):
        a, b = np.quantile(e_gpu, q), np.quantile(e_orc, q)
        print("fp32 sensitivities q%.1f: gpu %.3g oracle %.3g" % (q, a, b))
        assert a <= max(3 * b, 1e-3), (q, a, b)


def test_sens_full_size_sampled(orc):
    w = W.log_halo()
    g = U.forward_sens(w)
    assert np.all(g["status"] == 0)
    rng = np.random.default_rng(0)
    idx = np.unique(np.concatenate([[0, w.N - 1], rng.choice(w.N, size=24, replace=False)]))
    sub = W.subset(w, idx)
    r = _oracle(orc, sub)
    assert np.array_equal(g["S"][idx], r["S"])
    assert U.rel_rows(g["y1"][idx], r["y1"], w.atol).max() <= 1e-9
    assert U.rel_rows(g["sens"][idx], r["sens"], 1e-300).max() <= 1e-8


def test_sens_edges_and_argument_checks():
    import torch
    w = U.small("log_halo", 6)
    w.t1 = w.t0
    S0 = np.arange(6 * 6 * 2, dtype=np.float64).reshape(6, 6, 2)
    g = U.forward_sens(w, S0=S0)
    assert np.array_equal(g["y1"], w.y0) and np.array_equal(g["sens"], S0)
    assert np.all(g["S"] == 0)
    sys_ = U.gsys(w)
    z = torch.empty((0, 6), dtype=torch.float64, device="cuda")
    G.gs_solve_forward_sens(sys_, 0, U.dev(w.theta, torch.float64), z, 0.0, 1.0, 1e-6, 1e-6, z,
                            None)
    with pytest.raises(G.GradsolveError) as e:
        G.gs_solve_forward_sens(sys_, 6, U.dev(w.theta, torch.float64),
                                U.dev(w.y0, torch.float64), 0.0, 1.0, 1e-6, 1e-6,
                                torch.empty((6, 6), dtype=torch.float64, device="cuda"), None)
    assert e.value.code == G.GS_ERR_INVALID_ARG
    rob = W.robertson(N=4)
    out = torch.empty((4, 3), dtype=torch.float64, device="cuda")
    with pytest.raises(G.GradsolveError) as e:
        G.gs_solve_forward_sens(U.gsys(rob), 4, U.dev(rob.theta, torch.float64),
                                U.dev(rob.y0, torch.float64), 0.0, 1.0, 1e-6, 1e-6, out,
                                torch.empty((4, 3, 3), dtype=torch.float64, device="cuda"))
    assert e.value.code == G.GS_ERR_UNSUPPORTED


def test_start_order_changes_nothing_but_the_schedule():
    import torch
    w = U.small("log_halo", 2000)
    base = U.forward_sens(w)
    dt = torch.float64
    th, y0 = U.dev(w.theta, dt), U.dev(w.y0, dt)
    for order in (np.arange(w.N)[::-1], np.random.default_rng(4).permutation(w.N)):
        o = torch.as_tensor(order.astype(np.int32), device="cuda")
        y1 = torch.empty((w.N, w.d), dtype=dt, device="cuda")
        S1 = torch.empty((w.N, w.d, w.m), dtype=dt, device="cuda")
        S = torch.empty(w.N, dtype=torch.int32, device="cuda")
        G.gs_solve_forward_sens(U.gsys(w), w.N, th, y0, w.t0, w.t1, w.rtol, w.atol, y1, S1, None,
                                S, opts=G.options(start_order=o))
        y1f = torch.empty_like(y1)
        G.gs_solve_forward(U.gsys(w), w.N, th, y0, w.t0, w.t1, w.rtol, w.atol, y1f,
                           opts=G.options(start_order=o))
        torch.cuda.synchronize()
        assert np.array_equal(y1.cpu().numpy(), base["y1"])
        assert np.array_equal(y1f.cpu().numpy(), base["y1"])
        assert np.array_equal(S1.cpu().numpy(), base["sens"])
        assert np.array_equal(S.cpu().numpy(), base["S"])


def test_sens_non_finite_parameters_and_attempt_cap():
    # per-trajectory theta with a NaN: that trajectory ends at start-up with status 3 and its S is
    # the starting S0 (zero); the others are unaffected.  A cap of 5 attempts gives status 1.
    w = U.small("lorenz63", 16)
    w.theta = w.theta.copy()
    w.theta[5, 1] = np.nan
    g = U.forward_sens(w)
    assert g["status"][5] == 3 and np.all(np.delete(g["status"], 5) == 0)
    assert np.all(g["sens"][5] == 0)
    ok = U.forward_sens(U.small("lorenz63", 16))
    keep = np.delete(np.arange(16), 5)
    assert np.array_equal(g["sens"][keep], ok["sens"][keep])
    capped = U.forward_sens(U.small("lorenz63", 16), max_attempts=5)
    assert np.all(capped["status"] == 1) and np.all(capped["S"] + capped["rejected"] == 5)
