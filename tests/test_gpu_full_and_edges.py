"""GPU parity at the benchmark sizes (sampled trajectories the oracle computes one by one) and the
edge cases: empty and single-trajectory ensembles, a zero-length interval, non-finite parameters,
the attempt cap, record reuse, trajectories parked by a full pool and resumed, and zero-length
padding steps in an
imported record ([GS] = "gradsolve: fast exact gradients for ODE ensembles on GPUs", §3: a step of
size zero leaves the state and its derivative unchanged)."""
import numpy as np
import pytest

import gpu_util as U
from test_gpu_parity import _check_states
from differentiable_adaptive_ode_b200 import gradsolve as G
from differentiable_adaptive_ode_b200 import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    G.lib()


def _sample(N, n=24, seed=0):
    rng = np.random.default_rng(seed)
    return np.unique(np.concatenate([[0, N - 1], rng.choice(N, size=n, replace=False)]))


def _target(orc, w):
    """Loss targets: drawn (Lorenz, stellar) or solved at nominal parameters by the oracle."""
    if w.target is not None:
        return w.target
    if w.target_kind == "nominal_solve":
        r = orc.solve(w.field, w.method, w.nominal_theta[None, :], w.y0[:1], w.t0, w.t1, w.rtol,
                      w.atol)
        return np.repeat(r["y1"], w.N, axis=0)
    r = orc.solve(w.field, w.method, w.nominal_theta, w.y0, w.t0, w.t1, 1e-10, 1e-12,
                  theta_shared=True, nthreads=8)
    return r["y1"]


@pytest.mark.parametrize("name", ["lotka_volterra", "lorenz63", "robertson", "nfw_mn"])
def test_full_size_sampled_parity(orc, name):
    w = W.by_name(name)
    rec, out = U.record(w)
    info = rec.info()
    idx = _sample(w.N)
    sub = W.subset(w, idx)
    ref = orc.solve(sub.field, sub.method, sub.theta, sub.y0, sub.t0, sub.t1, sub.rtol, sub.atol,
                    nthreads=8)
    assert np.all(out["status"] == 0)
    # counts and final states of the sampled trajectories
    import torch
    off = torch.empty(w.N + 1, dtype=torch.int64, device="cuda")
    tot = int(info.total_steps)
    H = torch.empty(tot, dtype=torch.float64, device="cuda")
    G.gs_record_export(rec, None, H, None, off)
    torch.cuda.synchronize()
    off = off.cpu().numpy()
    S = np.diff(off)
    assert np.array_equal(S[idx], ref["S"])
    rel = U.rel_rows(out["y1"][idx], ref["y1"], w.atol)
    assert rel.max() <= 1e-9, rel.max()
    # gradient of the loss on the GPU mesh for the sampled trajectories
    tgt = _target(orc, w)
    lam = W.loss_cotangent(w, out["y1"], tgt)
    gy, gt = U.replay_grad(w, rec, lam)
    Hn = H.cpu().numpy()
    Hs = np.zeros((len(idx), S[idx].max()))
    for r_, k in enumerate(idx):
        Hs[r_, :S[k]] = Hn[off[k]:off[k + 1]]
    ry, rt = orc.replay_grad(sub.field, sub.method, sub.theta, sub.y0, Hs, S[idx], lam[idx],
                             nthreads=8)
    assert U.rel_rows(gy[idx], ry, 1e-300).max() <= 1e-8
    assert U.rel_rows(gt[idx], rt, 1e-300).max() <= 1e-8


def test_full_size_f32_stellar_sampled_parity(orc):
    # the fp32 stellar ensemble at its benchmark size (2^20 orbits, rtol 1e-5, atol 1e-6): a sample
    # of 256 orbits against the oracle in fp32 (counts and final states, held to the oracle's own
    # one-ulp spread), then on the GPU's fp32 mesh the fixed-mesh states (oracle fp32 replay) and
    # the gradient (the exact fp64 derivative of the replay over that mesh)
    import torch
    w = W.by_name("nfw_mn_f32")
    rec, out = U.record(w)
    assert np.all(out["status"] == 0)
    idx = _sample(w.N, n=254, seed=3)
    sub = W.subset(w, idx)
    info = rec.info()
    off = torch.empty(w.N + 1, dtype=torch.int64, device="cuda")
    H = torch.empty(int(info.total_steps), dtype=torch.float32, device="cuda")
    G.gs_record_export(rec, None, H, None, off)
    torch.cuda.synchronize()
    off = off.cpu().numpy()
    S = np.diff(off)
    Hn = H.cpu().numpy()
    Hs = np.zeros((len(idx), S[idx].max()), np.float32)
    for r_, k in enumerate(idx):
        Hs[r_, :S[k]] = Hn[off[k]:off[k + 1]]
    ref = orc.solve(sub.field, sub.method, sub.theta, sub.y0, sub.t0, sub.t1, sub.rtol, sub.atol,
                    dtype=np.float32, nthreads=8)
    _check_states(sub, dict(S=S[idx], y1=out["y1"][idx]), ref, orc)
    # fixed mesh: the oracle's fp32 replay of the GPU mesh (spec bar 1e-4 per trajectory)
    yrep = orc.replay(sub.field, sub.method, sub.theta, sub.y0, Hs, S[idx], dtype=np.float32,
                      nthreads=8)
    err = U.rel_rows(out["y1"][idx], yrep, sub.atol)
    print("fp32 stellar 2^20, fixed-mesh states: p50 %.3g p99 %.3g max %.3g"
          % (np.median(err), np.quantile(err, 0.99), err.max()))
    assert np.quantile(err, 0.99) <= 1e-4 and err.max() <= 1e-3, err.max()
    # gradient of the benchmark loss on the GPU mesh (spec bar 1e-3 per trajectory)
    lam = W.loss_cotangent(w, out["y1"], _target(orc, w))
    gy, gt = U.replay_grad(w, rec, lam)
    th64 = sub.theta.astype(np.float32).astype(np.float64)
    y064 = sub.y0.astype(np.float32).astype(np.float64)
    ry, rt = orc.replay_grad(sub.field, sub.method, th64, y064, Hs.astype(np.float64), S[idx],
                             lam[idx].astype(np.float32).astype(np.float64), nthreads=8)
    # the oracle's own fp32 reverse sweep over the same mesh: how far fp32 rounding alone carries
    # the gradient from the exact one on these orbits (amplified along the longer ones)
    oy, ot = orc.replay_grad(sub.field, sub.method, sub.theta, sub.y0, Hs, S[idx],
                             lam[idx].astype(np.float32), dtype=np.float32, nthreads=8)
    for name, got, own, want in (("dL/dy0", gy[idx], oy, ry), ("dL/dtheta", gt[idx], ot, rt)):
        rel = U.rel_rows(got, want, 1e-300)
        rel_o = U.rel_rows(own, want, 1e-300)
        print("fp32 stellar 2^20, %s against the exact derivative: GPU p50 %.3g p99 %.3g max %.3g;"
              " oracle fp32 p50 %.3g p99 %.3g max %.3g; north-star 1e-3: %.1f%% within"
              % (name, np.median(rel), np.quantile(rel, 0.99), rel.max(), np.median(rel_o),
                 np.quantile(rel_o, 0.99), rel_o.max(), 100 * np.mean(rel <= 1e-3)))
        assert np.median(rel) <= 1e-3
        assert np.quantile(rel, 0.99) <= max(1e-3, 3 * np.quantile(rel_o, 0.99))
        assert rel.max() <= max(1e-2, 3 * rel_o.max())


def test_full_size_mlp_sampled_shared_gradient(orc):
    # the ensemble weight gradient is linear in dL/dy1: zero the cotangent outside a sample and
    # the GPU returns the sample's weight gradient, which the oracle computes directly
    import torch
    w = W.mlp()
    rec, out = U.record(w)
    idx = _sample(w.N, n=126)
    sub = W.subset(w, idx)
    ref = orc.solve("mlp", "tsit5", w.theta, sub.y0, 0.0, 1.0, w.rtol, w.atol, dtype=np.float32,
                    theta_shared=True, nthreads=8)
    assert np.all(out["status"] == 0)
    info = rec.info()
    off = torch.empty(w.N + 1, dtype=torch.int64, device="cuda")
    H = torch.empty(int(info.total_steps), dtype=torch.float32, device="cuda")
    G.gs_record_export(rec, None, H, None, off)
    torch.cuda.synchronize()
    off = off.cpu().numpy()
    S = np.diff(off)
    # fp32: accept decisions near err = 1 sit on the rounding floor; counts and states are held to
    # the oracle's own spread under a one-ulp change of y0, measured on the same sample
    _check_states(sub, dict(S=S[idx], y1=out["y1"][idx]), ref, orc)
    tgt = _target(orc, w).astype(np.float32)
    lam = np.zeros((w.N, 4))
    lam[idx] = W.loss_cotangent(w, out["y1"], tgt)[idx]
    gy, gt = U.replay_grad(w, rec, lam)
    Hn = H.cpu().numpy().astype(np.float64)
    Hs = np.zeros((len(idx), S[idx].max()))
    for r_, k in enumerate(idx):
        Hs[r_, :S[k]] = Hn[off[k]:off[k + 1]]
    ry, rt = orc.replay_grad("mlp", "tsit5", w.theta, sub.y0, Hs, S[idx], lam[idx],
                             theta_shared=True, nthreads=8)
    want = rt.sum(0)
    assert np.linalg.norm(gt - want) <= 1e-3 * np.linalg.norm(want)
    others = np.setdiff1d(np.arange(w.N), idx)
    assert np.all(gy[others] == 0)


def test_empty_and_single_and_zero_interval():
    import torch
    w = W.lorenz63(N=1)
    rec, out = U.record(w)
    assert rec.info().N == 1 and out["status"][0] == 0
    # N = 0: nothing to do, success
    sys_ = U.gsys(w)
    z = torch.empty((0, 3), dtype=torch.float64, device="cuda")
    G.gs_solve_forward(sys_, 0, z, z, 0.0, 1.0, 1e-6, 1e-9, z)
    # t1 == t0: zero steps, y1 = y0, gradient = identity in y0 and zero in theta
    w0 = W.lorenz63(N=5)
    w0.t1 = 0.0
    rec0, out0 = U.record(w0)
    assert rec0.info().total_steps == 0
    assert np.array_equal(out0["y1"], w0.y0)
    lam = np.random.default_rng(0).normal(size=(5, 3))
    gy, gt = U.replay_grad(w0, rec0, lam)
    assert np.array_equal(gy, lam) and np.all(gt == 0)
    # ... and with no recorded step every output is y0 and the outputs' cotangents reach y0
    # unchanged (summed with dL/dy1), theta not at all
    tau = [0.0, 0.5]
    th, y0 = U.dev(w0.theta, torch.float64), U.dev(w0.y0, torch.float64)
    yo = torch.empty((5, 2, 3), dtype=torch.float64, device="cuda")
    G.gs_replay_outputs(rec0, th, y0, tau, yo)
    lo = np.random.default_rng(1).normal(size=(5, 2, 3))
    gy2 = torch.empty((5, 3), dtype=torch.float64, device="cuda")
    gt2 = torch.empty((5, 3), dtype=torch.float64, device="cuda")
    G.gs_replay_grad_outputs(rec0, th, tau, U.dev(lo, torch.float64), U.dev(lam, torch.float64),
                             gt2, gy2)
    torch.cuda.synchronize()
    assert np.array_equal(yo.cpu().numpy(), np.repeat(w0.y0[:, None, :], 2, axis=1))
    assert np.array_equal(gy2.cpu().numpy(), lam + lo[:, 0] + lo[:, 1])
    assert np.all(gt2.cpu().numpy() == 0)


def test_status_codes_and_failed_record():
    w = W.lorenz63(N=8)
    w.theta = w.theta.copy()
    w.theta[3, 0] = np.nan
    fw = U.forward(w)
    assert fw["status"][3] == 3 and np.all(np.delete(fw["status"], 3) == 0)
    with pytest.raises(G.GradsolveError) as e:
        U.record(w)
    assert e.value.code == G.GS_ERR_TRAJ_FAILED
    rec, out = U.record(w, allow_failed=True)
    assert out["status"][3] == 3
    w2 = W.lorenz63(N=8)
    fw2 = U.forward(w2, max_attempts=5)
    assert np.all(fw2["status"] == 1) and np.all(fw2["S"] + fw2["rejected"] == 5)


def test_record_reuse_and_overflow_rerun(orc):
    w = W.nfw_mn(N=700)
    # a pool far too small: the parked trajectories resume in later passes; results unchanged
    rec, out = U.record(w, capacity=50)
    ex = U.export_padded(w, rec)
    ref = orc.solve(w.field, w.method, w.theta, w.y0, w.t0, w.t1, w.rtol, w.atol, nthreads=8)
    assert np.array_equal(ex["S"], ref["S"])
    # reuse the record for another ensemble of a different size
    w2 = W.lorenz63(N=900)
    rec2, out2 = U.record(w2, rec=rec)
    ex2 = U.export_padded(w2, rec2)
    ref2 = orc.solve(w2.field, w2.method, w2.theta, w2.y0, w2.t0, w2.t1, w2.rtol, w2.atol,
                     nthreads=8)
    assert np.array_equal(ex2["S"], ref2["S"])
    assert U.rel_rows(out2["y1"], ref2["y1"], w2.atol).max() <= 1e-9


@pytest.mark.parametrize("name,N,capacity", [("nfw_mn", 700, 50),       # direct writes
                                             ("lorenz63", 900, 8),      # staged writes
                                             ("robertson", 300, 30),    # a Rosenbrock method
                                             ("lorenz63_vern7", 500, 20),
                                             ("mlp", 300, 16)])         # one warp per trajectory
def test_record_resumes_parked_trajectories(name, N, capacity):
    # A pool far too small: the trajectories that find it full are parked before their next
    # attempt and resumed by later passes once the pool has grown.  The record, the final states
    # and the gradient must equal those of a record made with room to spare, bit for bit.
    w = W.by_name(name, N=N)
    rec_a, out_a = U.record(w, capacity=capacity)
    rec_b, out_b = U.record(w, capacity=400 * N)
    ea, eb = U.export_padded(w, rec_a), U.export_padded(w, rec_b)
    assert np.all(out_a["status"] == 0)
    for key in ("S", "T", "H", "Y"):
        assert np.array_equal(ea[key], eb[key]), key
    assert np.array_equal(out_a["y1"], out_b["y1"])
    assert ea["info"].total_steps == eb["info"].total_steps
    assert ea["info"].max_steps == eb["info"].max_steps
    lam = np.random.default_rng(3).normal(size=(w.N, w.d)).astype(w.dtype)
    ga, gb = U.replay_grad(w, rec_a, lam), U.replay_grad(w, rec_b, lam)
    assert np.array_equal(ga[0], gb[0])
    if not w.theta_shared:   # a shared theta's sum is grouped by the visiting order
        assert np.array_equal(ga[1], gb[1])


@pytest.mark.parametrize("name,N", [("nfw_mn", 6000), ("lorenz63", 8192), ("robertson", 4500),
                                    ("nfw_mn_f32", 5000), ("hires", 4096)])
def test_first_record_in_slices_equals_ordered_record(name, N):
    # A first record of an ensemble (no order known) runs a slice of every trajectory, then
    # resumes them by decreasing estimate of their remaining steps, in a pool sized from that
    # estimate.  Scheduling only: it must equal, bit for bit, a record started from a caller's
    # order in one pass.
    import torch
    w = W.by_name(name, N=N)
    rec_a, out_a = U.record(w)
    dt = U.tdtype(w)
    y1 = torch.empty((w.N, w.d), dtype=dt, device="cuda")
    order = torch.arange(w.N, dtype=torch.int32, device="cuda")
    rec_b = G.gs_solve_record(U.gsys(w), w.N, U.dev(w.theta, dt), U.dev(w.y0, dt), w.t0, w.t1,
                              w.rtol, w.atol, y1,
                              opts=G.options(record_capacity_steps=400 * w.N, start_order=order))
    torch.cuda.synchronize()
    ea, eb = U.export_padded(w, rec_a), U.export_padded(w, rec_b)
    for key in ("S", "T", "H", "Y"):
        assert np.array_equal(ea[key], eb[key]), key
    assert np.array_equal(out_a["y1"], y1.cpu().numpy())
    assert ea["info"].max_steps == eb["info"].max_steps
    lam = np.random.default_rng(4).normal(size=(w.N, w.d)).astype(w.dtype)
    ga, gb = U.replay_grad(w, rec_a, lam), U.replay_grad(w, rec_b, lam)
    assert np.array_equal(ga[0], gb[0])
    if not w.theta_shared:
        assert np.array_equal(ga[1], gb[1])


def test_sliced_first_record_with_attempt_cap_and_failures():
    # a first record of 5,000 trajectories (sliced, then resumed) where the attempt cap (40) ends
    # most trajectories after they were parked and resumed, and a few fail at start-up (non-finite
    # theta): statuses, counts, final states and the record equal the plain forward solve's and
    # those of a record started from a caller's order (no slice)
    import torch
    w = W.nfw_mn(N=5000)
    w.theta = w.theta.copy()
    w.theta[[7, 4321], 1] = np.nan
    fw = U.forward(w, max_attempts=40)
    rec_a, out_a = U.record(w, allow_failed=True, max_attempts=40)
    ea = U.export_padded(w, rec_a)
    assert np.array_equal(out_a["status"], fw["status"])
    assert np.sum(fw["status"] == 1) > 1000 and np.all(fw["status"][[7, 4321]] == 3)
    assert np.array_equal(ea["S"], fw["S"])
    assert np.array_equal(out_a["y1"], fw["y1"])
    dt = U.tdtype(w)
    y1 = torch.empty((w.N, w.d), dtype=dt, device="cuda")
    order = torch.arange(w.N, dtype=torch.int32, device="cuda")
    rec_b = G.gs_solve_record(U.gsys(w), w.N, U.dev(w.theta, dt), U.dev(w.y0, dt), w.t0, w.t1,
                              w.rtol, w.atol, y1, opts=G.options(40, 400 * w.N, order),
                              allow_failed=True)
    eb = U.export_padded(w, rec_b)
    for key in ("S", "T", "H", "Y"):
        assert np.array_equal(ea[key], eb[key]), key


def test_record_storage_is_reused_and_trimmed():
    # a destroyed record's device storage goes back to the library's pool and the next record
    # takes it; gs_memory_trim hands the pool's idle storage back to the device; records made
    # before and after either are the same
    import torch
    w = W.lorenz63(N=1 << 16)
    rec, out = U.record(w)
    ref = U.export_padded(w, rec)
    rec.close()
    rec2, out2 = U.record(w)
    ex2 = U.export_padded(w, rec2)
    rec2.close()
    torch.cuda.synchronize()
    free_before = torch.cuda.mem_get_info()[0]
    G.gs_memory_trim(0)
    assert torch.cuda.mem_get_info()[0] > free_before   # the two records' storage was handed back
    rec3, out3 = U.record(w)
    ex3 = U.export_padded(w, rec3)
    for e in (ex2, ex3):
        for key in ("S", "H", "Y"):
            assert np.array_equal(e[key], ref[key]), key
    assert np.array_equal(out2["y1"], out["y1"]) and np.array_equal(out3["y1"], out["y1"])


def test_zero_steps_in_imported_record_change_nothing(orc):
    w = W.lorenz63(N=50)
    ref = orc.solve(w.field, w.method, w.theta, w.y0, w.t0, w.t1, w.rtol, w.atol, keep_record=True)
    lam = np.random.default_rng(1).normal(size=(w.N, 3))
    rec = U.import_record(w, ref["S"], ref["T"], ref["H"], ref["Y"])
    gy, gt = U.replay_grad(w, rec, lam)
    # append three h = 0 steps (state repeated) to every record
    S2 = ref["S"] + 3
    Smax = S2.max()
    T2 = np.zeros((w.N, Smax)); H2 = np.zeros((w.N, Smax)); Y2 = np.zeros((w.N, Smax, 3))
    for k in range(w.N):
        s = ref["S"][k]
        T2[k, :s], H2[k, :s], Y2[k, :s] = ref["T"][k, :s], ref["H"][k, :s], ref["Y"][k, :s]
        T2[k, s:s + 3] = w.t1
        Y2[k, s:s + 3] = ref["y1"][k]
    rec2 = U.import_record(w, S2, T2, H2, Y2)
    gy2, gt2 = U.replay_grad(w, rec2, lam)
    assert np.array_equal(gy, gy2) and np.array_equal(gt, gt2)


def test_rerecord_in_previous_order_is_bitwise_identical():
    # a record made again for the same ensemble visits the trajectories longest-first (the order
    # of the previous solve); the results may not depend on that order
    w = W.nfw_mn(N=3000)
    rec, out = U.record(w)
    ex1 = U.export_padded(w, rec)
    lam = np.random.default_rng(3).normal(size=(w.N, w.d))
    g1 = U.replay_grad(w, rec, lam)
    rec, out2 = U.record(w, rec=rec)
    ex2 = U.export_padded(w, rec)
    g2 = U.replay_grad(w, rec, lam)
    assert np.array_equal(out["y1"], out2["y1"])
    for key in ("S", "T", "H", "Y", "offsets"):
        assert np.array_equal(ex1[key], ex2[key]), key
    assert np.array_equal(g1[0], g2[0]) and np.array_equal(g1[1], g2[1])


def test_record_info_order_is_longest_first_permutation():
    w = W.lorenz63(N=777)
    rec, _ = U.record(w)
    ex = U.export_padded(w, rec)
    assert rec.info().order
    o = rec.order().cpu().numpy()
    assert np.array_equal(np.sort(o), np.arange(w.N))
    assert np.all(np.diff(ex["S"][o]) <= 0)
    # used as the start order of a forward solve: the same results
    f0 = U.forward(w)
    import torch
    y1 = torch.empty((w.N, w.d), dtype=torch.float64, device="cuda")
    G.gs_solve_forward(U.gsys(w), w.N, U.dev(w.theta, torch.float64), U.dev(w.y0, torch.float64),
                       w.t0, w.t1, w.rtol, w.atol, y1,
                       opts=G.options(start_order=rec.order().clone()))
    torch.cuda.synchronize()
    assert np.array_equal(y1.cpu().numpy(), f0["y1"])
