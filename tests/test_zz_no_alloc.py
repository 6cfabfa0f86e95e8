"""gs_replay_grad_noalloc: the replay gradient for callers that cannot allocate device memory.

Some callers may not call cudaMalloc at the moment they need a gradient -- for instance code
running while a stream is captured into a CUDA graph, code whose allocator forbids driver
allocations, or a loop in which an allocation would synchronise the device.  The no-alloc entry
point keeps its scratch in a fixed array inside the library instead.  These tests call it through
the C ABI and check that it returns what gs_replay_grad returns, on two calls in a row (the array
keeps the previous call's contents, so the second call shows that what must start at zero is
cleared), that the second call changes the device's free memory by nothing, and that a problem
too large for the array is refused with a clear error.  The no-alloc calls come first on each
record, so they cannot lean on anything gs_replay_grad allocated for it.

This file is collected last on purpose: it passes alone in a fresh process and after the others.
"""
import numpy as np
import pytest

import gpu_util as U
from differentiable_adaptive_ode_b200 import gradsolve as G
from differentiable_adaptive_ode_b200 import workloads as W

pytestmark = pytest.mark.gpu

GRAD_TOL = 1e-8   # the tests' fp64 gradient bar


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    G.lib()


def _both(w, rec, lam, theta=None):
    """Two no-alloc calls in a row on a record no other gradient call has touched, then
    gs_replay_grad for reference.  The second no-alloc call must leave the device's free memory
    exactly as it found it (the first may still load the variant's kernels)."""
    torch = U.torch()
    dt = U.tdtype(w)
    th = U.dev(w.theta if theta is None else theta, dt)
    lam_t = U.dev(lam, dt)
    shape_t = (w.m,) if w.theta_shared else (w.N, w.m)
    bufs = [(torch.full(shape_t, np.nan, dtype=dt, device="cuda"),
             torch.full((w.N, w.d), np.nan, dtype=dt, device="cuda")) for _ in range(2)]
    torch.cuda.synchronize()
    outs = []
    for i, (gt, gy) in enumerate(bufs):     # the two calls share the fixed scratch
        free_before = torch.cuda.mem_get_info()[0]
        G.gs_replay_grad_noalloc(rec, th, lam_t, gt, gy)
        torch.cuda.synchronize()
        if i == 1:
            assert torch.cuda.mem_get_info()[0] == free_before
        outs.append((gt.cpu().numpy(), gy.cpu().numpy()))
    ref_t = torch.empty(shape_t, dtype=dt, device="cuda")
    ref_y = torch.empty((w.N, w.d), dtype=dt, device="cuda")
    G.gs_replay_grad(rec, th, lam_t, ref_t, ref_y)
    torch.cuda.synchronize()
    return (ref_t.cpu().numpy(), ref_y.cpu().numpy()), outs


def _close(a, b):
    a = np.atleast_2d(a)
    b = np.atleast_2d(b)
    return U.rel_rows(a, b, 1e-300).max() <= GRAD_TOL


def test_no_alloc_matches_replay_grad_shared_theta():
    w = W.nfw_mn(N=2000)
    w.theta_shared = True
    w.theta = w.theta[0].copy()
    rec, _ = U.record(w)
    lam = np.random.default_rng(11).normal(size=(w.N, w.d))
    (rt, ry), outs = _both(w, rec, lam)
    for gt, gy in outs:
        assert np.all(np.isfinite(gt)) and np.all(np.isfinite(gy))
        assert _close(gt, rt) and _close(gy, ry)


def test_no_alloc_matches_replay_grad_per_trajectory_theta():
    w = W.lorenz63(N=500)
    rec, _ = U.record(w)
    lam = np.random.default_rng(12).normal(size=(w.N, w.d))
    (rt, ry), outs = _both(w, rec, lam)
    for gt, gy in outs:
        assert _close(gt, rt) and _close(gy, ry)


def test_no_alloc_at_a_theta_other_than_the_recorded_one():
    # the stored states were made at theta0; both entry points must differentiate the replay at
    # the theta they are given (the no-alloc one replays the states into the record's own slots)
    w = W.nfw_mn(N=700)
    rec, _ = U.record(w)
    lam = np.random.default_rng(13).normal(size=(w.N, w.d))
    (rt, ry), outs = _both(w, rec, lam, theta=w.theta * 1.01)
    for gt, gy in outs:
        assert _close(gt, rt) and _close(gy, ry)


def test_no_alloc_refuses_problems_beyond_its_scratch():
    torch = U.torch()
    w = W.lorenz63(N=400_000)       # shared theta: 400000 x 3 doubles > 8 MiB
    w.theta_shared = True
    w.theta = w.theta[0].copy()
    rec, _ = U.record(w)
    gt = torch.zeros(3, dtype=torch.float64, device="cuda")
    lam = torch.zeros((w.N, 3), dtype=torch.float64, device="cuda")
    th = U.dev(w.theta, torch.float64)
    with pytest.raises(G.GradsolveError) as e:
        G.gs_replay_grad_noalloc(rec, th, lam, gt, None)
    assert e.value.code == G.GS_ERR_CAPACITY
    assert "scratch" in str(e.value)
