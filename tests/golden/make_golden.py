"""Writes tests/golden/oracle_small_cases.json from the CPU oracle alone.

The pages print no worked numerical example for this method, so the stored values here are
regression anchors of the oracle (which is pinned separately against closed forms, order
conditions, invariants and finite differences): small seeded ensembles of every benchmark
field, their accepted/rejected step counts, final states and replay gradients.  Regenerate only
together with a change to the oracle's arithmetic whose commit names the passage (or the reading
of it) that justifies the change.

    python tests/golden/make_golden.py
"""
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

from differentiable_adaptive_ode_b200 import workloads as W  # noqa: E402
from oracle import oracle as orc  # noqa: E402

CASES = [("lotka_volterra", 4), ("lorenz63", 4), ("robertson", 2), ("nfw_mn", 4),
         ("nfw_mn_f32", 4), ("mlp", 2), ("lorenz63_vern7", 3), ("robertson_rb23", 2),
         ("hires", 1), ("log_halo", 3)]
SENS_CASES = [("log_halo", 3), ("lorenz63", 2)]


def compute(name, N):
    w = W.by_name(name, N=N)
    dt = w.dtype
    r = orc.solve(w.field, w.method, w.theta, w.y0, w.t0, w.t1, w.rtol, w.atol, dtype=dt,
                  keep_record=True, theta_shared=w.theta_shared)
    lam = np.random.default_rng(12345).normal(size=(N, w.d))
    gy, gt = orc.replay_grad(w.field, w.method, w.theta, w.y0, r["H"], r["S"], lam, dtype=dt,
                             theta_shared=w.theta_shared)
    if w.theta_shared:
        gt = gt.sum(0, keepdims=True)
    return dict(S=r["S"].tolist(), rejected=r["rejected"].tolist(), y1=r["y1"].tolist(),
                dL_dy0=gy.tolist(), dL_dtheta=gt.tolist())


def compute_sens(name, N):
    w = W.by_name(name, N=N)
    r = orc.solve_sens(w.field, w.theta, w.y0, w.t0, w.t1, w.rtol, w.atol,
                       theta_shared=w.theta_shared)
    return dict(S=r["S"].tolist(), rejected=r["rejected"].tolist(), y1=r["y1"].tolist(),
                sens=r["sens"].tolist())


def main():
    out = {"source": "oracle/ (CPU), seeds of differentiable_adaptive_ode_b200.workloads",
           "lam": "numpy default_rng(12345).normal(size=(N, d))", "cases": {}}
    for name, N in CASES:
        out["cases"][name] = dict(N=N, **compute(name, N))
    out["sens_cases"] = {}
    for name, N in SENS_CASES:
        out["sens_cases"][name] = dict(N=N, **compute_sens(name, N))
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "oracle_small_cases.json")
    with open(path, "w") as f:
        json.dump(out, f, indent=1)
    print(path)


if __name__ == "__main__":
    main()
