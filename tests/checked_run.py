"""Runs every record-reading path of the library once on small ensembles and prints, as JSON,
a checksum of each result and the library's count of out-of-range record accesses.  Executed by
tests/test_gpu_zchecked.py in a fresh process, once with the checked build of the library
(GRADSOLVE_B200_CHECKED=1) and once with the normal build."""
import json
import os
import sys

import numpy as np

sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

import gpu_util as U  # noqa: E402
from differentiable_adaptive_ode_b200 import gradsolve as G  # noqa: E402
from differentiable_adaptive_ode_b200 import workloads as W  # noqa: E402


def main():
    import torch
    out = {}
    for name, N in (("nfw_mn", 1500), ("lorenz63_vern7", 700), ("robertson", 300),
                    ("robertson_rb23", 300), ("mlp", 256), ("log_halo", 500)):
        w = W.by_name(name, N=N)
        dt = U.tdtype(w)
        rec, res = U.record(w)
        lam = np.random.default_rng(1).normal(size=(w.N, w.d))
        gy, gt = U.replay_grad(w, rec, lam)
        out[name + ":y1"] = float(np.abs(res["y1"]).sum())
        out[name + ":grad"] = float(np.abs(gy).sum() + np.abs(gt).sum())
        ex = U.export_padded(w, rec)
        out[name + ":export"] = float(np.abs(ex["H"]).sum() + np.abs(ex["Y"]).sum())
        tau = [w.t0 + (w.t1 - w.t0) * f for f in (0.25, 0.5, 0.9)]
        yo = torch.empty((w.N, 3, w.d), dtype=dt, device="cuda")
        G.gs_replay_outputs(rec, U.dev(w.theta, dt), U.dev(w.y0, dt), tau, yo)
        gy2 = torch.empty((w.N, w.d), dtype=dt, device="cuda")
        gt2 = torch.empty((w.m,) if w.theta_shared else (w.N, w.m), dtype=dt, device="cuda")
        G.gs_replay_grad_outputs(rec, U.dev(w.theta, dt), tau,
                                 U.dev(np.ones((w.N, 3, w.d)), dt), None, gt2, gy2)
        torch.cuda.synchronize()
        out[name + ":outputs"] = float(yo.abs().sum().item() + gy2.abs().sum().item() +
                                       gt2.abs().sum().item())
        if name != "mlp":
            # import the exported arrays and differentiate again
            rec2 = U.import_record(w, ex["S"], ex["T"], ex["H"], ex["Y"])
            gy3, _ = U.replay_grad(w, rec2, lam)
            out[name + ":import"] = float(np.abs(gy3).sum())
            # replay at the same parameters, then the allocation-free gradient
            G.gs_replay_forward(rec, U.dev(w.theta, dt), U.dev(w.y0, dt))
            g4 = torch.empty((w.N, w.d), dtype=dt, device="cuda")
            G.gs_replay_grad_noalloc(rec, U.dev(w.theta, dt), U.dev(lam, dt), None, g4)
            torch.cuda.synchronize()
            out[name + ":noalloc"] = float(g4.abs().sum().item())
    try:
        out["violations"] = G.checked_violations()
    except G.GradsolveError:
        out["violations"] = None
    print(json.dumps(out))


if __name__ == "__main__":
    main()
