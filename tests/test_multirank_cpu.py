"""The multi-rank path on CPU: two gloo ranks each take their shard of a shared-theta ensemble,
compute the shard's parameter cotangent with the oracle, and sum it over ranks; the result must
equal the single-process ensemble gradient.  Also the shard arithmetic and max-over-ranks."""
import os
import socket

import numpy as np
import pytest

from differentiable_adaptive_ode_b200.ensemble import shard_range


def test_shard_range_partitions():
    for N in (0, 1, 7, 1024, 1000003):
        for world in (1, 2, 3, 8):
            spans = [shard_range(N, r, world) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == N
            assert all(a[1] == b[0] for a, b in zip(spans, spans[1:]))
            sizes = [e - b for b, e in spans]
            assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        shard_range(10, 2, 2)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _rank_main(rank, world, port, out_dir):
    import torch
    import torch.distributed as dist
    from differentiable_adaptive_ode_b200 import workloads as W
    from differentiable_adaptive_ode_b200.ensemble import (allreduce_theta_bar, max_over_ranks,
                                                           shard_range)
    from oracle import oracle as orc
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    w = W.lotka_volterra(N=37)
    w.theta_shared = True
    w.theta = w.theta[0].copy()
    b, e = shard_range(w.N, rank, world)
    sub = W.subset(w, np.arange(b, e))
    r = orc.solve(sub.field, sub.method, sub.theta, sub.y0, sub.t0, sub.t1, sub.rtol, sub.atol,
                  keep_record=True, theta_shared=True)
    lam = np.random.default_rng(0).normal(size=(w.N, w.d))[b:e]
    _, gt = orc.replay_grad(sub.field, sub.method, sub.theta, sub.y0, r["H"], r["S"], lam,
                            theta_shared=True)
    t = torch.from_numpy(gt.sum(0))
    allreduce_theta_bar(t)
    slowest = max_over_ranks(float(rank + 1))
    np.save(os.path.join(out_dir, "rank%d.npy" % rank), np.append(t.numpy(), slowest))
    dist.barrier()
    dist.destroy_process_group()


def test_two_gloo_ranks_sum_the_shared_theta_cotangent(orc, tmp_path):
    import torch.multiprocessing as mp
    from differentiable_adaptive_ode_b200 import workloads as W
    port = _free_port()
    mp.spawn(_rank_main, args=(2, port, str(tmp_path)), nprocs=2, join=True)
    got = [np.load(os.path.join(tmp_path, "rank%d.npy" % r)) for r in range(2)]
    assert np.array_equal(got[0], got[1])            # every rank holds the same sum
    assert got[0][-1] == 2.0                          # max over ranks
    w = W.lotka_volterra(N=37)
    w.theta_shared = True
    w.theta = w.theta[0].copy()
    r = orc.solve(w.field, w.method, w.theta, w.y0, w.t0, w.t1, w.rtol, w.atol, keep_record=True,
                  theta_shared=True)
    lam = np.random.default_rng(0).normal(size=(w.N, w.d))
    _, gt = orc.replay_grad(w.field, w.method, w.theta, w.y0, r["H"], r["S"], lam,
                            theta_shared=True)
    want = gt.sum(0)
    assert np.max(np.abs(got[0][:-1] - want)) <= 1e-12 * np.max(np.abs(want))
