"""The per-step operation counts that bench.py divides by kernel time are re-derived here.

Per accepted step of the Tsit5 replay adjoint (recompute stages k1..k6 from y_n, reverse sweep):
  stage states Y_2..Y_6: sum_{i=2..6} (2i - 1) = 35 ops per component;
  kb_i = h (b_i lam + G_i): 2 + 5 * 3 = 17;  lam += Yb_i: 6;  G_j += a_ij Yb_i: 30
  => 88 d + 6 c_f + 6 c_v.
Per attempted step of the forward solve (k1 carried):
  stages 35, y_new 13, error 14, scale 2, quotient 1, square-accumulate 2 per component,
  plus mean, sqrt, pow, safety factor, h update (5) => 67 d + 6 c_f + 5.
c_f and c_v are the op counts (add/sub, mul, div, sqrt or rsqrt, log1p; an FMA counts as two) of the
field's f and vector-Jacobian product as written in csrc/gs_fields.cuh, tallied by compiling that
header with a counting scalar (tests/flop_counter.cpp)."""
import json

import numpy as np
import os
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def counts(tmp_path_factory):
    exe = str(tmp_path_factory.mktemp("fc") / "flop_counter")
    subprocess.run(["g++", "-std=c++17", "-O1", "-Wno-unknown-pragmas",
                    "-I" + os.path.join(ROOT, "differentiable_adaptive_ode_b200", "csrc"),
                    "-o", exe, os.path.join(ROOT, "tests", "flop_counter.cpp")], check=True)
    out = subprocess.run([exe], check=True, capture_output=True, text=True).stdout
    return {r["field"]: r for r in map(json.loads, out.splitlines())}


def ops(t):
    return t["add"] + t["mul"] + t["div"] + t["sqrt"] + t["log1p"]


@pytest.mark.parametrize("field", ["nfw_mn", "lorenz63", "lotka_volterra", "log_halo"])
def test_bench_constants_match_counts(counts, field):
    import bench
    c = counts[field]
    D = c["D"]
    adj = 88 * D + 6 * ops(c["f"]) + 6 * ops(c["vjp"])
    fwd = 67 * D + 6 * ops(c["f"]) + 5
    assert bench.FLOPS_ADJOINT_STEP[field] == adj
    assert bench.FLOPS_FORWARD_ATTEMPT[field] == fwd


def test_sens_constant_matches_counts(counts):
    # tangent of the Tsit5 step per column: stage tangents 35 d + result 13 d, plus six stage
    # evaluations of f's forward-mode rules beyond f itself (c_t = dual f - f)
    import bench
    c = counts["log_halo"]
    c_t = ops(c["fdual"]) - ops(c["f"])
    assert bench.FLOPS_SENS_STEP["log_halo"] == c["M"] * (48 * c["D"] + 6 * c_t)


def test_vern7_constants_match_counts(counts, orc):
    import bench
    A, b, bh = orc.vern7_tableau()
    nnz = [int(np.count_nonzero(A[i, :i])) for i in range(1, 10)]
    assert nnz == [1, 2, 2, 3, 4, 5, 6, 7, 6]
    nb, ne = int(np.count_nonzero(b[:9])), int(np.count_nonzero(b - bh))
    # attempt: stage states 2 nnz + 1 each, y_new 2 nb + 1, error 2 ne, scale/quotient/square 5
    per_c_fwd = sum(2 * n + 1 for n in nnz) + (2 * nb + 1) + 2 * ne + 5
    # adjoint: stage states 2..9, stage cotangents (3 with b_i != 0, else 1; the last stage 2),
    # G accumulation 2 per nonzero a_ij of rows 2..9, the nine lam increments and the final add
    kb = sum(3 if b[i] != 0 else 1 for i in range(8)) + 2
    per_c_adj = sum(2 * n + 1 for n in nnz[:8]) + kb + 2 * sum(nnz[:8]) + 9 + 1
    assert (per_c_fwd, per_c_adj) == (117, 160)
    for field in ("lorenz63", "nfw_mn"):
        c = counts[field]
        D = c["D"]
        assert bench.FLOPS_VERN7_ATTEMPT[field] == 117 * D + 10 * ops(c["f"]) + 5
        assert bench.FLOPS_VERN7_ADJOINT[field] == 160 * D + 8 * ops(c["f"]) + 9 * ops(c["vjp"])


def test_stiff_counts_and_formulas(counts):
    import bench
    for field in ("robertson", "hires"):
        c = counts[field]
        assert bench.STIFF_COUNTS[field] == (c["D"], ops(c["f"]), ops(c["vjp"]), c["jac"],
                                             c["jac_vjp"])
    # the 3 x 3 elimination: column 0: 1 reciprocal + 2 multipliers + 2 x 2 x 2; column 1:
    # 1 + 1 + 2; column 2: 1
    assert bench.lu_ops(3) == 16
    assert bench.stiff_flops("ros34pw2", "robertson") == (375, 895)
    assert bench.stiff_flops("rosenbrock23", "robertson") == (171, 250)
    # Rosenbrock23 on HIRES's declared pattern (25 entries, 2 of fill-in): 42 operations for the
    # elimination (dense 316), 46 per solve pair (dense 120); with the dense figures in their
    # place the same formula gives the dense count back
    assert bench.pattern_ops("hires", 8) == (25, 46, 42)
    assert bench.pattern_ops("robertson", 3) == (9, 15, bench.lu_ops(3))
    assert bench.stiff_flops("rosenbrock23", "hires") == (475, 722)
    saved = bench.JAC_PATTERN.pop("hires")
    try:
        assert bench.stiff_flops("rosenbrock23", "hires") == (1010, 1448)
    finally:
        bench.JAC_PATTERN["hires"] = saved


def test_mlp_hand_count():
    import bench
    H, D = 32, 4
    c_f = 2 * (H * D + H * H + D * H) + (H + H + D) + 2 * H      # products, biases, tanh
    c_v = 2 * (D * H + H * H + H * D) + 2 * (H * H + H * D + D * H) + 2 * 2 * H + (H + H + D)
    assert c_f == 2692 and c_v == 5316
    assert bench.FLOPS_ADJOINT_STEP["mlp"] == 88 * D + 6 * c_f + 6 * c_v
    assert bench.FLOPS_FORWARD_ATTEMPT["mlp"] == 67 * D + 6 * c_f + 5


def test_field_counts_are_plausible(counts):
    # Lorenz f: sigma (y - x), x (rho - z) - y, x y - beta z -> 4 add/sub + 4 mul
    assert ops(counts["lorenz63"]["f"]) == 8
    assert counts["nfw_mn"]["f"]["log1p"] == 1 and counts["nfw_mn"]["f"]["sqrt"] == 3
    assert counts["nfw_mn"]["f"]["div"] == 1


@pytest.mark.parametrize("field", ["nfw_mn", "lorenz63", "lotka_volterra", "log_halo",
                                   "robertson", "hires"])
def test_vjp_counts_within_the_plain_reverse_sweep(counts, orc, field):
    # The vector-Jacobian products the throughput figures charge (c_v, counted from the kernels'
    # own source) must not exceed what a plain reverse-mode sweep over the oracle's f costs: the
    # oracle tapes its own f and tallies the adjoint rules of every recorded operation.  A
    # hand-written pullback doing redundant work would exceed that bound and inflate the reported
    # fraction of peak; this pins c_v from outside the kernel source.
    D, M = orc.dims(field)
    rng = np.random.default_rng(4)
    rev = orc.count_ops(field, "vjp_reverse", rng.uniform(0.5, 1.5, M), rng.uniform(0.5, 1.5, D))
    kernel = ops(counts[field]["vjp"])
    print("%s: c_v kernel %d, plain reverse sweep %d" % (field, kernel, sum(rev.values())))
    assert kernel <= sum(rev.values())


def test_mlp_vjp_count_within_the_plain_reverse_sweep(orc):
    D, M = orc.dims("mlp")
    rng = np.random.default_rng(5)
    rev = orc.count_ops("mlp", "vjp_reverse", rng.normal(size=M) * 0.2, rng.normal(size=D))
    assert 5316 <= sum(rev.values())   # the hand count of test_mlp_hand_count
