"""Accuracy of the kernels' own fp64 arithmetic helpers: the step controller's factor
(gs::ctrl_factor), the refined reciprocal and reciprocal square root of the stellar field
(gs::rcp_nr, gs::rsqrt_nr) and its table-driven logarithm (gs::log_tab).

The I-controller ("gradsolve: fast exact gradients for ODE ensembles on GPUs", §2.1: a controller
proposes the next step from the error estimate) multiplies h by clamp(0.9 err^(-1/q), 0.2, 10).
The kernels take err^(-1/q) by two Newton steps on err y^q = 1 from a float estimate, after
clamping err to [1e-10, 1e10].  Bound: the float estimate is good to ~1e-7; each step squares the
relative error times (q + 1)/2, so the second leaves ~1e-26, and what remains is the rounding of
the last step and of the product with 0.9 -- within 2 ulps, checked against a long-double
reference with CUDA's pow beside it.  The clamp: below (0.09)^q the factor must be at least 10
and above 4.5^q at most 0.2, so that the controller's clamped factor is unchanged by it.
The reciprocal and reciprocal square root start from the hardware approximations (relative error
near 2^-22) and take one third-order correction (the residual's series to second order), whose
dropped terms are below 2^-63: what remains is the rounding of the few operations, within 1.5
ulps (checked over 2^-1000 .. 2^1000 against long double, CUDA's correctly rounded division and
its rsqrt beside).
The logarithm of the stellar field (gs::log_tab, Tang's table-driven method) is within half an
ulp plus its few roundings: the bar is 0.6 ulp (CUDA's log, beside it, within 1), with +inf,
+0, a negative argument, NaN and a subnormal mapped to +inf, -inf and NaN.
The LU of a patterned iteration matrix (HIRES's Jacobian pattern: only the entries the fill-in
reaches, no row exchange) reports a wanted exchange exactly when the dense LU makes one, gives
the dense solutions of W x = b and W^T x = b bit for bit otherwise, and a step run through
with_field_lu (patterned, else dense) gives the dense solution in every case: 20,000 random
matrices of that pattern, half of them made to need row exchanges; residuals at rounding level.
"""
import json
import os
import shutil
import subprocess

import pytest

pytestmark = pytest.mark.gpu
HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(os.path.dirname(HERE), "differentiable_adaptive_ode_b200", "csrc")


def test_kernel_math_helpers_within_bounds(tmp_path):
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    exe = str(tmp_path / "kernel_math_check")
    subprocess.run([nvcc, "-std=c++20", "-O3", "-gencode", "arch=compute_100a,code=sm_100a",
                    "-I", CSRC, "-o", exe, os.path.join(HERE, "kernel_math_check.cu")],
                   check=True, timeout=900)
    r = subprocess.run([exe], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    res = json.loads(r.stdout.strip().splitlines()[-1])
    assert res["n"] > 100000
    for q in ("q3", "q5", "q7"):
        assert res[q]["clamp_ok"] == 1, res
        assert res[q]["ulp"] <= 2.0, res
        # the comparison column: CUDA's pow takes the exponent -1/q rounded to a double, which
        # moves x^(-1/q) by |ln x| 2^-54 relative (up to ~1.6 ulp at the ends of [1e-14, 1e14])
        assert res[q]["pow_ulp"] <= 4.0, res
    assert res["n_recip"] > 100000
    for f in ("rcp", "rsqrt"):
        assert res[f]["ulp"] <= 1.5, res
        assert res[f]["cuda_ulp"] <= 1.5, res
    assert res["n_log"] > 500000
    assert res["log"]["ulp"] <= 0.6, res
    assert res["log"]["cuda_ulp"] <= 1.0, res
    assert res["log"]["special_ok"] == 1, res
    # the patterned LU asks for the dense one exactly when pivoting exchanges rows, equals it
    # otherwise, and a step through with_field_lu gives the dense solution in every case
    assert res["lu"]["n"] == 20000, res
    assert res["lu"]["fallback"] >= 2000 and res["lu"]["n"] - res["lu"]["fallback"] >= 2000, res
    assert res["lu"]["flag_mismatch"] == 0, res
    assert res["lu"]["mismatch"] == 0, res
    # backward error of partial pivoting: n 2^(n-1) u = 8 * 128 * 2^-53 ~ 1.1e-13 for n = 8 (the
    # growth bound), with the residual's own rounding: a decade of room
    assert res["lu"]["resid"] <= 1e-12, res
