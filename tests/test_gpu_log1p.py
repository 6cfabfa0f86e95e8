"""Accuracy of the fields' device log1p (gs::log1p_q) against a higher-precision host
reference, beside CUDA's own log1p on the same arguments.

fp64: w = fl(1 + x) with its exact rounding error c (TwoSum, Knuth), then
log(1 + x) = log(w) + c / w.  Bound: CUDA's log is within 1 ulp of log(w); the dropped term
(c / w)^2 / 2 is below 2^-107; c / w taken as c * (1 / (1 + x)) with a reciprocal good to 2 ulps
errs by under 2^-104 of |c / w| <= 2^-53 -- far below an ulp of the result wherever the result
is not itself below 2^-53 (and there w == 1, log(w) == 0 and the result is c * q = x to a few
ulps).  Adding the two terms rounds once more: within 2 ulps in all, checked here against 3.
fp32 is log1pf itself.
"""
import json
import os
import shutil
import subprocess

import pytest

pytestmark = pytest.mark.gpu
HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(os.path.dirname(HERE), "differentiable_adaptive_ode_b200", "csrc")


def test_log1p_q_within_3_ulps(tmp_path):
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    exe = str(tmp_path / "log1p_check")
    subprocess.run([nvcc, "-std=c++17", "-O3", "-gencode", "arch=compute_100a,code=sm_100a",
                    "-I", CSRC, "-o", exe, os.path.join(HERE, "log1p_check.cu")],
                   check=True, timeout=600)
    r = subprocess.run([exe], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    res = json.loads(r.stdout.strip().splitlines()[-1])
    assert res["n"] > 50000
    for prec in ("f64", "f32"):
        assert res[prec]["field_ulp"] <= 3.0, res
        assert res[prec]["cuda_ulp"] <= 2.0, res      # the comparison column itself is sane
