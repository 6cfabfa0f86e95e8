"""The Jacobian sparsity pattern that a field declares to the kernels (jac_nz; the LU of the
iteration matrices I - c J then takes only the entries that elimination can reach) must cover
every entry of the Jacobian that can be nonzero.  Pinned against the oracle's Jacobian: over
random states and parameters, the entries the oracle ever finds nonzero are exactly the declared
pattern -- none missing (which would make the kernels' LU wrong) and none extra."""
import os
import subprocess

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "differentiable_adaptive_ode_b200", "csrc")

PROGRAM = r"""
#include <cstdio>
#include "gs_fields.cuh"
int main() {
  for (int r = 0; r < 8; ++r)
    for (int c = 0; c < 8; ++c) std::printf("%d", gs::FHires::jac_nz(r, c) ? 1 : 0);
  std::printf("\n");
  return 0;
}
"""


@pytest.fixture(scope="module")
def declared(tmp_path_factory):
    d = tmp_path_factory.mktemp("jp")
    src, exe = str(d / "jp.cpp"), str(d / "jp")
    with open(src, "w") as f:
        f.write(PROGRAM)
    subprocess.run(["g++", "-std=c++17", "-O1", "-Wno-unknown-pragmas", "-I" + CSRC, "-o", exe,
                    src], check=True)
    out = subprocess.run([exe], check=True, capture_output=True, text=True).stdout.strip()
    return np.array([c == "1" for c in out]).reshape(8, 8)


def test_hires_pattern_is_the_oracles(declared, orc):
    rng = np.random.default_rng(7)
    seen = np.zeros((8, 8), bool)
    for _ in range(50):
        theta = rng.uniform(0.1, 10.0, 12)
        y = rng.uniform(-1.0, 1.0, 8)
        J = np.asarray(orc.jac("hires", theta, y[None], theta_shared=True)).reshape(8, 8)
        seen |= J != 0
    assert (seen & ~declared).sum() == 0, "entries the oracle finds nonzero outside the pattern"
    assert (declared & ~seen).sum() == 0, "declared entries the oracle never finds nonzero"
    # every diagonal entry is in the pattern (the iteration matrix's diagonal is never zero)
    assert declared.diagonal().all()


def test_bench_pattern_is_the_headers(declared):
    """bench.py counts the kernels' operations on the same pattern the header declares."""
    import bench
    rows = bench.JAC_PATTERN["hires"]
    mine = np.array([[(rows[r] >> c) & 1 for c in range(8)] for r in range(8)], bool)
    assert (mine == declared).all()
