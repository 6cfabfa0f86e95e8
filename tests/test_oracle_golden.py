"""The oracle reproduces its stored small-case anchors (tests/golden/oracle_small_cases.json,
written by tests/golden/make_golden.py from the oracle alone)."""
import json
import os

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))


def test_oracle_reproduces_golden_anchors():
    import sys
    sys.path.insert(0, os.path.join(HERE, "golden"))
    import make_golden
    with open(os.path.join(HERE, "golden", "oracle_small_cases.json")) as f:
        gold = json.load(f)
    for name, case in gold["cases"].items():
        got = make_golden.compute(name, case["N"])
        assert got["S"] == case["S"] and got["rejected"] == case["rejected"], name
        rtol = 1e-5 if name.endswith("f32") or name == "mlp" else 1e-12
        for key in ("y1", "dL_dy0", "dL_dtheta"):
            a, b = np.asarray(got[key]), np.asarray(case[key])
            assert np.max(np.abs(a - b)) <= rtol * max(1.0, np.max(np.abs(b))), (name, key)
    for name, case in gold.get("sens_cases", {}).items():
        got = make_golden.compute_sens(name, case["N"])
        assert got["S"] == case["S"] and got["rejected"] == case["rejected"], name
        for key in ("y1", "sens"):
            a, b = np.asarray(got[key]), np.asarray(case[key])
            assert np.max(np.abs(a - b)) <= 1e-12 * max(1.0, np.max(np.abs(b))), (name, key)
