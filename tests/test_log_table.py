"""The table of the kernels' logarithm (gs::log_tab, Tang's table-driven method; the device
function's accuracy is checked on the GPU by test_gpu_kernel_math.py).

Row j of differentiable_adaptive_ode_b200/csrc/gs_log_table.cuh holds g_j = RN(1/c_j),
c_j = 1 + j/128, and L_j = -log(g_j) as a head on the 2^-42 grid plus a tail.  Pinned here:
the committed header is what its generator writes; every g_j is the double nearest 1/c_j (exact
rational arithmetic); exp(-(head + tail)) returns g_j to 2^-94 (the generator takes a logarithm,
the check an exponential); the special rows (g_0 = 1, L_0 = 0; g_128 = 1/2, L_128 = ln 2 split
as the ln 2 constants); the exactness of e ln2_hi + head for every binary exponent; and the
reduction bound |m g_j - 1| <= 2^-8 + 2^-53 over each breakpoint's interval, which the degree-7
polynomial of the method relies on."""
import math
import os
import re
import subprocess
import sys
from decimal import Decimal, getcontext
from fractions import Fraction

CSRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                    "differentiable_adaptive_ode_b200", "csrc")
HEADER = os.path.join(CSRC, "gs_log_table.cuh")


def _rows():
    text = open(HEADER).read()
    consts = dict(re.findall(r"constexpr double (LOG_LN2_\w+) = (\S+);", text))
    rows = re.findall(r"\{(\S+), (\S+), (\S+), 0\.0\},", text)
    hx = float.fromhex
    return ({k: hx(v) for k, v in consts.items()},
            [(hx(g), hx(hi), hx(lo)) for g, hi, lo in rows])


def test_header_is_the_generators_output():
    out = subprocess.run([sys.executable, os.path.join(CSRC, "gen_log_table.py")], check=True,
                         capture_output=True, text=True).stdout
    assert out == open(HEADER).read()


def test_rows_match_their_definition():
    getcontext().prec = 50
    consts, rows = _rows()
    assert len(rows) == 129
    for j, (g, hi, lo) in enumerate(rows):
        c = 1 + Fraction(j, 128)
        # g is the double nearest 1/c: neither neighbouring double is closer (exact rationals)
        d = abs(Fraction(g) - 1 / c)
        for nb in (math.nextafter(g, 0.0), math.nextafter(g, 2.0)):
            assert d <= abs(Fraction(nb) - 1 / c), j
        # the head is on the 2^-42 grid and the tail below its spacing
        assert (Fraction(hi) * 2 ** 42).denominator == 1, j
        assert abs(lo) <= 2.0 ** -43, j
        # exp(-(head + tail)) gives back g to 2^-94
        back = (-(Decimal(hi) + Decimal(lo))).exp()
        assert abs(back - Decimal(g)) <= Decimal(2) ** -94, j
    assert rows[0] == (1.0, 0.0, 0.0)
    assert rows[128] == (0.5, consts["LOG_LN2_HI"], consts["LOG_LN2_LO"])
    ln2 = Decimal(consts["LOG_LN2_HI"]) + Decimal(consts["LOG_LN2_LO"])
    assert abs(ln2.exp() - 2) <= Decimal(2) ** -100
    assert (Fraction(consts["LOG_LN2_HI"]) * 2 ** 42).denominator == 1


def test_head_sum_is_exact_for_every_exponent():
    consts, rows = _rows()
    h2 = Fraction(consts["LOG_LN2_HI"]) * 2 ** 42
    for _, hi, _ in rows:
        hj = Fraction(hi) * 2 ** 42
        for e in (-1022, -1, 0, 1, 1023):
            n = e * h2 + hj                       # an integer: the sum on the 2^-42 grid
            assert n.denominator == 1 and abs(n) < 2 ** 53


def test_reduction_bound():
    _, rows = _rows()
    bound = Fraction(1, 256) + Fraction(1, 2 ** 53)
    for j, (g, _, _) in enumerate(rows):
        c = 1 + Fraction(j, 128)
        lo = max(Fraction(1), c - Fraction(1, 256))
        hi = min(Fraction(2), c + Fraction(1, 256))
        for m in (lo, hi):
            assert abs(m * Fraction(g) - 1) <= bound, j
    # the first term the polynomial leaves out, r^8 / 8, is about 2^-67 at most
    assert bound ** 8 / 8 < Fraction(1, 2 ** 67) * (1 + Fraction(1, 2 ** 40))
