"""The density pass evaluates the cosine cutoff f_c(r) = (cos(pi r / r_c) + 1) / 2
of section "REANN Architecture" ("Efficient Parallelization of Message Passing
Neural Network Potentials for Large-Scale Molecular Dynamics") as cos^2(theta),
theta = pi r / (2 r_c), with the cosine's Taylor series to theta^14 in fp32
Horner form (edge.cu, cutoff_cos2).  These checks bound its error from the
mathematics: the truncation on [0, pi/2], and the fp32 evaluation (each fused
multiply-add rounded once, emulated exactly in fp64) against fp64 cos on a dense
grid of distances for r_c = 6 A.
"""
import math
import re
from pathlib import Path

import numpy as np

SRC = Path(__file__).resolve().parent.parent / "molecular_dynamics_b200" / "csrc" / "edge.cu"


def _series_coefficients():
    """The Horner coefficients as written in the kernel source, highest first."""
    body = SRC.read_text().split("float cutoff_cos2(float theta)")[1].split("}")[0]
    return [(-1.0 if sign else 1.0) * float(num) / float(den)
            for sign, num, den in re.findall(r"(-?)(\d+\.\d+)f\s*/\s*(\d+\.\d+)f", body)]


def test_source_holds_the_taylor_coefficients():
    c = _series_coefficients()
    # -1/14!, 1/12!, ..., 1/4! as divisions, then -0.5 and 1 as literals
    expect = [(-1) ** k / math.factorial(2 * k) for k in range(7, 1, -1)]
    assert len(c) == len(expect)
    assert np.allclose(c, expect, rtol=1e-12)


def test_truncation_error_on_the_cutoff_range():
    th = np.linspace(0.0, np.pi / 2, 20001)
    series = sum((-1) ** k * th ** (2 * k) / math.factorial(2 * k) for k in range(8))
    assert np.abs(series - np.cos(th)).max() < 7e-11


def test_fp32_evaluation_error():
    f32 = np.float32
    coef = [f32(v) for v in _series_coefficients()] + [f32(-0.5), f32(1.0)]

    def fma(a, b, c):   # exact product and sum of float32 values, rounded once
        return f32(np.float64(a) * np.float64(b) + np.float64(c))

    r_c = 6.0
    k = f32(0.5) * f32(np.pi / r_c)
    r = np.linspace(0.3, 5.9999, 40001).astype(np.float32)
    worst = 0.0
    for x in r:
        th = f32(x * k)
        z = f32(th * th)
        c = coef[0]
        for a in coef[1:]:
            c = fma(c, z, a)
        fc = f32(c * c)
        exact = 0.5 * (math.cos(math.pi * float(x) / r_c) + 1.0)
        worst = max(worst, abs(float(fc) - exact))
    # the argument's own fp32 rounding contributes ~1e-7; the series adds little
    assert worst < 3e-7, worst
