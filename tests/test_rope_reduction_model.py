"""The RoPE angle arithmetic of the kernels, modelled exactly on the CPU, against the oracle's.

The kernels form theta = pos * f_k in fp64 (f_k = base^(-2k/d_R) from a host fp64 table),
reduce it modulo 2 pi by subtracting n * 2pi with 2pi split into its fp64 value and the
remainder (each step one fused multiply-add, i.e. one rounding), and take cos/sin of the
reduced angle in fp32.  Here the fused multiply-adds are evaluated exactly with rationals and
rounded once; cos/sin of the fp32 angle are taken in fp64 and rounded to fp32, standing in for
an fp32 sincos of at most a few ulps.  The result must match fp64 cos/sin of the oracle's fp64
angle pos * f_k to within a few fp32 ulps for positions up to 2^31 - 1.
"""
from fractions import Fraction

import numpy as np
import pytest

TWO_PI = 6.283185307179586           # 2pi rounded to fp64 (the kernels' constant)
TWO_PI_REM = 2.4492935982947064e-16  # 2pi - TWO_PI
INV_TWO_PI = 0.15915494309189535


def fma(a: float, b: float, c: float) -> float:
    """a * b + c with one rounding to fp64."""
    return float(Fraction(a) * Fraction(b) + Fraction(c))


TWO_PI_EXACT = Fraction("6.28318530717958647692528676655900576839433879875021164194988918")


def kernel_reduced_angle(pos: int, f: float):
    theta = float(pos) * f
    n = float(np.rint(theta * INV_TWO_PI))
    return theta, n, fma(-n, TWO_PI_REM, fma(-n, TWO_PI, theta))


def kernel_cos_sin(pos: int, f: float):
    r32 = np.float32(kernel_reduced_angle(pos, f)[2])
    return np.float32(np.cos(np.float64(r32))), np.float32(np.sin(np.float64(r32)))


def test_constants_split_two_pi():
    # TWO_PI is the fp64 nearest to 2pi, TWO_PI_REM the rest to ~1e-32
    two_pi_30 = Fraction("6.283185307179586476925286766559005768394338798750")
    assert Fraction(TWO_PI) == Fraction(float(two_pi_30))
    assert abs(Fraction(TWO_PI) + Fraction(TWO_PI_REM) - two_pi_30) < Fraction(1, 10 ** 30)


def test_reduction_is_exact_to_fp64_rounding():
    """theta - n * 2pi of the fp64 angle, exactly: the two fused steps land within an ulp or
    two of it (dropping the remainder term would be off by n * 2.4e-16, up to ~1e-7)."""
    rng = np.random.default_rng(7)
    for p in [1, 4095, (1 << 31) - 1] + [int(x) for x in rng.integers(0, 1 << 31, 200)]:
        for f in (1.0, 0.749894209332456, 1e-4 ** (31 / 32)):
            theta, n, r = kernel_reduced_angle(p, f)
            exact = Fraction(theta) - Fraction(n) * TWO_PI_EXACT
            assert abs(Fraction(r) - exact) <= Fraction(2) * Fraction(np.spacing(abs(r)) if r else 2 ** -1074)
            assert abs(r) <= 3.1416


@pytest.mark.parametrize("base,d_r", [(1e4, 64), (1e4, 32), (5e5, 64)])
def test_reduced_angle_cos_sin_match_fp64(base, d_r):
    rng = np.random.default_rng(int(base) + d_r)
    positions = [0, 1, 2, 63, 64, 4095, 131071, 1 << 20, (1 << 31) - 1] + \
        [int(x) for x in rng.integers(0, 1 << 31, 40)]
    worst = 0.0
    for k in range(d_r // 2):
        f = float(base ** (-(2.0 * k) / d_r))  # the host table's fp64 value
        for p in positions:
            theta = float(p) * f
            c, s = kernel_cos_sin(p, f)
            worst = max(worst, abs(float(c) - np.cos(theta)), abs(float(s) - np.sin(theta)))
    # fp32 rounding of the reduced angle (|r| <= pi: half an ulp is 1.2e-7) plus that of cos/sin
    assert worst < 3e-7, worst
