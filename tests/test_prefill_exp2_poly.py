"""The FMA-pipe 2^x of the prefill softmax (ex2_poly2 in csrc/prefill_tc.cu), modelled on the CPU.

The kernel takes part of the softmax exponentials off the MUFU unit: x = j + f, j = rint(x) by
adding 1.5 * 2^23, 2^f by a degree-3 polynomial, 2^j added into the exponent field.  The model
reads the four coefficients from the kernel source and repeats its fp32 steps; pinned:
* the coefficients are the minimax (Remez) fit of the relative error of 2^f on [-1/2, 1/2],
  re-derived here from the definition, to fp32 rounding;
* over x in [-125, 9] (the softmax's range: scores minus a running max that lags by at most
  2^8) the relative error stays below 7.6e-5, well under the 2^-9 rounding of bf16 P;
* below -126 (masked or vanishing keys) the result is finite, non-negative and at most 2^-126;
* a planted mistake (the rounding constant 2^23 instead of 1.5 * 2^23, which breaks rint for
  negative x) fails the error bound.
"""
import pathlib
import re

import numpy as np

SRC = pathlib.Path(__file__).resolve().parents[1] / "mla_latent_kv_mqa_b200" / "csrc" / "prefill_tc.cu"


def coefficients():
    text = SRC.read_text()
    c = [float(re.search(rf"kEx2C{i}\s*=\s*([0-9.eE+-]+)f", text).group(1)) for i in range(4)]
    return np.array(c, dtype=np.float32)


def f32(x):
    return np.asarray(x, dtype=np.float32)


def fma32(a, b, c):
    """fp32 fused multiply-add: the fp32 product is exact in fp64, one rounding to fp32 after."""
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def ex2_model(x, c, rnd=12582912.0):
    x = np.maximum(f32(x), np.float32(-126.0))
    t = (x + np.float32(rnd)).astype(np.float32)
    f = (x - (t - np.float32(rnd)).astype(np.float32)).astype(np.float32)
    p = fma32(f32(c[3]), f, f32(c[2]))
    p = fma32(p, f, f32(c[1]))
    p = fma32(p, f, f32(c[0]))
    bits = p.view(np.uint32) + (t.view(np.uint32) << np.uint32(23))
    return bits.astype(np.uint32).view(np.float32)


def remez(deg=3, a=-0.5, b=0.5, iters=20):
    """Minimax polynomial for the relative error of 2^f on [a, b] (Remez exchange)."""
    n = deg + 2
    x = (a + b) / 2 + (b - a) / 2 * np.cos(np.pi * np.arange(n)[::-1] / (n - 1))
    g = np.linspace(a, b, 100001)
    for _ in range(iters):
        A = np.array([[xi ** k for k in range(deg + 1)] + [(-1) ** i * 2.0 ** xi] for i, xi in enumerate(x)])
        c = np.linalg.solve(A, 2.0 ** x)[:deg + 1]
        e = (np.polyval(c[::-1], g) - 2.0 ** g) / 2.0 ** g
        segs = np.split(np.arange(len(g)), np.where(np.diff(np.sign(e)) != 0)[0] + 1)
        if len(segs) == n:
            x = g[[s[np.argmax(np.abs(e[s]))] for s in segs]]
    return c


def test_coefficients_are_the_minimax_fit():
    c = coefficients()
    ref = remez()
    assert np.allclose(c.astype(np.float64), ref, rtol=0, atol=2e-7), (c, ref)


def test_relative_error_over_the_softmax_range():
    c = coefficients()
    x = np.concatenate([np.linspace(-125.0, 9.0, 2_000_001), -np.arange(0, 126, dtype=np.float64),
                        np.arange(-125, 9) + 0.5]).astype(np.float32)
    got = ex2_model(x, c).astype(np.float64)
    exact = np.exp2(x.astype(np.float64))
    rel = np.abs(got - exact) / exact
    assert rel.max() < 7.6e-5, float(rel.max())
    assert rel.max() > 5e-5  # the fit's equioscillation level is reached (not some other formula)


def test_below_the_normal_range():
    c = coefficients()
    x = np.array([-126.0, -126.4, -127.0, -200.0, -1e30, -np.inf], dtype=np.float32)
    got = ex2_model(x, c)
    assert np.all(np.isfinite(got)) and np.all(got >= 0) and np.all(got <= np.float32(2.0 ** -126) * 1.0001)


def test_planted_rounding_constant_fails():
    c = coefficients()
    x = np.linspace(-20.0, 0.0, 10001).astype(np.float32)
    rel = np.abs(ex2_model(x, c, rnd=8388608.0).astype(np.float64) - np.exp2(x.astype(np.float64))) / np.exp2(x.astype(np.float64))
    assert rel.max() > 1e-2
