"""The e4m3 query split of the FP8 tensor-core scores (MLA_FLAG_FP8_MMA), modelled on the CPU.

Per head the kernel forms alpha = max|q_lat| / 448 (at least FLT_MIN), hi = e4m3(q / alpha)
and lo = e4m3(q / alpha - hi) (fp32 arithmetic, round to nearest even, saturating), and the
tensor core accumulates (hi + lo) . c8 exactly in fp32.  The model pins, on V3-shaped query
rows (d_c = 512, N(0, 1) and log-normal magnitudes):
* alpha (hi + lo) reproduces q to about 7 significant bits (relative error <= 2^-7 for the
  entries that carry the dot product), where one e4m3 rounding alone gives only 2^-4;
* the content score (hi + lo) . c8 * alpha * s_j then sits within the error a bf16 query
  (the default path's operand) already has, so the split keeps the FP8 path's bound;
* a zero row gives alpha = FLT_MIN and zero codes (no division by zero, no NaN).
A model that drops the low part fails the second point by an order of magnitude.
"""
import numpy as np
import pytest
import torch

FLT_MIN = np.float32(1.1754943508222875e-38)


def e4m3(x32):
    """fp32 -> e4m3 value (nearest even, saturating at 448), as fp64."""
    x = np.clip(np.asarray(x32, dtype=np.float32), -448.0, 448.0)
    return torch.from_numpy(x).to(torch.float8_e4m3fn).to(torch.float64).numpy()


def split(q):
    """alpha, hi, lo of one query row (fp32 arithmetic as in the kernel)."""
    q = np.asarray(q, dtype=np.float32)
    alpha = np.float32(max(np.float32(np.abs(q).max()) / np.float32(448.0), FLT_MIN))
    ia = np.float32(1.0) / alpha
    y = (q * ia).astype(np.float32)
    hi = e4m3(y)
    lo = e4m3((y - hi.astype(np.float32)).astype(np.float32))
    return np.float64(alpha), hi, lo


def bf16(x):
    return torch.from_numpy(np.asarray(x, dtype=np.float32)).to(torch.bfloat16).to(torch.float64).numpy()


@pytest.mark.parametrize("dist", ["normal", "lognormal"])
def test_hi_lo_reproduces_the_query_to_seven_bits(dist):
    rng = np.random.default_rng(7)
    for _ in range(64):
        q = rng.standard_normal(512).astype(np.float32)
        if dist == "lognormal":
            q *= rng.lognormal(0.0, 1.0, 512).astype(np.float32)
        alpha, hi, lo = split(q)
        rec = alpha * (hi + lo)
        big = np.abs(q) >= np.abs(q).max() / 64  # the entries that carry the dot product
        rel = np.abs(rec - q)[big] / np.abs(q)[big]
        assert rel.max() <= 2.0 ** -7, rel.max()
        one = np.abs(alpha * hi - q)[big] / np.abs(q)[big]
        assert one.max() > 2.0 ** -6  # one e4m3 rounding alone is far coarser


def test_content_scores_stay_at_the_bf16_query_error():
    rng = np.random.default_rng(11)
    codes = rng.standard_normal((64, 512)).astype(np.float32)
    c8 = e4m3(codes * 40.0)                   # cache codes of a page
    s = rng.uniform(0.002, 0.02, 64)          # per-token scales
    errs_split, errs_bf16, errs_hi = [], [], []
    for _ in range(32):
        q = rng.standard_normal(512).astype(np.float32)
        exact = (c8 @ q.astype(np.float64)) * s
        alpha, hi, lo = split(q)
        errs_split.append(np.abs((c8 @ (hi + lo)) * alpha * s - exact).max())
        errs_hi.append(np.abs((c8 @ hi) * alpha * s - exact).max())
        errs_bf16.append(np.abs((c8 @ bf16(q)) * s - exact).max())
    split_e, bf16_e, hi_e = np.median(errs_split), np.median(errs_bf16), np.median(errs_hi)
    assert split_e <= 2.0 * bf16_e, (split_e, bf16_e)
    assert hi_e >= 5.0 * bf16_e, (hi_e, bf16_e)   # the planted mistake: no low part


def test_zero_row():
    alpha, hi, lo = split(np.zeros(512, dtype=np.float32))
    assert alpha == np.float64(FLT_MIN)
    assert not np.any(hi) and not np.any(lo) and np.all(np.isfinite(hi))
