"""The arithmetic the decode kernels are built on, modelled in fp64 on the CPU.

1. Split-KV with lazy rescaling.  Each segment of a row's tokens runs an online softmax over
   64-token pages in log2 units, moving its running max only when a page's max exceeds it by
   more than a threshold (8 in the kernel); O and l are rescaled only then.  The combine step
   merges the segments' (m, l, O) with M = max m, w = 2^(m - M), L = sum w l, o = sum w O / L,
   lse = (M + log2 L) ln 2.  The result must equal the direct softmax-weighted sum exactly (up
   to fp64 rounding), for any split and threshold, including empty segments (m = -inf).
2. The output projection carries o_lat (fp32) as bf16 hi + bf16 lo, ~16 mantissa bits.
"""
import numpy as np
import pytest
import torch

LOG2E = 1.4426950408889634


def _segment(s2, v, thresh, page=64):
    """Online softmax of one segment (scores already in log2 units, s2 = s * log2(e))."""
    m, l, o = -np.inf, 0.0, np.zeros(v.shape[1])
    for p0 in range(0, len(s2), page):
        sp, vp = s2[p0:p0 + page], v[p0:p0 + page]
        mx = sp.max()
        if m == -np.inf:
            m_new = mx
        elif mx > m + thresh:
            m_new = mx
        else:
            m_new = m
        fac = 2.0 ** (m - m_new) if m != -np.inf else 0.0
        p = 2.0 ** (sp - m_new)
        l = l * fac + p.sum()
        o = o * fac + p @ vp
        m = m_new
    return m, l, o


def _combine(parts):
    ms = np.array([m for m, _, _ in parts])
    M = ms.max()
    w = np.where(ms == -np.inf, 0.0, 2.0 ** (ms - M))
    L = sum(wi * l for wi, (_, l, _) in zip(w, parts))
    o = sum(wi * oi for wi, (_, _, oi) in zip(w, parts)) / L
    return o, (M + np.log2(L)) / LOG2E


@pytest.mark.parametrize("seed", range(12))
def test_split_kv_with_lazy_rescale_equals_softmax(seed):
    rng = np.random.default_rng(seed)
    n = int(rng.integers(1, 900))
    # scores with drifts, so the running max moves by more than the threshold now and then
    s = rng.standard_normal(n) * rng.uniform(0.5, 6) + np.cumsum(rng.standard_normal(n)) * rng.uniform(0, 0.5)
    v = rng.standard_normal((n, 8))
    want = np.exp(s - s.max()) @ v / np.exp(s - s.max()).sum()
    want_lse = s.max() + np.log(np.exp(s - s.max()).sum())
    cuts = sorted(set(int(x) for x in rng.integers(0, n + 1, int(rng.integers(0, 6))))) + [n]
    parts, a = [], 0
    for b in cuts:
        seg = _segment(s[a:b] * LOG2E, v[a:b], thresh=float(rng.choice([0.0, 8.0, 30.0])))
        parts.append(seg)  # empty segments give m = -inf, l = 0: weight 0 in the combine
        a = b
    o, lse = _combine(parts)
    assert np.max(np.abs(o - want)) < 1e-12 * max(1.0, np.max(np.abs(want)))
    assert abs(lse - want_lse) < 1e-12 * max(1.0, abs(want_lse))


def test_lazy_rescale_keeps_unnormalised_weights_bounded():
    # with threshold t, every p = 2^(s2 - m_used) of a page is at most 2^t (t = 8: P <= 256)
    rng = np.random.default_rng(5)
    s2 = np.cumsum(rng.uniform(0, 0.3, 2000))  # steadily rising scores
    m = -np.inf
    for p0 in range(0, len(s2), 64):
        mx = s2[p0:p0 + 64].max()
        if m == -np.inf or mx > m + 8.0:
            m = mx
        assert np.max(2.0 ** (s2[p0:p0 + 64] - m)) <= 2.0 ** 8


def test_hi_lo_bf16_split_keeps_sixteen_bits():
    rng = np.random.default_rng(6)
    x = np.float32(rng.standard_normal(200000) * np.exp(rng.uniform(-20, 20, 200000)))
    hi = torch.from_numpy(x).to(torch.bfloat16)
    lo = (torch.from_numpy(x) - hi.float()).to(torch.bfloat16)
    rec = hi.double() + lo.double()
    rel = (rec - torch.from_numpy(x).double()).abs() / torch.from_numpy(x).double().abs()
    assert float(rel.max()) <= 2.0 ** -16
