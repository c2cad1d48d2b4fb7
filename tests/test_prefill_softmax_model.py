"""The prefill attention kernel's softmax scheme, modelled on the CPU (fp32 where the kernel is
fp32) and held to exact causal attention in fp64.

Per query row the kernel walks 128-key tiles.  Two warps own the row, each 64 of the tile's
keys: each takes the max of its raw scores, the two exchange them, and the row's running max
m (log2 units, scores times scale * log2 e) moves only when the tile's max exceeds it by more
than 8; then O and both halves' running sums are scaled by 2^(m_old - m_new).  P = 2^(s - m)
goes to the tensor core rounded to bf16, while each half sums its own fp32 P; a quarter of the
exponentials (pairs c with c % 4 == 3, tiles without masked keys) come from the FMA-pipe
polynomial of `test_prefill_exp2_poly.py`.  At the end o = O / (l_0 + l_1) and
lse = (m + log2(l_0 + l_1)) ln 2.

Pinned: each row stays within the bf16 rounding of P (relative error at most 2^-8, which is
also the 4e-3 rel-L2 bound of the GPU tests) and the lse within fp32 rounding, with scores
that drift enough for the running max to move several times; planted mistakes fail: a half that rescales O but not its own
sum, halves that skip the max exchange, and a running max taken before the scale.
"""
import numpy as np
import pytest
import torch

from tests.test_prefill_exp2_poly import coefficients, ex2_model

LN2 = 0.6931471805599453
LOG2E = 1.4426950408889634


def bf16(x):
    return torch.from_numpy(np.asarray(x, dtype=np.float32)).to(torch.bfloat16).to(torch.float32).numpy()


def kernel_row(s_raw, v, qi, scale, mistake=None):
    """One query row at position qi over keys 0..qi (s_raw: raw fp32 scores of keys 0..L-1).
    Half h is warp h of the row: its keys are columns 64 h .. 64 h + 63 of each tile, and it
    rescales and finally normalises its half of O's value columns."""
    c = coefficients()
    sl2 = np.float32(scale * LOG2E)
    m = [-np.inf, -np.inf]                      # running max of each half (equal after the exchange)
    l = [np.float32(0.0), np.float32(0.0)]      # each half's sum over its own keys
    o = np.zeros(v.shape[1], dtype=np.float64)  # fp32 tensor-core accumulation, kept exact here
    cols = [slice(0, v.shape[1] // 2), slice(v.shape[1] // 2, v.shape[1])]
    for j in range(qi // 128 + 1):
        keys = np.arange(j * 128, j * 128 + 128)
        vis = keys <= qi
        tile = np.where(vis, s_raw[np.minimum(keys, len(s_raw) - 1)], -np.inf).astype(np.float32)
        halves = [tile[:64], tile[64:]]
        pm = [hv.max() for hv in halves]
        ps = []
        for h in range(2):
            raw = pm[h] if mistake == "no_exchange" else max(pm)
            mt = np.float32(raw) if mistake == "max_before_scale" else np.float32(np.float32(raw) * sl2)
            if mt > m[h] + 8:  # also the first visible key (m = -inf)
                fac = np.float32(np.exp2(np.float64(m[h] - mt))) if m[h] != -np.inf else np.float32(0.0)
                m[h] = mt
                if mistake != "sum_not_rescaled":
                    l[h] = np.float32(l[h] * fac)
                o[cols[h]] *= fac
            x = (halves[h] * sl2 - np.float32(m[h])).astype(np.float32)
            p = np.exp2(x.astype(np.float64)).astype(np.float32)
            if vis.all():  # the polynomial takes pairs c % 4 == 3 (elements 6, 7, 14, 15, ...)
                sel = ((np.arange(64) // 2) % 4) == 3
                p[sel] = ex2_model(x[sel], c)
            l[h] = np.float32(l[h] + p.sum(dtype=np.float32))
            ps.append(p)
        for h in range(2):  # O += P V over all of O's columns (one MMA per tile)
            kh = np.minimum(keys[h * 64:(h + 1) * 64], len(v) - 1)
            o += bf16(ps[h]).astype(np.float64) @ v[kh]
    lt = np.float64(l[0]) + np.float64(l[1])
    return o / lt, (np.float64(m[0]) + np.log2(lt)) * LN2


def exact_row(s_raw, v, qi, scale):
    s = s_raw[:qi + 1].astype(np.float64) * scale
    w = np.exp(s - s.max())
    return w @ v[:qi + 1] / w.sum(), s.max() + np.log(w.sum())


def _case(seed, L=700):
    rng = np.random.default_rng(seed)
    d = 192
    scale = 1.0 / np.sqrt(d)
    # raw scores q.k for d = 192 with a drift, so the running max jumps by more than 2^8 at times
    drift = np.cumsum(rng.standard_normal(L)) * 6.0
    s_raw = (rng.standard_normal(L) * np.sqrt(d) + drift).astype(np.float32)
    v = bf16(rng.standard_normal((L, 16))).astype(np.float64)
    return s_raw, v, scale


@pytest.mark.parametrize("seed", range(6))
def test_scheme_matches_exact_attention(seed):
    s_raw, v, scale = _case(seed)
    for qi in (0, 63, 127, 128, 255, 400, 699):
        got, got_lse = kernel_row(s_raw, v, qi, scale)
        want, want_lse = exact_row(s_raw, v, qi, scale)
        rel = np.linalg.norm(got - want) / np.linalg.norm(want)
        # each P is rounded to bf16 (relative error <= 2^-8) while l sums the unrounded values,
        # so one row's output can be off by up to 2^-8 when a few keys carry the weight
        assert rel <= 2.0 ** -8, (qi, rel)
        assert abs(got_lse - want_lse) < 1e-4 * max(1.0, abs(want_lse)), (qi, got_lse, want_lse)


@pytest.mark.parametrize("mistake", ["sum_not_rescaled", "no_exchange", "max_before_scale"])
def test_planted_mistakes_fail(mistake):
    worst = 0.0
    for seed in range(6):
        s_raw, v, scale = _case(seed)
        for qi in (255, 400, 699):
            with np.errstate(divide="ignore", invalid="ignore", over="ignore"):
                got, got_lse = kernel_row(s_raw, v, qi, scale, mistake)
                want, want_lse = exact_row(s_raw, v, qi, scale)
                rel = np.linalg.norm(got - want) / np.linalg.norm(want)
            err = max(rel if np.isfinite(rel) else np.inf, abs(got_lse - want_lse) if np.isfinite(got_lse) else np.inf)
            worst = max(worst, err)
    assert worst > 1e-2, worst
