"""Brute-force pure-Python loops for tiny MLA decode problems.

TEST INFRASTRUCTURE (like the rest of ``oracle/``).  A second, independent
restatement of the itwiki article "멀티 헤드 잠재 어텐션" (Multi-head latent
attention): section 분리 RoPE (scores over [q^C; q^R] . [k^C; k^R] scaled by
1/sqrt(d_h + d_R), causal softmax, value sum) and section 구현 (half-split RoPE,
base 1e4).  Nothing here calls numpy for arithmetic: every sum is a Python loop.
Only sizes of a few hundred multiply-adds per score are practical.
"""
from __future__ import annotations

import math


def rope(x, pos, base=1e4):
    d = len(x)
    half = d // 2
    out = [0.0] * d
    for k in range(half):
        theta = pos * base ** (-(2.0 * k) / d)
        out[k] = x[k] * math.cos(theta) - x[k + half] * math.sin(theta)
        out[k + half] = x[k + half] * math.cos(theta) + x[k] * math.sin(theta)
    return out


def _matvec_head(w, h, d_h, x):
    """W_h x for rows h*d_h .. h*d_h+d_h-1 of w (w given as nested lists)."""
    return [sum(w[h * d_h + d][c] * x[c] for c in range(len(x))) for d in range(d_h)]


def decode(q_c, q_r, q_pos, c_kv, k_r, w_uk, w_uv, *, mode="absorbed", base=1e4):
    """One sequence.  q_c [s_q][n_h][d_h], q_r [s_q][n_h][d_R] (before RoPE), q_pos [s_q],
    c_kv [L][d_c], k_r [L][d_R] (before RoPE, token j at position j), weights
    [n_h*d_h][d_c] as nested lists.  Returns (o [s_q][n_h][d_h], lse [s_q][n_h])."""
    s_q, n_h, d_h = len(q_c), len(q_c[0]), len(q_c[0][0])
    d_r = len(q_r[0][0])
    d_c = len(c_kv[0])
    L = len(c_kv)
    scale = 1.0 / math.sqrt(d_h + d_r)
    k_rot = [rope(k_r[j], j, base) for j in range(L)]
    o_all, lse_all = [], []
    for i in range(s_q):
        o_i, lse_i = [], []
        for h in range(n_h):
            q_rot = rope(q_r[i][h], q_pos[i], base)
            n = min(L, q_pos[i] + 1)
            scores = []
            if mode == "absorbed":
                q_lat = [sum(w_uk[h * d_h + k][c] * q_c[i][h][k] for k in range(d_h))
                         for c in range(d_c)]
                for j in range(n):
                    s = sum(q_lat[c] * c_kv[j][c] for c in range(d_c))
                    s += sum(q_rot[k] * k_rot[j][k] for k in range(d_r))
                    scores.append(s * scale)
            else:
                for j in range(n):
                    k_c = _matvec_head(w_uk, h, d_h, c_kv[j])
                    s = sum(q_c[i][h][k] * k_c[k] for k in range(d_h))
                    s += sum(q_rot[k] * k_rot[j][k] for k in range(d_r))
                    scores.append(s * scale)
            m = max(scores)
            e = [math.exp(s - m) for s in scores]
            z = sum(e)
            p = [x / z for x in e]
            if mode == "absorbed":
                o_lat = [sum(p[j] * c_kv[j][c] for j in range(n)) for c in range(d_c)]
                o = _matvec_head(w_uv, h, d_h, o_lat)
            else:
                vs = [_matvec_head(w_uv, h, d_h, c_kv[j]) for j in range(n)]
                o = [sum(p[j] * vs[j][d] for j in range(n)) for d in range(d_h)]
            o_i.append(o)
            lse_i.append(m + math.log(z))
        o_all.append(o_i)
        lse_all.append(lse_i)
    return o_all, lse_all
