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


def linear(w, x):
    """y = W x for W given as rows [out][in] (the nn.Linear weight convention), by loops."""
    return [sum(w[o][k] * x[k] for k in range(len(x))) for o in range(len(w))]


def toy_projections(h, W):
    """Projections of the simplified layer for one sequence h [T][d], by loops, written from
    the notation of sections 구조 and 분리 RoPE rather than from any reshape:
        c^KV_t = W^DKV h_t,   k^R_t = W^KR h_t   (the shared RoPE key comes from h_t),
        c^Q_t  = W^DQ h_t,
        q^C_{t,i} = W^UQ_i c^Q_t,   q^R_{t,i} = W^QR_i c^Q_t,
    where W^UQ_i (W^QR_i) is the i-th block of d_h (d_R) consecutive rows of W^UQ (W^QR): head i
    owns output features i*d_h .. i*d_h + d_h - 1 (section 행렬 흡수's per-head W_i).
    Returns (c_kv [T][d_c], k_r [T][d_R], q_c [T][n_h][d_h], q_r [T][n_h][d_R]); keys and
    queries before RoPE."""
    n_h, d_h, d_r = W["n_h"], W["d_h"], W["d_r"]
    c_kv, k_r, q_c, q_r = [], [], [], []
    for x in h:
        c_kv.append(linear(W["w_dkv"], x))
        k_r.append(linear(W["w_kr"], x))
        cq = linear(W["w_dq"], x)
        q_c.append([linear(W["w_uq"][i * d_h:(i + 1) * d_h], cq) for i in range(n_h)])
        q_r.append([linear(W["w_qr"][i * d_r:(i + 1) * d_r], cq) for i in range(n_h)])
    return c_kv, k_r, q_c, q_r


def output_projection(o_heads, w_o):
    """u_t = W^O [o_{t,1}; ...; o_{t,n_h}] for one token: the heads' outputs concatenated in
    head order (section 분리 RoPE, output equation), then W^O [d][n_h*d_h]."""
    cat = [v for head in o_heads for v in head]
    return linear(w_o, cat)
