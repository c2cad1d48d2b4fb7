"""Pins of the fp64 CPU oracle against facts it does not compute itself.

Each test ties one part of ``oracle/`` to something independent: a library routine
(torch's scaled_dot_product_attention, torch's float8_e4m3fn cast), a closed form
(uniform attention, a single cached token), an invariant of the method (rotations
preserve norms and compose; absorbed and naive modes agree to rounding, as the
implementation section of the itwiki "멀티 헤드 잠재 어텐션" article reports at
the 1e-15 level in float64), brute-force loops, or numbers the pages print
(``tests/golden/cache_sizes.txt``).
"""
import math
import os

import numpy as np
import pytest
import torch

from oracle import brute
from mla_latent_kv_mqa_b200 import workloads as wl

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rng(seed=0):
    return np.random.default_rng(seed)


# ---------------------------------------------------------------------------------------------
# RoPE (구현 section: half-split pairs, angle pos * base^(-2k/d_R))
# ---------------------------------------------------------------------------------------------

def test_rope_identity_at_position_zero(oracle_mod):
    x = _rng(1).standard_normal(64)
    assert np.array_equal(oracle_mod.rope(x, 0.0), x)


def test_rope_preserves_norm_and_composes(oracle_mod):
    x = _rng(2).standard_normal(64)
    for a, b in [(3.0, 5.0), (1000.0, 77.0), (131071.0, 1.0)]:
        ra = oracle_mod.rope(x, a)
        assert abs(np.linalg.norm(ra) - np.linalg.norm(x)) < 1e-12
        # rotating by a then by b equals rotating by a + b
        assert np.max(np.abs(oracle_mod.rope(ra, b) - oracle_mod.rope(x, a + b))) < 1e-9


def test_rope_is_a_complex_rotation_of_half_split_pairs(oracle_mod):
    # Pair k couples x[k] with x[k + d/2]; as a complex number x[k] + i x[k + d/2] it is
    # multiplied by exp(i * theta_k).
    d = 8
    x = _rng(3).standard_normal(d)
    pos = 7.0
    z = x[: d // 2] + 1j * x[d // 2:]
    theta = pos * 1e4 ** (-np.arange(0, d, 2) / d)
    w = z * np.exp(1j * theta)
    want = np.concatenate([w.real, w.imag])
    assert np.max(np.abs(oracle_mod.rope(x, pos) - want)) < 1e-14


def test_rope_frequencies_by_periodicity(oracle_mod):
    # Pair k turns half-way (x -> -x) at pos = pi * base^(2k/d) and returns to the identity
    # at twice that.  A wrong frequency for any pair fails one of the two.
    d = 16
    x = _rng(4).standard_normal(d)
    for k in range(d // 2):
        half_turn = math.pi * 1e4 ** (2 * k / d)
        y = oracle_mod.rope(x, half_turn)
        assert abs(y[k] + x[k]) < 1e-9 and abs(y[k + d // 2] + x[k + d // 2]) < 1e-9
        y = oracle_mod.rope(x, 2 * half_turn)
        assert abs(y[k] - x[k]) < 1e-9 and abs(y[k + d // 2] - x[k + d // 2]) < 1e-9


def test_rope_scores_depend_only_on_relative_position(oracle_mod):
    rng = _rng(5)
    q, k = rng.standard_normal(64), rng.standard_normal(64)
    ref = oracle_mod.rope(q, 100.0) @ oracle_mod.rope(k, 60.0)
    for shift in (0.0, 1.0, 4000.0, 120000.0):
        s = oracle_mod.rope(q, 100.0 + shift) @ oracle_mod.rope(k, 60.0 + shift)
        assert abs(s - ref) < 1e-9


# ---------------------------------------------------------------------------------------------
# Softmax and closed forms
# ---------------------------------------------------------------------------------------------

def _small_problem(seed, n_h=4, d_h=16, d_c=32, d_r=8, lens=(5, 9), s_q=1, qscale=1.0):
    rng = _rng(seed)
    B = len(lens)
    T = B * s_q
    q_c = rng.standard_normal((T, n_h, d_h)) * qscale
    q_r = rng.standard_normal((T, n_h, d_r)) * qscale
    q_pos = np.array([L - s_q + i for L in lens for i in range(s_q)], dtype=np.int64)
    c = [rng.standard_normal((L, d_c)) for L in lens]
    k = [rng.standard_normal((L, d_r)) for L in lens]
    w_uk = rng.standard_normal((n_h * d_h, d_c)) / math.sqrt(d_c)
    w_uv = rng.standard_normal((n_h * d_h, d_c)) / math.sqrt(d_c)
    return q_c, q_r, q_pos, c, k, w_uk, w_uv


def test_softmax_rows_sum_to_one(oracle_mod):
    args = _small_problem(6, lens=(2, 7, 33), s_q=2)
    r = oracle_mod.decode_absorbed(*args, s_q=2, want_probs=True)
    sums = r.probs.sum(-1)
    assert np.max(np.abs(sums - 1.0)) < 1e-14
    assert np.all(r.probs >= 0)


def test_softmax_lse_of_equal_scores_is_log_n(oracle_mod):
    p, lse = oracle_mod.softmax(np.full(10, 2.5))
    assert np.allclose(p, 0.1, atol=1e-16) and abs(lse - (2.5 + math.log(10))) < 1e-14


def test_single_cached_token_returns_its_value(oracle_mod):
    q_c, q_r, q_pos, c, k, w_uk, w_uv = _small_problem(7, lens=(1,))
    r = oracle_mod.decode_absorbed(q_c, q_r, q_pos, c, k, w_uk, w_uv)
    n_h, d_h = q_c.shape[1], q_c.shape[2]
    want = (w_uv.reshape(n_h, d_h, -1) @ c[0][0])  # W_UV,h c_0 for every head
    assert np.max(np.abs(r.o[0] - want)) < 1e-13
    assert np.max(np.abs(r.o_lat[0] - c[0][0][None, :])) < 1e-15


def test_zero_query_attends_uniformly(oracle_mod):
    q_c, q_r, q_pos, c, k, w_uk, w_uv = _small_problem(8, lens=(6, 11), s_q=2)
    q_c[:] = 0
    q_r[:] = 0
    r = oracle_mod.decode_absorbed(q_c, q_r, q_pos, c, k, w_uk, w_uv, s_q=2)
    n_h, d_h = q_c.shape[1], q_c.shape[2]
    for t in range(q_c.shape[0]):
        b = t // 2
        n = int(q_pos[t]) + 1
        mean = c[b][:n].mean(0)
        assert np.max(np.abs(r.o_lat[t] - mean[None])) < 1e-14
        assert np.max(np.abs(r.o[t] - w_uv.reshape(n_h, d_h, -1) @ mean)) < 1e-13
        assert np.max(np.abs(r.lse[t] - math.log(n))) < 1e-14


# ---------------------------------------------------------------------------------------------
# Absorbed mode == naive mode (the implementation section's float64 experiment)
# ---------------------------------------------------------------------------------------------

def test_page_experiment_absorbed_equals_naive(oracle_mod):
    # Default toy dims of the implementation section, h ~ N(0,1) of shape (2, 12, 1024),
    # positions 0..11, every token querying with the causal mask.
    h, W = wl.toy_layer_inputs(seed=11, B=2, T=12)
    a = oracle_mod.toy_layer(h.astype(np.float64), W, mode="absorbed")
    n = oracle_mod.toy_layer(h.astype(np.float64), W, mode="naive")
    assert np.max(np.abs(a.u - n.u)) < 1e-12
    assert np.max(np.abs(a.o - n.o)) < 1e-12
    assert np.max(np.abs(a.lse - n.lse)) < 1e-12


def test_absorbed_equals_naive_decode_shapes(oracle_mod):
    for seed, kw in [(12, dict(lens=(3, 64, 65), s_q=1)), (13, dict(lens=(70, 2), s_q=2)),
                     (14, dict(n_h=2, d_h=128, d_c=512, d_r=64, lens=(40,), s_q=1))]:
        s_q = kw["s_q"]
        args = _small_problem(seed, **kw)
        a = oracle_mod.decode_absorbed(*args, s_q=s_q)
        n = oracle_mod.decode_naive(*args, s_q=s_q)
        assert np.max(np.abs(a.o - n.o)) < 1e-12
        assert np.max(np.abs(a.lse - n.lse)) < 1e-12


# ---------------------------------------------------------------------------------------------
# Naive mode against a library attention routine
# ---------------------------------------------------------------------------------------------

def _rope_complex(x, pos, base=1e4):
    d = x.shape[-1]
    z = x[..., : d // 2] + 1j * x[..., d // 2:]
    theta = np.asarray(pos, dtype=np.float64)[..., None] * base ** (-np.arange(0, d, 2) / d)
    w = z * np.exp(1j * theta)
    return np.concatenate([w.real, w.imag], -1)


def test_naive_mode_matches_torch_sdpa(oracle_mod):
    n_h, d_h, d_c, d_r, s_q = 3, 16, 24, 8, 2
    lens = (9, 17)
    q_c, q_r, q_pos, c, k, w_uk, w_uv = _small_problem(15, n_h, d_h, d_c, d_r, lens, s_q)
    r = oracle_mod.decode_naive(q_c, q_r, q_pos, c, k, w_uk, w_uv, s_q=s_q)
    import torch.nn.functional as F
    for b, L in enumerate(lens):
        K_c = np.einsum("hdc,jc->hjd", w_uk.reshape(n_h, d_h, d_c), c[b])       # [n_h, L, d_h]
        V = np.einsum("hdc,jc->hjd", w_uv.reshape(n_h, d_h, d_c), c[b])
        K_r = _rope_complex(k[b], np.arange(L))                                 # [L, d_r]
        K = np.concatenate([K_c, np.broadcast_to(K_r, (n_h, L, d_r))], -1)
        Q = np.concatenate([q_c[b * s_q:(b + 1) * s_q].transpose(1, 0, 2),
                            _rope_complex(q_r[b * s_q:(b + 1) * s_q].transpose(1, 0, 2),
                                          q_pos[b * s_q:(b + 1) * s_q])], -1)   # [n_h, s_q, .]
        mask = np.arange(L)[None, :] <= q_pos[b * s_q:(b + 1) * s_q][:, None]
        out = F.scaled_dot_product_attention(torch.from_numpy(Q), torch.from_numpy(K.copy()),
                                             torch.from_numpy(V), attn_mask=torch.from_numpy(mask),
                                             scale=1.0 / math.sqrt(d_h + d_r)).numpy()
        got = r.o[b * s_q:(b + 1) * s_q]                                        # [s_q, n_h, d_h]
        assert np.max(np.abs(got - out.transpose(1, 0, 2))) < 1e-12


# ---------------------------------------------------------------------------------------------
# Brute force on tiny inputs
# ---------------------------------------------------------------------------------------------

@pytest.mark.parametrize("mode", ["absorbed", "naive"])
def test_brute_force_loops_match_oracle(oracle_mod, mode):
    n_h, d_h, d_c, d_r, s_q = 2, 4, 8, 4, 2
    lens = (1 + 1, 7, 5)
    q_c, q_r, q_pos, c, k, w_uk, w_uv = _small_problem(16, n_h, d_h, d_c, d_r, lens, s_q)
    fn = oracle_mod.decode_absorbed if mode == "absorbed" else oracle_mod.decode_naive
    r = fn(q_c, q_r, q_pos, c, k, w_uk, w_uv, s_q=s_q)
    for b in range(len(lens)):
        sl = slice(b * s_q, (b + 1) * s_q)
        o, lse = brute.decode(q_c[sl].tolist(), q_r[sl].tolist(), q_pos[sl].tolist(),
                              c[b].tolist(), k[b].tolist(), w_uk.tolist(), w_uv.tolist(), mode=mode)
        assert np.max(np.abs(np.array(o) - r.o[sl])) < 1e-13
        assert np.max(np.abs(np.array(lse) - r.lse[sl])) < 1e-13


# ---------------------------------------------------------------------------------------------
# FP8 e4m3 codec against torch's float8_e4m3fn
# ---------------------------------------------------------------------------------------------

def _tiny_toy_weights(seed):
    """Tiny simplified-layer weights with d_cq == d, so that taking k^R from c^Q instead of h
    (or any other mix-up of the two inputs) still runs and shows up only in the values."""
    rng = np.random.default_rng(seed)
    d, n_h, d_h, d_c, d_cq, d_r = 5, 3, 2, 4, 5, 4
    w = lambda o, i: rng.standard_normal((o, i)) / np.sqrt(i)
    return dict(n_h=n_h, d_h=d_h, d_r=d_r, d_c=d_c, d=d, d_cq=d_cq,
                w_dq=w(d_cq, d), w_uq=w(n_h * d_h, d_cq), w_qr=w(n_h * d_r, d_cq), w_dkv=w(d_c, d),
                w_kr=w(d_r, d), w_uk=w(n_h * d_h, d_c), w_uv=w(n_h * d_h, d_c), w_o=w(d, n_h * d_h))


def test_toy_projections_match_per_head_loops(oracle_mod):
    """The oracle's up projections split the n_h*d_h features head by head (head i owns rows
    i*d_h ..), and the RoPE key is projected from h, as the loops written from the sections'
    notation do.  A feature split in the other order, or k^R taken from c^Q, fails here."""
    Wt = _tiny_toy_weights(11)
    h = np.random.default_rng(12).standard_normal((1, 4, Wt["d"]))
    c_kv, k_r, q_c, q_r = oracle_mod.toy_projections(h, Wt)
    bc, bk, bq, br = brute.toy_projections(h[0].tolist(), {k: (v.tolist() if hasattr(v, "tolist") else v)
                                                          for k, v in Wt.items()})
    for got, want in ((c_kv[0], bc), (k_r[0], bk), (q_c[0], bq), (q_r[0], br)):
        assert np.max(np.abs(np.asarray(got) - np.asarray(want))) <= 1e-13
    # the planted mistakes really differ
    n_h, d_h, d_r = Wt["n_h"], Wt["d_h"], Wt["d_r"]
    cq = h[0] @ Wt["w_dq"].T
    wrong_split = (cq @ Wt["w_uq"].T).reshape(4, d_h, n_h).transpose(0, 2, 1)
    assert np.max(np.abs(wrong_split - np.asarray(bq))) > 1e-2
    assert np.max(np.abs(cq @ Wt["w_kr"].T - np.asarray(bk))) > 1e-2


def test_toy_layer_output_projection_matches_loops(oracle_mod):
    """u = W^O [o_1; ...; o_{n_h}] over the whole simplified layer (prefill form, every token
    querying): the oracle against the loops end to end (projections, decode, W^O)."""
    Wt = _tiny_toy_weights(13)
    T = 5
    h = np.random.default_rng(14).standard_normal((1, T, Wt["d"]))
    res = oracle_mod.toy_layer(h, Wt, mode="absorbed", last_only=False)
    L = {k: (v.tolist() if hasattr(v, "tolist") else v) for k, v in Wt.items()}
    bc, bk, bq, br = brute.toy_projections(h[0].tolist(), L)
    o, _ = brute.decode(bq, br, list(range(T)), bc, bk, L["w_uk"], L["w_uv"], mode="naive")
    u = [brute.output_projection(o[t], L["w_o"]) for t in range(T)]
    assert np.max(np.abs(res.u[0] - np.asarray(u))) <= 1e-12
    # a head-interleaved concatenation (feature d of every head, then d + 1, ...) differs
    o_arr = np.asarray(o)
    wrong = o_arr.transpose(0, 2, 1).reshape(T, -1) @ Wt["w_o"].T
    assert np.max(np.abs(wrong - np.asarray(u))) > 1e-2


def test_e4m3_table_matches_library(oracle_mod):
    lib_vals = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    mine = np.array([oracle_mod.e4m3_value(c) for c in range(256)])
    nan = np.isnan(lib_vals)
    assert np.array_equal(np.isnan(mine), nan)
    assert set(np.nonzero(nan)[0].tolist()) == {0x7F, 0xFF}
    assert np.array_equal(mine[~nan], lib_vals[~nan])
    assert np.nanmax(mine) == 448.0


def test_e4m3_rounding_matches_library(oracle_mod):
    rng = _rng(17)
    vals = np.concatenate([rng.uniform(-448, 448, 3000), rng.standard_normal(3000) * 0.05,
                           rng.standard_normal(1000) * 1e-3]).astype(np.float32)
    # midpoints between neighbouring codes exercise ties-to-even
    pos_codes = np.arange(0, 0x7E)
    table = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    mids = ((table[pos_codes] + table[pos_codes + 1]) / 2).astype(np.float32)
    vals = np.concatenate([vals, mids, -mids])
    want = torch.from_numpy(vals).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([oracle_mod.e4m3_quantize(float(v)) for v in vals], dtype=np.uint8)
    assert np.array_equal(got, want)
    assert oracle_mod.e4m3_quantize(1e6) == 0x7E and oracle_mod.e4m3_quantize(-1e6) == 0xFE


def test_per_token_quantisation_scale(oracle_mod):
    rng = _rng(18)
    rows = wl.round_bf16(rng.standard_normal((50, 512)).astype(np.float32))
    rows[3] = 0.0
    codes, scales = oracle_mod.quantize_rows(rows)
    amax = np.abs(rows).max(1)
    assert scales[3] == 1.0 and not codes[3].any()
    nz = amax > 0
    assert np.array_equal(scales[nz], (amax[nz] / np.float32(448.0)).astype(np.float32))
    # the largest element of every row lands on the largest code, 448
    for i in np.nonzero(nz)[0]:
        j = int(np.argmax(np.abs(rows[i])))
        assert codes[i, j] & 0x7F == 0x7E
    deq = oracle_mod.dequantize_rows(codes, scales)
    rel = np.abs(deq - rows) / np.maximum(amax[:, None], 1e-30)
    assert rel.max() <= 2.0 ** -4 + 1e-12  # half an e4m3 ulp at the top binade, relative to amax


# ---------------------------------------------------------------------------------------------
# Cache width (numbers the pages print)
# ---------------------------------------------------------------------------------------------

def _golden_cache_sizes():
    rows = {}
    with open(os.path.join(GOLDEN, "cache_sizes.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            name, params, value, unit, _src = [s.strip() for s in line.split("|")]
            kv = dict(p.split("=") for p in params.split())
            rows[name] = ({k: int(v) for k, v in kv.items()}, int(value), unit)
    return rows


def test_cache_row_width_matches_printed_sizes(oracle_mod):
    g = _golden_cache_sizes()
    row = oracle_mod.cache_row_elems
    assert row(512, 64) == g["mla_v2"][1] == wl.V3_DIMS.row
    assert row(512, 64) * 61 == g["mla_v3_61l"][1]
    assert round(row(512, 64) * 61 * 2 / 1000) - 1 <= g["mla_v3_61l_kb"][1] <= round(row(512, 64) * 61 * 2 / 1024) + 1
    assert 2 * 128 * 128 == g["mha_v2"][1] and 2 * 128 == g["mqa_v2"][1]
    assert 80 * 2 * 8 * 128 == g["llama3_70b"][1] and 80 * 2 * 8 * 128 * 2 // 1024 == g["llama3_70b_kb"][1]
    assert row(512, 64) * 2 == g["mla_576"][1]
    assert 2 * 32 * 128 * 2 == g["mha_32h"][1] and 2 * 8 * 128 * 2 == g["gqa8_32h"][1]
    assert 2 * 128 * 2 == g["mqa_32h"][1]
    assert row(512, 64) * 2 * 32 // 1024 == g["mla_32l_kib"][1]
    assert 2 * 32 * 128 * 2 * 32 // 1024 == g["mha_32l_kib"][1]
    # toy dims of the implementation section: 128 + 32 per token
    assert row(128, 32) == wl.TOY_DIMS.row == 160
