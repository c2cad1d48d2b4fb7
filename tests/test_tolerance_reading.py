"""What the parity bounds can ask of a kernel whose boundary fixes bf16 operands.

The bf16 path's operands are bf16 by definition of the C ABI: the absorbed query
q_abs = [W^UK_h^T q^C ; RoPE(q^R)] that mla_absorb_q writes and mla_decode reads, and the
cached row [c^KV ; RoPE(k^R)] that mla_cache_append writes (MLA article, 분리 RoPE section:
the cache holds c^KV and the rotated shared key).  This test runs the fp64 oracle on those
operands, rounded exactly as the boundary rounds them and with every other step exact, and
compares it with the oracle on the unrounded inputs.  The difference is the error floor of
ANY kernel behind this boundary, before a single rounding of its own.

Findings pinned here, which decide how tests/harness.check_step applies the bounds:
* N(0,1) latents (the DeepSeek-V3-shaped workload): max |err| of o_lat and o stays far below
  the flat 2e-2 bound and |err(lse)| far below 1e-2, so those cases use the flat bounds.
* Per-token norms LogNormal(0, 0.5) (the long-context workload's recipe): outputs reach
  |o_lat| ~ 20 and lse ~ 9..22, and the rounding alone moves single elements of o_lat by more
  than 2e-2 and lse by more than 1e-2.  No kernel can meet the flat bounds there, so those
  cases (and only those) use max |err| <= 2e-2 * max(1, max |ref|) and
  |err(lse)| <= 1e-2 * max(1, |lse|).  The relative L2 of the rounding alone is 3.5e-3 on
  seed 23 but 4.4e-3 on seed 64, above the 4e-3 bound: on these cases the relative bound
  is held against the oracle on the rounded operands (the kernel's own error).

The rounding is applied to the oracle's INPUTS only (oracle/ is unchanged):
* q_lat: the oracle forms q_lat = W^UK_h^T q^C itself, so W^UK_h gets the rank-one update
  q^C (bf16(q_lat) - q_lat)^T / |q^C|^2, after which W'^T q^C = bf16(q_lat) (one query row
  per head: B = 1, s_q = 1).
* the rotated query and key: the oracle rotates q^R and k^R itself, so it is given
  RoPE(bf16(RoPE(x, p)), -p), whose rotation by p is bf16(RoPE(x, p)).
"""
import numpy as np
import pytest

from mla_latent_kv_mqa_b200 import workloads as W

FLAT_ABS, REL, LSE_ABS = 2e-2, 4e-3, 1e-2


from tests.harness import bf16_round as _bf16
from tests.harness import rope_rows as _rope_np


def _floor(orc, L, lognormal, seed, heads):
    wl = W.make_decode(seed, [L], lognormal_tokens=lognormal)
    d = wl.dims
    hs = np.asarray(heads)
    wsel = (hs[:, None] * d.d_h + np.arange(d.d_h)[None, :]).reshape(-1)
    qc = wl.q_c[:, hs].astype(np.float64)
    qr = wl.q_r[:, hs].astype(np.float64)
    c = wl.c_kv.astype(np.float64)
    k = wl.k_r.astype(np.float64)
    wuk = wl.w_uk[wsel].astype(np.float64)
    wuv = wl.w_uv[wsel].astype(np.float64)
    exact = orc.decode_absorbed(qc, qr, wl.q_pos, [c], [k], wuk, wuv)

    w2 = wuk.reshape(len(hs), d.d_h, d.d_c).copy()
    tgt = _bf16(exact.q_lat)
    for i in range(len(hs)):
        q = qc[0, i]
        w2[i] += np.outer(q, tgt[0, i] - exact.q_lat[0, i]) / (q @ q)
    w2 = w2.reshape(-1, d.d_c)
    pos = int(wl.q_pos[0])
    pq = np.full(len(hs), pos)
    qr2 = _rope_np(_bf16(_rope_np(qr[0], pq)), -pq)[None]
    j = np.arange(L)
    k2 = _rope_np(_bf16(_rope_np(k, j)), -j)
    rounded = orc.decode_absorbed(qc, qr2, wl.q_pos, [c], [k2], w2, wuv)
    # the rank-one update reproduces bf16(q_lat) to fp64 rounding
    assert np.max(np.abs(rounded.q_lat - tgt)) <= 1e-12 * max(1.0, float(np.abs(tgt).max()))
    return exact, rounded


def _errors(exact, rounded):
    e = {}
    for nm in ("o_lat", "o"):
        x, r = getattr(rounded, nm), getattr(exact, nm)
        err = np.abs(x - r)
        e[nm + "_abs"] = float(err.max())
        e[nm + "_scaled"] = float(err.max() / max(1.0, float(np.abs(r).max())))
        e[nm + "_rel"] = float(np.linalg.norm(x - r) / np.linalg.norm(r))
        e[nm + "_max"] = float(np.abs(r).max())
    dl = np.abs(rounded.lse - exact.lse)
    e["lse_abs"] = float(dl.max())
    e["lse_scaled"] = float((dl / np.maximum(1.0, np.abs(exact.lse))).max())
    return e


def test_normal_latents_meet_the_flat_bounds_with_margin(oracle_mod):
    """DeepSeek-V3-shaped N(0,1) workload, one 4096-token sequence, all 128 heads."""
    e = _errors(*_floor(oracle_mod, 4096, False, 2, range(128)))
    assert e["o_lat_abs"] < FLAT_ABS / 10 and e["o_abs"] < FLAT_ABS / 10, e
    assert e["lse_abs"] < LSE_ABS / 10, e
    assert e["o_lat_rel"] < REL and e["o_rel"] < REL, e


@pytest.mark.parametrize("L,seed,heads", [(3000, 23, 128), (131072, 4, 8)],
                         ids=["parity_case_3000", "long_context_131072"])
def test_lognormal_norms_exceed_the_flat_bounds_by_rounding_alone(oracle_mod, L, seed, heads):
    """Per-token norms LogNormal(0, 0.5): the 3000-token case is the GPU parity case of this
    recipe; the 131072-token sequence has the long-context workload's length."""
    e = _errors(*_floor(oracle_mod, L, True, seed, range(heads)))
    assert e["o_lat_max"] > 15.0, e                       # outputs reach ~20
    assert e["o_lat_abs"] > FLAT_ABS, e                   # the flat bound is out of reach ...
    assert e["lse_abs"] > LSE_ABS, e
    assert e["o_lat_scaled"] <= FLAT_ABS / 2, e           # ... the scaled one is met with margin
    assert e["o_scaled"] <= FLAT_ABS / 2, e
    assert e["lse_scaled"] <= LSE_ABS / 2, e
    assert e["o_lat_rel"] < REL and e["o_rel"] < REL, e


def test_lognormal_rounding_alone_can_exceed_the_relative_bound(oracle_mod):
    """Seed 64 of the same recipe (3000 tokens, all heads): rounding alone moves o_lat and o
    by more than 4e-3 in relative L2.  So on log-normal norms the relative bound is applied to
    the kernel's own error, against the oracle on the rounded operands (the `rounded` result
    here, tests/harness.rounded_operand_ref in the GPU tests)."""
    e = _errors(*_floor(oracle_mod, 3000, True, 64, range(128)))
    assert e["o_lat_rel"] > REL and e["o_rel"] > REL, e
    assert e["o_lat_scaled"] <= FLAT_ABS and e["lse_scaled"] <= LSE_ABS, e
