"""Shared helpers for the GPU tests: run the CUDA path on a workload, run the oracle on a
subset of it, and compare."""
from __future__ import annotations

import numpy as np
import torch

from mla_latent_kv_mqa_b200 import workloads as W


def rel_l2(x, ref) -> float:
    x = np.asarray(x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    return float(np.linalg.norm(x - ref) / max(np.linalg.norm(ref), 1e-300))


def max_abs(x, ref) -> float:
    return float(np.max(np.abs(np.asarray(x, dtype=np.float64) - np.asarray(ref, dtype=np.float64))))


# Tolerances of the bf16 path: relative L2 <= 4e-3 and max |err| <= 2e-2 on o_lat and o, and
# |err(lse)| <= 1e-2.  Workloads whose per-token norms are log-normal (the long-context recipe)
# use max |err| <= 2e-2 * max(1, max |ref|) and |err(lse)| <= 1e-2 * max(1, |lse|) instead:
# tests/test_tolerance_reading.py shows that exact arithmetic on the bf16 operands the C ABI
# defines already exceeds the flat bounds there, and stays far inside them on N(0,1) latents.
# FP8 content cache: relative L2 <= 3e-2 against the oracle on its own dequantised cache.
BF16_REL, BF16_ABS, FP8_REL, LSE_ABS = 4e-3, 2e-2, 3e-2, 1e-2


def scaled_max_abs(x, ref):
    """max |x - ref| / max(1, max |ref|)."""
    x = np.asarray(x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    return float(np.abs(x - ref).max() / max(1.0, float(np.abs(ref).max())))


def check_step(got, ref, rows, heads, rel_tol, abs_tol, *, lognormal=False):
    """Compare one step's (o_lat, lse, o) on the given rows and heads with the oracle's.

    ``lognormal``: the workload's per-token norms are log-normal; the max-abs and lse bounds
    scale with the output (see the tolerance note above).  Both the plain and the scaled
    errors are always reported in the assertion message."""
    q_abs, o_lat, lse, o = got
    o_lat = o_lat.cpu().numpy()[rows][:, heads]
    o = o.float().cpu().numpy()[rows][:, heads]
    lse = lse.cpu().numpy()[rows][:, heads]
    dl = np.abs(lse.astype(np.float64) - ref.lse)
    e = dict(o_lat_rel=rel_l2(o_lat, ref.o_lat), o_rel=rel_l2(o, ref.o),
             o_lat_abs=max_abs(o_lat, ref.o_lat), o_abs=max_abs(o, ref.o),
             o_lat_scaled=scaled_max_abs(o_lat, ref.o_lat), o_scaled=scaled_max_abs(o, ref.o),
             lse_abs=float(dl.max()), lse_scaled=float(np.max(dl / np.maximum(1.0, np.abs(ref.lse)))),
             bounds="scaled (log-normal norms)" if lognormal else "flat")
    assert e["o_lat_rel"] <= rel_tol and e["o_rel"] <= rel_tol, e
    k = "_scaled" if lognormal else "_abs"
    if abs_tol is not None:
        assert e["o_lat" + k] <= abs_tol and e["o" + k] <= abs_tol, e
    assert e["lse" + k] <= LSE_ABS, e
    return e


def _act(x: np.ndarray, act: str, dev):
    t = torch.from_numpy(np.ascontiguousarray(x))
    return t.to(device=dev, dtype=torch.bfloat16 if act == "bf16" else torch.float32)


class GpuRun:
    """Device state of one workload: cache filled through mla_cache_append, then one step."""

    def __init__(self, wl: W.DecodeWorkload, flags: int = 0, poison: bool = True, dev="cuda",
                 block_table=None):
        from mla_latent_kv_mqa_b200 import layer as Lyr
        self.wl = wl
        d = wl.dims
        self.dims = Lyr.dims_for(d.n_h, d.d_h, d.d_c, d.d_r, act=wl.act_dtype, kv=wl.kv_dtype,
                                 page=d.page, rope_base=d.rope_base, flags=flags)
        self.layer = Lyr.MLADecodeLayer(self.dims, _act(wl.w_uk, wl.act_dtype, dev),
                                        _act(wl.w_uv, wl.act_dtype, dev))
        bt = wl.block_table if block_table is None else block_table
        self.block_table = torch.from_numpy(np.ascontiguousarray(bt)).to(dev)
        self.cache = Lyr.PagedLatentCache(self.dims, wl.num_blocks, dev, poison=poison)
        self.seq_lens = torch.from_numpy(wl.seq_lens.astype(np.int32)).to(dev)
        self.max_seq_len = int(wl.seq_lens.max())
        seq, pos = wl.token_seq_pos()
        self.tok_seq = torch.from_numpy(seq).to(dev)
        self.tok_pos = torch.from_numpy(pos).to(dev)
        self.c_kv = _act(wl.c_kv, wl.act_dtype, dev)
        self.k_r = _act(wl.k_r, wl.act_dtype, dev)
        self.q_c = _act(wl.q_c, wl.act_dtype, dev)
        self.q_r = _act(wl.q_r, wl.act_dtype, dev)
        self.q_pos = torch.from_numpy(wl.q_pos.astype(np.int32)).to(dev)

    def fill_cache(self):
        self.layer.append(self.cache, self.c_kv, self.k_r, self.tok_seq, self.tok_pos, self.block_table)

    def step(self, out_dtype="f32"):
        q_abs = self.layer.absorb(self.q_c, self.q_r, self.q_pos)
        o_lat, lse = self.layer.decode(self.cache, q_abs, self.block_table, self.seq_lens,
                                       self.wl.s_q, self.max_seq_len)
        o = self.layer.out_proj(o_lat, out_dtype)
        torch.cuda.synchronize()
        return q_abs, o_lat, lse, o


def oracle_cache_rows(wl: W.DecodeWorkload, orc, seqs):
    """Per-sequence cache content as the oracle sees it (FP8: its own quantise/dequantise)."""
    cs, ks = [], []
    for b in seqs:
        c = wl.seq_c_kv(b)
        if wl.kv_dtype == "fp8":
            codes, scales = orc.quantize_rows(c)
            c = orc.dequantize_rows(codes, scales)
        cs.append(np.asarray(c, dtype=np.float64))
        ks.append(np.asarray(wl.seq_k_r(b), dtype=np.float64))
    return cs, ks


def oracle_ref(wl: W.DecodeWorkload, orc, seqs=None, heads=None, naive=False):
    """Oracle (absorbed mode; naive on request) for sequences ``seqs`` and heads ``heads``."""
    seqs = list(range(wl.B)) if seqs is None else list(seqs)
    d = wl.dims
    heads = np.arange(d.n_h) if heads is None else np.asarray(heads)
    rows = np.array([b * wl.s_q + i for b in seqs for i in range(wl.s_q)])
    wsel = (heads[:, None] * d.d_h + np.arange(d.d_h)[None, :]).reshape(-1)
    cs, ks = oracle_cache_rows(wl, orc, seqs)
    args = (wl.q_c[rows][:, heads], wl.q_r[rows][:, heads], wl.q_pos[rows], cs, ks,
            wl.w_uk[wsel], wl.w_uv[wsel])
    if naive:
        return rows, heads, orc.decode_naive(*args, s_q=wl.s_q, rope_base=d.rope_base)
    return rows, heads, orc.decode_absorbed(*args, s_q=wl.s_q, rope_base=d.rope_base)
