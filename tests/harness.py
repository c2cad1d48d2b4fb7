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
# use max |err| <= 2e-2 * max(1, max |ref|) and |err(lse)| <= 1e-2 * max(1, |lse|) instead, and
# hold the relative L2 bound against the oracle run on the bf16 operands the C ABI defines
# (rounded_operand_ref): tests/test_tolerance_reading.py shows that exact arithmetic on those
# operands already exceeds the flat bounds there -- and on some seeds the relative L2 bound as
# well -- while it stays far inside all of them on N(0,1) latents.
# FP8 content cache: relative L2 <= 3e-2 against the oracle on its own dequantised cache.
BF16_REL, BF16_ABS, FP8_REL, LSE_ABS = 4e-3, 2e-2, 3e-2, 1e-2


def scaled_max_abs(x, ref):
    """max |x - ref| / max(1, max |ref|)."""
    x = np.asarray(x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    return float(np.abs(x - ref).max() / max(1.0, float(np.abs(ref).max())))


def check_step(got, ref, rows, heads, rel_tol, abs_tol, *, lognormal=False, ref_ops=None):
    """Compare one step's (o_lat, lse, o) on the given rows and heads with the oracle's.

    ``lognormal``: the workload's per-token norms are log-normal; the max-abs and lse bounds
    scale with the output (see the tolerance note above).  ``ref_ops``: the oracle on the
    boundary's bf16 operands (rounded_operand_ref); when given, the relative L2 bound applies
    against it (the kernel's own error) and is also reported against ``ref``.  Both the plain
    and the scaled errors are always reported in the assertion message."""
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
    rel = (e["o_lat_rel"], e["o_rel"])
    if ref_ops is not None:
        e["o_lat_rel_vs_operands"] = rel_l2(o_lat, ref_ops.o_lat)
        e["o_rel_vs_operands"] = rel_l2(o, ref_ops.o)
        rel = (e["o_lat_rel_vs_operands"], e["o_rel_vs_operands"])
    assert rel[0] <= rel_tol and rel[1] <= rel_tol, e
    k = "_scaled" if lognormal else "_abs"
    if abs_tol is not None:
        assert e["o_lat" + k] <= abs_tol and e["o" + k] <= abs_tol, e
    assert e["lse" + k] <= LSE_ABS, e
    return e


def bf16_round(x):
    """Round to bf16 (nearest even) and return float64."""
    return torch.from_numpy(np.asarray(x, dtype=np.float32)).to(torch.bfloat16).double().numpy()


def rope_rows(x, pos, base=1e4):
    """Half-split rotation of the rows of x [n, d] by angles pos[n] * base^(-2k/d) (the MLA
    article's implementation-section pairing), vectorised; used only to prepare rounded
    oracle inputs."""
    d = x.shape[1]
    half = d // 2
    ang = np.asarray(pos, dtype=np.float64)[:, None] * base ** (-2.0 * np.arange(half) / d)[None, :]
    c, s = np.cos(ang), np.sin(ang)
    a, b = x[:, :half], x[:, half:]
    return np.concatenate([a * c - b * s, b * c + a * s], 1)


def rounded_operand_ref(wl: W.DecodeWorkload, orc, seqs, heads):
    """The fp64 oracle on the operands the C ABI fixes for the bf16 path: the absorbed query
    q_lat and the rotated RoPE query rounded to bf16 (what mla_absorb_q writes), the rotated
    RoPE key rounded to bf16 (what mla_cache_append stores); every other step exact.  s_q = 1:
    q_lat is rounded by a rank-one update of each head's W^UK (one query row per head), the
    rotations by handing the oracle RoPE(bf16(RoPE(x, p)), -p).  Returns (rows, heads, result)
    like oracle_ref."""
    from oracle.oracle import DecodeResult
    assert wl.s_q == 1 and wl.kv_dtype == "bf16"
    d = wl.dims
    heads = np.asarray(heads)
    wsel = (heads[:, None] * d.d_h + np.arange(d.d_h)[None, :]).reshape(-1)
    wuk = wl.w_uk[wsel].astype(np.float64)
    wuv = wl.w_uv[wsel].astype(np.float64)
    outs = []
    for b in seqs:
        qc = wl.q_c[[b]][:, heads].astype(np.float64)
        qr = wl.q_r[[b]][:, heads].astype(np.float64)
        c = wl.seq_c_kv(b).astype(np.float64)
        k = wl.seq_k_r(b).astype(np.float64)
        qp = wl.q_pos[[b]]
        exact = orc.decode_absorbed(qc, qr, qp, [c], [k], wuk, wuv, rope_base=d.rope_base)
        tgt = bf16_round(exact.q_lat)
        w2 = wuk.reshape(len(heads), d.d_h, d.d_c).copy()
        for i in range(len(heads)):
            q = qc[0, i]
            w2[i] += np.outer(q, tgt[0, i] - exact.q_lat[0, i]) / (q @ q)
        pq = np.full(len(heads), int(qp[0]))
        qr2 = rope_rows(bf16_round(rope_rows(qr[0], pq, d.rope_base)), -pq, d.rope_base)[None]
        j = np.arange(c.shape[0])
        k2 = rope_rows(bf16_round(rope_rows(k, j, d.rope_base)), -j, d.rope_base)
        outs.append(orc.decode_absorbed(qc, qr2, qp, [c], [k2], w2.reshape(-1, d.d_c), wuv, rope_base=d.rope_base))
    res = DecodeResult(o=np.concatenate([r.o for r in outs]), lse=np.concatenate([r.lse for r in outs]),
                       o_lat=np.concatenate([r.o_lat for r in outs]))
    return np.asarray(list(seqs)), heads, res


def operands_ref(wl: W.DecodeWorkload, orc, rows, heads):
    """rounded_operand_ref where the relative bound is applied against it (bf16 cache, s_q = 1,
    log-normal norms), else None."""
    if wl.extra.get("lognormal_norms", False) and wl.kv_dtype == "bf16" and wl.s_q == 1:
        return rounded_operand_ref(wl, orc, list(rows), heads)[2]
    return None


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


class PrefillRun:
    """Device state of one prefill workload and the call through the C ABI."""

    def __init__(self, wl: W.PrefillWorkload, dev="cuda"):
        from mla_latent_kv_mqa_b200 import layer as Lyr
        self.wl = wl
        d = wl.dims
        self.dims = Lyr.dims_for(d.n_h, d.d_h, d.d_c, d.d_r, act="bf16", kv="bf16", page=d.page,
                                 rope_base=d.rope_base)
        self.layer = Lyr.MLADecodeLayer(self.dims, _act(wl.w_uk, "bf16", dev), _act(wl.w_uv, "bf16", dev))
        self.cu = torch.from_numpy(wl.cu_seqlens.astype(np.int32)).to(dev)
        self.max_len = int(wl.seq_lens.max())
        self.q_c = _act(wl.q_c, "bf16", dev)
        self.q_r = _act(wl.q_r, "bf16", dev)
        self.c_kv = _act(wl.c_kv, "bf16", dev)
        self.k_r = _act(wl.k_r, "bf16", dev)

    def run(self, o=None, lse=None):
        o, lse = self.layer.prefill(self.q_c, self.q_r, self.c_kv, self.k_r, self.cu, self.max_len, o=o, lse=lse)
        torch.cuda.synchronize()
        return o, lse


def prefill_oracle_rows(wl: W.PrefillWorkload, orc, rows, heads):
    """Naive-mode (MHA) oracle for the given (prompt, token) rows and heads: each sampled row is
    a one-query problem whose context is its prompt's tokens 0..t."""
    d = wl.dims
    heads = np.asarray(heads)
    wsel = (heads[:, None] * d.d_h + np.arange(d.d_h)[None, :]).reshape(-1)
    glob = np.array([wl.cu_seqlens[b] + t for b, t in rows])
    cs = [np.asarray(wl.c_kv[wl.cu_seqlens[b]:wl.cu_seqlens[b] + t + 1], dtype=np.float64) for b, t in rows]
    ks = [np.asarray(wl.k_r[wl.cu_seqlens[b]:wl.cu_seqlens[b] + t + 1], dtype=np.float64) for b, t in rows]
    pos = np.array([t for _, t in rows], dtype=np.int64)
    ref = orc.decode_naive(wl.q_c[glob][:, heads], wl.q_r[glob][:, heads], pos, cs, ks, wl.w_uk[wsel],
                           wl.w_uv[wsel], s_q=1, rope_base=d.rope_base)
    return glob, heads, ref
