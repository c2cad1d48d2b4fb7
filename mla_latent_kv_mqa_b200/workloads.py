"""Seeded synthetic workloads for MLA decode.

This module only draws random numbers, rounds them to the storage format
(bf16 by round-to-nearest-even, or leaves fp32), and lays out sequence lengths
and block tables.  It holds none of the method's arithmetic (no RoPE, no
projection, no softmax, no quantisation), so both the CUDA path and the CPU
oracle can consume the same inputs.

The five workloads are the decode shapes the MLA pages discuss: the toy layer
of the itwiki "멀티 헤드 잠재 어텐션" implementation section (d=1024, n_h=8,
d_h=64, d_c=128, d_cq=256, d_R=32), and four DeepSeek-V3-shaped single-layer
decode batches (n_h=128, d_h=128, d_c=512, d_R=64; the V2/V3 settings table of
the same article) with a 64-token page.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

PAGE = 64


@dataclass
class MLADims:
    n_h: int
    d_h: int
    d_c: int
    d_r: int
    page: int = PAGE
    rope_base: float = 1e4

    @property
    def row(self) -> int:
        return self.d_c + self.d_r


V3_DIMS = MLADims(n_h=128, d_h=128, d_c=512, d_r=64)
TOY_DIMS = MLADims(n_h=8, d_h=64, d_c=128, d_r=32)


@dataclass
class DecodeWorkload:
    """One decode step of one layer.

    Arrays are float32 holding exactly-representable values of the storage dtype
    (bf16 values for the bf16 configs).  Context token j of sequence b sits at
    position j; the cache rows are given before RoPE (k_r) and are written into the
    paged cache by the append call.  The last ``s_q`` tokens of every sequence are
    the current (query) tokens, so the context includes them."""
    name: str
    dims: MLADims
    kv_dtype: str                     # "bf16", "fp8" (content e4m3 + bf16 RoPE key), "f32"
    act_dtype: str                    # "bf16" or "f32"
    s_q: int
    seq_lens: np.ndarray              # [B] int32, includes the current tokens
    q_c: np.ndarray                   # [B*s_q, n_h, d_h]
    q_r: np.ndarray                   # [B*s_q, n_h, d_r]  (before RoPE)
    q_pos: np.ndarray                 # [B*s_q] int32
    c_kv: np.ndarray                  # [sum L, d_c]
    k_r: np.ndarray                   # [sum L, d_r]  (before RoPE)
    ctx_off: np.ndarray               # [B+1] int64
    w_uk: np.ndarray                  # [n_h*d_h, d_c]
    w_uv: np.ndarray                  # [n_h*d_h, d_c]
    block_table: np.ndarray           # [B, max_blocks] int32
    num_blocks: int                   # physical blocks in the pool
    extra: dict = field(default_factory=dict)

    @property
    def B(self) -> int:
        return int(self.seq_lens.shape[0])

    @property
    def T(self) -> int:
        return self.B * self.s_q

    @property
    def max_blocks(self) -> int:
        return int(self.block_table.shape[1])

    def seq_c_kv(self, b: int) -> np.ndarray:
        return self.c_kv[self.ctx_off[b]:self.ctx_off[b + 1]]

    def seq_k_r(self, b: int) -> np.ndarray:
        return self.k_r[self.ctx_off[b]:self.ctx_off[b + 1]]

    def token_seq_pos(self) -> tuple[np.ndarray, np.ndarray]:
        """(sequence index, position) of every context token, in ctx order."""
        L = self.seq_lens.astype(np.int64)
        seq = np.repeat(np.arange(self.B, dtype=np.int32), L)
        pos = (np.arange(int(L.sum()), dtype=np.int64) - np.repeat(self.ctx_off[:-1], L)).astype(np.int32)
        return seq, pos


def round_bf16(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (nearest, ties to even), returned as float32."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    bits = x.view(np.uint32)
    lsb = (bits >> 16) & 1
    r = ((bits + np.uint32(0x7FFF) + lsb) & np.uint32(0xFFFF0000)).astype(np.uint32)
    return r.view(np.float32)


def _normal(rng, shape, std=1.0, bf16=True):
    x = rng.standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        x *= np.float32(std)
    return round_bf16(x) if bf16 else x


def make_block_table(rng, seq_lens, page=PAGE, permute=False, spare=0):
    """Block table [B, max_blocks] of distinct physical block ids.

    Contiguous: sequence b's pages take consecutive ids.  Permuted: every needed id
    and ``spare`` unreferenced ids are shuffled by a seeded permutation.  Unused table
    slots hold -1."""
    nblk = [(int(L) + page - 1) // page for L in seq_lens]
    max_blocks = max(nblk)
    total = sum(nblk) + spare
    ids = rng.permutation(total).astype(np.int32) if permute else np.arange(total, dtype=np.int32)
    bt = np.full((len(seq_lens), max_blocks), -1, dtype=np.int32)
    k = 0
    for b, n in enumerate(nblk):
        bt[b, :n] = ids[k:k + n]
        k += n
    return bt, total


def _decode_workload(name, dims, seq_lens, s_q, kv_dtype, act_dtype, rng, *, permute=False,
                     spare=0, token_scale=None, w_std=None):
    bf16 = act_dtype == "bf16"
    seq_lens = np.asarray(seq_lens, dtype=np.int32)
    B = len(seq_lens)
    T = B * s_q
    total = int(seq_lens.astype(np.int64).sum())
    ctx_off = np.zeros(B + 1, dtype=np.int64)
    ctx_off[1:] = np.cumsum(seq_lens.astype(np.int64))
    w_std = (1.0 / np.sqrt(dims.d_c)) if w_std is None else w_std
    w_uk = _normal(rng, (dims.n_h * dims.d_h, dims.d_c), w_std, bf16)
    w_uv = _normal(rng, (dims.n_h * dims.d_h, dims.d_c), w_std, bf16)
    q_c = _normal(rng, (T, dims.n_h, dims.d_h), 1.0, bf16)
    q_r = _normal(rng, (T, dims.n_h, dims.d_r), 1.0, bf16)
    rows = rng.standard_normal(size=(total, dims.row), dtype=np.float32)
    if token_scale is not None:
        rows *= token_scale(rng, total)[:, None].astype(np.float32)
    rows = round_bf16(rows) if (bf16 or kv_dtype != "f32") else rows
    c_kv = np.ascontiguousarray(rows[:, :dims.d_c])
    k_r = np.ascontiguousarray(rows[:, dims.d_c:])
    del rows
    q_pos = (np.repeat(seq_lens.astype(np.int64), s_q) - s_q + np.tile(np.arange(s_q), B)).astype(np.int32)
    bt, nb = make_block_table(rng, seq_lens, dims.page, permute=permute, spare=spare)
    return DecodeWorkload(name=name, dims=dims, kv_dtype=kv_dtype, act_dtype=act_dtype, s_q=s_q,
                          seq_lens=seq_lens, q_c=q_c, q_r=q_r, q_pos=q_pos, c_kv=c_kv, k_r=k_r,
                          ctx_off=ctx_off, w_uk=w_uk, w_uv=w_uv, block_table=bt, num_blocks=nb)


# ----------------------------------------------------------------------------------------------
# The five workloads.  ``scale`` < 1 shrinks batch/context for fast parity cases while keeping
# the structure (ragged tails, permuted tables, length mix).
# ----------------------------------------------------------------------------------------------

def toy_layer_inputs(seed: int = 1, B: int = 1, T: int = 256):
    """Toy layer: h ~ N(0,1) [B, T, 1024] and nn.Linear-shaped weights ~ N(0, 1/fan_in), fp32."""
    rng = np.random.default_rng(seed)
    d, n_h, d_h, d_c, d_cq, d_r = 1024, 8, 64, 128, 256, 32

    def w(out_f, in_f):
        return rng.standard_normal(size=(out_f, in_f), dtype=np.float32) * np.float32(1.0 / np.sqrt(in_f))

    W = dict(n_h=n_h, d_h=d_h, d_r=d_r, d_c=d_c, d=d, d_cq=d_cq,
             w_dq=w(d_cq, d), w_uq=w(n_h * d_h, d_cq), w_qr=w(n_h * d_r, d_cq),
             w_dkv=w(d_c, d), w_kr=w(d_r, d), w_uk=w(n_h * d_h, d_c), w_uv=w(n_h * d_h, d_c),
             w_o=w(d, n_h * d_h))
    h = rng.standard_normal(size=(B, T, d), dtype=np.float32)
    return h, W


def v3_decode(seed: int = 2, B: int = 16, L: int = 4096, permute: bool = False) -> DecodeWorkload:
    """DeepSeek-V3-shaped decode: uniform context, bf16 cache, N(0,1) latents."""
    rng = np.random.default_rng(seed)
    return _decode_workload("v3_b%d_l%d" % (B, L), V3_DIMS, [L] * B, 1, "bf16", "bf16", rng,
                            permute=permute)


def varlen_decode(seed: int = 3, B: int = 64, lo: int = 1024, hi: int = 16384,
                  spare: int = 8) -> DecodeWorkload:
    """Variable-length paged batch: L_b ~ U[lo, hi] integers, randomly permuted block table,
    ``spare`` unreferenced blocks."""
    rng = np.random.default_rng(seed)
    lens = rng.integers(lo, hi + 1, size=B)
    return _decode_workload("varlen_b%d_%d_%d" % (B, lo, hi), V3_DIMS, lens, 1, "bf16", "bf16",
                            rng, permute=True, spare=spare)


def long_decode(seed: int = 4, B: int = 4, L: int = 131072) -> DecodeWorkload:
    """Long-context decode: rows [c_kv; k_R] = s_t z with z ~ N(0,1), s_t ~ LogNormal(0, 0.5)."""
    rng = np.random.default_rng(seed)
    wl = _decode_workload("long_b%d_l%d" % (B, L), V3_DIMS, [L] * B, 1, "bf16", "bf16", rng,
                          token_scale=lambda r, n: r.lognormal(0.0, 0.5, size=n))
    wl.extra["lognormal_norms"] = True
    return wl


def mtp_fp8_decode(seed: int = 5, B: int = 128, L: int = 8192, s_q: int = 2) -> DecodeWorkload:
    """MTP/speculative decode: s_q=2 causal queries, content cache stored as FP8 e4m3 with a
    per-token fp32 scale (quantised by the append call), RoPE key kept bf16."""
    rng = np.random.default_rng(seed)
    return _decode_workload("mtp_fp8_b%d_l%d_sq%d" % (B, L, s_q), V3_DIMS, [L] * B, s_q, "fp8",
                            "bf16", rng)


def make_decode(seed: int, seq_lens, *, s_q: int = 1, kv_dtype: str = "bf16",
                act_dtype: str = "bf16", permute: bool = False, spare: int = 0,
                lognormal_tokens: bool = False, dims: MLADims = V3_DIMS,
                name: str = "custom") -> DecodeWorkload:
    """Any decode batch with the structure of the five workloads (ragged lengths, permuted
    tables, spare blocks, per-token norm spread)."""
    rng = np.random.default_rng(seed)
    ts = (lambda r, n: r.lognormal(0.0, 0.5, size=n)) if lognormal_tokens else None
    wl = _decode_workload(name, dims, list(seq_lens), s_q, kv_dtype, act_dtype, rng,
                          permute=permute, spare=spare, token_scale=ts)
    wl.extra["lognormal_norms"] = bool(lognormal_tokens)
    return wl


@dataclass
class PrefillWorkload:
    """Causal prefill of B prompts packed into T tokens (prompt b is tokens cu_seqlens[b] ..
    cu_seqlens[b+1]-1, token i of a prompt at position i).  Arrays as in DecodeWorkload:
    float32 holding bf16 values; q_r and k_r before RoPE."""
    name: str
    dims: MLADims
    seq_lens: np.ndarray              # [B] int32
    cu_seqlens: np.ndarray            # [B+1] int32
    q_c: np.ndarray                   # [T, n_h, d_h]
    q_r: np.ndarray                   # [T, n_h, d_r]
    c_kv: np.ndarray                  # [T, d_c]
    k_r: np.ndarray                   # [T, d_r]
    w_uk: np.ndarray                  # [n_h*d_h, d_c]
    w_uv: np.ndarray                  # [n_h*d_h, d_c]

    @property
    def B(self) -> int:
        return int(self.seq_lens.shape[0])

    @property
    def T(self) -> int:
        return int(self.cu_seqlens[-1])


def make_prefill(seed: int, seq_lens, dims: MLADims = V3_DIMS, name: str = "prefill") -> PrefillWorkload:
    """Prompts of the given lengths, V3-shaped by default: weights ~ N(0, 1/d_c), activations
    and latents ~ N(0, 1), all rounded to bf16 (the decode workloads' recipe)."""
    rng = np.random.default_rng(seed)
    seq_lens = np.asarray(seq_lens, dtype=np.int32)
    cu = np.zeros(len(seq_lens) + 1, dtype=np.int32)
    cu[1:] = np.cumsum(seq_lens)
    T = int(cu[-1])
    w_std = 1.0 / np.sqrt(dims.d_c)
    w_uk = _normal(rng, (dims.n_h * dims.d_h, dims.d_c), w_std)
    w_uv = _normal(rng, (dims.n_h * dims.d_h, dims.d_c), w_std)
    q_c = _normal(rng, (T, dims.n_h, dims.d_h))
    q_r = _normal(rng, (T, dims.n_h, dims.d_r))
    c_kv = _normal(rng, (T, dims.d_c))
    k_r = _normal(rng, (T, dims.d_r))
    return PrefillWorkload(name=name, dims=dims, seq_lens=seq_lens, cu_seqlens=cu, q_c=q_c, q_r=q_r,
                           c_kv=c_kv, k_r=k_r, w_uk=w_uk, w_uv=w_uv)


CONFIGS = {
    "toy": dict(desc="Toy MLA layer d=1024 n_h=8 d_h=64 d_c=128 d_cq=256 d_R=32, B=1, ctx 256, fp32"),
    "v3": dict(desc="DeepSeek-V3-shaped decode n_h=128 d_h=128 d_c=512 d_R=64, bf16, B=16, ctx 4096, page 64"),
    "varlen": dict(desc="V3 dims, B=64, ctx U[1024,16384], permuted block table, bf16"),
    "long": dict(desc="V3 dims, B=4, ctx 131072, per-token norms LogNormal(0,0.5), bf16"),
    "mtp_fp8": dict(desc="V3 dims, B=128, ctx 8192, s_q=2 causal, FP8 e4m3 content + bf16 RoPE key"),
}
