"""Sequence split of a long-context decode across GPUs: one process per GPU, each holding a
contiguous range of every sequence's pages.

The MLA article's 한계 (limitations) section notes that every head reads the whole latent
cache, so splitting heads across GPUs (tensor parallelism) cannot shard it.  Splitting the
context can: rank i runs mla_decode (s_q = 1) over its own pages and the ranks' results merge
exactly by their log-sum-exp (include/mla.h, mla_lse_merge_prepare / _finish).  The RoPE key
is cached already rotated at its absolute position, so a rank's pages need no adjustment;
the query is the same on every rank.

What crosses ranks per step: one all-reduce(max) of lse [rows, n_h] and one all-reduce(sum)
of [rows, n_h, d_c + 1] fp32 (w o_lat and w), through torch.distributed (NCCL on GPUs).
"""
from __future__ import annotations

import numpy as np

from . import native as N


def page_bounds(seq_lens, world: int, page: int = 64) -> np.ndarray:
    """[world + 1, B] page boundaries: rank i holds pages bounds[i, b] .. bounds[i + 1, b] - 1 of
    sequence b, a near-even contiguous split of its ceil(L_b / page) pages.  Every rank must hold
    at least one page of every sequence (the split is meant for long contexts)."""
    L = np.asarray(seq_lens, dtype=np.int64)
    P = (L + page - 1) // page
    if world < 1 or (P < world).any():
        raise ValueError(f"every sequence needs at least {world} pages to split over {world} ranks")
    r = np.arange(world + 1, dtype=np.int64)[:, None]
    return (r * P[None, :]) // world


def token_ranges(seq_lens, bounds: np.ndarray, rank: int, page: int = 64):
    """(first token, token count) of every sequence on ``rank``: tokens page*bounds[rank] ..
    min(page*bounds[rank+1], L) - 1."""
    L = np.asarray(seq_lens, dtype=np.int64)
    t0 = bounds[rank] * page
    t1 = np.minimum(bounds[rank + 1] * page, L)
    return t0, t1 - t0


def local_block_table(global_table: np.ndarray, bounds: np.ndarray, rank: int) -> np.ndarray:
    """The rows of a block table restricted to this rank's pages, left-aligned and padded with
    -1: the table mla_decode takes for the rank's share of each sequence."""
    p0, p1 = bounds[rank], bounds[rank + 1]
    n = int((p1 - p0).max())
    out = np.full((global_table.shape[0], n), -1, dtype=np.int32)
    for b in range(global_table.shape[0]):
        out[b, :p1[b] - p0[b]] = global_table[b, p0[b]:p1[b]]
    return out


def merge(o_lat, lse, group=None, stream=None, prepare=None, finish=None):
    """Exact merge over the ranks of ``group`` of this rank's (o_lat [rows, n_h, d_c], lse
    [rows, n_h]) from mla_decode over its own pages; returns the merged (o_lat, lse), the same
    on every rank.  The two per-rank steps run in libmla's kernels on CUDA tensors;
    ``prepare`` / ``finish`` replace them only where the caller supplies its own."""
    import torch
    import torch.distributed as dist
    rows, n_h, d_c = o_lat.shape
    if prepare is None or finish is None:
        if not (o_lat.is_cuda and lse.is_cuda):
            raise ValueError("merge: the library's kernels need CUDA tensors")
        prepare = lambda o, l, m, a: N.mla_lse_merge_prepare(rows, n_h, d_c, o, l, m, a, stream)
        finish = lambda a, m, o, l: N.mla_lse_merge_finish(rows, n_h, d_c, a, m, o, l, stream)
    lse = lse.contiguous()
    lse_max = lse.clone()
    dist.all_reduce(lse_max, op=dist.ReduceOp.MAX, group=group)
    acc = torch.empty(rows * n_h * (d_c + 1), dtype=torch.float32, device=o_lat.device)
    prepare(o_lat.contiguous(), lse, lse_max, acc)
    dist.all_reduce(acc, op=dist.ReduceOp.SUM, group=group)
    out = torch.empty_like(o_lat)
    out_lse = torch.empty_like(lse)
    finish(acc, lse_max, out, out_lse)
    return out, out_lse
