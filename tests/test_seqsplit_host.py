"""Sequence split of a decode across ranks, host side, on CPU ranks over gloo.

Each rank attends over a contiguous range of every sequence's pages; the ranks' partial
(o_lat, lse) merge by their log-sum-exp (MLA article, 한계 section: the cache cannot be
sharded by heads, so long contexts split by tokens).  Here the partials come from the fp64
oracle run on each rank's tokens alone, the per-rank merge steps are torch stand-ins of the
library's two kernels, and the collectives are gloo's: the merged result must equal the
oracle's decode over whole sequences.

The oracle places token j of the sequences it is given at position j; a rank's tokens start
at t0, so it is given the query position q_pos - t0.  RoPE scores depend on the distance
between positions only, and every token of the rank stays visible (q_pos - t0 >= its last
local index), so the rank's scores are those of the full decode.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from mla_latent_kv_mqa_b200 import seqsplit as S
from mla_latent_kv_mqa_b200 import workloads as W

SEQ_LENS = [1000, 650, 1300]   # ragged tails; 16, 11 and 21 pages of 64


def _prepare(o, l, m, acc):
    rows, n_h, d_c = o.shape
    w = torch.where(torch.isneginf(l) | torch.isneginf(m), torch.zeros_like(l), torch.exp(l - m))
    acc[:rows * n_h * d_c] = (w[..., None] * o).reshape(-1)
    acc[rows * n_h * d_c:] = w.reshape(-1)


def _finish(acc, m, o, l):
    rows, n_h, d_c = o.shape
    s = acc[rows * n_h * d_c:].reshape(rows, n_h)
    inv = torch.where(s > 0, 1.0 / s, torch.zeros_like(s))
    o.copy_(acc[:rows * n_h * d_c].reshape(rows, n_h, d_c) * inv[..., None])
    l.copy_(torch.where(s > 0, m + torch.log(s), torch.full_like(s, -float("inf"))))


def _workload():
    return W.make_decode(31, SEQ_LENS, dims=W.TOY_DIMS, act_dtype="f32", kv_dtype="f32", name="split")


def _partial(orc, wl, bounds, rank):
    """The fp64 oracle over this rank's tokens of every sequence."""
    t0, n = S.token_ranges(wl.seq_lens, bounds, rank, wl.dims.page)
    cs = [wl.seq_c_kv(b)[t0[b]:t0[b] + n[b]] for b in range(wl.B)]
    ks = [wl.seq_k_r(b)[t0[b]:t0[b] + n[b]] for b in range(wl.B)]
    r = orc.decode_absorbed(wl.q_c, wl.q_r, wl.q_pos - t0, cs, ks, wl.w_uk, wl.w_uv,
                            rope_base=wl.dims.rope_base)
    return r


def _full(orc, wl):
    return orc.decode_absorbed(wl.q_c, wl.q_r, wl.q_pos, [wl.seq_c_kv(b) for b in range(wl.B)],
                               [wl.seq_k_r(b) for b in range(wl.B)], wl.w_uk, wl.w_uv,
                               rope_base=wl.dims.rope_base)


def test_page_bounds_cover_every_page_once_near_evenly():
    L = [64 * 5, 64 * 7 + 1, 64 * 64, 10000]
    for world in (1, 2, 3, 4, 5):
        b = S.page_bounds(L, world)
        P = (np.asarray(L) + 63) // 64
        assert b.shape == (world + 1, len(L))
        assert (b[0] == 0).all() and (b[-1] == P).all()
        cnt = np.diff(b, axis=0)
        assert (cnt >= 1).all() and (cnt.max(0) - cnt.min(0) <= 1).all()
        tot = sum(S.token_ranges(L, b, r)[1] for r in range(world))
        assert (tot == np.asarray(L)).all()
    with pytest.raises(ValueError):
        S.page_bounds([64 * 3], 4)


def test_local_block_table_is_the_ranks_slice_left_aligned():
    rng = np.random.default_rng(0)
    L = [64 * 9 + 5, 64 * 4]
    bt, _ = W.make_block_table(rng, L, permute=True)
    b = S.page_bounds(L, 3)
    for r in range(3):
        loc = S.local_block_table(bt, b, r)
        for s in range(2):
            k = b[r + 1, s] - b[r, s]
            assert (loc[s, :k] == bt[s, b[r, s]:b[r + 1, s]]).all()
            assert (loc[s, k:] == -1).all()


def test_partials_reproduce_the_full_decode_on_one_process(oracle_mod):
    """No process group: the same merge arithmetic over all ranks' partials at once."""
    wl = _workload()
    full = _full(oracle_mod, wl)
    for world in (2, 3):
        b = S.page_bounds(wl.seq_lens, world)
        parts = [_partial(oracle_mod, wl, b, r) for r in range(world)]
        lse = np.stack([p.lse for p in parts])
        m = lse.max(0)
        w = np.exp(lse - m)
        o = sum(w[r][..., None] * parts[r].o_lat for r in range(world)) / w.sum(0)[..., None]
        assert np.abs(o - full.o_lat).max() <= 1e-11
        assert np.abs(m + np.log(w.sum(0)) - full.lse).max() <= 1e-11
        # each rank alone is NOT the answer (the split is real)
        assert np.abs(parts[0].o_lat - full.o_lat).max() > 1e-3


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_o, out_l):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from oracle import oracle as orc
        wl = _workload()
        b = S.page_bounds(wl.seq_lens, world)
        p = _partial(orc, wl, b, rank)
        o, l = S.merge(torch.from_numpy(p.o_lat).float(), torch.from_numpy(p.lse).float(),
                       prepare=_prepare, finish=_finish)
        out_o[rank].copy_(o)
        out_l[rank].copy_(l)
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_gloo_ranks_merge_to_the_full_decode(oracle_mod, world):
    wl = _workload()
    d = wl.dims
    out_o = torch.zeros(world, wl.B, d.n_h, d.d_c).share_memory_()
    out_l = torch.zeros(world, wl.B, d.n_h).share_memory_()
    mp.spawn(_rank_main, args=(world, _free_port(), out_o, out_l), nprocs=world, join=True)
    full = _full(oracle_mod, wl)
    for r in range(world):
        assert torch.equal(out_o[r], out_o[0]) and torch.equal(out_l[r], out_l[0])
    # fp32 merge of fp64 partials: a few ulp of fp32 on values of order 1
    assert np.abs(out_o[0].double().numpy() - full.o_lat).max() <= 1e-5
    assert np.abs(out_l[0].double().numpy() - full.lse).max() <= 1e-5


def test_merge_without_kernels_on_cpu_tensors_refuses():
    with pytest.raises(ValueError):
        S.merge(torch.zeros(1, 1, 4), torch.zeros(1, 1))
