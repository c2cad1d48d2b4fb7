"""Sequence split of a decode on the GPU, through the C ABI.

A deployment runs one rank per GPU, each holding a contiguous range of every sequence's pages
(MLA article, 한계 section: heads cannot shard the latent cache, tokens can).  With one GPU
here, the ranks are emulated one after another on the same device: each runs mla_decode with
its own block table (its slice of the sequence's pages) and token count, then
mla_lse_merge_prepare; torch's elementwise max and sum stand in for the two all-reduces; and
mla_lse_merge_finish completes the merge.  No kernel waits on another.  The merged result is
held to the same bounds against the fp64 oracle (whole sequences) as the unsplit decode.
"""
import os
import socket

import numpy as np
import pytest
import torch

from mla_latent_kv_mqa_b200 import native as N
from mla_latent_kv_mqa_b200 import seqsplit as S
from mla_latent_kv_mqa_b200 import workloads as W
from tests.harness import BF16_ABS, BF16_REL, FP8_REL, GpuRun, check_step, operands_ref, oracle_ref, rel_l2

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from mla_latent_kv_mqa_b200 import build
    build.build()
    torch.backends.cuda.matmul.allow_tf32 = False


def _split_decode(run, q_abs, world):
    """o_lat, lse of every emulated rank, and the merged pair."""
    wl = run.wl
    d = run.dims
    rows = wl.B
    bounds = S.page_bounds(wl.seq_lens, world, wl.dims.page)
    parts = []
    for r in range(world):
        _, n = S.token_ranges(wl.seq_lens, bounds, r, wl.dims.page)
        bt = torch.from_numpy(S.local_block_table(wl.block_table, bounds, r)).cuda()
        lens = torch.from_numpy(n.astype(np.int32)).cuda()
        o, l = run.layer.decode(run.cache, q_abs, bt, lens, 1, int(n.max()))
        parts.append((o.clone(), l.clone()))
    lse_max = torch.stack([p[1] for p in parts]).amax(0).contiguous()        # all-reduce(max)
    accs = []
    for o, l in parts:
        acc = torch.empty(rows * d.n_h * (d.d_c + 1), dtype=torch.float32, device="cuda")
        N.mla_lse_merge_prepare(rows, d.n_h, d.d_c, o, l, lse_max, acc)
        accs.append(acc)
    acc = torch.stack(accs).sum(0).contiguous()                             # all-reduce(sum)
    o_lat = torch.empty_like(parts[0][0])
    lse = torch.empty_like(parts[0][1])
    N.mla_lse_merge_finish(rows, d.n_h, d.d_c, acc, lse_max, o_lat, lse)
    torch.cuda.synchronize()
    return parts, o_lat, lse


CASES = {
    "bf16_2ranks": dict(seed=61, seq_lens=[5000, 3000, 4100], world=2),
    "bf16_4ranks_ragged_permuted": dict(seed=62, seq_lens=[64 * 4 + 1, 2049, 6000], world=4,
                                        permute=True, spare=6),
    "fp8_3ranks": dict(seed=63, seq_lens=[4096, 2500], world=3, kv_dtype="fp8"),
    "bf16_lognormal_2ranks": dict(seed=64, seq_lens=[3000], world=2, lognormal_tokens=True),
}


@pytest.mark.parametrize("case", sorted(CASES))
def test_split_decode_matches_the_oracle_on_whole_sequences(oracle_mod, case):
    kw = dict(CASES[case])
    world = kw.pop("world")
    wl = W.make_decode(name=case, **kw)
    run = GpuRun(wl)
    run.fill_cache()
    q_abs = run.layer.absorb(run.q_c, run.q_r, run.q_pos)
    parts, o_lat, lse = _split_decode(run, q_abs, world)
    o = run.layer.out_proj(o_lat)
    torch.cuda.synchronize()
    rows, heads, ref = oracle_ref(wl, oracle_mod)
    fp8 = wl.kv_dtype == "fp8"
    check_step((q_abs, o_lat, lse, o), ref, rows, heads, FP8_REL if fp8 else BF16_REL,
               None if fp8 else BF16_ABS, lognormal=wl.extra.get("lognormal_norms", False),
               ref_ops=operands_ref(wl, oracle_mod, rows, heads))
    # the split is real: one rank's partial alone is far from the answer
    assert rel_l2(parts[0][0].cpu().numpy(), ref.o_lat) > 0.05
    # and the merge agrees with the unsplit decode of the same cache
    _, o1, l1, _ = run.step()
    assert rel_l2(o_lat.cpu().numpy(), o1.cpu().numpy()) <= (FP8_REL if fp8 else BF16_REL)
    assert float((lse - l1).abs().max()) <= 1e-2 * max(1.0, float(l1.abs().max()))


def test_merge_kernels_ignore_ranks_without_tokens():
    """A rank that saw no token of a (row, head) reports lse = -inf; the merge must give the
    other ranks' result bit for bit, and 0 / -inf where no rank saw a token."""
    g = torch.Generator(device="cpu").manual_seed(65)
    rows, n_h, d_c = 3, 5, 72
    o = [torch.randn(rows, n_h, d_c, generator=g).cuda() for _ in range(3)]
    l = [torch.randn(rows, n_h, generator=g).mul(4).cuda() for _ in range(3)]
    l[2][:] = -float("inf")
    o[2][:] = 0.0                     # a rank with no tokens reports zeros, as mla_decode does
    l[1][0, :] = -float("inf")
    l[0][0, :] = -float("inf")
    o[0][0], o[1][0] = 0.0, 0.0

    def merge(ks):
        m = torch.stack([l[k] for k in ks]).amax(0).contiguous()
        accs = []
        for k in ks:
            a = torch.empty(rows * n_h * (d_c + 1), device="cuda")
            N.mla_lse_merge_prepare(rows, n_h, d_c, o[k], l[k], m, a)
            accs.append(a)
        acc = accs[0]
        for a in accs[1:]:
            acc = acc + a
        out_o, out_l = torch.empty(rows, n_h, d_c, device="cuda"), torch.empty(rows, n_h, device="cuda")
        N.mla_lse_merge_finish(rows, n_h, d_c, acc, m, out_o, out_l)
        torch.cuda.synchronize()
        return out_o, out_l

    o3, l3 = merge([0, 1, 2])
    o2, l2 = merge([0, 1])
    assert torch.equal(o3, o2) and torch.equal(l3, l2)
    assert torch.equal(o3[0], torch.zeros_like(o3[0])) and bool(torch.isneginf(l3[0]).all())
    assert bool(torch.isfinite(o3[1:]).all()) and bool(torch.isfinite(l3[1:]).all())
    # one rank alone merges to itself exactly: w = 1
    o1, l1 = merge([1])
    assert torch.equal(o1[1:], o[1][1:]) and torch.equal(l1[1:], l[1][1:])


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_merge_through_a_one_rank_nccl_group_is_the_identity():
    """seqsplit.merge with its real collectives (NCCL, one rank) and the library's kernels."""
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_free_port()))
    dist.init_process_group("nccl", rank=0, world_size=1, device_id=torch.device("cuda:0"))
    try:
        g = torch.Generator(device="cpu").manual_seed(66)
        o = torch.randn(4, 16, 512, generator=g).cuda()
        l = torch.randn(4, 16, generator=g).cuda()
        mo, ml = S.merge(o, l)
        torch.cuda.synchronize()
        assert torch.equal(mo, o) and torch.equal(ml, l)
    finally:
        dist.destroy_process_group()

