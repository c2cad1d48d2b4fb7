"""MHA-mode prefill (mla_prefill) on the GPU against the fp64 naive-mode oracle.

The oracle reconstructs k = W^UK_h c and v = W^UV_h c per head and token (MLA article, 구조
section) and runs the causal softmax for each sampled (prompt, token) row over the prompt's
tokens 0..t.  Bounds as for the bf16 decode: relative L2 <= 4e-3 and max |err| <= 2e-2 on o,
|err(lse)| <= 1e-2 (bf16 operands: q, K and V after reconstruction, P).
"""
import numpy as np
import pytest
import torch

from mla_latent_kv_mqa_b200 import native as N
from mla_latent_kv_mqa_b200 import workloads as W
from tests.harness import BF16_ABS, BF16_REL, LSE_ABS, PrefillRun, max_abs, prefill_oracle_rows, rel_l2

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from mla_latent_kv_mqa_b200 import build
    build.build()


def _check(wl, o, lse, orc, rows, heads):
    glob, heads, ref = prefill_oracle_rows(wl, orc, rows, heads)
    got_o = o.float().cpu().numpy()[glob][:, heads]
    got_l = lse.cpu().numpy()[glob][:, heads]
    e = dict(rel=rel_l2(got_o, ref.o), abs=max_abs(got_o, ref.o), lse=max_abs(got_l, ref.lse))
    assert e["rel"] <= BF16_REL and e["abs"] <= BF16_ABS and e["lse"] <= LSE_ABS, e
    return e


def _rows(wl, per_prompt):
    """Sampled rows: the first and last token of every prompt, the tile edges 127/128/255/256
    where present, and a few seeded others."""
    rng = np.random.default_rng(5)
    out = []
    for b, L in enumerate(wl.seq_lens):
        ts = {0, int(L) - 1} | {t for t in (63, 127, 128, 129, 255, 256) if t < L}
        ts |= set(int(x) for x in rng.integers(0, L, size=per_prompt))
        out += [(b, t) for t in sorted(ts)]
    return out


def test_prefill_every_row_of_small_prompts(oracle_mod):
    """All rows, 8 heads: one-token prompt, prompts ending inside / right after a tile."""
    wl = W.make_prefill(81, [1, 130, 64, 200])
    run = PrefillRun(wl)
    o, lse = run.run()
    rows = [(b, t) for b, L in enumerate(wl.seq_lens) for t in range(L)]
    _check(wl, o, lse, oracle_mod, rows, np.arange(0, 128, 16))


@pytest.mark.parametrize("lens", [[700, 1500], [2048], [129, 1, 1000, 383]], ids=["two", "one_2048", "mixed"])
def test_prefill_sampled_rows_many_tiles(oracle_mod, lens):
    wl = W.make_prefill(82 + len(lens), lens)
    run = PrefillRun(wl)
    o, lse = run.run()
    heads = np.random.default_rng(len(lens)).choice(128, size=12, replace=False)
    _check(wl, o, lse, oracle_mod, _rows(wl, 4), heads)


@pytest.mark.parametrize("lens", [[4096] * 4, [16384]], ids=["bench_4x4096", "one_16384"])
def test_prefill_full_size_sampled_rows(oracle_mod, lens):
    """The benchmark's prefill workloads, in the same single mla_prefill call: the last token of
    every prompt (the longest causal rows), a token on a tile edge and a seeded one, on a few
    heads (each sampled row costs the oracle a K/V reconstruction over its whole prefix)."""
    wl = W.make_prefill(88 + len(lens), lens)
    run = PrefillRun(wl)
    o, lse = run.run()
    rng = np.random.default_rng(9)
    rows = []
    for b, L in enumerate(wl.seq_lens):
        rows += [(b, int(L) - 1), (b, 1023), (b, int(rng.integers(0, L)))]
    heads = rng.choice(128, size=3 if len(lens) > 1 else 2, replace=False)
    _check(wl, o, lse, oracle_mod, rows, heads)


def test_prefill_empty_prompts_among_others(oracle_mod):
    """Zero-length prompts in the table (first, middle, last): their CTAs have no rows and exit,
    the others are computed as if alone; every row of the call is written."""
    wl = W.make_prefill(89, [0, 70, 0, 129, 0])
    run = PrefillRun(wl)
    o = torch.full((wl.T, 128, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((wl.T, 128), float("nan"), device="cuda")
    run.run(o, lse)
    assert bool(torch.isfinite(o.float()).all()) and bool(torch.isfinite(lse).all())
    rows = [(b, t) for b, L in enumerate(wl.seq_lens) for t in range(L)]
    _check(wl, o, lse, oracle_mod, rows, np.arange(3, 128, 25))


def test_prefill_is_deterministic_and_writes_every_row():
    wl = W.make_prefill(86, [300, 77, 513])
    run = PrefillRun(wl)
    o1 = torch.full((wl.T, 128, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
    l1 = torch.full((wl.T, 128), float("nan"), device="cuda")
    run.run(o1, l1)
    assert bool(torch.isfinite(o1.float()).all()) and bool(torch.isfinite(l1).all())
    o2, l2 = run.run()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_bad_prompt_table_is_reported_without_faults():
    """cu_seqlens must start at 0, not decrease and end at T: a table that breaks this is
    reported as MLA_ERR_BAD_SEQ_LEN, and nothing outside the buffers is touched."""
    wl = W.make_prefill(87, [100, 100, 100])
    run = PrefillRun(wl)
    N.mla_get_last_device_error()
    run.cu = torch.tensor([0, 150, 90, 300], dtype=torch.int32, device="cuda")
    run.run()
    assert N.mla_get_last_device_error() == N.MLA_ERR_BAD_SEQ_LEN
    run.cu = torch.from_numpy(wl.cu_seqlens).cuda()
    run.run()
    assert N.mla_get_last_device_error() == N.MLA_OK
