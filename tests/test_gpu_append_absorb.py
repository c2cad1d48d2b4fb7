"""mla_append_absorb: the cache append and the query absorption in one call must give, bit for
bit, what mla_cache_append followed by mla_absorb_q gives: the whole cache pool (every slot,
the NaN-poisoned unreferenced ones included) and q_abs."""
import numpy as np
import pytest
import torch

from mla_latent_kv_mqa_b200 import workloads as W
from tests.harness import GpuRun

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from mla_latent_kv_mqa_b200 import build
    build.build()


def _pools(run):
    c = run.cache
    return [t.clone() for t in (c.kv_pool, c.kr_pool, c.kv_scale) if t is not None]


def _same(a, b):
    # NaN slots compare equal through their bits
    return all(torch.equal(x.view(torch.uint8), y.view(torch.uint8)) for x, y in zip(a, b))


CASES = {
    "bf16_16": dict(seed=91, seq_lens=[700, 33, 1000, 64 * 5, 2, 90, 65, 1, 300, 129, 64, 200, 400, 77, 128, 9],
                    permute=True, spare=5),
    "fp8_sq2": dict(seed=92, seq_lens=[300, 2, 65, 128], s_q=2, kv_dtype="fp8"),
    # 150 new tokens: more appending CTAs than SMs left free by the absorption's 128
    "bf16_150": dict(seed=93, seq_lens=[int(x) for x in np.random.default_rng(93).integers(1, 200, 150)]),
    "simt": dict(seed=94, seq_lens=[200, 64, 1, 129, 65]),
}


@pytest.mark.parametrize("case", sorted(CASES))
def test_one_call_equals_the_two(case):
    wl = W.make_decode(name=case, **CASES[case])
    flags = 2 if case == "simt" else 0  # 2: CUDA-core projections (the two-launch path)
    a, b = GpuRun(wl, flags=flags), GpuRun(wl, flags=flags)
    # the step's new tokens: the last s_q of every sequence; the rest appended beforehand
    idx = np.concatenate([np.arange(wl.ctx_off[i + 1] - wl.s_q, wl.ctx_off[i + 1]) for i in range(wl.B)])
    rest = np.setdiff1d(np.arange(int(wl.ctx_off[-1])), idx)
    for run in (a, b):
        sel = torch.from_numpy(rest).cuda()
        run.layer.append(run.cache, run.c_kv[sel], run.k_r[sel], run.tok_seq[sel], run.tok_pos[sel], run.block_table)
    sel = torch.from_numpy(idx).cuda()
    a.layer.append(a.cache, a.c_kv[sel], a.k_r[sel], a.tok_seq[sel], a.tok_pos[sel], a.block_table)
    qa = a.layer.absorb(a.q_c, a.q_r, a.q_pos)
    qb = b.layer.append_absorb(b.cache, b.c_kv[sel], b.k_r[sel], b.tok_seq[sel], b.tok_pos[sel], b.block_table,
                               b.q_c, b.q_r, b.q_pos)
    torch.cuda.synchronize()
    assert torch.equal(qa, qb)
    assert _same(_pools(a), _pools(b))


def test_either_part_may_be_empty():
    wl = W.make_decode(95, [100, 64])
    run = GpuRun(wl)
    run.fill_cache()
    before = _pools(run)
    q0 = run.layer.absorb(run.q_c, run.q_r, run.q_pos)
    e = torch.empty(0, dtype=run.c_kv.dtype, device="cuda")
    ei = torch.empty(0, dtype=torch.int32, device="cuda")
    q1 = run.layer.append_absorb(run.cache, e.view(0, 512), e.view(0, 64), ei, ei, run.block_table,
                                 run.q_c, run.q_r, run.q_pos)
    torch.cuda.synchronize()
    assert torch.equal(q0, q1) and _same(before, _pools(run))
