"""mla_decode_project: the decode with its split-merge fused into the output projection.

The call must give, bit for bit, what mla_decode followed by mla_out_proj gives (o, o_lat and
lse), on the bf16 and FP8 caches, for tiles of query rows that are full, ragged and several,
with the workspace poisoned, and on the CUDA-core path (where it is the two calls in a row).
The unfused pair is held to the oracle by tests/test_gpu_parity.py; one bf16 and one FP8
case are also compared with the oracle here directly.
"""
import numpy as np
import pytest
import torch

from mla_latent_kv_mqa_b200 import workloads as W
from tests.harness import BF16_ABS, BF16_REL, FP8_REL, GpuRun, check_step, oracle_ref

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from mla_latent_kv_mqa_b200 import build
    build.build()
    torch.backends.cuda.matmul.allow_tf32 = False


def _lens(seed, n, lo, hi):
    return [int(x) for x in np.random.default_rng(seed).integers(lo, hi, n)]


CASES = {
    "v3_ragged": dict(seed=71, seq_lens=[200, 64, 1, 129, 65]),
    "v3_permuted": dict(seed=72, seq_lens=[700, 33, 1000, 64 * 5], permute=True, spare=8),
    "bf16_sq2": dict(seed=73, seq_lens=[513, 3, 64, 1000], s_q=2),
    "fp8_sq2": dict(seed=74, seq_lens=[300, 2, 65, 128], s_q=2, kv_dtype="fp8"),
    "fp8_lognormal": dict(seed=75, seq_lens=[2000], lognormal_tokens=True, kv_dtype="fp8"),
    # 40 rows: one full tile of 32 and a ragged one of 8
    "rows_40": dict(seed=76, seq_lens=_lens(76, 40, 1, 700)),
    # 256 rows (s_q = 2): eight tiles
    "rows_256_sq2": dict(seed=77, seq_lens=_lens(77, 128, 2, 300), s_q=2),
}


def _unfused(run, q_abs, out_dtype):
    o_lat, lse = run.layer.decode(run.cache, q_abs, run.block_table, run.seq_lens, run.wl.s_q, run.max_seq_len)
    o = run.layer.out_proj(o_lat, out_dtype)
    torch.cuda.synchronize()
    return o, o_lat, lse


def _fused(run, q_abs, out_dtype, poison=False):
    if poison:
        ws = run.layer.workspace(run.wl.B, run.wl.s_q, run.max_seq_len)
        ws.fill_(0xFF)  # NaN patterns everywhere
    o, o_lat, lse = run.layer.decode_project(run.cache, q_abs, run.block_table, run.seq_lens, run.wl.s_q,
                                             run.max_seq_len, out_dtype)
    torch.cuda.synchronize()
    return o, o_lat, lse


@pytest.mark.parametrize("out_dtype", ["f32", "bf16"])
@pytest.mark.parametrize("case", sorted(CASES))
def test_fused_equals_decode_then_out_proj(case, out_dtype):
    wl = W.make_decode(name=case, **CASES[case])
    run = GpuRun(wl)
    run.fill_cache()
    q_abs = run.layer.absorb(run.q_c, run.q_r, run.q_pos)
    ref = _unfused(run, q_abs, out_dtype)
    got = _fused(run, q_abs, out_dtype, poison=True)
    for name, a, b in zip(("o", "o_lat", "lse"), got, ref):
        assert torch.equal(a, b), (name, float((a.float() - b.float()).abs().max()))
    again = _fused(run, q_abs, out_dtype)
    assert all(torch.equal(a, b) for a, b in zip(again, got))


@pytest.mark.parametrize("case", ["v3_permuted", "fp8_sq2"])
def test_fused_matches_the_oracle(oracle_mod, case):
    wl = W.make_decode(name=case, **CASES[case])
    run = GpuRun(wl)
    run.fill_cache()
    q_abs = run.layer.absorb(run.q_c, run.q_r, run.q_pos)
    o, o_lat, lse = _fused(run, q_abs, "f32")
    rows, heads, ref = oracle_ref(wl, oracle_mod)
    fp8 = wl.kv_dtype == "fp8"
    check_step((q_abs, o_lat, lse, o), ref, rows, heads, FP8_REL if fp8 else BF16_REL,
               None if fp8 else BF16_ABS, lognormal=wl.extra.get("lognormal_norms", False))


def test_cuda_core_path_is_the_two_calls():
    """With the CUDA-core flags the call runs the CUDA-core decode and projection in a row."""
    wl = W.make_decode(name="simt", **CASES["v3_ragged"])
    run = GpuRun(wl, flags=3)
    run.fill_cache()
    q_abs = run.layer.absorb(run.q_c, run.q_r, run.q_pos)
    ref = _unfused(run, q_abs, "f32")
    got = _fused(run, q_abs, "f32")
    assert all(torch.equal(a, b) for a, b in zip(got, ref))
