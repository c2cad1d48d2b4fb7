"""Parity at the full workload sizes, in the launch configuration bench.py times (the default
path of mla_decode: the tensor-core kernel, for the bf16 and the FP8 cache).

The whole decode step runs on the GPU for every query row.  The fp64 oracle is run on a seeded
sample of sequences and heads that it computes in seconds; the tolerances are those of
test_gpu_parity.py.  Marked slow: the inputs are generated on the host at full size.
"""
import numpy as np
import pytest
import torch

from mla_latent_kv_mqa_b200 import workloads as W
from tests.harness import BF16_ABS, BF16_REL, FP8_REL, GpuRun, check_step, operands_ref, oracle_ref

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from mla_latent_kv_mqa_b200 import build
    build.build()


# workload, number of sampled sequences, number of sampled heads
CONFIGS = {
    "v3_b16_l4096": (lambda: W.v3_decode(), 4, 32),
    "varlen_b64": (lambda: W.varlen_decode(), 4, 16),
    "long_b4_l131072": (lambda: W.long_decode(), 2, 8),
    "mtp_fp8_b128": (lambda: W.mtp_fp8_decode(), 4, 16),
}


@pytest.mark.parametrize("cfg", sorted(CONFIGS))
def test_full_size_sampled_rows(oracle_mod, cfg):
    make, n_seq, n_head = CONFIGS[cfg]
    wl = make()
    run = GpuRun(wl)
    run.fill_cache()
    got = run.step()
    rng = np.random.default_rng(1234)
    # the first and last sequences (block-table edges) and random ones in between
    seqs = sorted({0, wl.B - 1} | set(int(x) for x in rng.choice(wl.B, n_seq, replace=False)))[:n_seq + 1]
    heads = np.sort(rng.choice(wl.dims.n_h, n_head, replace=False))
    rows, heads, ref = oracle_ref(wl, oracle_mod, seqs, heads)
    fp8 = wl.kv_dtype == "fp8"
    check_step(got, ref, rows, heads, FP8_REL if fp8 else BF16_REL, None if fp8 else BF16_ABS,
               lognormal=wl.extra.get("lognormal_norms", False),
               ref_ops=operands_ref(wl, oracle_mod, rows, heads))
