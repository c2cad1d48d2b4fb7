"""Failure detection of the tensor-core decode, on the GPU, without a fault.

Every wait of the decode kernel is bounded.  When one gives up, the cluster raises an abort
flag in both of its CTAs, records MLA_ERR_DEVICE_TIMEOUT in the device error word, waits
(with a bound) for the copies and MMAs it has started, and exits through the normal teardown.
MLA_FLAG_TEST_GIVE_UP plants such a give-up: after the first page's copies have started,
one short wait on a barrier that nothing completes runs out.  The test checks that the call
returns, that the error word reports the timeout, and that the next normal call on the same
buffers is bitwise the result of a normal call made before (the context stays usable and the
workspace holds nothing that a later call reads).
"""
import ctypes
import time

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


@pytest.mark.parametrize("kv", ["bf16", "fp8"])
def test_timed_out_wait_is_reported_and_the_next_call_is_exact(kv):
    from mla_latent_kv_mqa_b200 import native as N
    N.mla_get_last_device_error()
    # 64 + 47 + 40 = 151 pages: every cluster of the grid gets at least two
    wl = W.make_decode(51, [4096, 3000, 2500], kv_dtype=kv)
    run = GpuRun(wl)
    run.fill_cache()
    q_abs = run.layer.absorb(run.q_c, run.q_r, run.q_pos)
    ref_o, ref_lse = run.layer.decode(run.cache, q_abs, run.block_table, run.seq_lens, wl.s_q,
                                      run.max_seq_len)
    ref_o, ref_lse = ref_o.clone(), ref_lse.clone()
    assert N.mla_get_last_device_error() == N.MLA_OK

    d = run.dims
    bad = N.mla_dims_t(d.n_h, d.d_h, d.d_c, d.d_r, d.page_size, d.rope_base, d.act_dtype, d.kv_dtype,
                       d.flags | N.MLA_FLAG_TEST_GIVE_UP)
    c = run.cache
    ws = run.layer.workspace(wl.B, wl.s_q, run.max_seq_len)
    o = torch.empty_like(ref_o)
    lse = torch.empty_like(ref_lse)
    t0 = time.perf_counter()
    N.mla_decode(bad, wl.B, wl.s_q, q_abs, c.kv_pool, c.kr_pool, c.kv_scale, run.block_table,
                 run.block_table.shape[1], c.num_blocks, run.seq_lens, run.max_seq_len, ws, ws.numel(),
                 o, lse)
    torch.cuda.synchronize()
    assert time.perf_counter() - t0 < 10.0  # the drains are bounded (2 s each at most)
    assert N.mla_get_last_device_error() == N.MLA_ERR_DEVICE_TIMEOUT
    assert N.mla_get_last_device_error() == N.MLA_OK  # reading clears the word

    o2, lse2 = run.layer.decode(run.cache, q_abs, run.block_table, run.seq_lens, wl.s_q,
                                run.max_seq_len)
    torch.cuda.synchronize()
    assert N.mla_get_last_device_error() == N.MLA_OK
    assert torch.equal(o2, ref_o) and torch.equal(lse2, ref_lse)
