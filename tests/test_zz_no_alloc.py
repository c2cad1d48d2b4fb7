"""mla_decode_fixed_scratch (decode on the library's static scratch array, no caller workspace)
against mla_decode with a caller workspace, through the C ABI.

The entry point is for callers that cannot allocate device memory when they decode: a service
whose device-memory budget is reserved up front, where a late allocation may find none left,
or a latency-critical path on which an allocation's possible device synchronisation is not
acceptable.

The file name sorts last so that the test also runs after every other test in one session;
it passes alone in a fresh process as well (the first call on the device does the scratch
set-up).  Both entry points run the same kernels on the same inputs, so their results must
agree bit for bit.  The scratch array keeps the previous call's contents; the test first
fills it with a call on a larger, different batch, so that a kernel that read a partial slot
or a slot range it did not write in the current call would show up as a difference.  The
target batch has fewer pages than the kernel has clusters, so some clusters sit inside a
row's slot range with no pages of it and must mark their slot empty in every call.
"""
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


def _fixed_scratch_decode(run, q_abs):
    from mla_latent_kv_mqa_b200 import native as N
    d = run.dims
    rows = run.wl.B * run.wl.s_q
    o_lat = torch.full((rows, d.n_h, d.d_c), float("nan"), dtype=torch.float32, device="cuda")
    lse = torch.full((rows, d.n_h), float("nan"), dtype=torch.float32, device="cuda")
    c = run.cache
    N.mla_decode_fixed_scratch(d, run.wl.B, run.wl.s_q, q_abs, c.kv_pool, c.kr_pool, c.kv_scale,
                               run.block_table, run.block_table.shape[1], c.num_blocks, run.seq_lens,
                               run.max_seq_len, o_lat, lse)
    torch.cuda.synchronize()
    return o_lat, lse


@pytest.mark.parametrize("flags", [0, 1], ids=["tensor_core", "simt"])
def test_fixed_scratch_matches_workspace_decode_twice(flags):
    from mla_latent_kv_mqa_b200 import native as N
    # a different, larger batch first: every slot it writes holds stale values afterwards
    other = W.make_decode(43, [int(x) for x in np.random.default_rng(43).integers(1, 2500, 40)],
                          permute=True, spare=3)
    orun = GpuRun(other, flags=flags)
    orun.fill_cache()
    oq = orun.layer.absorb(orun.q_c, orun.q_r, orun.q_pos)
    o_other, _ = _fixed_scratch_decode(orun, oq)
    assert torch.isfinite(o_other).all()

    wl = W.make_decode(41, [700, 33, 1000, 64 * 5, 1], permute=True, spare=8)
    run = GpuRun(wl, flags=flags)
    run.fill_cache()
    q_abs = run.layer.absorb(run.q_c, run.q_r, run.q_pos)
    ref_o, ref_lse = run.layer.decode(run.cache, q_abs, run.block_table, run.seq_lens, wl.s_q,
                                      run.max_seq_len)
    torch.cuda.synchronize()
    assert torch.isfinite(ref_o).all() and torch.isfinite(ref_lse).all()
    for _ in range(2):  # two calls in a row share the scratch array
        o, lse = _fixed_scratch_decode(run, q_abs)
        assert torch.equal(o, ref_o)
        assert torch.equal(lse, ref_lse)
    assert N.mla_get_last_device_error() == N.MLA_OK


def test_fixed_scratch_rejects_batches_beyond_its_size():
    from mla_latent_kv_mqa_b200 import native as N
    wl = W.make_decode(42, [64, 65], permute=False)
    run = GpuRun(wl)
    limit = 32 << 20
    B = 2
    while N.mla_decode_workspace_size(run.dims, B, 1, 4096) <= limit:
        B *= 2
        assert B <= 1 << 20
    # The size check comes before anything is launched, so the small workload's buffers serve
    # as stand-ins for a batch of B sequences.
    d, c = run.dims, run.cache
    o_lat = torch.empty((wl.B, d.n_h, d.d_c), dtype=torch.float32, device="cuda")
    q_abs = run.layer.absorb(run.q_c, run.q_r, run.q_pos)
    with pytest.raises(N.MLAError) as e:
        N.mla_decode_fixed_scratch(d, B, 1, q_abs, c.kv_pool, c.kr_pool, c.kv_scale, run.block_table,
                                   run.block_table.shape[1], c.num_blocks, run.seq_lens, 4096, o_lat)
    assert e.value.status == N.MLA_ERR_WORKSPACE_TOO_SMALL
