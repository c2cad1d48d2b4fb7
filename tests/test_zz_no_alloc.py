"""mla_decode_fixed_scratch (decode on the library's static scratch array, no caller workspace)
against mla_decode with a caller workspace, through the C ABI.

The file name sorts last so that the test also runs after every other test in one session;
it passes alone in a fresh process as well (the first call on the device does the scratch
set-up).  Tolerance: the bf16 parity bound of the other GPU tests (relative L2 <= 4e-3);
both calls run the same kernels, so in practice the results agree bit for bit.
"""
import numpy as np
import pytest
import torch

from mla_latent_kv_mqa_b200 import workloads as W
from tests.harness import GpuRun, rel_l2

pytestmark = pytest.mark.gpu

REL = 4e-3


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
    wl = W.make_decode(41, [700, 33, 1000, 64 * 5, 1], permute=True, spare=8)
    run = GpuRun(wl, flags=flags)
    run.fill_cache()
    q_abs = run.layer.absorb(run.q_c, run.q_r, run.q_pos)
    ref_o, ref_lse = run.layer.decode(run.cache, q_abs, run.block_table, run.seq_lens, wl.s_q,
                                      run.max_seq_len)
    torch.cuda.synchronize()
    ref_o, ref_lse = ref_o.cpu().numpy(), ref_lse.cpu().numpy()
    for _ in range(2):  # two calls in a row share the scratch array
        o, lse = _fixed_scratch_decode(run, q_abs)
        o, lse = o.cpu().numpy(), lse.cpu().numpy()
        assert np.isfinite(o).all() and np.isfinite(lse).all()
        assert rel_l2(o, ref_o) <= REL
        assert rel_l2(lse, ref_lse) <= REL
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
