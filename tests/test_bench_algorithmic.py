"""The algorithmic work the benchmark divides by, against the method's per-token definition:
1152 B per cached token for the bf16 cache (576 bf16 values), 644 B for the FP8 cache (512
codes + a bf16 RoPE key of 64 + a 4-byte scale), and 2 * n_h * ((d_c + d_R) + d_c) FLOPs per
head-shared visible token and query row.  Also which roofline binds at the measured B200 peaks."""
import types

import numpy as np
import pytest

import bench
from mla_latent_kv_mqa_b200 import workloads as W

HBM_GBS, TC_TFLOPS = 6539.5, 1606.3


def _wl(seq_lens, s_q=1, kv="bf16"):
    return types.SimpleNamespace(dims=W.V3_DIMS, seq_lens=np.asarray(seq_lens, np.int32), s_q=s_q, kv_dtype=kv)


@pytest.mark.parametrize("name,seq_lens,s_q,kv,bytes_,flops,bound,t_us", [
    ("v3", [4096] * 16, 1, "bf16", 75_497_472, 18_253_611_008, "hbm", 11.54),
    ("long", [131072] * 4, 1, "bf16", 603_979_776, 146_028_888_064, "hbm", 92.36),
    ("mtp_fp8", [8192] * 128, 2, "fp8", 675_282_944, 584_079_900_672, "tensor", 363.6),
])
def test_algorithmic_work_per_config(name, seq_lens, s_q, kv, bytes_, flops, bound, t_us):
    b, f = bench.algorithmic(_wl(seq_lens, s_q, kv))
    assert (b, f) == (bytes_, flops)
    t_hbm, t_tc = b / (HBM_GBS * 1e3), f / (TC_TFLOPS * 1e6)  # microseconds
    assert ("hbm" if t_hbm >= t_tc else "tensor") == bound
    assert abs(max(t_hbm, t_tc) - t_us) < 0.05


def test_per_token_figures():
    one = bench.algorithmic(_wl([1]))
    assert one == (1152, 2 * 128 * (576 + 512))
    assert bench.algorithmic(_wl([1], kv="fp8"))[0] == 512 + 2 * 64 + 4
    # s_q = 2: the first query sees one token fewer than the second (causal within the pair)
    assert bench.algorithmic(_wl([10], s_q=2))[1] == (9 + 10) * 2 * 128 * 1088


def test_varlen_lengths_and_bytes():
    rng = np.random.default_rng(3)  # the varlen workload's own draw of its lengths
    lens = rng.integers(1024, 16384 + 1, size=64)
    b, f = bench.algorithmic(_wl(lens))
    assert b == int(lens.sum()) * 1152
    assert 0.55e9 < b < 0.75e9  # about 642 MB for U[1024, 16384] at B = 64


def test_prefill_flops_count_every_visible_pair():
    """Brute force over (query t, key j <= t) pairs of small prompts, and the benchmark's
    4 x 4096 prompts: 2 (d_h + d_R) + 2 d_h FLOPs per head and pair, plus 2 d_c d_h per head,
    token and reconstructed matrix (K and V)."""
    d = W.V3_DIMS
    lens = [1, 5, 130]
    pairs = sum(1 for L in lens for t in range(L) for j in range(t + 1))
    wl = types.SimpleNamespace(dims=d, seq_lens=np.asarray(lens, np.int32), T=sum(lens))
    attn, up = bench.prefill_flops(wl)
    assert attn == pairs * d.n_h * 2 * (192 + 128)
    assert up == 2 * sum(lens) * 2 * 512 * 128 * 128
    wl = types.SimpleNamespace(dims=d, seq_lens=np.asarray(bench.PREFILL_LENS, np.int32), T=4 * 4096)
    attn, up = bench.prefill_flops(wl)
    assert attn == 4 * (4096 * 4097 // 2) * 128 * 640 and up == 549_755_813_888
