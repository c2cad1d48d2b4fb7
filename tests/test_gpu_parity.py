"""GPU parity of the CUDA path (through the C ABI) against the fp64 CPU oracle.

Tolerances.  bf16 path: relative L2 <= 4e-3, max |err| <= 2e-2 on o_lat and o, |err(lse)|
<= 1e-2.  Cases whose per-token norms are log-normal use max |err| <= 2e-2 * max(1, max |ref|)
and |err(lse)| <= 1e-2 * max(1, |lse|): exact arithmetic on the bf16 operands of the C ABI
already moves single elements of o_lat by ~0.1 and lse by ~0.02 there
(tests/test_tolerance_reading.py).  FP8 content cache: relative L2 <= 3e-2 against the oracle
run on its own dequantised cache (the same codes, checked bit-exact below).  The fp32 toy
layer accumulates in fp32 over at most 256 tokens x 160 dims: relative L2 <= 1e-5.
"""
import numpy as np
import pytest
import torch

from mla_latent_kv_mqa_b200 import workloads as W
from tests.harness import (BF16_ABS, BF16_REL, FP8_REL, LSE_ABS, GpuRun, check_step, max_abs, operands_ref,
                           oracle_ref, rel_l2, scaled_max_abs)

pytestmark = pytest.mark.gpu



@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from mla_latent_kv_mqa_b200 import build
    build.build()
    torch.backends.cuda.matmul.allow_tf32 = False


def _check(wl, got, ref, rows, heads, rel_tol, abs_tol, orc=None):
    return check_step(got, ref, rows, heads, rel_tol, abs_tol,
                      lognormal=wl.extra.get("lognormal_norms", False),
                      ref_ops=operands_ref(wl, orc, rows, heads) if orc is not None else None)


# ---------------------------------------------------------------------------------------------
# small cases: several tiles, ragged tails, permuted tables, both kernels
# ---------------------------------------------------------------------------------------------

SMALL = {
    "v3_ragged": dict(seed=21, seq_lens=[200, 64, 1, 129, 65]),
    "v3_permuted": dict(seed=22, seq_lens=[700, 33, 1000, 64 * 5], permute=True, spare=8),
    "v3_lognormal": dict(seed=23, seq_lens=[3000], lognormal_tokens=True),
    "fp8_sq2": dict(seed=24, seq_lens=[300, 2, 65, 128], s_q=2, kv_dtype="fp8"),
    "fp8_ragged_permuted": dict(seed=27, seq_lens=[200, 64, 1, 129, 700], kv_dtype="fp8", permute=True, spare=4),
    "fp8_lognormal": dict(seed=28, seq_lens=[2000], lognormal_tokens=True, kv_dtype="fp8"),
    "bf16_sq2": dict(seed=25, seq_lens=[513, 3], s_q=2),
    # more query rows than the tensor-core kernel has clusters: the scheduler's contiguous split
    "many_rows": dict(seed=26, seq_lens=[int(x) for x in np.random.default_rng(26).integers(1, 300, 96)]),
}


@pytest.mark.parametrize("simt", [False, True], ids=["default", "simt"])
@pytest.mark.parametrize("case", sorted(SMALL))
def test_decode_matches_oracle_small(oracle_mod, case, simt):
    kw = dict(SMALL[case])
    wl = W.make_decode(name=case, **kw)
    run = GpuRun(wl, flags=3 if simt else 0)  # 3: CUDA-core decode and projections
    run.fill_cache()
    got = run.step()
    rows, heads, ref = oracle_ref(wl, oracle_mod)
    tol = FP8_REL if wl.kv_dtype == "fp8" else BF16_REL
    _check(wl, got, ref, rows, heads, tol, None if wl.kv_dtype == "fp8" else BF16_ABS, oracle_mod)
    # q_abs = [W_UK^T q_C ; RoPE(q_R)] against the oracle's q_lat and rotation
    q_abs = got[0].float().cpu().numpy()
    assert rel_l2(q_abs[:, :, :wl.dims.d_c], ref.q_lat) <= 4e-3


def test_toy_layer_fp32(oracle_mod):
    """The implementation section's toy layer: decode of the last of 256 tokens, fp32."""
    from mla_latent_kv_mqa_b200 import layer as Lyr
    h, Wt = W.toy_layer_inputs(seed=1)
    ref = oracle_mod.toy_layer(h.astype(np.float64), Wt, mode="absorbed", last_only=True)
    dev = "cuda"
    f = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(dev)
    # upstream projections (outside the decode path) in fp32 on the GPU
    hd = f(h[0])
    c_kv = hd @ f(Wt["w_dkv"]).T
    k_r = hd @ f(Wt["w_kr"]).T
    c_q = hd[-1:] @ f(Wt["w_dq"]).T
    q_c = (c_q @ f(Wt["w_uq"]).T).reshape(1, 8, 64).contiguous()
    q_r = (c_q @ f(Wt["w_qr"]).T).reshape(1, 8, 32).contiguous()
    dims = Lyr.dims_for(8, 64, 128, 32, act="f32", kv="f32")
    layer = Lyr.MLADecodeLayer(dims, f(Wt["w_uk"]), f(Wt["w_uv"]))
    cache = Lyr.PagedLatentCache(dims, 4, dev, poison=True)
    bt = torch.tensor([[2, 0, 3, 1]], dtype=torch.int32, device=dev)
    T = 256
    layer.append(cache, c_kv.contiguous(), k_r.contiguous(), torch.zeros(T, dtype=torch.int32, device=dev),
                 torch.arange(T, dtype=torch.int32, device=dev), bt)
    q_abs = layer.absorb(q_c, q_r, torch.tensor([T - 1], dtype=torch.int32, device=dev))
    o_lat, lse = layer.decode(cache, q_abs, bt, torch.tensor([T], dtype=torch.int32, device=dev), 1, T)
    o = layer.out_proj(o_lat, "f32")
    u = o.reshape(1, -1) @ f(Wt["w_o"]).T
    torch.cuda.synchronize()
    assert rel_l2(o_lat.cpu().numpy(), ref.o_lat[0]) <= 1e-5
    assert rel_l2(o.cpu().numpy(), ref.o[0]) <= 1e-5
    assert max_abs(lse.cpu().numpy(), ref.lse[0]) <= 1e-5
    assert rel_l2(u.cpu().numpy(), ref.u[0]) <= 1e-5


# ---------------------------------------------------------------------------------------------
# bit-exact indexing
# ---------------------------------------------------------------------------------------------

def _bf16_bits(x):
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16).view(torch.int16).numpy()


def test_append_bf16_scatter_is_bit_exact(oracle_mod):
    wl = W.make_decode(31, [130, 64, 5, 200], permute=True, spare=5)
    run = GpuRun(wl)
    run.fill_cache()
    torch.cuda.synchronize()
    pool = run.cache.kv_pool.cpu()
    bits = pool.view(torch.int16).numpy()
    touched = np.zeros(pool.shape[:2], dtype=bool)
    d_c = wl.dims.d_c
    for b in range(wl.B):
        L = int(wl.seq_lens[b])
        j = np.arange(L)
        blk = wl.block_table[b, j // 64]
        slot = j % 64
        touched[blk, slot] = True
        assert np.array_equal(bits[blk, slot, :d_c], _bf16_bits(wl.seq_c_kv(b)))
        # RoPE at position 0 is the identity: bit-exact
        assert np.array_equal(bits[blk[0], 0, d_c:], _bf16_bits(wl.seq_k_r(b)[0]))
        # every rotated key within one bf16 rounding (2^-9 relative) of the fp64 rotation, plus
        # the fp32 rotation's own error, which scales with the pair (x_k, x_{k+d/2}) it mixes
        got = pool[blk, slot, d_c:].float().numpy()
        x = wl.seq_k_r(b).astype(np.float64)
        want = np.stack([oracle_mod.rope(x[p], float(p)) for p in range(L)])
        half = x.shape[1] // 2
        pair = np.abs(x[:, :half]) + np.abs(x[:, half:])
        pair = np.concatenate([pair, pair], 1)
        assert np.all(np.abs(got - want) <= np.abs(want) * 2.0 ** -8 + pair * 2.0 ** -20)
    assert torch.isnan(pool[torch.from_numpy(~touched)].float()).all()


def test_append_fp8_codes_and_scales_are_bit_exact(oracle_mod):
    wl = W.make_decode(32, [100, 64, 1], kv_dtype="fp8", permute=True, spare=2)
    run = GpuRun(wl)
    run.fill_cache()
    torch.cuda.synchronize()
    codes = run.cache.kv_pool.cpu().numpy()
    scales = run.cache.kv_scale.cpu().numpy()
    for b in range(wl.B):
        L = int(wl.seq_lens[b])
        j = np.arange(L)
        blk, slot = wl.block_table[b, j // 64], j % 64
        want_codes, want_scales = oracle_mod.quantize_rows(wl.seq_c_kv(b))
        assert np.array_equal(codes[blk, slot], want_codes)
        assert np.array_equal(scales[blk, slot].view(np.uint32), want_scales.view(np.uint32))


@pytest.mark.parametrize("kv", ["bf16", "fp8"])
def test_permuted_block_table_is_bitwise_identical(kv):
    wl = W.make_decode(33, [1000, 77, 640, 2048], kv_dtype=kv)
    a = GpuRun(wl)
    a.fill_cache()
    ga = a.step()
    rng = np.random.default_rng(5)
    perm = rng.permutation(wl.num_blocks + 3).astype(np.int32)
    bt = np.where(wl.block_table >= 0, perm[np.maximum(wl.block_table, 0)], -1).astype(np.int32)
    wl2 = W.make_decode(33, [1000, 77, 640, 2048], kv_dtype=kv)
    wl2.num_blocks = wl.num_blocks + 3
    b = GpuRun(wl2, block_table=bt)
    b.fill_cache()
    gb = b.step()
    for x, y in zip(ga[1:], gb[1:]):
        assert torch.equal(x, y)


@pytest.mark.parametrize("simt", [False, True], ids=["default", "simt"])
def test_out_proj_bf16_output_is_the_rounded_f32_output(oracle_mod, simt):
    """mla_out_proj with a bf16 output: the same fp32 accumulation, rounded once to bf16."""
    wl = W.make_decode(38, [300, 65, 1], name="bf16_out")
    run = GpuRun(wl, flags=3 if simt else 0)
    run.fill_cache()
    q_abs, o_lat, lse, o32 = run.step("f32")
    o16 = run.layer.out_proj(o_lat, "bf16")
    torch.cuda.synchronize()
    assert o16.dtype == torch.bfloat16
    assert torch.equal(o16, o32.to(torch.bfloat16))
    rows, heads, ref = oracle_ref(wl, oracle_mod)
    assert rel_l2(o16.float().cpu().numpy(), ref.o) <= BF16_REL


@pytest.mark.parametrize("kv", ["bf16", "fp8"])
def test_repeated_decode_is_deterministic(kv):
    wl = W.make_decode(34, [4096, 100, 3000], kv_dtype=kv)
    run = GpuRun(wl)
    run.fill_cache()
    g1 = run.step()
    g2 = run.step()
    for x, y in zip(g1, g2):
        assert torch.equal(x, y)


# ---------------------------------------------------------------------------------------------
# device-side error reporting (no faults: the kernels skip the bad access)
# ---------------------------------------------------------------------------------------------

def test_bad_block_id_is_reported_not_faulted():
    from mla_latent_kv_mqa_b200 import native as N
    N.mla_get_last_device_error()
    wl = W.make_decode(35, [130, 64])
    bt = wl.block_table.copy()
    bt[0, 1] = wl.num_blocks + 1000  # outside the pool
    run = GpuRun(wl, block_table=bt)
    run.fill_cache()
    assert N.mla_get_last_device_error() == N.MLA_ERR_BAD_BLOCK_TABLE
    run.step()
    assert N.mla_get_last_device_error() == N.MLA_ERR_BAD_BLOCK_TABLE
    assert N.mla_get_last_device_error() == N.MLA_OK


def test_bad_seq_len_is_reported_not_faulted():
    from mla_latent_kv_mqa_b200 import native as N
    N.mla_get_last_device_error()
    wl = W.make_decode(36, [130, 64])
    run = GpuRun(wl)
    run.fill_cache()
    run.seq_lens[1] = 0  # shorter than s_q
    run.step()
    assert N.mla_get_last_device_error() == N.MLA_ERR_BAD_SEQ_LEN


@pytest.mark.parametrize("fill", [float("nan"), 12345.0])
def test_workspace_contents_do_not_matter(fill):
    """mla_decode must not read partial slots it did not write in this call (e.g. the slots
    of clusters that received no pages of a row when pages are fewer than clusters)."""
    wl = W.make_decode(37, [700, 33, 1000, 320], permute=True, spare=8)
    run = GpuRun(wl)
    run.fill_cache()
    ref = run.step()
    ws = run.layer.workspace(wl.B, wl.s_q, run.max_seq_len)
    ws.view(torch.float32)[: ws.numel() // 4].fill_(fill)
    got = run.step()
    for x, y in zip(ref[1:], got[1:]):
        assert torch.equal(x, y)


# ---------------------------------------------------------------------------------------------
# FP8 cache with the content scores on the FP8 tensor core (MLA_FLAG_FP8_MMA): the same
# bounds as the FP8 cache (relative L2 <= 3e-2 against the oracle on its own dequantised cache)
# ---------------------------------------------------------------------------------------------

FP8_MMA = {
    "fp8_mma_sq2": dict(seed=41, seq_lens=[300, 2, 65, 128], s_q=2, kv_dtype="fp8"),
    "fp8_mma_ragged_permuted": dict(seed=42, seq_lens=[200, 64, 1, 129, 700], kv_dtype="fp8", permute=True,
                                    spare=4),
    "fp8_mma_lognormal": dict(seed=43, seq_lens=[2000], lognormal_tokens=True, kv_dtype="fp8"),
    "fp8_mma_long_rows": dict(seed=44, seq_lens=[5000, 3000], s_q=2, kv_dtype="fp8"),
}


@pytest.mark.parametrize("case", sorted(FP8_MMA))
def test_fp8_tensor_core_scores_match_oracle(oracle_mod, case):
    import mla_latent_kv_mqa_b200.native as Nat
    wl = W.make_decode(name=case, **FP8_MMA[case])
    run = GpuRun(wl, flags=Nat.MLA_FLAG_FP8_MMA)
    run.fill_cache()
    got = run.step()
    assert Nat.mla_get_last_device_error() == 0
    rows, heads, ref = oracle_ref(wl, oracle_mod)
    e = _check(wl, got, ref, rows, heads, FP8_REL, None)
    # and against the default FP8 path (bf16 dequantisation) on the same cache
    run2 = GpuRun(wl)
    run2.fill_cache()
    got2 = run2.step()
    assert rel_l2(got[1].cpu().numpy(), got2[1].cpu().numpy()) <= FP8_REL, e
    # bitwise reproducible
    again = run.step()
    assert torch.equal(again[1], got[1]) and torch.equal(again[2], got[2])
