"""The C-ABI library loads, exports every symbol include/mla.h declares, and rejects bad
arguments on the host before touching the GPU (no compute calls here)."""
import ctypes
import subprocess

import pytest

from mla_latent_kv_mqa_b200 import build as B


@pytest.fixture(scope="module")
def N():
    B.build()
    from mla_latent_kv_mqa_b200 import native
    return native


def test_exports_every_declared_symbol(N):
    names = N.declared_functions()
    assert {"mla_absorb_q", "mla_cache_append", "mla_decode", "mla_decode_workspace_size",
            "mla_out_proj", "mla_get_last_device_error", "mla_status_string",
            "mla_version"} <= set(names)
    out = subprocess.run(["nm", "-D", "--defined-only", N.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if line.strip()}
    for n in names:
        assert n in exported, n
        assert hasattr(N.library(), n)


def test_status_strings_and_version(N):
    assert N.version() == 100
    assert N.status_string(0) == "MLA_OK"
    assert N.status_string(N.MLA_ERR_WORKSPACE_TOO_SMALL) == "MLA_ERR_WORKSPACE_TOO_SMALL"
    assert N.status_string(99) == "MLA_ERR_UNKNOWN"


def _v3(N, **kw):
    return N.make_dims(128, 128, 512, 64, **kw)


def test_host_argument_checks(N):
    L = N.library()
    d = _v3(N)
    dp = ctypes.byref(d)
    # null pointers with work to do
    assert L.mla_absorb_q(dp, 4, None, None, None, None, None, None) == N.MLA_ERR_INVALID_ARG
    # zero tokens is a no-op even with null pointers
    assert L.mla_absorb_q(dp, 0, None, None, None, None, None, None) == N.MLA_OK
    assert L.mla_out_proj(dp, -1, None, None, None, 0, None) == N.MLA_ERR_INVALID_ARG
    # odd RoPE width, bad dtype
    bad = _v3(N)
    bad.d_r = 63
    assert L.mla_out_proj(ctypes.byref(bad), 1, 8, 8, 8, 0, None) == N.MLA_ERR_INVALID_ARG
    bad = _v3(N, act_dtype=N.MLA_DTYPE_FP8_E4M3)
    assert L.mla_out_proj(ctypes.byref(bad), 1, 8, 8, 8, 0, None) == N.MLA_ERR_UNSUPPORTED
    # fp8 cache needs the RoPE pool and the scales, and only then
    f8 = _v3(N, kv_dtype=N.MLA_DTYPE_FP8_E4M3)
    assert L.mla_cache_append(ctypes.byref(f8), 1, 8, 8, 8, 8, 8, 1, 1, 1, 8, None, None,
                              None) == N.MLA_ERR_INVALID_ARG
    assert L.mla_cache_append(dp, 1, 8, 8, 8, 8, 8, 1, 1, 1, 8, 8, None, None) == N.MLA_ERR_INVALID_ARG
    # decode: s_q < 1, max_seq_len beyond the table, workspace too small / misaligned
    args = [dp, 2, 0, 16, 16, None, None, 16, 4, 8, 16, 256, 256, 1 << 30, 16, 16, None]
    assert L.mla_decode(*args) == N.MLA_ERR_INVALID_ARG
    args = [dp, 2, 1, 16, 16, None, None, 16, 4, 8, 16, 257, 256, 1 << 30, 16, 16, None]
    assert L.mla_decode(*args) == N.MLA_ERR_INVALID_ARG
    simt = _v3(N, flags=N.MLA_FLAG_SIMT_DECODE)  # its size needs no device query
    args = [ctypes.byref(simt), 2, 1, 16, 16, None, None, 16, 4, 8, 16, 256, 256, 0, 16, 16, None]
    assert L.mla_decode(*args) == N.MLA_ERR_WORKSPACE_TOO_SMALL
    args = [dp, 2, 1, 16, 16, None, None, 16, 4, 8, 16, 256, 8, 1 << 30, 16, 16, None]
    assert L.mla_decode(*args) == N.MLA_ERR_INVALID_ARG
    # query rows (B * s_q) and table positions (max_blocks * page) must fit in int
    sp = ctypes.byref(simt)
    args = [sp, 1 << 20, 1 << 12, 16, 16, None, None, 16, 4, 8, 16, 256, 256, 1 << 40, 16, 16, None]
    assert L.mla_decode(*args) == N.MLA_ERR_INVALID_ARG
    args = [sp, 2, 1, 16, 16, None, None, 16, 1 << 26, 8, 16, 256, 256, 1 << 40, 16, 16, None]
    assert L.mla_decode(*args) == N.MLA_ERR_INVALID_ARG
    assert N.mla_decode_workspace_size(simt, 1 << 20, 1 << 12, 4096) == 0
    assert L.mla_cache_append(dp, 1, 8, 8, 8, 8, 8, 1, 1 << 26, 1, 8, None, None, None) == N.MLA_ERR_INVALID_ARG
    # decode + projection: the decode's checks, plus w_uv, o, and a 16-byte aligned o_lat
    def dp_call(w_uv=16, o=16, out_dtype=0, o_lat=16, q_abs=16, B=2):
        return L.mla_decode_project(dp, B, 1, q_abs, 16, None, None, 16, 4, 8, 16, 256, 256, 1 << 30,
                                    w_uv, o, out_dtype, o_lat, 16, None)
    assert dp_call(w_uv=None) == N.MLA_ERR_INVALID_ARG
    assert dp_call(o=None) == N.MLA_ERR_INVALID_ARG
    assert dp_call(o_lat=None) == N.MLA_ERR_INVALID_ARG
    assert dp_call(o_lat=8) == N.MLA_ERR_INVALID_ARG
    assert dp_call(q_abs=None) == N.MLA_ERR_INVALID_ARG
    assert dp_call(out_dtype=N.MLA_DTYPE_FP8_E4M3) == N.MLA_ERR_UNSUPPORTED
    assert dp_call(B=0, w_uv=None) == N.MLA_OK
    # append + absorb in one call: each part's checks, before anything is launched
    def aa(T_new=4, c_kv=16, T=4, q_c=16, kr=None):
        return L.mla_append_absorb(dp, T_new, c_kv, 16, 16, 16, 16, 2, 4, 8, 16, kr, None, T, q_c, 16, 16, 16, 16,
                                   None)
    assert aa(c_kv=None) == N.MLA_ERR_INVALID_ARG and aa(q_c=None) == N.MLA_ERR_INVALID_ARG
    assert aa(T_new=-1) == N.MLA_ERR_INVALID_ARG and aa(T=-1) == N.MLA_ERR_INVALID_ARG
    assert aa(kr=16) == N.MLA_ERR_INVALID_ARG  # a RoPE pool only with the FP8 cache
    assert aa(T_new=0, c_kv=None, T=0, q_c=None) == N.MLA_OK
    # prefill: the supported shape, sizes, null and misaligned pointers, workspace size
    def pf(B=2, T=256, max_len=128, cu=16, q_c=16, q_r=16, o=16, ws=256, ws_bytes=1 << 40, d=dp):
        return L.mla_prefill(d, B, cu, T, max_len, q_c, q_r, 16, 16, 16, 16, ws, ws_bytes, o, None, None)
    assert pf(B=0) == N.MLA_OK and pf(T=0) == N.MLA_OK
    assert pf(B=-1) == N.MLA_ERR_INVALID_ARG and pf(max_len=0) == N.MLA_ERR_INVALID_ARG
    assert pf(cu=None) == N.MLA_ERR_INVALID_ARG and pf(q_c=8) == N.MLA_ERR_INVALID_ARG
    assert pf(q_r=8) == N.MLA_ERR_INVALID_ARG
    assert pf(o=8) == N.MLA_ERR_INVALID_ARG and pf(ws=16) == N.MLA_ERR_INVALID_ARG
    assert pf(ws_bytes=1024) == N.MLA_ERR_WORKSPACE_TOO_SMALL
    assert pf(B=70000) == N.MLA_ERR_INVALID_ARG
    odd = _v3(N)
    odd.n_h = 3
    assert pf(d=ctypes.byref(odd)) == N.MLA_ERR_UNSUPPORTED
    assert N.mla_prefill_workspace_size(odd, 256) == 0
    w1, w2 = N.mla_prefill_workspace_size(d, 256), N.mla_prefill_workspace_size(d, 257)
    assert 0 < w1 < w2
    # sequence-split merge: sizes, null pointers with work to do, (rows, n_h) within int
    for f in (L.mla_lse_merge_prepare, L.mla_lse_merge_finish):
        for rows, n_h, d_c in [(-1, 1, 1), (1, 0, 1), (1, 1, 0), (1 << 20, 1 << 12, 8)]:
            assert f(rows, n_h, d_c, 16, 16, 16, 16, None) == N.MLA_ERR_INVALID_ARG
        assert f(0, 1, 1, None, None, None, None, None) == N.MLA_OK
    assert L.mla_lse_merge_prepare(1, 1, 1, None, 16, 16, 16, None) == N.MLA_ERR_INVALID_ARG
    assert L.mla_lse_merge_prepare(1, 1, 1, 16, 16, 16, None, None) == N.MLA_ERR_INVALID_ARG
    assert L.mla_lse_merge_finish(1, 1, 1, 16, 16, None, 16, None) == N.MLA_ERR_INVALID_ARG


def test_workspace_size_is_positive_and_monotone(N):
    d = _v3(N, flags=N.MLA_FLAG_SIMT_DECODE)
    a = N.mla_decode_workspace_size(d, 16, 1, 4096)
    b = N.mla_decode_workspace_size(d, 64, 1, 16384)
    assert 0 < a <= b
    assert N.mla_decode_workspace_size(d, 4, 0, 4096) == 0
