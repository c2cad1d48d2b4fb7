"""ctypes binding of libmla (include/mla.h): same names, argument marshalling only.

Every function takes torch CUDA tensors (or raw device addresses as ints) and the
stream to enqueue on (default: torch's current stream), passes their device
pointers to the C ABI and raises :class:`MLAError` on a non-OK status.  All
computation happens in libmla's CUDA kernels; there is no fallback: if the
library is not built, importing this module fails.
"""
from __future__ import annotations

import ctypes
import os
import re

_PKG = os.path.dirname(os.path.abspath(__file__))
# MLA_LIBRARY may point at another build of the same library (e.g. an instrumented one).
LIB_PATH = os.environ.get("MLA_LIBRARY") or os.path.join(_PKG, "libmla.so")
HEADER = os.path.join(os.path.dirname(_PKG), "include", "mla.h")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is not built; run `python -m mla_latent_kv_mqa_b200.build`")

_lib = ctypes.CDLL(LIB_PATH)

# mla_status_t
MLA_OK = 0
MLA_ERR_INVALID_ARG = 1
MLA_ERR_UNSUPPORTED = 2
MLA_ERR_WORKSPACE_TOO_SMALL = 3
MLA_ERR_BAD_BLOCK_TABLE = 4
MLA_ERR_BAD_SEQ_LEN = 5
MLA_ERR_DEVICE_TIMEOUT = 6
MLA_ERR_CUDA = 7
# mla_dtype_t
MLA_DTYPE_F32 = 0
MLA_DTYPE_BF16 = 1
MLA_DTYPE_FP8_E4M3 = 2
MLA_FLAG_SIMT_DECODE = 1
MLA_FLAG_SIMT_PROJ = 2
MLA_FLAG_TEST_GIVE_UP = 4
MLA_FLAG_FP8_MMA = 8


class MLAError(RuntimeError):
    def __init__(self, status: int, call: str):
        self.status = status
        super().__init__(f"{call} -> {status_string(status)}")


class mla_dims_t(ctypes.Structure):
    _fields_ = [("n_h", ctypes.c_int), ("d_h", ctypes.c_int), ("d_c", ctypes.c_int),
                ("d_r", ctypes.c_int), ("page_size", ctypes.c_int), ("rope_base", ctypes.c_float),
                ("act_dtype", ctypes.c_int), ("kv_dtype", ctypes.c_int), ("flags", ctypes.c_uint)]


def make_dims(n_h, d_h, d_c, d_r, page_size=64, rope_base=1e4, act_dtype=MLA_DTYPE_BF16,
              kv_dtype=MLA_DTYPE_BF16, flags=0) -> mla_dims_t:
    return mla_dims_t(n_h, d_h, d_c, d_r, page_size, rope_base, act_dtype, kv_dtype, flags)


_vp, _i, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
_dp = ctypes.POINTER(mla_dims_t)
_lib.mla_absorb_q.argtypes = [_dp, _i, _vp, _vp, _vp, _vp, _vp, _vp]
_lib.mla_cache_append.argtypes = [_dp, _i, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _vp, _vp, _vp, _vp]
_lib.mla_decode_workspace_size.argtypes = [_dp, _i, _i, _i]
_lib.mla_decode_workspace_size.restype = _sz
_lib.mla_decode.argtypes = [_dp, _i, _i, _vp, _vp, _vp, _vp, _vp, _i, _i, _vp, _i, _vp, _sz, _vp,
                            _vp, _vp]
_lib.mla_decode_fixed_scratch.argtypes = [_dp, _i, _i, _vp, _vp, _vp, _vp, _vp, _i, _i, _vp, _i,
                                          _vp, _vp, _vp]
_lib.mla_out_proj.argtypes = [_dp, _i, _vp, _vp, _vp, _i, _vp]
_lib.mla_append_absorb.argtypes = [_dp, _i, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _vp, _vp, _vp, _i, _vp, _vp, _vp,
                                   _vp, _vp, _vp]
_lib.mla_decode_project.argtypes = [_dp, _i, _i, _vp, _vp, _vp, _vp, _vp, _i, _i, _vp, _i, _vp, _sz,
                                    _vp, _vp, _i, _vp, _vp, _vp]
_lib.mla_prefill_workspace_size.argtypes = [_dp, _i]
_lib.mla_prefill_workspace_size.restype = _sz
_lib.mla_prefill.argtypes = [_dp, _i, _vp, _i, _i, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp, _vp, _vp]
_lib.mla_lse_merge_prepare.argtypes = [_i, _i, _i, _vp, _vp, _vp, _vp, _vp]
_lib.mla_lse_merge_finish.argtypes = [_i, _i, _i, _vp, _vp, _vp, _vp, _vp]
_lib.mla_get_last_device_error.argtypes = []
_lib.mla_status_string.argtypes = [_i]
_lib.mla_status_string.restype = ctypes.c_char_p
_lib.mla_version.restype = _i
for _f in ("mla_absorb_q", "mla_cache_append", "mla_decode", "mla_decode_fixed_scratch", "mla_out_proj",
           "mla_decode_project", "mla_prefill", "mla_append_absorb", "mla_get_last_device_error",
           "mla_lse_merge_prepare",
           "mla_lse_merge_finish"):
    getattr(_lib, _f).restype = _i


def declared_functions() -> list[str]:
    """Names of the functions include/mla.h declares."""
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(mla_[a-z_0-9]+)\s*\(", src)))


def library() -> ctypes.CDLL:
    return _lib


def _ptr(x):
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(rc: int, call: str):
    if rc != MLA_OK:
        raise MLAError(rc, call)


def status_string(status: int) -> str:
    return _lib.mla_status_string(status).decode()


def version() -> int:
    return _lib.mla_version()


def mla_absorb_q(dims, T, q_c, q_r, pos, w_uk, q_abs, stream=None):
    _check(_lib.mla_absorb_q(ctypes.byref(dims), T, _ptr(q_c), _ptr(q_r), _ptr(pos), _ptr(w_uk),
                             _ptr(q_abs), _stream(stream)), "mla_absorb_q")


def mla_cache_append(dims, T, c_kv, k_r, seq_idx, pos, block_table, num_seqs, max_blocks_per_seq,
                     num_blocks, kv_pool, kr_pool=None, kv_scale=None, stream=None):
    _check(_lib.mla_cache_append(ctypes.byref(dims), T, _ptr(c_kv), _ptr(k_r), _ptr(seq_idx),
                                 _ptr(pos), _ptr(block_table), num_seqs, max_blocks_per_seq,
                                 num_blocks, _ptr(kv_pool), _ptr(kr_pool), _ptr(kv_scale),
                                 _stream(stream)), "mla_cache_append")


def mla_append_absorb(dims, T_new, c_kv, k_r, seq_idx, pos_new, block_table, num_seqs, max_blocks_per_seq,
                      num_blocks, kv_pool, kr_pool, kv_scale, T, q_c, q_r, pos, w_uk, q_abs, stream=None):
    """mla_cache_append then mla_absorb_q (one launch where the tensor-core absorption applies)."""
    _check(_lib.mla_append_absorb(ctypes.byref(dims), T_new, _ptr(c_kv), _ptr(k_r), _ptr(seq_idx), _ptr(pos_new),
                                  _ptr(block_table), num_seqs, max_blocks_per_seq, num_blocks, _ptr(kv_pool),
                                  _ptr(kr_pool), _ptr(kv_scale), T, _ptr(q_c), _ptr(q_r), _ptr(pos), _ptr(w_uk),
                                  _ptr(q_abs), _stream(stream)), "mla_append_absorb")


def mla_decode_workspace_size(dims, B, s_q, max_seq_len) -> int:
    return int(_lib.mla_decode_workspace_size(ctypes.byref(dims), B, s_q, max_seq_len))


def mla_decode(dims, B, s_q, q_abs, kv_pool, kr_pool, kv_scale, block_table, max_blocks_per_seq,
               num_blocks, seq_lens, max_seq_len, workspace, workspace_bytes, o_lat, lse=None,
               stream=None):
    _check(_lib.mla_decode(ctypes.byref(dims), B, s_q, _ptr(q_abs), _ptr(kv_pool), _ptr(kr_pool),
                           _ptr(kv_scale), _ptr(block_table), max_blocks_per_seq, num_blocks,
                           _ptr(seq_lens), max_seq_len, _ptr(workspace), workspace_bytes,
                           _ptr(o_lat), _ptr(lse), _stream(stream)), "mla_decode")


def mla_decode_fixed_scratch(dims, B, s_q, q_abs, kv_pool, kr_pool, kv_scale, block_table,
                             max_blocks_per_seq, num_blocks, seq_lens, max_seq_len, o_lat, lse=None,
                             stream=None):
    """mla_decode on the library's static scratch array (no workspace argument)."""
    _check(_lib.mla_decode_fixed_scratch(ctypes.byref(dims), B, s_q, _ptr(q_abs), _ptr(kv_pool),
                                         _ptr(kr_pool), _ptr(kv_scale), _ptr(block_table),
                                         max_blocks_per_seq, num_blocks, _ptr(seq_lens), max_seq_len,
                                         _ptr(o_lat), _ptr(lse), _stream(stream)),
           "mla_decode_fixed_scratch")


def mla_out_proj(dims, T, o_lat, w_uv, o, out_dtype=MLA_DTYPE_F32, stream=None):
    _check(_lib.mla_out_proj(ctypes.byref(dims), T, _ptr(o_lat), _ptr(w_uv), _ptr(o), out_dtype,
                             _stream(stream)), "mla_out_proj")


def mla_decode_project(dims, B, s_q, q_abs, kv_pool, kr_pool, kv_scale, block_table, max_blocks_per_seq,
                       num_blocks, seq_lens, max_seq_len, workspace, workspace_bytes, w_uv, o, out_dtype,
                       o_lat, lse=None, stream=None):
    """mla_decode followed by mla_out_proj (one fused merge + projection kernel where it applies)."""
    _check(_lib.mla_decode_project(ctypes.byref(dims), B, s_q, _ptr(q_abs), _ptr(kv_pool), _ptr(kr_pool),
                                   _ptr(kv_scale), _ptr(block_table), max_blocks_per_seq, num_blocks,
                                   _ptr(seq_lens), max_seq_len, _ptr(workspace), workspace_bytes, _ptr(w_uv),
                                   _ptr(o), out_dtype, _ptr(o_lat), _ptr(lse), _stream(stream)),
           "mla_decode_project")


def mla_prefill_workspace_size(dims, total_tokens) -> int:
    return int(_lib.mla_prefill_workspace_size(ctypes.byref(dims), total_tokens))


def mla_prefill(dims, B, cu_seqlens, total_tokens, max_seq_len, q_c, q_r, c_kv, k_r, w_uk, w_uv, workspace,
                workspace_bytes, o, lse=None, stream=None):
    _check(_lib.mla_prefill(ctypes.byref(dims), B, _ptr(cu_seqlens), total_tokens, max_seq_len, _ptr(q_c), _ptr(q_r),
                            _ptr(c_kv), _ptr(k_r), _ptr(w_uk), _ptr(w_uv), _ptr(workspace), workspace_bytes, _ptr(o),
                            _ptr(lse), _stream(stream)), "mla_prefill")


def mla_lse_merge_prepare(rows, n_h, d_c, o_lat, lse, lse_max, acc, stream=None):
    _check(_lib.mla_lse_merge_prepare(rows, n_h, d_c, _ptr(o_lat), _ptr(lse), _ptr(lse_max), _ptr(acc),
                                      _stream(stream)), "mla_lse_merge_prepare")


def mla_lse_merge_finish(rows, n_h, d_c, acc, lse_max, o_lat, lse=None, stream=None):
    _check(_lib.mla_lse_merge_finish(rows, n_h, d_c, _ptr(acc), _ptr(lse_max), _ptr(o_lat), _ptr(lse),
                                     _stream(stream)), "mla_lse_merge_finish")


def mla_get_last_device_error() -> int:
    return int(_lib.mla_get_last_device_error())
