"""Python front end of the fp64 CPU oracle (``mla_oracle.c``).

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU
baseline leg of ``bench.py`` may import this module.  The product path never
does; it shares no code with the CUDA library.

What the oracle computes follows the itwiki article "멀티 헤드 잠재 어텐션"
(Multi-head latent attention):

* ``decode_absorbed`` -- MQA mode (sections 행렬 흡수 "matrix absorption" and
  구현 "implementation", forward_absorbed): ``q_lat = W_UK,h^T q_C``, scores
  over the (d_c + d_R)-wide cached row scaled by ``1/sqrt(d_h + d_R)``
  (section 분리 RoPE, output equation), softmax, ``o_lat = sum_j p_j c_j``,
  ``o = W_UV,h o_lat``.
* ``decode_naive`` -- MHA mode (section 구조 and 구현 forward_naive): keys and
  values reconstructed per head from the cached latent.
* ``toy_layer`` -- the whole simplified layer of the 구현 section, with the
  down/up projections of section 구조 and the output projection ``u = W_O o``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "mla_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libmla_oracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile ``libmla_oracle.so`` with gcc (-O2, OpenMP) if it is missing or stale."""
    stale = (not os.path.exists(_LIB_PATH)) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC)
    if force or stale:
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB_PATH)
        dp = ctypes.POINTER(ctypes.c_double)
        i64p = ctypes.POINTER(ctypes.c_int64)
        u8p = ctypes.POINTER(ctypes.c_uint8)
        fp = ctypes.POINTER(ctypes.c_float)
        ci, cd = ctypes.c_int, ctypes.c_double
        L.mla_oracle_rope.argtypes = [ci, cd, cd, dp, dp]
        L.mla_oracle_softmax.argtypes = [ci, dp, dp]
        L.mla_oracle_softmax.restype = cd
        L.mla_oracle_decode_absorbed.argtypes = [ci] * 6 + [cd, dp, dp, i64p, i64p, dp, dp, dp, dp,
                                                           dp, dp, dp, dp, dp, ci]
        L.mla_oracle_decode_absorbed.restype = ci
        L.mla_oracle_decode_naive.argtypes = [ci] * 6 + [cd, dp, dp, i64p, i64p, dp, dp, dp, dp,
                                                        dp, dp]
        L.mla_oracle_decode_naive.restype = ci
        L.mla_oracle_e4m3_value.argtypes = [ctypes.c_uint8]
        L.mla_oracle_e4m3_value.restype = cd
        L.mla_oracle_e4m3_quantize.argtypes = [ctypes.c_float]
        L.mla_oracle_e4m3_quantize.restype = ctypes.c_uint8
        L.mla_oracle_quantize_rows.argtypes = [ctypes.c_int64, ci, fp, u8p, fp]
        L.mla_oracle_dequantize_rows.argtypes = [ctypes.c_int64, ci, u8p, fp, dp]
        L.mla_oracle_cache_row_elems.argtypes = [ci, ci]
        L.mla_oracle_cache_row_elems.restype = ci
        L.mla_oracle_num_threads.restype = ci
        L.mla_oracle_set_num_threads.argtypes = [ci]
        _lib = L
    return _lib


def _dp(a: np.ndarray):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.float64)


def num_threads() -> int:
    return int(lib().mla_oracle_num_threads())


def set_num_threads(n: int) -> None:
    """Host threads of the following oracle calls (results are independent of it)."""
    lib().mla_oracle_set_num_threads(int(n))


def rope(x, pos: float, base: float = 1e4) -> np.ndarray:
    """Half-split RoPE of one vector (구현 section, ``rope``)."""
    x = _f64(x)
    out = np.empty_like(x)
    lib().mla_oracle_rope(x.shape[-1], base, float(pos), _dp(x), _dp(out))
    return out


def softmax(s) -> tuple[np.ndarray, float]:
    s = _f64(s)
    p = np.empty_like(s)
    lse = lib().mla_oracle_softmax(s.shape[0], _dp(s), _dp(p))
    return p, lse


@dataclass
class DecodeResult:
    o: np.ndarray            # [T, n_h, d_h]
    lse: np.ndarray          # [T, n_h], natural log
    o_lat: np.ndarray | None = None   # [T, n_h, d_c] (absorbed mode only)
    q_lat: np.ndarray | None = None   # [T, n_h, d_c] (absorbed mode only)
    probs: np.ndarray | None = None   # [T, n_h, max_L] (absorbed mode, on request)


def _ctx_offsets(ctx_lens) -> np.ndarray:
    off = np.zeros(len(ctx_lens) + 1, dtype=np.int64)
    off[1:] = np.cumsum(np.asarray(ctx_lens, dtype=np.int64))
    return off


def decode_absorbed(q_c, q_r, q_pos, c_kv_seqs, k_r_seqs, w_uk, w_uv, *, s_q: int = 1,
                    rope_base: float = 1e4, want_probs: bool = False) -> DecodeResult:
    """MQA-mode decode.

    q_c [T, n_h, d_h], q_r [T, n_h, d_R] (before RoPE), q_pos [T] with T = B*s_q;
    c_kv_seqs / k_r_seqs: lists of B arrays [L_b, d_c] / [L_b, d_R] (k_R before RoPE;
    token j sits at position j).  Query t of sequence t // s_q sees tokens j <= q_pos[t].
    """
    q_c, q_r = _f64(q_c), _f64(q_r)
    T, n_h, d_h = q_c.shape
    d_r = q_r.shape[-1]
    B = len(c_kv_seqs)
    assert T == B * s_q
    d_c = c_kv_seqs[0].shape[-1]
    off = _ctx_offsets([c.shape[0] for c in c_kv_seqs])
    c_all = _f64(np.concatenate([np.asarray(c, dtype=np.float64) for c in c_kv_seqs], 0))
    k_all = _f64(np.concatenate([np.asarray(k, dtype=np.float64) for k in k_r_seqs], 0))
    pos = np.ascontiguousarray(q_pos, dtype=np.int64)
    w_uk, w_uv = _f64(w_uk), _f64(w_uv)
    q_lat = np.empty((T, n_h, d_c))
    o_lat = np.empty((T, n_h, d_c))
    lse = np.empty((T, n_h))
    o = np.empty((T, n_h, d_h))
    maxL = int(max(c.shape[0] for c in c_kv_seqs))
    probs = np.empty((T, n_h, maxL)) if want_probs else None
    i64p = ctypes.POINTER(ctypes.c_int64)
    rc = lib().mla_oracle_decode_absorbed(
        B, s_q, n_h, d_h, d_c, d_r, rope_base, _dp(q_c), _dp(q_r), pos.ctypes.data_as(i64p),
        off.ctypes.data_as(i64p), _dp(c_all), _dp(k_all), _dp(w_uk), _dp(w_uv), _dp(q_lat),
        _dp(o_lat), _dp(lse), _dp(o), _dp(probs) if want_probs else None, maxL)
    if rc != 0:
        raise ValueError(f"oracle decode_absorbed failed with code {rc}")
    return DecodeResult(o=o, lse=lse, o_lat=o_lat, q_lat=q_lat, probs=probs)


def decode_naive(q_c, q_r, q_pos, c_kv_seqs, k_r_seqs, w_uk, w_uv, *, s_q: int = 1,
                 rope_base: float = 1e4) -> DecodeResult:
    """MHA-mode decode with the same arguments as :func:`decode_absorbed`."""
    q_c, q_r = _f64(q_c), _f64(q_r)
    T, n_h, d_h = q_c.shape
    d_r = q_r.shape[-1]
    B = len(c_kv_seqs)
    assert T == B * s_q
    d_c = c_kv_seqs[0].shape[-1]
    off = _ctx_offsets([c.shape[0] for c in c_kv_seqs])
    c_all = _f64(np.concatenate([np.asarray(c, dtype=np.float64) for c in c_kv_seqs], 0))
    k_all = _f64(np.concatenate([np.asarray(k, dtype=np.float64) for k in k_r_seqs], 0))
    pos = np.ascontiguousarray(q_pos, dtype=np.int64)
    w_uk, w_uv = _f64(w_uk), _f64(w_uv)
    lse = np.empty((T, n_h))
    o = np.empty((T, n_h, d_h))
    i64p = ctypes.POINTER(ctypes.c_int64)
    rc = lib().mla_oracle_decode_naive(
        B, s_q, n_h, d_h, d_c, d_r, rope_base, _dp(q_c), _dp(q_r), pos.ctypes.data_as(i64p),
        off.ctypes.data_as(i64p), _dp(c_all), _dp(k_all), _dp(w_uk), _dp(w_uv), _dp(lse), _dp(o))
    if rc != 0:
        raise ValueError(f"oracle decode_naive failed with code {rc}")
    return DecodeResult(o=o, lse=lse)


# --------------------------------------------------------------------------------------------
# FP8 e4m3 content cache (QuantMLA review page, "Motivation & Problem Statement").
# --------------------------------------------------------------------------------------------

def e4m3_value(code: int) -> float:
    return float(lib().mla_oracle_e4m3_value(ctypes.c_uint8(code)))


def e4m3_quantize(v: float) -> int:
    return int(lib().mla_oracle_e4m3_quantize(ctypes.c_float(v)))


def quantize_rows(c) -> tuple[np.ndarray, np.ndarray]:
    """Per-token e4m3 codes and fp32 scales of rows ``c`` [n, d_c] (float32 values)."""
    c = np.ascontiguousarray(c, dtype=np.float32)
    n, d_c = c.shape
    codes = np.empty((n, d_c), dtype=np.uint8)
    scales = np.empty(n, dtype=np.float32)
    lib().mla_oracle_quantize_rows(n, d_c, c.ctypes.data_as(ctypes.POINTER(ctypes.c_float)),
                                   codes.ctypes.data_as(ctypes.POINTER(ctypes.c_uint8)),
                                   scales.ctypes.data_as(ctypes.POINTER(ctypes.c_float)))
    return codes, scales


def dequantize_rows(codes, scales) -> np.ndarray:
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.float32)
    n, d_c = codes.shape
    out = np.empty((n, d_c))
    lib().mla_oracle_dequantize_rows(n, d_c, codes.ctypes.data_as(ctypes.POINTER(ctypes.c_uint8)),
                                     scales.ctypes.data_as(ctypes.POINTER(ctypes.c_float)), _dp(out))
    return out


def cache_row_elems(d_c: int, d_r: int) -> int:
    return int(lib().mla_oracle_cache_row_elems(d_c, d_r))


# --------------------------------------------------------------------------------------------
# The simplified layer of the 구현 section (projections of section 구조 and 분리 RoPE).
# --------------------------------------------------------------------------------------------

@dataclass
class ToyLayerResult:
    c_kv: np.ndarray   # [B, T, d_c]
    k_r: np.ndarray    # [B, T, d_R]  (before RoPE)
    q_c: np.ndarray    # [B, T, n_h, d_h]
    q_r: np.ndarray    # [B, T, n_h, d_R] (before RoPE)
    o: np.ndarray      # [B, T_q, n_h, d_h]
    lse: np.ndarray    # [B, T_q, n_h]
    u: np.ndarray      # [B, T_q, d]
    o_lat: np.ndarray | None = None


def toy_projections(h, W):
    """Down/up projections of the 구조 and 분리 RoPE sections, in fp64:
    c_kv = W_DKV h, k_R = W_KR h, c_q = W_DQ h, q_C = W_UQ c_q, q_R = W_QR c_q."""
    h = _f64(h)
    B, T, _ = h.shape
    n_h, d_h, d_r = W["n_h"], W["d_h"], W["d_r"]
    c_kv = h @ _f64(W["w_dkv"]).T
    k_r = h @ _f64(W["w_kr"]).T
    c_q = h @ _f64(W["w_dq"]).T
    q_c = (c_q @ _f64(W["w_uq"]).T).reshape(B, T, n_h, d_h)
    q_r = (c_q @ _f64(W["w_qr"]).T).reshape(B, T, n_h, d_r)
    return c_kv, k_r, q_c, q_r


def toy_layer(h, W, *, mode: str = "absorbed", last_only: bool = False,
              rope_base: float = 1e4) -> ToyLayerResult:
    """Whole simplified layer for input ``h`` [B, T, d] at positions 0..T-1.

    ``last_only``: decode form -- only the last token queries (over all T cached tokens);
    otherwise every token queries with the causal mask (the page's prefill form)."""
    c_kv, k_r, q_c, q_r = toy_projections(h, W)
    B, T = c_kv.shape[:2]
    qsel = slice(T - 1, T) if last_only else slice(0, T)
    s_q = 1 if last_only else T
    pos = np.tile(np.arange(T)[qsel], B)
    qc = q_c[:, qsel].reshape(B * s_q, W["n_h"], W["d_h"])
    qr = q_r[:, qsel].reshape(B * s_q, W["n_h"], W["d_r"])
    args = (qc, qr, pos, [c_kv[b] for b in range(B)], [k_r[b] for b in range(B)],
            W["w_uk"], W["w_uv"])
    if mode == "absorbed":
        r = decode_absorbed(*args, s_q=s_q, rope_base=rope_base)
    elif mode == "naive":
        r = decode_naive(*args, s_q=s_q, rope_base=rope_base)
    else:
        raise ValueError(mode)
    o = r.o.reshape(B, s_q, W["n_h"], W["d_h"])
    u = o.reshape(B, s_q, -1) @ _f64(W["w_o"]).T
    return ToyLayerResult(c_kv=c_kv, k_r=k_r, q_c=q_c, q_r=q_r, o=o,
                          lse=r.lse.reshape(B, s_q, W["n_h"]), u=u,
                          o_lat=None if r.o_lat is None else r.o_lat.reshape(B, s_q, W["n_h"], -1))
