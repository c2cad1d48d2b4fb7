"""User-facing objects over the C ABI: the paged latent cache and one MLA decode layer.

PyTorch only allocates device memory and supplies streams here; each step of the
decode path runs in libmla's kernels through :mod:`.native`.

A decode step of one layer (itwiki "멀티 헤드 잠재 어텐션", sections 분리 RoPE and
행렬 흡수) is::

    layer.append(cache, c_kv_new, k_r_new, seq_idx, pos, block_table)   # cache rows
    q_abs = layer.absorb(q_c, q_r, pos_q)                                # [W_UK^T q_C ; RoPE(q_R)]
    o_lat, lse = layer.decode(cache, q_abs, block_table, seq_lens, s_q)  # attention over the cache
    o = layer.out_proj(o_lat)                                            # W_UV o_lat
"""
from __future__ import annotations

import torch

from . import native as N

DTYPE = {"f32": N.MLA_DTYPE_F32, "bf16": N.MLA_DTYPE_BF16, "fp8": N.MLA_DTYPE_FP8_E4M3}
TORCH_ACT = {N.MLA_DTYPE_F32: torch.float32, N.MLA_DTYPE_BF16: torch.bfloat16}


def dims_for(n_h, d_h, d_c, d_r, *, act="bf16", kv="bf16", page=64, rope_base=1e4, flags=0):
    return N.make_dims(n_h, d_h, d_c, d_r, page, rope_base, DTYPE[act], DTYPE[kv], flags)


class PagedLatentCache:
    """Device buffers of a paged latent cache with ``num_blocks`` blocks of ``page_size`` tokens.

    bf16 / f32: ``kv_pool`` [num_blocks, page, d_c + d_r] rows [c_kv ; RoPE(k_r)].
    fp8: ``kv_pool`` [num_blocks, page, d_c] e4m3 codes, ``kr_pool`` [num_blocks, page, d_r]
    bf16, ``kv_scale`` [num_blocks, page] fp32.  ``poison`` fills every slot with NaN first."""

    def __init__(self, dims: N.mla_dims_t, num_blocks: int, device="cuda", poison: bool = False):
        self.dims = dims
        self.num_blocks = int(num_blocks)
        page = dims.page_size
        self.kr_pool = None
        self.kv_scale = None
        if dims.kv_dtype == N.MLA_DTYPE_FP8_E4M3:
            self.kv_pool = torch.empty((num_blocks, page, dims.d_c), dtype=torch.uint8, device=device)
            self.kr_pool = torch.empty((num_blocks, page, dims.d_r), dtype=torch.bfloat16, device=device)
            self.kv_scale = torch.empty((num_blocks, page), dtype=torch.float32, device=device)
            if poison:
                self.kv_pool.fill_(0x7F)
                self.kr_pool.fill_(float("nan"))
                self.kv_scale.fill_(float("nan"))
        else:
            dt = torch.float32 if dims.kv_dtype == N.MLA_DTYPE_F32 else torch.bfloat16
            self.kv_pool = torch.empty((num_blocks, page, dims.d_c + dims.d_r), dtype=dt, device=device)
            if poison:
                self.kv_pool.fill_(float("nan"))

    @property
    def nbytes(self) -> int:
        n = self.kv_pool.numel() * self.kv_pool.element_size()
        if self.kr_pool is not None:
            n += self.kr_pool.numel() * self.kr_pool.element_size()
            n += self.kv_scale.numel() * self.kv_scale.element_size()
        return n


class MLADecodeLayer:
    """Weights of one MLA layer (W_UK, W_UV as [n_h*d_h, d_c]) plus reusable decode and
    prefill workspaces."""

    def __init__(self, dims: N.mla_dims_t, w_uk: torch.Tensor, w_uv: torch.Tensor):
        self.dims = dims
        self.w_uk = w_uk.contiguous()
        self.w_uv = w_uv.contiguous()
        self.device = w_uk.device
        self._ws = None
        self._ws_key = None
        self._pf_ws = None

    # -- the four calls ----------------------------------------------------------------------
    def append(self, cache: PagedLatentCache, c_kv, k_r, seq_idx, pos, block_table, stream=None):
        T = c_kv.shape[0]
        B, max_blocks = block_table.shape
        N.mla_cache_append(self.dims, T, c_kv, k_r, seq_idx, pos, block_table, B, max_blocks,
                           cache.num_blocks, cache.kv_pool, cache.kr_pool, cache.kv_scale, stream)

    def absorb(self, q_c, q_r, pos, out=None, stream=None):
        T = q_c.shape[0]
        d = self.dims
        if out is None:
            out = torch.empty((T, d.n_h, d.d_c + d.d_r), dtype=TORCH_ACT[d.act_dtype], device=self.device)
        N.mla_absorb_q(d, T, q_c, q_r, pos, self.w_uk, out, stream)
        return out

    def append_absorb(self, cache: PagedLatentCache, c_kv, k_r, seq_idx, pos_new, block_table, q_c, q_r, pos,
                      out=None, stream=None):
        """append then absorb in one library call; returns q_abs."""
        T_new = c_kv.shape[0]
        B, max_blocks = block_table.shape
        T = q_c.shape[0]
        d = self.dims
        if out is None:
            out = torch.empty((T, d.n_h, d.d_c + d.d_r), dtype=TORCH_ACT[d.act_dtype], device=self.device)
        N.mla_append_absorb(d, T_new, c_kv, k_r, seq_idx, pos_new, block_table, B, max_blocks, cache.num_blocks,
                            cache.kv_pool, cache.kr_pool, cache.kv_scale, T, q_c, q_r, pos, self.w_uk, out, stream)
        return out

    def workspace(self, B, s_q, max_seq_len):
        key = (B, s_q, max_seq_len)
        if self._ws_key != key:
            n = N.mla_decode_workspace_size(self.dims, B, s_q, max_seq_len)
            if self._ws is None or self._ws.numel() < n:
                self._ws = torch.empty(max(n, 256), dtype=torch.uint8, device=self.device)
            self._ws_key = key
        return self._ws

    def decode(self, cache: PagedLatentCache, q_abs, block_table, seq_lens, s_q, max_seq_len,
               o_lat=None, lse=None, stream=None):
        d = self.dims
        B, max_blocks = block_table.shape
        rows = B * s_q
        if o_lat is None:
            o_lat = torch.empty((rows, d.n_h, d.d_c), dtype=torch.float32, device=self.device)
        if lse is None:
            lse = torch.empty((rows, d.n_h), dtype=torch.float32, device=self.device)
        ws = self.workspace(B, s_q, max_seq_len)
        N.mla_decode(d, B, s_q, q_abs, cache.kv_pool, cache.kr_pool, cache.kv_scale, block_table,
                     max_blocks, cache.num_blocks, seq_lens, max_seq_len, ws, ws.numel(), o_lat,
                     lse, stream)
        return o_lat, lse

    def decode_project(self, cache: PagedLatentCache, q_abs, block_table, seq_lens, s_q, max_seq_len,
                       out_dtype="f32", o=None, o_lat=None, lse=None, stream=None):
        """decode followed by out_proj in one library call; returns (o, o_lat, lse)."""
        d = self.dims
        B, max_blocks = block_table.shape
        rows = B * s_q
        dt = DTYPE[out_dtype]
        if o is None:
            o = torch.empty((rows, d.n_h, d.d_h), dtype=TORCH_ACT[dt], device=self.device)
        if o_lat is None:
            o_lat = torch.empty((rows, d.n_h, d.d_c), dtype=torch.float32, device=self.device)
        if lse is None:
            lse = torch.empty((rows, d.n_h), dtype=torch.float32, device=self.device)
        ws = self.workspace(B, s_q, max_seq_len)
        N.mla_decode_project(d, B, s_q, q_abs, cache.kv_pool, cache.kr_pool, cache.kv_scale, block_table,
                             max_blocks, cache.num_blocks, seq_lens, max_seq_len, ws, ws.numel(), self.w_uv,
                             o, dt, o_lat, lse, stream)
        return o, o_lat, lse

    def prefill(self, q_c, q_r, c_kv, k_r, cu_seqlens, max_seq_len, o=None, lse=None, stream=None):
        """Causal MHA-mode attention over packed prompts (cu_seqlens [B + 1] int32 on the
        device); returns (o [T, n_h, d_h] bf16, lse [T, n_h])."""
        d = self.dims
        T = q_c.shape[0]
        B = cu_seqlens.numel() - 1
        if o is None:
            o = torch.empty((T, d.n_h, d.d_h), dtype=torch.bfloat16, device=self.device)
        if lse is None:
            lse = torch.empty((T, d.n_h), dtype=torch.float32, device=self.device)
        n = N.mla_prefill_workspace_size(d, T)
        if self._pf_ws is None or self._pf_ws.numel() < n:
            self._pf_ws = torch.empty(max(n, 256), dtype=torch.uint8, device=self.device)
        N.mla_prefill(d, B, cu_seqlens, T, max_seq_len, q_c, q_r, c_kv, k_r, self.w_uk, self.w_uv, self._pf_ws,
                      self._pf_ws.numel(), o, lse, stream)
        return o, lse

    def out_proj(self, o_lat, out_dtype="f32", out=None, stream=None):
        d = self.dims
        T = o_lat.shape[0]
        dt = DTYPE[out_dtype]
        if out is None:
            out = torch.empty((T, d.n_h, d.d_h), dtype=TORCH_ACT[dt], device=self.device)
        N.mla_out_proj(d, T, o_lat, self.w_uv, out, dt, stream)
        return out
