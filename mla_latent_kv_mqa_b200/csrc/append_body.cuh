// The per-token work of mla_cache_append, shared by the append kernel and by the fused
// append + query absorption kernel.
//
// MLA article (itwiki "멀티 헤드 잠재 어텐션"), section 분리 RoPE: the cache holds c^KV_t and
// the shared RoPE key k^R_t = RoPE(W^KR h_t), d_c + d_R values per token.  The FP8 content
// cache with a bf16 RoPE-key cache is the layout the QuantMLA review page ("Motivation &
// Problem Statement") describes as existing practice.
#pragma once
#include <float.h>

#include "mla_internal.cuh"

namespace mla {

struct AppendArgs {
    int T, d_c, d_r, page;
    const void *c_kv, *k_r;
    const int32_t *seq_idx, *pos, *bt;
    int num_seqs, max_blocks, num_blocks;
    void *kv_pool;
    __nv_bfloat16 *kr_pool;
    float *kv_scale;
};

AppendArgs append_args(const mla_dims_t &d, int T, const void *c_kv, const void *k_r, const int32_t *seq_idx,
                       const int32_t *pos, const int32_t *bt, int num_seqs, int max_blocks, int num_blocks,
                       void *kv_pool, void *kr_pool, float *kv_scale);

// One warp writes token t's cache row.  KV: 0 = f32 cache, 1 = bf16 cache, 2 = fp8 content
// cache.  Bad sequence indices, positions or block ids are recorded, never dereferenced.
template <typename Tin, int KV>
__device__ __forceinline__ void append_token(const AppendArgs &a, const RopeFreqs &rope, int t, int lane,
                                             unsigned *err) {
    const int d_c = a.d_c, d_r = a.d_r, page = a.page;
    const Tin *c_kv = reinterpret_cast<const Tin *>(a.c_kv);
    const Tin *k_r = reinterpret_cast<const Tin *>(a.k_r);
    const int32_t *seq_idx = a.seq_idx, *pos = a.pos, *bt = a.bt;
    const int num_seqs = a.num_seqs, max_blocks = a.max_blocks, num_blocks = a.num_blocks;
    void *kv_pool = a.kv_pool;
    __nv_bfloat16 *kr_pool = a.kr_pool;
    float *kv_scale = a.kv_scale;
    const int s = seq_idx[t];
    const int p = pos[t];
    if (s < 0 || s >= num_seqs || p < 0 || p / page >= max_blocks) {
        if (lane == 0) record_error(err, kErrBadBlock);
        return;
    }
    const int blk = bt[(size_t)s * max_blocks + p / page];
    if (blk < 0 || blk >= num_blocks) {
        if (lane == 0) record_error(err, kErrBadBlock);
        return;
    }
    const size_t slot = (size_t)blk * page + (p % page);
    const Tin *c_in = c_kv + (size_t)t * d_c;
    const Tin *k_in = k_r + (size_t)t * d_r;

    // RoPE of the shared key (pairs k, k + d_r/2).
    const int half = d_r >> 1;
    for (int k = lane; k < half; k += 32) {
        float cs, sn;
        rope_cos_sin(rope, k, p, &cs, &sn);
        float x0 = to_f32(k_in[k]), x1 = to_f32(k_in[k + half]);
        float y0 = x0 * cs - x1 * sn;
        float y1 = x1 * cs + x0 * sn;
        if (KV == 0) {
            float *row = reinterpret_cast<float *>(kv_pool) + slot * (d_c + d_r) + d_c;
            row[k] = y0;
            row[k + half] = y1;
        } else if (KV == 1) {
            __nv_bfloat16 *row = reinterpret_cast<__nv_bfloat16 *>(kv_pool) + slot * (d_c + d_r) + d_c;
            row[k] = __float2bfloat16_rn(y0);
            row[k + half] = __float2bfloat16_rn(y1);
        } else {
            __nv_bfloat16 *row = kr_pool + slot * d_r;
            row[k] = __float2bfloat16_rn(y0);
            row[k + half] = __float2bfloat16_rn(y1);
        }
    }

    if (KV == 0) {
        float *row = reinterpret_cast<float *>(kv_pool) + slot * (d_c + d_r);
        for (int k = lane; k < d_c; k += 32) row[k] = to_f32(c_in[k]);
    } else if (KV == 1) {
        __nv_bfloat16 *row = reinterpret_cast<__nv_bfloat16 *>(kv_pool) + slot * (d_c + d_r);
        for (int k = lane; k < d_c; k += 32) row[k] = __float2bfloat16_rn(to_f32(c_in[k]));
    } else {
        float amax = 0.f;
        for (int k = lane; k < d_c; k += 32) amax = fmaxf(amax, fabsf(to_f32(c_in[k])));
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        float sc = 1.f;
        if (amax > 0.f) sc = fmaxf(__fdiv_rn(amax, 448.f), FLT_MIN);
        uint8_t *row = reinterpret_cast<uint8_t *>(kv_pool) + slot * d_c;
        for (int k = lane; k < d_c; k += 32) {
            float x = __fdiv_rn(to_f32(c_in[k]), sc);
            row[k] = (uint8_t)__nv_cvt_float_to_fp8(x, __NV_SATFINITE, __NV_E4M3);
        }
        if (lane == 0) kv_scale[slot] = sc;
    }
}

}  // namespace mla
