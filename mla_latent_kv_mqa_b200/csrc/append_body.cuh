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
// The token's inputs depend only on t, so all of a lane's loads (up to AP_BATCH content values
// and its RoPE pair) are issued before the sequence / position / block-table lookups and travel
// together with them; loads interleaved with the row's stores would each wait for the previous
// store (the compiler cannot prove the input and the pool apart), one trip to memory apiece.
constexpr int AP_BATCH = 16;  // content values per lane in the first batch: d_c <= 512

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
    const Tin *c_in = c_kv + (size_t)t * d_c;
    const Tin *k_in = k_r + (size_t)t * d_r;
    const int half = d_r >> 1;

    float cv[AP_BATCH];
#pragma unroll
    for (int i = 0; i < AP_BATCH; ++i) {
        const int k = lane + 32 * i;
        cv[i] = k < d_c ? to_f32(c_in[k]) : 0.f;
    }
    const float x0 = lane < half ? to_f32(k_in[lane]) : 0.f;
    const float x1 = lane < half ? to_f32(k_in[lane + half]) : 0.f;
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

    // RoPE of the shared key (pairs k, k + d_r/2).
    auto put_rope = [&](int k, float a0, float a1) {
        float cs, sn;
        rope_cos_sin(rope, k, p, &cs, &sn);
        const float y0 = a0 * cs - a1 * sn;
        const float y1 = a1 * cs + a0 * sn;
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
    };
    if (lane < half) put_rope(lane, x0, x1);
    for (int k = lane + 32; k < half; k += 32) put_rope(k, to_f32(k_in[k]), to_f32(k_in[k + half]));

    constexpr int kRest = 32 * AP_BATCH;  // content values past the first batch (d_c > 512)
    if (KV == 0) {
        float *row = reinterpret_cast<float *>(kv_pool) + slot * (d_c + d_r);
#pragma unroll
        for (int i = 0; i < AP_BATCH; ++i)
            if (lane + 32 * i < d_c) row[lane + 32 * i] = cv[i];
        for (int k = kRest + lane; k < d_c; k += 32) row[k] = to_f32(c_in[k]);
    } else if (KV == 1) {
        __nv_bfloat16 *row = reinterpret_cast<__nv_bfloat16 *>(kv_pool) + slot * (d_c + d_r);
#pragma unroll
        for (int i = 0; i < AP_BATCH; ++i)
            if (lane + 32 * i < d_c) row[lane + 32 * i] = __float2bfloat16_rn(cv[i]);
        for (int k = kRest + lane; k < d_c; k += 32) row[k] = __float2bfloat16_rn(to_f32(c_in[k]));
    } else {
        float amax = 0.f;
#pragma unroll
        for (int i = 0; i < AP_BATCH; ++i) amax = fmaxf(amax, fabsf(cv[i]));
        for (int k = kRest + lane; k < d_c; k += 32) amax = fmaxf(amax, fabsf(to_f32(c_in[k])));
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        float sc = 1.f;
        if (amax > 0.f) sc = fmaxf(__fdiv_rn(amax, 448.f), FLT_MIN);
        uint8_t *row = reinterpret_cast<uint8_t *>(kv_pool) + slot * d_c;
#pragma unroll
        for (int i = 0; i < AP_BATCH; ++i)
            if (lane + 32 * i < d_c)
                row[lane + 32 * i] = (uint8_t)__nv_cvt_float_to_fp8(__fdiv_rn(cv[i], sc), __NV_SATFINITE, __NV_E4M3);
        for (int k = kRest + lane; k < d_c; k += 32) {
            float x = __fdiv_rn(to_f32(c_in[k]), sc);
            row[k] = (uint8_t)__nv_cvt_float_to_fp8(x, __NV_SATFINITE, __NV_E4M3);
        }
        if (lane == 0) kv_scale[slot] = sc;
    }
}

}  // namespace mla
