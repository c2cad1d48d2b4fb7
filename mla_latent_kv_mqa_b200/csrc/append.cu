// mla_cache_append: scatter new tokens' [c^KV ; RoPE(k^R)] rows into the paged latent cache.
//
// MLA article (itwiki "멀티 헤드 잠재 어텐션"), section 분리 RoPE: the cache holds c^KV_t and
// the shared RoPE key k^R_t = RoPE(W^KR h_t), d_c + d_R values per token.  The FP8 content
// cache with a bf16 RoPE-key cache is the layout the QuantMLA review page ("Motivation &
// Problem Statement") describes as existing practice.
//
// One warp per token.  The work is a few KB per token, bound by its HBM writes; the only
// arithmetic is the RoPE rotation (angle in fp64) and, for FP8, a warp max and the e4m3
// conversion (cvt.rn.satfinite through cuda_fp8.h).
#include "append_body.cuh"

namespace mla {
namespace {

constexpr int kWarpsPerBlock = 8;

template <typename Tin, int KV>  // KV: 0 = f32 cache, 1 = bf16 cache, 2 = fp8 content cache
__global__ void __launch_bounds__(kWarpsPerBlock * 32)
append_kernel(const __grid_constant__ AppendArgs a, const __grid_constant__ RopeFreqs rope, unsigned *err) {
    // The query absorption that usually follows may start now: it waits for this kernel on the
    // device before it reads anything that could depend on it.
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const int t = blockIdx.x * kWarpsPerBlock + (threadIdx.x >> 5);
    if (t >= a.T) return;
    append_token<Tin, KV>(a, rope, t, threadIdx.x & 31, err);
}

}  // namespace

AppendArgs append_args(const mla_dims_t &d, int T, const void *c_kv, const void *k_r, const int32_t *seq_idx,
                       const int32_t *pos, const int32_t *bt, int num_seqs, int max_blocks, int num_blocks,
                       void *kv_pool, void *kr_pool, float *kv_scale) {
    AppendArgs a;
    a.T = T;
    a.d_c = d.d_c;
    a.d_r = d.d_r;
    a.page = d.page_size;
    a.c_kv = c_kv;
    a.k_r = k_r;
    a.seq_idx = seq_idx;
    a.pos = pos;
    a.bt = bt;
    a.num_seqs = num_seqs;
    a.max_blocks = max_blocks;
    a.num_blocks = num_blocks;
    a.kv_pool = kv_pool;
    a.kr_pool = reinterpret_cast<__nv_bfloat16 *>(kr_pool);
    a.kv_scale = kv_scale;
    return a;
}

cudaError_t launch_append(const mla_dims_t &d, int T, const void *c_kv, const void *k_r,
                          const int32_t *seq_idx, const int32_t *pos, const int32_t *bt,
                          int num_seqs, int max_blocks, int num_blocks, void *kv_pool,
                          void *kr_pool, float *kv_scale, cudaStream_t st) {
    if (T == 0) return cudaSuccess;
    dim3 grid((T + kWarpsPerBlock - 1) / kWarpsPerBlock), block(kWarpsPerBlock * 32);
    const RopeFreqs rope = make_rope_freqs((double)d.rope_base, d.d_r);
    unsigned *err = device_error_word();
    const AppendArgs a = append_args(d, T, c_kv, k_r, seq_idx, pos, bt, num_seqs, max_blocks, num_blocks, kv_pool,
                                     kr_pool, kv_scale);
#define MLA_APPEND(TIN, KV) append_kernel<TIN, KV><<<grid, block, 0, st>>>(a, rope, err)
    const bool in_bf16 = d.act_dtype == MLA_DTYPE_BF16;
    switch (d.kv_dtype) {
        case MLA_DTYPE_F32:
            if (in_bf16) MLA_APPEND(__nv_bfloat16, 0); else MLA_APPEND(float, 0);
            break;
        case MLA_DTYPE_BF16:
            if (in_bf16) MLA_APPEND(__nv_bfloat16, 1); else MLA_APPEND(float, 1);
            break;
        default:
            if (in_bf16) MLA_APPEND(__nv_bfloat16, 2); else MLA_APPEND(float, 2);
            break;
    }
#undef MLA_APPEND
    return cudaGetLastError();
}

}  // namespace mla
