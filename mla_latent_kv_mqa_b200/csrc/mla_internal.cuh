// Internal declarations of libmla (not part of the ABI).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <stdint.h>

#include "../../include/mla.h"

namespace mla {

// Device error word codes (first condition wins, see record_error).
enum : unsigned {
    kErrNone = 0,
    kErrBadBlock = MLA_ERR_BAD_BLOCK_TABLE,
    kErrBadSeqLen = MLA_ERR_BAD_SEQ_LEN,
    kErrTimeout = MLA_ERR_DEVICE_TIMEOUT,
};

// Address of this device's error word (set up once per device by the API layer).
unsigned *device_error_word();

__device__ __forceinline__ void record_error(unsigned *err, unsigned code) {
    if (err) atomicCAS(err, 0u, code);
}

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }
template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

// RoPE angles (구현 section of the MLA article: pair k of a d_r-wide vector is rotated by
// pos * base^(-2k/d_r)).  The per-pair frequencies are computed once on the host in fp64 and
// passed by value; on the device the angle pos * f_k is formed in fp64 and reduced to [-pi, pi]
// by Cody-Waite subtraction of n * 2pi (2pi split into its fp64 value and the remainder, each
// subtracted with one fused multiply-add), and cos/sin of the reduced angle are taken in fp32.
// Positions up to 2^31 keep cos/sin within a few fp32 ulps.
constexpr int kRopeTab = 64;  // pairs held in the table (d_r <= 128); wider d_r computes f_k on the fly
struct RopeFreqs {
    double inv_freq[kRopeTab];
    double base;
    int d_r;
};
inline RopeFreqs make_rope_freqs(double base, int d_r) {
    RopeFreqs f = {};
    f.base = base;
    f.d_r = d_r;
    for (int k = 0; k < kRopeTab && k < d_r / 2; ++k) f.inv_freq[k] = pow(base, -(double)(2 * k) / (double)d_r);
    return f;
}
__device__ __forceinline__ void rope_cos_sin(const RopeFreqs &f, int k, int pos, float *c, float *s) {
    constexpr double kTwoPi = 6.283185307179586;        // 2pi rounded to fp64
    constexpr double kTwoPiRem = 2.4492935982947064e-16;  // 2pi - kTwoPi
    constexpr double kInvTwoPi = 0.15915494309189535;
    const double inv = k < kRopeTab ? f.inv_freq[k] : pow(f.base, -(double)(2 * k) / (double)f.d_r);
    const double theta = (double)pos * inv;
    const double n = rint(theta * kInvTwoPi);
    const double r = fma(-n, kTwoPiRem, fma(-n, kTwoPi, theta));
    sincosf((float)r, s, c);
}

// Partial results of one split segment, shared by the decode kernels and the combine kernel.
//   o_part [slot][n_h][d_c] fp32: sum_j exp2(s2_j - m) c_j   (not normalised)
//   m_part [slot][n_h]      fp32: running max m in log2 units (s2 = s * log2(e)); -inf = empty
//   l_part [slot][n_h]      fp32: sum_j exp2(s2_j - m)
struct Partials {
    float *o;
    float *m;
    float *l;
};

// ---- launchers (host) --------------------------------------------------------------------
cudaError_t launch_append(const mla_dims_t &d, int T, const void *c_kv, const void *k_r,
                          const int32_t *seq_idx, const int32_t *pos, const int32_t *bt,
                          int num_seqs, int max_blocks, int num_blocks, void *kv_pool,
                          void *kr_pool, float *kv_scale, cudaStream_t st);

cudaError_t launch_absorb_q(const mla_dims_t &d, int T, const void *q_c, const void *q_r,
                            const int32_t *pos, const void *w_uk, void *q_abs, cudaStream_t st);

cudaError_t launch_out_proj(const mla_dims_t &d, int T, const float *o_lat, const void *w_uv,
                            void *o, mla_dtype_t out_dtype, cudaStream_t st);

// Tensor-core projections (d_h = 128, d_c = 512, d_R = 64, bf16).
bool proj_tc_supported(const mla_dims_t &d);
cudaError_t launch_absorb_q_tc(const mla_dims_t &d, int T, const void *q_c, const void *q_r,
                               const int32_t *pos, const void *w_uk, void *q_abs, cudaStream_t st);
cudaError_t launch_out_proj_tc(const mla_dims_t &d, int T, const float *o_lat, const void *w_uv, void *o,
                               mla_dtype_t out_dtype, cudaStream_t st);

// mla_cache_append + mla_absorb_q in one launch (tensor-core absorption, bf16 or FP8 cache).
struct AppendArgs;
bool append_absorb_tc_supported(const mla_dims_t &d);
cudaError_t launch_append_absorb_tc(const mla_dims_t &d, const AppendArgs &job, int T, const void *q_c,
                                    const void *q_r, const int32_t *pos, const void *w_uk, void *q_abs,
                                    cudaStream_t st);
// CUDA-core split-KV decode.  Splits every query row into n_split segments of seg_len tokens.
struct SimtPlan {
    int n_split;
    int seg_len;
};
SimtPlan simt_plan(const mla_dims_t &d, int B, int s_q, int max_seq_len);
size_t simt_workspace_bytes(const mla_dims_t &d, int B, int s_q, int max_seq_len);
cudaError_t launch_decode_simt(const mla_dims_t &d, int B, int s_q, const void *q_abs,
                               const void *kv_pool, const void *kr_pool, const float *kv_scale,
                               const int32_t *bt, int max_blocks, int num_blocks,
                               const int32_t *seq_lens, int max_seq_len, void *ws,
                               float *o_lat, float *lse, cudaStream_t st);

// Log-sum-exp merge of split partials.  Row r (= query row t) owns slots
// seg_range[2r] .. seg_range[2r+1]-1 when seg_range != nullptr, else r*uniform .. r*uniform+uniform-1.
cudaError_t launch_combine(int rows, int n_h, int d_c, Partials p, const int32_t *seg_range,
                           int uniform, float *o_lat, float *lse, cudaStream_t st);

// Tensor-core (tcgen05) decode for the DeepSeek-V3 shape.  With `fuse`, the split partials
// are merged by the fused combine + output projection kernel instead of the combine kernel.
struct FusedOutProj {
    const void *w_uv;
    void *o;
    mla_dtype_t out_dtype;
};
bool tc_supported(const mla_dims_t &d);
size_t tc_workspace_bytes(const mla_dims_t &d, int B, int s_q, int max_seq_len);
cudaError_t launch_decode_tc(const mla_dims_t &d, int B, int s_q, const void *q_abs,
                             const void *kv_pool, const void *kr_pool, const float *kv_scale,
                             const int32_t *bt, int max_blocks, int num_blocks,
                             const int32_t *seq_lens, int max_seq_len, void *ws,
                             size_t ws_bytes, float *o_lat, float *lse, cudaStream_t st,
                             const FusedOutProj *fuse = nullptr);
// The fused kernel: partials in the tensor-core decode's layout ([slot][d_c / 2][n_h] bf16
// pairs, m and l per slot and head, per-row slot ranges) -> o_lat, lse (either may be null)
// and o = W^UV_h o_lat.  o_lat, when given, must be 16-byte aligned.
cudaError_t launch_combine_out_proj_tc(const mla_dims_t &d, int T, const int32_t *seg_range,
                                       const uint32_t *o_part, const float *m_part, const float *l_part,
                                       float *o_lat, float *lse, const void *w_uv, void *o,
                                       mla_dtype_t out_dtype, cudaStream_t st);

// MHA-mode prefill (d_h = 128, d_c = 512, d_R = 64, bf16, even n_h): K / V reconstruction
// GEMM + causal tcgen05 attention over packed prompts (cu_seqlens [B + 1], T tokens).
bool prefill_supported(const mla_dims_t &d);
size_t prefill_workspace_bytes(const mla_dims_t &d, int T);
cudaError_t launch_prefill(const mla_dims_t &d, int B, const int32_t *cu_seqlens, int T, int max_seq_len,
                           const void *q_c, const void *q_r, const void *c_kv, const void *k_r, const void *w_uk,
                           const void *w_uv, void *ws, size_t ws_bytes, void *o, float *lse, cudaStream_t st);
// Sequence split across GPUs: the per-rank steps of the exact log-sum-exp merge.
cudaError_t launch_lse_merge_prepare(int rows, int n_h, int d_c, const float *o_lat, const float *lse,
                                     const float *lse_max, float *acc, cudaStream_t st);
cudaError_t launch_lse_merge_finish(int rows, int n_h, int d_c, const float *acc, const float *lse_max,
                                    float *o_lat, float *lse, cudaStream_t st);

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

}  // namespace mla
