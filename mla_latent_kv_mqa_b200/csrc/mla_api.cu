// C ABI entry points of libmla: host-side argument checks, then the launches.
// The operations are documented in include/mla.h.
#include <limits.h>
#include <math.h>
#include <mutex>
#include <stdio.h>

#include "append_body.cuh"
#include "mla_internal.cuh"

namespace mla {

// The library's only device allocation: one error word per device (static storage).
__device__ unsigned g_device_error;

namespace {
constexpr int kMaxDevices = 64;
unsigned *g_err_addr[kMaxDevices] = {};
std::mutex g_err_mu;
}  // namespace

unsigned *device_error_word() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lk(g_err_mu);
    if (!g_err_addr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_device_error) != cudaSuccess) return nullptr;
        g_err_addr[dev] = reinterpret_cast<unsigned *>(p);
    }
    return g_err_addr[dev];
}

// Scratch of mla_decode_fixed_scratch: file-scope device storage, so that entry point never
// allocates.  Every call on a device uses this one array.
constexpr size_t kDecodeScratchBytes = (size_t)MLA_DECODE_FIXED_SCRATCH_BYTES;
static __device__ __align__(256) unsigned char g_decode_scratch[kDecodeScratchBytes];

namespace {
void *g_scratch_addr[kMaxDevices] = {};
std::mutex g_scratch_mu;
}  // namespace

// Device address of the scratch array on the current device.  The first call on a device
// resolves it (and may load the module there); later calls return the cached pointer.
void *decode_scratch() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lk(g_scratch_mu);
    if (!g_scratch_addr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress((void **)&p, g_decode_scratch) != cudaSuccess || !p) return nullptr;
        g_scratch_addr[dev] = p;
    }
    return g_scratch_addr[dev];
}

}  // namespace mla

using namespace mla;

namespace {

bool act_ok(mla_dtype_t t) { return t == MLA_DTYPE_F32 || t == MLA_DTYPE_BF16; }

mla_status_t check_dims(const mla_dims_t *d) {
    if (!d) return MLA_ERR_INVALID_ARG;
    if (d->n_h < 1 || d->d_h < 1 || d->d_c < 1 || d->d_r < 2 || (d->d_r & 1) || d->page_size < 1)
        return MLA_ERR_INVALID_ARG;
    if (!(d->rope_base > 0.f) || !isfinite(d->rope_base)) return MLA_ERR_INVALID_ARG;
    if (!act_ok(d->act_dtype)) return MLA_ERR_UNSUPPORTED;
    if (d->kv_dtype != MLA_DTYPE_F32 && d->kv_dtype != MLA_DTYPE_BF16 &&
        d->kv_dtype != MLA_DTYPE_FP8_E4M3)
        return MLA_ERR_UNSUPPORTED;
    if (d->d_c > 1024 || d->d_c + d->d_r > 2048) return MLA_ERR_UNSUPPORTED;
    return MLA_OK;
}

mla_status_t from_cuda(cudaError_t e) { return e == cudaSuccess ? MLA_OK : MLA_ERR_CUDA; }

bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

}  // namespace

extern "C" {

int mla_version(void) { return 100; }

const char *mla_status_string(mla_status_t s) {
    switch (s) {
        case MLA_OK: return "MLA_OK";
        case MLA_ERR_INVALID_ARG: return "MLA_ERR_INVALID_ARG";
        case MLA_ERR_UNSUPPORTED: return "MLA_ERR_UNSUPPORTED";
        case MLA_ERR_WORKSPACE_TOO_SMALL: return "MLA_ERR_WORKSPACE_TOO_SMALL";
        case MLA_ERR_BAD_BLOCK_TABLE: return "MLA_ERR_BAD_BLOCK_TABLE";
        case MLA_ERR_BAD_SEQ_LEN: return "MLA_ERR_BAD_SEQ_LEN";
        case MLA_ERR_DEVICE_TIMEOUT: return "MLA_ERR_DEVICE_TIMEOUT";
        case MLA_ERR_CUDA: return "MLA_ERR_CUDA";
    }
    return "MLA_ERR_UNKNOWN";
}

mla_status_t mla_get_last_device_error(void) {
    unsigned *w = device_error_word();
    if (!w) return MLA_ERR_CUDA;
    if (cudaDeviceSynchronize() != cudaSuccess) return MLA_ERR_CUDA;
    unsigned v = 0;
    if (cudaMemcpy(&v, w, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess) return MLA_ERR_CUDA;
    unsigned zero = 0;
    if (cudaMemcpy(w, &zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess) return MLA_ERR_CUDA;
    return (mla_status_t)v;
}

// Host checks of mla_absorb_q (MLA_OK with *work = false: nothing to do).
static mla_status_t check_absorb(const mla_dims_t *dims, int T, const void *q_c, const void *q_r,
                                 const int32_t *pos, const void *w_uk, void *q_abs, bool *work) {
    *work = false;
    mla_status_t s = check_dims(dims);
    if (s != MLA_OK) return s;
    if (T < 0) return MLA_ERR_INVALID_ARG;
    if (T == 0) return MLA_OK;
    if (!q_c || !q_r || !pos || !w_uk || !q_abs) return MLA_ERR_INVALID_ARG;
    *work = true;
    return MLA_OK;
}

mla_status_t mla_absorb_q(const mla_dims_t *dims, int T, const void *q_c, const void *q_r,
                          const int32_t *pos, const void *w_uk, void *q_abs,
                          mla_stream_t stream) {
    bool work;
    mla_status_t s = check_absorb(dims, T, q_c, q_r, pos, w_uk, q_abs, &work);
    if (s != MLA_OK || !work) return s;
    return from_cuda(launch_absorb_q(*dims, T, q_c, q_r, pos, w_uk, q_abs, (cudaStream_t)stream));
}

// Host checks of mla_cache_append.
static mla_status_t check_append(const mla_dims_t *dims, int T, const void *c_kv, const void *k_r,
                                 const int32_t *seq_idx, const int32_t *pos, const int32_t *block_table,
                                 int num_seqs, int max_blocks_per_seq, int num_blocks, void *kv_pool,
                                 void *kr_pool, float *kv_scale, bool *work) {
    *work = false;
    mla_status_t s = check_dims(dims);
    if (s != MLA_OK) return s;
    if (T < 0 || num_seqs < 0 || max_blocks_per_seq < 0 || num_blocks < 0) return MLA_ERR_INVALID_ARG;
    if (T == 0) return MLA_OK;
    if (!c_kv || !k_r || !seq_idx || !pos || !block_table || !kv_pool) return MLA_ERR_INVALID_ARG;
    if (num_seqs == 0 || max_blocks_per_seq == 0 || num_blocks == 0) return MLA_ERR_INVALID_ARG;
    if ((int64_t)max_blocks_per_seq * dims->page_size > INT_MAX) return MLA_ERR_INVALID_ARG;
    const bool fp8 = dims->kv_dtype == MLA_DTYPE_FP8_E4M3;
    if (fp8 != (kr_pool != nullptr) || fp8 != (kv_scale != nullptr)) return MLA_ERR_INVALID_ARG;
    *work = true;
    return MLA_OK;
}

mla_status_t mla_cache_append(const mla_dims_t *dims, int T, const void *c_kv, const void *k_r,
                              const int32_t *seq_idx, const int32_t *pos,
                              const int32_t *block_table, int num_seqs, int max_blocks_per_seq,
                              int num_blocks, void *kv_pool, void *kr_pool, float *kv_scale,
                              mla_stream_t stream) {
    bool work;
    mla_status_t s = check_append(dims, T, c_kv, k_r, seq_idx, pos, block_table, num_seqs, max_blocks_per_seq,
                                  num_blocks, kv_pool, kr_pool, kv_scale, &work);
    if (s != MLA_OK || !work) return s;
    return from_cuda(launch_append(*dims, T, c_kv, k_r, seq_idx, pos, block_table, num_seqs,
                                   max_blocks_per_seq, num_blocks, kv_pool, kr_pool, kv_scale,
                                   (cudaStream_t)stream));
}

mla_status_t mla_append_absorb(const mla_dims_t *dims, int T_new, const void *c_kv, const void *k_r,
                               const int32_t *seq_idx, const int32_t *pos_new, const int32_t *block_table,
                               int num_seqs, int max_blocks_per_seq, int num_blocks, void *kv_pool,
                               void *kr_pool, float *kv_scale, int T, const void *q_c, const void *q_r,
                               const int32_t *pos, const void *w_uk, void *q_abs, mla_stream_t stream) {
    bool wa, wq;
    mla_status_t s = check_append(dims, T_new, c_kv, k_r, seq_idx, pos_new, block_table, num_seqs,
                                  max_blocks_per_seq, num_blocks, kv_pool, kr_pool, kv_scale, &wa);
    if (s != MLA_OK) return s;
    s = check_absorb(dims, T, q_c, q_r, pos, w_uk, q_abs, &wq);
    if (s != MLA_OK) return s;
    cudaStream_t st = (cudaStream_t)stream;
    // one launch where the tensor-core absorption applies (the conditions of launch_absorb_q)
    if (wa && wq && append_absorb_tc_supported(*dims) && !(dims->flags & MLA_FLAG_SIMT_PROJ) &&
        aligned(q_c, 16) && aligned(q_r, 16) && aligned(w_uk, 16) && aligned(q_abs, 16)) {
        const AppendArgs job = append_args(*dims, T_new, c_kv, k_r, seq_idx, pos_new, block_table, num_seqs,
                                           max_blocks_per_seq, num_blocks, kv_pool, kr_pool, kv_scale);
        return from_cuda(launch_append_absorb_tc(*dims, job, T, q_c, q_r, pos, w_uk, q_abs, st));
    }
    if (wa) {
        s = from_cuda(launch_append(*dims, T_new, c_kv, k_r, seq_idx, pos_new, block_table, num_seqs,
                                    max_blocks_per_seq, num_blocks, kv_pool, kr_pool, kv_scale, st));
        if (s != MLA_OK) return s;
    }
    if (wq) return from_cuda(launch_absorb_q(*dims, T, q_c, q_r, pos, w_uk, q_abs, st));
    return MLA_OK;
}

static bool use_tc(const mla_dims_t *d) {
    return !(d->flags & MLA_FLAG_SIMT_DECODE) && tc_supported(*d);
}

size_t mla_decode_workspace_size(const mla_dims_t *dims, int B, int s_q, int max_seq_len) {
    if (check_dims(dims) != MLA_OK || B < 0 || s_q < 1 || max_seq_len < 1) return 0;
    if ((int64_t)B * s_q > INT_MAX) return 0;  // query rows are counted in int
    if (use_tc(dims)) return tc_workspace_bytes(*dims, B, s_q, max_seq_len);
    return simt_workspace_bytes(*dims, B, s_q, max_seq_len);
}

// mla_decode and mla_decode_project: `fuse` (may be null) routes the merge of the split
// partials through the fused combine + output projection kernel.
static mla_status_t decode_impl(const mla_dims_t *dims, int B, int s_q, const void *q_abs,
                                const void *kv_pool, const void *kr_pool, const float *kv_scale,
                                const int32_t *block_table, int max_blocks_per_seq, int num_blocks,
                                const int32_t *seq_lens, int max_seq_len, void *workspace,
                                size_t workspace_bytes, float *o_lat, float *lse, mla_stream_t stream,
                                const FusedOutProj *fuse) {
    mla_status_t s = check_dims(dims);
    if (s != MLA_OK) return s;
    if (B < 0 || s_q < 1 || max_blocks_per_seq < 1 || num_blocks < 1 || max_seq_len < 1)
        return MLA_ERR_INVALID_ARG;
    if (B == 0) return MLA_OK;
    // The kernels count query rows (B * s_q) and table positions (max_blocks * page) in int.
    if ((int64_t)B * s_q > INT_MAX || (int64_t)max_blocks_per_seq * dims->page_size > INT_MAX)
        return MLA_ERR_INVALID_ARG;
    if (max_seq_len > max_blocks_per_seq * dims->page_size || max_seq_len < s_q)
        return MLA_ERR_INVALID_ARG;
    if (!q_abs || !kv_pool || !block_table || !seq_lens || !workspace || !o_lat)
        return MLA_ERR_INVALID_ARG;
    const bool fp8 = dims->kv_dtype == MLA_DTYPE_FP8_E4M3;
    if (fp8 != (kr_pool != nullptr) || fp8 != (kv_scale != nullptr)) return MLA_ERR_INVALID_ARG;
    if (!aligned(workspace, 256)) return MLA_ERR_INVALID_ARG;
    const size_t need = mla_decode_workspace_size(dims, B, s_q, max_seq_len);
    if (need == 0) return MLA_ERR_CUDA;  // the device could not be queried
    if (workspace_bytes < need) return MLA_ERR_WORKSPACE_TOO_SMALL;
    cudaStream_t st = (cudaStream_t)stream;
    if (use_tc(dims)) {
        // The tensor-core kernel reads the cache and q_abs with TMA: 16-byte aligned bases.
        if (!aligned(q_abs, 16) || !aligned(kv_pool, 16) || (kr_pool && !aligned(kr_pool, 16)) ||
            (kv_scale && !aligned(kv_scale, 16)))
            return MLA_ERR_INVALID_ARG;
        return from_cuda(launch_decode_tc(*dims, B, s_q, q_abs, kv_pool, kr_pool, kv_scale,
                                          block_table, max_blocks_per_seq, num_blocks, seq_lens,
                                          max_seq_len, workspace, workspace_bytes, o_lat, lse, st, fuse));
    }
    if (fuse) return MLA_ERR_UNSUPPORTED;  // callers fuse only where the tensor-core path applies
    return from_cuda(launch_decode_simt(*dims, B, s_q, q_abs, kv_pool, kr_pool, kv_scale,
                                        block_table, max_blocks_per_seq, num_blocks, seq_lens,
                                        max_seq_len, workspace, o_lat, lse, st));
}

mla_status_t mla_decode(const mla_dims_t *dims, int B, int s_q, const void *q_abs,
                        const void *kv_pool, const void *kr_pool, const float *kv_scale,
                        const int32_t *block_table, int max_blocks_per_seq, int num_blocks,
                        const int32_t *seq_lens, int max_seq_len, void *workspace,
                        size_t workspace_bytes, float *o_lat, float *lse, mla_stream_t stream) {
    return decode_impl(dims, B, s_q, q_abs, kv_pool, kr_pool, kv_scale, block_table, max_blocks_per_seq,
                       num_blocks, seq_lens, max_seq_len, workspace, workspace_bytes, o_lat, lse, stream,
                       nullptr);
}

mla_status_t mla_decode_project(const mla_dims_t *dims, int B, int s_q, const void *q_abs,
                                const void *kv_pool, const void *kr_pool, const float *kv_scale,
                                const int32_t *block_table, int max_blocks_per_seq, int num_blocks,
                                const int32_t *seq_lens, int max_seq_len, void *workspace,
                                size_t workspace_bytes, const void *w_uv, void *o,
                                mla_dtype_t out_dtype, float *o_lat, float *lse,
                                mla_stream_t stream) {
    mla_status_t s = check_dims(dims);
    if (s != MLA_OK) return s;
    if (B < 0 || s_q < 1) return MLA_ERR_INVALID_ARG;
    if (B == 0) return MLA_OK;
    if (!w_uv || !o || !o_lat || !aligned(o_lat, 16)) return MLA_ERR_INVALID_ARG;
    if (!act_ok(out_dtype)) return MLA_ERR_UNSUPPORTED;
    if ((int64_t)B * s_q > INT_MAX) return MLA_ERR_INVALID_ARG;
    if (use_tc(dims) && proj_tc_supported(*dims) && !(dims->flags & MLA_FLAG_SIMT_PROJ)) {
        const FusedOutProj fuse{w_uv, o, out_dtype};
        return decode_impl(dims, B, s_q, q_abs, kv_pool, kr_pool, kv_scale, block_table, max_blocks_per_seq,
                           num_blocks, seq_lens, max_seq_len, workspace, workspace_bytes, o_lat, lse, stream,
                           &fuse);
    }
    s = decode_impl(dims, B, s_q, q_abs, kv_pool, kr_pool, kv_scale, block_table, max_blocks_per_seq,
                    num_blocks, seq_lens, max_seq_len, workspace, workspace_bytes, o_lat, lse, stream, nullptr);
    if (s != MLA_OK) return s;
    return mla_out_proj(dims, B * s_q, o_lat, w_uv, o, out_dtype, stream);
}

// mla_decode on the library's fixed scratch array instead of a caller workspace, for callers
// that cannot allocate device memory when they decode: a service whose device-memory budget
// is reserved up front (a late allocation may find none left), or a latency-critical path on
// which an allocation's possible device synchronisation is not acceptable.  The size check
// comes first; every other argument is checked by mla_decode itself.  The scratch holds
// nothing between calls: the decode kernels write every workspace value before they read it.
mla_status_t mla_decode_fixed_scratch(const mla_dims_t *dims, int B, int s_q, const void *q_abs,
                                      const void *kv_pool, const void *kr_pool,
                                      const float *kv_scale, const int32_t *block_table,
                                      int max_blocks_per_seq, int num_blocks,
                                      const int32_t *seq_lens, int max_seq_len, float *o_lat,
                                      float *lse, mla_stream_t stream) {
    void *scratch = decode_scratch();
    if (!scratch) return MLA_ERR_CUDA;
    if (mla_decode_workspace_size(dims, B, s_q, max_seq_len) > kDecodeScratchBytes)
        return MLA_ERR_WORKSPACE_TOO_SMALL;
    return mla_decode(dims, B, s_q, q_abs, kv_pool, kr_pool, kv_scale, block_table,
                      max_blocks_per_seq, num_blocks, seq_lens, max_seq_len, scratch,
                      kDecodeScratchBytes, o_lat, lse, stream);
}

size_t mla_prefill_workspace_size(const mla_dims_t *dims, int total_tokens) {
    if (check_dims(dims) != MLA_OK || !prefill_supported(*dims) || total_tokens < 0) return 0;
    return prefill_workspace_bytes(*dims, total_tokens);
}

mla_status_t mla_prefill(const mla_dims_t *dims, int B, const int32_t *cu_seqlens, int total_tokens,
                         int max_seq_len, const void *q_c, const void *q_r, const void *c_kv,
                         const void *k_r, const void *w_uk, const void *w_uv, void *workspace,
                         size_t workspace_bytes, void *o, float *lse, mla_stream_t stream) {
    mla_status_t s = check_dims(dims);
    if (s != MLA_OK) return s;
    if (!prefill_supported(*dims)) return MLA_ERR_UNSUPPORTED;
    if (B < 0 || total_tokens < 0 || max_seq_len < 1) return MLA_ERR_INVALID_ARG;
    if (B == 0 || total_tokens == 0) return MLA_OK;
    // grid limits (heads, prompts, 128-token tiles) and int TMA coordinates over n_h * T rows
    const int64_t T_pad = ((int64_t)total_tokens + 127) / 128 * 128;
    if (B > 65535 || (int64_t)dims->n_h > 65535 || T_pad / 128 > 65535 ||
        (int64_t)dims->n_h * T_pad > INT_MAX)
        return MLA_ERR_INVALID_ARG;
    if (!cu_seqlens || !q_c || !q_r || !c_kv || !k_r || !w_uk || !w_uv || !workspace || !o)
        return MLA_ERR_INVALID_ARG;
    if (!aligned(q_c, 16) || !aligned(q_r, 16) || !aligned(c_kv, 16) || !aligned(w_uk, 16) || !aligned(w_uv, 16) || !aligned(o, 16) ||
        !aligned(workspace, 256))
        return MLA_ERR_INVALID_ARG;
    if (workspace_bytes < prefill_workspace_bytes(*dims, total_tokens)) return MLA_ERR_WORKSPACE_TOO_SMALL;
    return from_cuda(launch_prefill(*dims, B, cu_seqlens, total_tokens, max_seq_len, q_c, q_r, c_kv, k_r, w_uk, w_uv,
                                    workspace, workspace_bytes, o, lse, (cudaStream_t)stream));
}

mla_status_t mla_lse_merge_prepare(int rows, int n_h, int d_c, const float *o_lat, const float *lse,
                                   const float *lse_max, float *acc, mla_stream_t stream) {
    if (rows < 0 || n_h < 1 || d_c < 1 || (int64_t)rows * n_h > INT_MAX) return MLA_ERR_INVALID_ARG;
    if (rows == 0) return MLA_OK;
    if (!o_lat || !lse || !lse_max || !acc) return MLA_ERR_INVALID_ARG;
    return from_cuda(launch_lse_merge_prepare(rows, n_h, d_c, o_lat, lse, lse_max, acc, (cudaStream_t)stream));
}

mla_status_t mla_lse_merge_finish(int rows, int n_h, int d_c, const float *acc, const float *lse_max,
                                  float *o_lat, float *lse, mla_stream_t stream) {
    if (rows < 0 || n_h < 1 || d_c < 1 || (int64_t)rows * n_h > INT_MAX) return MLA_ERR_INVALID_ARG;
    if (rows == 0) return MLA_OK;
    if (!acc || !lse_max || !o_lat) return MLA_ERR_INVALID_ARG;
    return from_cuda(launch_lse_merge_finish(rows, n_h, d_c, acc, lse_max, o_lat, lse, (cudaStream_t)stream));
}

mla_status_t mla_out_proj(const mla_dims_t *dims, int T, const float *o_lat, const void *w_uv,
                          void *o, mla_dtype_t out_dtype, mla_stream_t stream) {
    mla_status_t s = check_dims(dims);
    if (s != MLA_OK) return s;
    if (T < 0) return MLA_ERR_INVALID_ARG;
    if (T == 0) return MLA_OK;
    if (!o_lat || !w_uv || !o) return MLA_ERR_INVALID_ARG;
    if (!act_ok(out_dtype)) return MLA_ERR_UNSUPPORTED;
    return from_cuda(launch_out_proj(*dims, T, o_lat, w_uv, o, out_dtype, (cudaStream_t)stream));
}

}  // extern "C"
