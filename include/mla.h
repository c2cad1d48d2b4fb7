/*
 * mla.h -- C ABI of libmla: absorbed (MQA-mode) Multi-head Latent Attention decode
 * over a paged latent KV cache, for NVIDIA B200 (sm_100a).
 *
 * The method is the one of the itwiki article "멀티 헤드 잠재 어텐션"
 * (Multi-head latent attention):
 *   - section 구조 (structure): the cache holds the joint latent c^KV_t = W^DKV h_t
 *     (d_c wide); keys and values are W^UK c and W^UV c with W^UK, W^UV of shape
 *     [n_h*d_h, d_c].
 *   - section 행렬 흡수 (matrix absorption): the score q^T W^UK c is computed as
 *     (W^UK^T q)^T c, so each head's query is moved into the latent space and all
 *     heads score the same cached c^KV; W^UV is applied after the weighted sum.
 *   - section 분리 RoPE (decoupled RoPE): a per-head RoPE query q^R and one shared
 *     RoPE key k^R_t are concatenated to the content parts; the cache stores
 *     [c^KV_t ; k^R_t], d_c + d_R values per token; scores are divided by
 *     sqrt(d_h + d_R) and softmaxed over the tokens j <= t.
 *   - section 구현 (implementation): half-split RoPE, angle pos * base^(-2k/d_R).
 * The lecture page "MHA · GQA · MQA · MLA", section "Why Projection Absorption
 * Helps", gives the same identity q^T W_UK c_t = (W_UK^T q)^T c_t.
 *
 * One decode step of one layer is four calls, in this order on one stream:
 *   mla_cache_append  -- write the new tokens' [c^KV ; RoPE(k^R)] rows into the cache
 *   mla_absorb_q      -- q_abs = [W^UK_h^T q^C ; RoPE(q^R)]  per token and head
 *   mla_decode        -- split-KV attention over the cache + log-sum-exp combine
 *   mla_out_proj      -- o = W^UV_h o_lat per token and head
 *
 * Conventions shared by every call
 *   Memory     The caller owns every buffer; all pointers are device pointers of one
 *              device (the current device) unless a comment says otherwise.  The
 *              library allocates no device memory.  Its only device storage is static:
 *              one error word per device (see mla_get_last_device_error) and the scratch
 *              array of mla_decode_fixed_scratch.
 *   Streams    Calls only enqueue work on `stream` (NULL = the legacy default stream)
 *              and return; results are ready in stream order.  mla_absorb_q, mla_decode
 *              and mla_out_proj launch their kernels as programmatic dependents of the
 *              kernel ahead of them on the stream (CUDA programmatic dependent launch):
 *              their blocks may start while that kernel drains, and they wait for it on
 *              the device before reading any activation, cache or table or writing any
 *              output.
 *   Weights    w_uk and w_uv are treated as constants of the layer: mla_absorb_q and
 *              mla_out_proj start reading them before that wait.  Write the weights
 *              before the first call that uses them and make that write complete
 *              (synchronize the stream or device, or wait on an event recorded after
 *              it); do not produce them in the kernel that immediately precedes the call.
 *   Layouts    Row-major, contiguous, as each argument states.
 *   Errors     Arguments are checked on the host before anything is launched; a bad
 *              argument returns an error and launches nothing.  A launch failure
 *              returns MLA_ERR_CUDA.  Conditions only the device can see (a block id
 *              outside the pool, a sequence length outside its table) make the kernel
 *              skip the offending access and set the device error word, which
 *              mla_get_last_device_error reports.  Nothing throws across the ABI.
 *   Softmax    The scale is 1/sqrt(d_h + d_R) (분리 RoPE section, output equation).
 */
#ifndef MLA_H_
#define MLA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t; declared here so the header needs no CUDA include. */
typedef struct CUstream_st *mla_stream_t;

typedef enum {
    MLA_OK = 0,
    MLA_ERR_INVALID_ARG = 1,         /* null pointer, negative size, misaligned pointer */
    MLA_ERR_UNSUPPORTED = 2,         /* dims / dtype combination not built into the library */
    MLA_ERR_WORKSPACE_TOO_SMALL = 3, /* workspace_bytes < mla_decode_workspace_size(...) */
    MLA_ERR_BAD_BLOCK_TABLE = 4,     /* device saw a block id outside [0, num_blocks) */
    MLA_ERR_BAD_SEQ_LEN = 5,         /* device saw a length < s_q or > max_blocks*page */
    MLA_ERR_DEVICE_TIMEOUT = 6,      /* a bounded device-side wait gave up */
    MLA_ERR_CUDA = 7                 /* a CUDA runtime call failed */
} mla_status_t;

typedef enum {
    MLA_DTYPE_F32 = 0,
    MLA_DTYPE_BF16 = 1,
    MLA_DTYPE_FP8_E4M3 = 2 /* cache only: e4m3 content + per-token fp32 scale + bf16 RoPE key */
} mla_dtype_t;

/* flags */
#define MLA_FLAG_SIMT_DECODE 1u /* run mla_decode on the CUDA-core kernel even where the
                                   tensor-core kernel applies (cross-checks) */
#define MLA_FLAG_SIMT_PROJ 2u   /* same for mla_absorb_q and mla_out_proj */
/* FP8 cache only: compute the content part of the scores on the FP8 tensor core
 * (tcgen05 kind::f8f6f4) from the cached e4m3 codes as they are, instead of dequantising every
 * page to bf16 first.  The absorbed query is split per head into two e4m3 parts,
 * q_lat ~ alpha_h (hi + lo) with alpha_h = max|q_lat| / 448, hi = e4m3(q_lat / alpha_h),
 * lo = e4m3(q_lat / alpha_h - hi) (about 7 significant bits, near bf16's 8), and the RoPE part
 * runs in bf16 on (q_R / alpha_h) . (k_R / s_j), so each score is
 *     s_j = alpha_h s_j [ (hi + lo) . c8_j + (q_R / alpha_h) . (k_R,j / s_j) ] / sqrt(d_h + d_R).
 * The value product P . V keeps bf16 V (dequantised on chip).  QuantMLA review, Motivation
 * & Problem Statement (an FP8 content cache next to a high-precision RoPE-key cache). */
#define MLA_FLAG_FP8_MMA 8u
#define MLA_FLAG_TEST_GIVE_UP 4u /* test of the failure path of the tensor-core decode: in
                                    every cluster with two or more pages, after the copies of
                                    the first page have started, one bounded wait (20 us) on a
                                    barrier that nothing completes gives up.  The cluster then
                                    does what any timed-out wait does: it flags both of its CTAs,
                                    records MLA_ERR_DEVICE_TIMEOUT in the device error word,
                                    waits (2 s bound) for the copies and MMAs it has started, and
                                    exits.  The call's outputs are invalid; nothing faults. */

typedef struct {
    int n_h;            /* heads */
    int d_h;            /* head dim of the content query q^C and of the output o */
    int d_c;            /* latent width of c^KV */
    int d_r;            /* RoPE width d_R (even) */
    int page_size;      /* tokens per cache block (64) */
    float rope_base;    /* RoPE base (1e4) */
    mla_dtype_t act_dtype; /* q_c, q_r, q_abs, c_kv/k_r append inputs, w_uk, w_uv: F32 or BF16 */
    mla_dtype_t kv_dtype;  /* cache: F32, BF16 or FP8_E4M3 */
    unsigned flags;
} mla_dims_t;

/* ----------------------------------------------------------------------------------------
 * mla_absorb_q -- the query side of the absorbed form (행렬 흡수 section; 분리 RoPE section
 * for q^R).  For every token t < T and head h:
 *     q_abs[t, h, 0:d_c]         = W^UK_h^T q_c[t, h, :]      (W^UK_h = rows h*d_h .. of w_uk)
 *     q_abs[t, h, d_c:d_c+d_r]   = RoPE(q_r[t, h, :], pos[t])
 *   q_c   [T, n_h, d_h]   act dtype
 *   q_r   [T, n_h, d_r]   act dtype, before rotation
 *   pos   [T]             int32 position of each token (>= 0)
 *   w_uk  [n_h*d_h, d_c]  act dtype (the nn.Linear(d_c, n_h*d_h) weight)
 *   q_abs [T, n_h, d_c+d_r] act dtype, written
 * Accumulation is fp32.  The rotation angle pos * base^(-2k/d_r) is formed in fp64 and reduced
 * modulo 2 pi in fp64; cos and sin of the reduced angle are fp32.  T == 0 is a no-op.
 * ---------------------------------------------------------------------------------------- */
mla_status_t mla_absorb_q(const mla_dims_t *dims, int T, const void *q_c, const void *q_r,
                          const int32_t *pos, const void *w_uk, void *q_abs,
                          mla_stream_t stream);

/* ----------------------------------------------------------------------------------------
 * mla_cache_append -- write new tokens into the paged latent cache (분리 RoPE section: the
 * cache holds c^KV_t and k^R_t = RoPE(W^KR h_t), d_c + d_R values per token).
 * Token t goes to sequence s = seq_idx[t] at position p = pos[t]:
 *     block = block_table[s * max_blocks_per_seq + p / page_size],  slot = p % page_size.
 *   c_kv [T, d_c] act dtype;  k_r [T, d_r] act dtype, before rotation.
 *   BF16 / F32 cache: kv_pool [num_blocks, page_size, d_c + d_r] of that dtype, row =
 *       [c_kv ; RoPE(k_r, p)].  kr_pool and kv_scale must be NULL.
 *   FP8_E4M3 cache: kv_pool [num_blocks, page_size, d_c] uint8 e4m3 codes,
 *       kr_pool [num_blocks, page_size, d_r] bf16 RoPE(k_r, p),
 *       kv_scale [num_blocks, page_size] fp32.  Per token s = amax|c_kv|/448 computed in
 *       fp32 (at least FLT_MIN; 1 when amax = 0); codes = e4m3(c_kv / s), nearest-even,
 *       saturating.
 * A token whose block id or table index is out of range is skipped and sets
 * MLA_ERR_BAD_BLOCK_TABLE on the device.  Never reads the pool.
 * ---------------------------------------------------------------------------------------- */
mla_status_t mla_cache_append(const mla_dims_t *dims, int T, const void *c_kv, const void *k_r,
                              const int32_t *seq_idx, const int32_t *pos,
                              const int32_t *block_table, int num_seqs, int max_blocks_per_seq,
                              int num_blocks, void *kv_pool, void *kr_pool, float *kv_scale,
                              mla_stream_t stream);

/* ----------------------------------------------------------------------------------------
 * mla_append_absorb -- mla_cache_append followed by mla_absorb_q, in one call.  The two
 * write different buffers (the cache; q_abs) and neither reads the other's output, so where
 * the tensor-core absorption applies (n_h any, d_h = 128, d_c = 512, d_r = 64, bf16
 * activations, bf16 or FP8 cache, no MLA_FLAG_SIMT_PROJ, 16-byte aligned q_c, q_r, w_uk,
 * q_abs) both run in ONE launch, the cache writes overlapping the absorption's weight fetch;
 * elsewhere the two are launched one after the other.  The results are bit for bit those of
 * the two calls.
 *   Arguments: those of mla_cache_append (T_new new tokens, pos_new their positions), then
 *   those of mla_absorb_q (T query tokens, pos their positions).
 * Errors: those of either call, checked before anything is launched.
 * ---------------------------------------------------------------------------------------- */
mla_status_t mla_append_absorb(const mla_dims_t *dims, int T_new, const void *c_kv, const void *k_r,
                               const int32_t *seq_idx, const int32_t *pos_new,
                               const int32_t *block_table, int num_seqs, int max_blocks_per_seq,
                               int num_blocks, void *kv_pool, void *kr_pool, float *kv_scale, int T,
                               const void *q_c, const void *q_r, const int32_t *pos, const void *w_uk,
                               void *q_abs, mla_stream_t stream);

/* ----------------------------------------------------------------------------------------
 * mla_decode_workspace_size -- bytes of device workspace mla_decode needs for B sequences of
 * s_q queries each and sequence lengths up to max_seq_len, on the current device.  Returns 0
 * for invalid arguments or when the current device cannot be queried.
 * ---------------------------------------------------------------------------------------- */
size_t mla_decode_workspace_size(const mla_dims_t *dims, int B, int s_q, int max_seq_len);

/* ----------------------------------------------------------------------------------------
 * mla_decode -- absorbed attention over the paged cache (분리 RoPE section output equation
 * in the latent form of the 행렬 흡수 section).  Query i < s_q of sequence b (row
 * t = b*s_q + i) sits at position P = seq_lens[b] - s_q + i and, for every head h,
 *     s_j     = (q_abs[t,h,0:d_c] . c_j + q_abs[t,h,d_c:] . kR_j) / sqrt(d_h + d_r),  j <= P
 *     o_lat   = sum_j softmax(s)_j c_j,       lse = ln sum_j exp(s_j)
 * where (c_j ; kR_j) is cache row j of sequence b (FP8: c_j = e4m3(code) * scale_j).
 * Precision: bf16 operands, fp32 accumulation and softmax.  With an FP8 cache the kernel
 * dequantises each page on chip to bf16(e4m3(code) * scale_j), one rounding per value, the
 * same a bf16 cache applies when it is written.
 * The tokens are split into segments processed in parallel; the partial results are merged
 * exactly by a log-sum-exp combine kernel.
 *   q_abs       [B*s_q, n_h, d_c+d_r] act dtype (from mla_absorb_q)
 *   kv_pool, kr_pool, kv_scale: the cache, as in mla_cache_append (read only)
 *   block_table [B, max_blocks_per_seq] int32
 *   seq_lens    [B] int32 device array; each in [s_q, max_seq_len]
 *   max_seq_len host-side upper bound of seq_lens (<= max_blocks_per_seq * page_size)
 *   workspace   device scratch of workspace_bytes >= mla_decode_workspace_size(...);
 *               its content on entry does not matter.
 *   o_lat       [B*s_q, n_h, d_c] fp32, written
 *   lse         [B*s_q, n_h] fp32 natural-log normaliser, written (may be NULL)
 * Deterministic: the result depends only on the logical cache content, not on which
 * physical blocks hold it.
 * ---------------------------------------------------------------------------------------- */
mla_status_t mla_decode(const mla_dims_t *dims, int B, int s_q, const void *q_abs,
                        const void *kv_pool, const void *kr_pool, const float *kv_scale,
                        const int32_t *block_table, int max_blocks_per_seq, int num_blocks,
                        const int32_t *seq_lens, int max_seq_len, void *workspace,
                        size_t workspace_bytes, float *o_lat, float *lse, mla_stream_t stream);

/* ----------------------------------------------------------------------------------------
 * mla_decode_fixed_scratch -- mla_decode without a caller workspace.  This call is a
 * library convenience: the pages describe no counterpart to it.  It computes exactly what
 * mla_decode computes, with the same arguments minus workspace / workspace_bytes.
 *
 * Who it is for: callers that cannot allocate device memory at decode time.  Examples are
 * services with a fixed device-memory budget that is reserved up front (a decode-time
 * allocation may fail once that budget is taken), and code on a latency-critical path where
 * cudaFree / cudaMalloc are not acceptable because they may synchronise the device.
 * Instead of a workspace argument, the call uses a scratch array of
 * MLA_DECODE_FIXED_SCRATCH_BYTES that lives in the library's own static device storage.
 * It allocates nothing itself.
 *
 *   Set-up     The first call on a device looks up that device's scratch address (the CUDA
 *              runtime may load the library's device code at that moment).  Make the first
 *              call on each device before any stream capture begins.  Later calls only read
 *              a cached pointer.
 *   Limit      If mla_decode_workspace_size(dims, B, s_q, max_seq_len) exceeds
 *              MLA_DECODE_FIXED_SCRATCH_BYTES, the call returns MLA_ERR_WORKSPACE_TOO_SMALL
 *              and launches nothing.  Use mla_decode with your own workspace instead.
 *   Sharing    Every call on a device uses the same scratch array.  Calls whose executions
 *              overlap on the device (on different streams without ordering between them)
 *              race on it and produce wrong results.  Serialize them, for example on one
 *              stream.  The scratch needs no clearing: every value the kernels read from it
 *              is written earlier in the same call.
 *   Errors     As for mla_decode; MLA_ERR_CUDA also when the scratch address cannot be
 *              obtained.
 * ---------------------------------------------------------------------------------------- */
#define MLA_DECODE_FIXED_SCRATCH_BYTES (32u << 20) /* 32 MiB per device */
mla_status_t mla_decode_fixed_scratch(const mla_dims_t *dims, int B, int s_q, const void *q_abs,
                                      const void *kv_pool, const void *kr_pool,
                                      const float *kv_scale, const int32_t *block_table,
                                      int max_blocks_per_seq, int num_blocks,
                                      const int32_t *seq_lens, int max_seq_len, float *o_lat,
                                      float *lse, mla_stream_t stream);

/* ----------------------------------------------------------------------------------------
 * mla_out_proj -- value up-projection after the aggregation (행렬 흡수 section):
 *     o[t, h, :] = W^UV_h o_lat[t, h, :]      (d_h <- d_c; W^UV_h = rows h*d_h .. of w_uv)
 *   o_lat [T, n_h, d_c] fp32;  w_uv [n_h*d_h, d_c] act dtype;
 *   o     [T, n_h, d_h] of out_dtype (F32 or BF16), written.  fp32 accumulation.
 * ---------------------------------------------------------------------------------------- */
mla_status_t mla_out_proj(const mla_dims_t *dims, int T, const float *o_lat, const void *w_uv,
                          void *o, mla_dtype_t out_dtype, mla_stream_t stream);

/* ----------------------------------------------------------------------------------------
 * mla_decode_project -- mla_decode followed by mla_out_proj in one call: the attention of
 * mla_decode, then o = W^UV_h o_lat (행렬 흡수 section: the value up-projection applied after
 * the aggregation).  Where the tensor-core kernels apply (n_h = 128, d_h = 128, d_c = 512,
 * d_r = 64, page 64, bf16 activations, bf16 or FP8 cache, no MLA_FLAG_SIMT_* flag), the merge
 * of the split partials and the projection run as ONE kernel, which never reads o_lat back;
 * elsewhere the call runs mla_decode and mla_out_proj one after the other.  Either way o,
 * o_lat and lse are bit for bit those of mla_decode followed by mla_out_proj.
 *   Arguments as for mla_decode, plus
 *   w_uv       [n_h*d_h, d_c] act dtype (as for mla_out_proj; written before the call)
 *   o          [B*s_q, n_h, d_h] of out_dtype (F32 or BF16), written
 *   o_lat      [B*s_q, n_h, d_c] fp32, written; 16-byte aligned
 *   lse        as for mla_decode (may be NULL)
 *   workspace  as for mla_decode (mla_decode_workspace_size)
 * Errors: those of mla_decode and mla_out_proj; MLA_ERR_INVALID_ARG also for a null w_uv or
 * o, or an o_lat that is not 16-byte aligned.
 * ---------------------------------------------------------------------------------------- */
mla_status_t mla_decode_project(const mla_dims_t *dims, int B, int s_q, const void *q_abs,
                                const void *kv_pool, const void *kr_pool, const float *kv_scale,
                                const int32_t *block_table, int max_blocks_per_seq, int num_blocks,
                                const int32_t *seq_lens, int max_seq_len, void *workspace,
                                size_t workspace_bytes, const void *w_uv, void *o,
                                mla_dtype_t out_dtype, float *o_lat, float *lse,
                                mla_stream_t stream);

/* ----------------------------------------------------------------------------------------
 * mla_prefill -- causal attention over whole prompts in MHA ("naive") mode: the keys and
 * values are reconstructed per head from the latent (구조 section), k_{j,h} = [W^UK_h c_j ;
 * RoPE(k^R_j, j)] and v_{j,h} = W^UV_h c_j, and for every prompt token t and head h
 *     o[t,h,:] = sum_{j <= t} softmax_j( [q^C ; RoPE(q^R, t)]_{t,h} . k_{j,h} / sqrt(d_h + d_r) ) v_{j,h}
 * (분리 RoPE section output equation).  The 한계 section and the mode remarks of the 행렬 흡수
 * section: with as many queries as keys, reconstructing K and V once costs less than the
 * 576-wide latent scores of the absorbed form, which pays off in decode only.
 * Positions are token indices within each prompt (0 .. L_b - 1).  The call does not write the
 * cache: append the prompt with mla_cache_append for the decode steps that follow.
 * Supported shape: d_h = 128, d_c = 512, d_r = 64, even n_h, bf16 activations and weights
 * (MLA_ERR_UNSUPPORTED otherwise).  Precision: bf16 operands (K and V rounded to bf16 once,
 * P to bf16), fp32 accumulation and softmax.
 *   B            number of prompts
 *   cu_seqlens   [B+1] int32 device array: prompt b is tokens cu_seqlens[b] .. cu_seqlens[b+1]-1
 *                of the packed inputs; cu_seqlens[0] = 0, cu_seqlens[B] = total_tokens
 *   total_tokens T, the packed token count
 *   max_seq_len  host-side upper bound of the prompt lengths
 *   q_c [T, n_h, d_h], q_r [T, n_h, d_r] (before RoPE), c_kv [T, d_c], k_r [T, d_r] (before
 *                RoPE): bf16, row-major; q_c, q_r, c_kv 16-byte aligned
 *   w_uk, w_uv   [n_h*d_h, d_c] bf16, 16-byte aligned (written before the call)
 *   workspace    device scratch of workspace_bytes >= mla_prefill_workspace_size(dims, T),
 *                256-byte aligned; its content on entry does not matter
 *   o            [T, n_h, d_h] bf16, 16-byte aligned, written
 *   lse          [T, n_h] fp32 natural-log normaliser, written (may be NULL)
 * Errors: MLA_ERR_INVALID_ARG for bad sizes, null or misaligned pointers; a prompt table that
 * is not as stated (or a prompt longer than max_seq_len) is reported by the device as
 * MLA_ERR_BAD_SEQ_LEN through mla_get_last_device_error, with no access outside the buffers.
 * ---------------------------------------------------------------------------------------- */
size_t mla_prefill_workspace_size(const mla_dims_t *dims, int total_tokens);
mla_status_t mla_prefill(const mla_dims_t *dims, int B, const int32_t *cu_seqlens, int total_tokens,
                         int max_seq_len, const void *q_c, const void *q_r, const void *c_kv,
                         const void *k_r, const void *w_uk, const void *w_uv, void *workspace,
                         size_t workspace_bytes, void *o, float *lse, mla_stream_t stream);

/* ----------------------------------------------------------------------------------------
 * Sequence split across GPUs (long contexts): exact merge of decode results.
 *
 * MLA article, section 한계 (limitations): every head reads the whole latent cache, so tensor
 * parallelism over heads cannot shard it.  The context can be split instead: each rank holds
 * a contiguous range of every sequence's pages, runs mla_decode (s_q = 1) over its own pages
 * only, and the ranks' results merge exactly.  For query row r and head h, with rank i's
 * (o_lat_i, lse_i) from mla_decode:
 *     M = max_i lse_i,  w_i = e^{lse_i - M},
 *     o_lat = sum_i w_i o_lat_i / sum_i w_i,   lse = M + ln sum_i w_i.
 * One step per rank before the cross-rank sum and one after it:
 *   1. lse_max = all-reduce(max) of lse over the ranks       (the caller's collective)
 *   2. mla_lse_merge_prepare: acc = [w o_lat ; w]            (this rank)
 *   3. acc = all-reduce(sum) of acc over the ranks            (the caller's collective)
 *   4. mla_lse_merge_finish: o_lat = acc_o / acc_w, lse = M + ln acc_w
 * Arguments (device pointers, fp32, row-major):
 *   o_lat   [rows, n_h, d_c]  this rank's mla_decode output (prepare) / the merged one (finish)
 *   lse     [rows, n_h]       this rank's lse (prepare, natural log; -inf: no token) / merged
 *                             (finish; may be NULL)
 *   lse_max [rows, n_h]       the maximum of lse over the ranks
 *   acc     [rows * n_h * (d_c + 1)]  w o_lat for every (row, head), then the rows*n_h weights
 *                             w; the caller owns it and sums it over the ranks between the calls
 * A row and head that no rank saw (every lse -inf) merge to o_lat = 0, lse = -inf.  Errors:
 * MLA_ERR_INVALID_ARG for a negative or oversized count or a null pointer (rows = 0 is a no-op).
 * ---------------------------------------------------------------------------------------- */
mla_status_t mla_lse_merge_prepare(int rows, int n_h, int d_c, const float *o_lat, const float *lse,
                                   const float *lse_max, float *acc, mla_stream_t stream);
mla_status_t mla_lse_merge_finish(int rows, int n_h, int d_c, const float *acc, const float *lse_max,
                                  float *o_lat, float *lse, mla_stream_t stream);

/* Reads and clears the device error word of the current device.  Synchronises the device.
 * Returns MLA_OK, MLA_ERR_BAD_BLOCK_TABLE, MLA_ERR_BAD_SEQ_LEN or MLA_ERR_DEVICE_TIMEOUT
 * (the first condition seen since the last call), or MLA_ERR_CUDA. */
mla_status_t mla_get_last_device_error(void);

/* Static, human-readable name of a status code. */
const char *mla_status_string(mla_status_t status);

/* Library ABI version (major * 100 + minor). */
int mla_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MLA_H_ */
