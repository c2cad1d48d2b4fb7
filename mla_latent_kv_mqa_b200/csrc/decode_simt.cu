// CUDA-core split-KV decode (any dims, f32 / bf16 / fp8 caches) and the log-sum-exp combine.
//
// MLA article (itwiki "멀티 헤드 잠재 어텐션"), section 분리 RoPE, output equation, in the
// absorbed form of section 행렬 흡수: per query row t and head h
//   s_j = (q_lat . c_j + q^R . k^R_j) / sqrt(d_h + d_R),  j <= pos(t)
//   o_lat = sum_j softmax(s)_j c_j   (every head reads the same c^KV row as key and value).
// The softmax runs online in log2 units (exp2 with log2(e)/sqrt(d_h+d_R) folded into the
// scale), one warp per head.  Each block handles one query row, one split segment of its
// tokens and 8 heads; the segment's partial (o, m, l) is merged by the combine kernel.
//
// This kernel is the general path (the toy layer's fp32 shape, any other shape) and an
// independent cross-check of the tensor-core kernel; it re-reads the cache once per head
// group, so it is far from the HBM roofline on the 128-head shape.
#include <float.h>
#include <math.h>

#include "mla_internal.cuh"

namespace mla {
namespace {

constexpr int kHeadsPerBlock = 8;  // one warp per head
constexpr int kTileTok = 32;       // one token per lane in the score step
constexpr int kMaxColsPerLane = 32;  // d_c <= 1024

template <int KV>  // 0 = f32 pool, 1 = bf16 pool, 2 = fp8 content pool + bf16 RoPE pool
__device__ __forceinline__ float load_cache(const void *kv_pool, const __nv_bfloat16 *kr_pool,
                                            const float *kv_scale, size_t slot, int k, int d_c,
                                            int d_r) {
    if (KV == 0) return reinterpret_cast<const float *>(kv_pool)[slot * (d_c + d_r) + k];
    if (KV == 1) return __bfloat162float(reinterpret_cast<const __nv_bfloat16 *>(kv_pool)[slot * (d_c + d_r) + k]);
    if (k < d_c) {
        uint8_t code = reinterpret_cast<const uint8_t *>(kv_pool)[slot * d_c + k];
        __half_raw hr = __nv_cvt_fp8_to_halfraw((__nv_fp8_storage_t)code, __NV_E4M3);
        return __half2float(__half(hr)) * kv_scale[slot];
    }
    return __bfloat162float(kr_pool[slot * d_r + (k - d_c)]);
}

template <typename Ta, int KV>
__global__ void __launch_bounds__(kHeadsPerBlock * 32)
decode_simt_kernel(int s_q, int n_h, int d_c, int d_r, float scale_log2, int page,
                   const Ta *__restrict__ q_abs, const void *__restrict__ kv_pool,
                   const __nv_bfloat16 *__restrict__ kr_pool, const float *__restrict__ kv_scale,
                   const int32_t *__restrict__ bt, int max_blocks, int num_blocks,
                   const int32_t *__restrict__ seq_lens, int max_seq_len, int seg_len,
                   int n_split, Partials part, unsigned *err) {
    extern __shared__ float smem[];
    const int row = d_c + d_r;
    const int kv_stride = row + 1;  // padding: lanes reading different rows hit different banks
    float *q_s = smem;                                  // [8][row]
    float *kv_s = smem + kHeadsPerBlock * row;          // [32][row+1]

    const int r = blockIdx.x;        // query row t = b*s_q + i
    const int split = blockIdx.y;
    const int h0 = blockIdx.z * kHeadsPerBlock;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int h = h0 + warp;
    const int b = r / s_q, i = r % s_q;
    const size_t slot_id = (size_t)r * n_split + split;

    const int L = seq_lens[b];
    bool bad = L < s_q || L > max_seq_len || L > max_blocks * page;
    if (bad && threadIdx.x == 0 && split == 0 && blockIdx.z == 0) record_error(err, kErrBadSeqLen);
    const int n_vis = bad ? 0 : L - s_q + i + 1;
    const int j_begin = split * seg_len;
    const int j_end = min(n_vis, j_begin + seg_len);
    if (j_begin >= j_end) {
        if (lane == 0 && h < n_h) {
            part.m[slot_id * n_h + h] = -INFINITY;
            part.l[slot_id * n_h + h] = 0.f;
        }
        return;
    }

    for (int idx = threadIdx.x; idx < kHeadsPerBlock * row; idx += blockDim.x) {
        int g = idx / row, k = idx % row;
        q_s[idx] = (h0 + g < n_h) ? to_f32(q_abs[((size_t)r * n_h + h0 + g) * row + k]) : 0.f;
    }

    float o[kMaxColsPerLane];
#pragma unroll
    for (int q = 0; q < kMaxColsPerLane; ++q) o[q] = 0.f;
    float m = -INFINITY, l = 0.f;

    for (int j0 = j_begin; j0 < j_end; j0 += kTileTok) {
        __syncthreads();
        for (int idx = threadIdx.x; idx < kTileTok * row; idx += blockDim.x) {
            int jj = idx / row, k = idx % row;
            int j = j0 + jj;
            float v = 0.f;
            if (j < j_end) {
                int blk = bt[(size_t)b * max_blocks + j / page];
                if (blk >= 0 && blk < num_blocks)
                    v = load_cache<KV>(kv_pool, kr_pool, kv_scale, (size_t)blk * page + j % page, k, d_c, d_r);
                else if (k == 0)
                    record_error(err, kErrBadBlock);
            }
            kv_s[jj * kv_stride + k] = v;
        }
        __syncthreads();
        if (h >= n_h) continue;

        // scores: lane = token
        const float *qh = q_s + warp * row;
        const float *kvj = kv_s + lane * kv_stride;
        float s = 0.f;
        for (int k = 0; k < row; ++k) s = fmaf(qh[k], kvj[k], s);
        const bool valid = j0 + lane < j_end;
        float s2 = valid ? s * scale_log2 : -INFINITY;
        float mt = s2;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, off));
        const float m_new = fmaxf(m, mt);
        const float corr = exp2f(m - m_new);
        const float p = valid ? exp2f(s2 - m_new) : 0.f;
        float ps = p;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, off);
        l = l * corr + ps;
        m = m_new;
#pragma unroll
        for (int q = 0; q < kMaxColsPerLane; ++q) o[q] *= corr;
        for (int jj = 0; jj < kTileTok; ++jj) {
            const float pj = __shfl_sync(0xffffffffu, p, jj);
            const float *kvr = kv_s + jj * kv_stride;
#pragma unroll
            for (int q = 0; q < kMaxColsPerLane; ++q) {
                int c = lane + 32 * q;
                if (c < d_c) o[q] = fmaf(pj, kvr[c], o[q]);
            }
        }
    }
    if (h >= n_h) return;
    float *op = part.o + (slot_id * n_h + h) * d_c;
#pragma unroll
    for (int q = 0; q < kMaxColsPerLane; ++q) {
        int c = lane + 32 * q;
        if (c < d_c) op[c] = o[q];
    }
    if (lane == 0) {
        part.m[slot_id * n_h + h] = m;
        part.l[slot_id * n_h + h] = l;
    }
}

// Log-sum-exp merge: block per (row, head).  The per-slot weights 2^(m_s - M) are computed once
// into shared memory, then each thread sweeps its columns across the slots with float4 loads.
constexpr int kCombineThreads = 128;
constexpr int kCombineMaxSlots = 1024;

__global__ void __launch_bounds__(kCombineThreads)
combine_kernel(int n_h, int d_c, Partials p, const int32_t *__restrict__ seg_range, int uniform,
               float *__restrict__ o_lat, float *__restrict__ lse) {
    __shared__ float w_s[kCombineMaxSlots];
    __shared__ float red[kCombineThreads / 32];
    const int r = blockIdx.x, h = blockIdx.y, tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const int s0 = seg_range ? seg_range[2 * r] : r * uniform;
    int s1 = seg_range ? seg_range[2 * r + 1] : s0 + uniform;
    if (s1 - s0 > kCombineMaxSlots) s1 = s0 + kCombineMaxSlots;  // never reached: slots <= clusters + rows
    const int S = s1 - s0;
    float mloc = -INFINITY;
    for (int s = tid; s < S; s += kCombineThreads) mloc = fmaxf(mloc, p.m[(size_t)(s0 + s) * n_h + h]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mloc = fmaxf(mloc, __shfl_xor_sync(0xffffffffu, mloc, o));
    if (lane == 0) red[wid] = mloc;
    __syncthreads();
    float M = red[0];
#pragma unroll
    for (int i = 1; i < kCombineThreads / 32; ++i) M = fmaxf(M, red[i]);
    __syncthreads();
    float lloc = 0.f;
    for (int s = tid; s < S; s += kCombineThreads) {
        const float ms = p.m[(size_t)(s0 + s) * n_h + h];
        const float w = ms == -INFINITY ? 0.f : exp2f(ms - M);  // empty slot: weight 0, never read
        w_s[s] = w;
        if (w != 0.f) lloc += w * p.l[(size_t)(s0 + s) * n_h + h];
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) lloc += __shfl_xor_sync(0xffffffffu, lloc, o);
    if (lane == 0) red[wid] = lloc;
    __syncthreads();
    float Lsum = 0.f;
#pragma unroll
    for (int i = 0; i < kCombineThreads / 32; ++i) Lsum += red[i];
    const float inv = Lsum > 0.f ? 1.f / Lsum : 0.f;
    const size_t row_stride = (size_t)n_h * d_c;
    const float *obase = p.o + ((size_t)s0 * n_h + h) * d_c;
    float *dst = o_lat + ((size_t)r * n_h + h) * d_c;
    if ((d_c & 3) == 0 && (reinterpret_cast<uintptr_t>(o_lat) & 15) == 0) {
        for (int c4 = tid; c4 < d_c / 4; c4 += kCombineThreads) {
            float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
            for (int s = 0; s < S; ++s) {
                const float w = w_s[s];
                if (w == 0.f) continue;
                const float4 v = reinterpret_cast<const float4 *>(obase + s * row_stride)[c4];
                acc.x = fmaf(w, v.x, acc.x);
                acc.y = fmaf(w, v.y, acc.y);
                acc.z = fmaf(w, v.z, acc.z);
                acc.w = fmaf(w, v.w, acc.w);
            }
            reinterpret_cast<float4 *>(dst)[c4] = make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
        }
    } else {
        for (int c = tid; c < d_c; c += kCombineThreads) {
            float acc = 0.f;
            for (int s = 0; s < S; ++s) {
                const float w = w_s[s];
                if (w != 0.f) acc = fmaf(w, obase[s * row_stride + c], acc);
            }
            dst[c] = acc * inv;
        }
    }
    if (lse && tid == 0)
        lse[(size_t)r * n_h + h] = Lsum > 0.f ? (M + log2f(Lsum)) * 0.69314718055994531f : -INFINITY;
}

int sm_count() {
    int dev = 0, n = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n;
}

}  // namespace

SimtPlan simt_plan(const mla_dims_t &d, int B, int s_q, int max_seq_len) {
    const int rows = B * s_q;
    const int hg = (d.n_h + kHeadsPerBlock - 1) / kHeadsPerBlock;
    const long per_split = (long)rows * hg;
    const long target = 4L * sm_count();
    int n_split = (int)((target + per_split - 1) / per_split);
    const int max_split = (max_seq_len + kTileTok - 1) / kTileTok;
    n_split = n_split < 1 ? 1 : (n_split > max_split ? max_split : n_split);
    if (n_split < 1) n_split = 1;
    int seg = (max_seq_len + n_split - 1) / n_split;
    seg = (seg + kTileTok - 1) / kTileTok * kTileTok;
    if (seg < kTileTok) seg = kTileTok;
    n_split = (max_seq_len + seg - 1) / seg;
    if (n_split < 1) n_split = 1;
    return {n_split, seg};
}

size_t simt_workspace_bytes(const mla_dims_t &d, int B, int s_q, int max_seq_len) {
    SimtPlan pl = simt_plan(d, B, s_q, max_seq_len);
    size_t slots = (size_t)B * s_q * pl.n_split;
    return align_up(slots * d.n_h * d.d_c * sizeof(float), 256) +
           2 * align_up(slots * d.n_h * sizeof(float), 256);
}

cudaError_t launch_decode_simt(const mla_dims_t &d, int B, int s_q, const void *q_abs,
                               const void *kv_pool, const void *kr_pool, const float *kv_scale,
                               const int32_t *bt, int max_blocks, int num_blocks,
                               const int32_t *seq_lens, int max_seq_len, void *ws,
                               float *o_lat, float *lse, cudaStream_t st) {
    const int rows = B * s_q;
    if (rows == 0) return cudaSuccess;
    SimtPlan pl = simt_plan(d, B, s_q, max_seq_len);
    size_t slots = (size_t)rows * pl.n_split;
    char *w = reinterpret_cast<char *>(ws);
    Partials part;
    part.o = reinterpret_cast<float *>(w);
    w += align_up(slots * d.n_h * d.d_c * sizeof(float), 256);
    part.m = reinterpret_cast<float *>(w);
    w += align_up(slots * d.n_h * sizeof(float), 256);
    part.l = reinterpret_cast<float *>(w);

    const int row = d.d_c + d.d_r;
    const size_t smem = sizeof(float) * ((size_t)kHeadsPerBlock * row + (size_t)kTileTok * (row + 1));
    dim3 grid(rows, pl.n_split, (d.n_h + kHeadsPerBlock - 1) / kHeadsPerBlock);
    dim3 block(kHeadsPerBlock * 32);
    const float scale_log2 = (float)(1.4426950408889634 / sqrt((double)(d.d_h + d.d_r)));
    unsigned *err = device_error_word();
    const auto *krp = reinterpret_cast<const __nv_bfloat16 *>(kr_pool);
    cudaError_t e = cudaSuccess;
#define MLA_SIMT(TA, KV)                                                                          \
    do {                                                                                          \
        auto kern = decode_simt_kernel<TA, KV>;                                                   \
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);   \
        if (e != cudaSuccess) return e;                                                           \
        kern<<<grid, block, smem, st>>>(s_q, d.n_h, d.d_c, d.d_r, scale_log2, d.page_size,        \
                                        reinterpret_cast<const TA *>(q_abs), kv_pool, krp,        \
                                        kv_scale, bt, max_blocks, num_blocks, seq_lens,           \
                                        max_seq_len, pl.seg_len, pl.n_split, part, err);          \
    } while (0)
    const bool ab = d.act_dtype == MLA_DTYPE_BF16;
    if (d.kv_dtype == MLA_DTYPE_F32) {
        if (ab) MLA_SIMT(__nv_bfloat16, 0); else MLA_SIMT(float, 0);
    } else if (d.kv_dtype == MLA_DTYPE_BF16) {
        if (ab) MLA_SIMT(__nv_bfloat16, 1); else MLA_SIMT(float, 1);
    } else {
        if (ab) MLA_SIMT(__nv_bfloat16, 2); else MLA_SIMT(float, 2);
    }
#undef MLA_SIMT
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    return launch_combine(rows, d.n_h, d.d_c, part, nullptr, pl.n_split, o_lat, lse, st);
}

cudaError_t launch_combine(int rows, int n_h, int d_c, Partials p, const int32_t *seg_range,
                           int uniform, float *o_lat, float *lse, cudaStream_t st) {
    if (rows == 0) return cudaSuccess;
    combine_kernel<<<dim3(rows, n_h), kCombineThreads, 0, st>>>(n_h, d_c, p, seg_range, uniform, o_lat, lse);
    return cudaGetLastError();
}

}  // namespace mla
