// mla_absorb_q and mla_out_proj: the per-head small GEMMs around the absorbed attention.
//
// MLA article (itwiki "멀티 헤드 잠재 어텐션"), section 행렬 흡수 (matrix absorption):
//   absorb:   q_lat[t,h,:] = W^UK_h^T q^C[t,h,:]   (d_c <- d_h), then [q_lat ; RoPE(q^R)]
//   out_proj: o[t,h,:]     = W^UV_h o_lat[t,h,:]   (d_h <- d_c)
// W^UK, W^UV are [n_h*d_h, d_c] row-major (section 구조), head h owning rows h*d_h...
//
// CUDA-core kernels: every weight element is read from HBM once per launch and reused for a
// tile of tokens held in shared memory / registers.  At decode batch sizes (T = 16..256 query
// tokens) these two calls are bound by the 2 x 16.8 MB of bf16 weights.
#include "mla_internal.cuh"

namespace mla {
namespace {

constexpr int kAbsorbCols = 128;  // latent columns per block (one per thread)
constexpr int kAbsorbTok = 16;    // tokens per block

// grid (n_h, ceil(d_c/128), ceil(T/16)); block 128.  Thread = one latent column c of head h.
template <typename Ta>
__global__ void __launch_bounds__(kAbsorbCols)
absorb_q_kernel(int T, int n_h, int d_h, int d_c, int d_r, const __grid_constant__ RopeFreqs rope,
                const Ta *__restrict__ q_c, const Ta *__restrict__ q_r,
                const int32_t *__restrict__ pos, const Ta *__restrict__ w_uk, Ta *__restrict__ q_abs) {
    extern __shared__ float q_s[];  // [kAbsorbTok][d_h]
    const int h = blockIdx.x;
    const int c = blockIdx.y * kAbsorbCols + threadIdx.x;
    const int t0 = blockIdx.z * kAbsorbTok;
    const int nt = min(kAbsorbTok, T - t0);
    const int row = d_c + d_r;
    for (int i = threadIdx.x; i < nt * d_h; i += blockDim.x) {
        int tt = i / d_h, k = i % d_h;
        q_s[tt * d_h + k] = to_f32(q_c[((size_t)(t0 + tt) * n_h + h) * d_h + k]);
    }
    __syncthreads();
    if (c < d_c) {
        float acc[kAbsorbTok];
#pragma unroll
        for (int tt = 0; tt < kAbsorbTok; ++tt) acc[tt] = 0.f;
        const Ta *w = w_uk + (size_t)h * d_h * d_c + c;
        for (int k = 0; k < d_h; ++k) {
            float wk = to_f32(w[(size_t)k * d_c]);
#pragma unroll
            for (int tt = 0; tt < kAbsorbTok; ++tt) acc[tt] = fmaf(q_s[tt * d_h + k], wk, acc[tt]);
        }
#pragma unroll
        for (int tt = 0; tt < kAbsorbTok; ++tt)
            if (tt < nt) q_abs[((size_t)(t0 + tt) * n_h + h) * row + c] = from_f32<Ta>(acc[tt]);
    }
    // RoPE part of the query (분리 RoPE section), written by the first column block.
    if (blockIdx.y == 0) {
        const int half = d_r >> 1;
        for (int i = threadIdx.x; i < nt * half; i += blockDim.x) {
            int tt = i / half, k = i % half;
            int t = t0 + tt;
            float cs, sn;
            rope_cos_sin(rope, k, pos[t], &cs, &sn);
            const Ta *x = q_r + ((size_t)t * n_h + h) * d_r;
            float x0 = to_f32(x[k]), x1 = to_f32(x[k + half]);
            Ta *y = q_abs + ((size_t)t * n_h + h) * row + d_c;
            y[k] = from_f32<Ta>(x0 * cs - x1 * sn);
            y[k + half] = from_f32<Ta>(x1 * cs + x0 * sn);
        }
    }
}

constexpr int kOutRowsPerBlock = 8;  // one warp per output row d
constexpr int kOutTok = 8;

// grid (n_h, ceil(d_h/8), ceil(T/8)); block 256.  Warp = one output row d of head h.
template <typename Tw, typename To>
__global__ void __launch_bounds__(kOutRowsPerBlock * 32)
out_proj_kernel(int T, int n_h, int d_h, int d_c, const float *__restrict__ o_lat,
                const Tw *__restrict__ w_uv, To *__restrict__ o) {
    const int h = blockIdx.x;
    const int d = blockIdx.y * kOutRowsPerBlock + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    const int t0 = blockIdx.z * kOutTok;
    const int nt = min(kOutTok, T - t0);
    if (d >= d_h) return;
    const Tw *w = w_uv + ((size_t)h * d_h + d) * d_c;
    float acc[kOutTok];
#pragma unroll
    for (int tt = 0; tt < kOutTok; ++tt) acc[tt] = 0.f;
    for (int c = lane; c < d_c; c += 32) {
        float wc = to_f32(w[c]);
#pragma unroll
        for (int tt = 0; tt < kOutTok; ++tt)
            if (tt < nt) acc[tt] = fmaf(wc, o_lat[((size_t)(t0 + tt) * n_h + h) * d_c + c], acc[tt]);
    }
#pragma unroll
    for (int tt = 0; tt < kOutTok; ++tt) {
        float v = acc[tt];
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
        if (lane == 0 && tt < nt) o[((size_t)(t0 + tt) * n_h + h) * d_h + d] = from_f32<To>(v);
    }
}

}  // namespace

static bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

cudaError_t launch_absorb_q(const mla_dims_t &d, int T, const void *q_c, const void *q_r,
                            const int32_t *pos, const void *w_uk, void *q_abs, cudaStream_t st) {
    if (T == 0) return cudaSuccess;
    if (!(d.flags & MLA_FLAG_SIMT_PROJ) && proj_tc_supported(d) && aligned16(q_c) && aligned16(q_r) &&
        aligned16(w_uk) && aligned16(q_abs))
        return launch_absorb_q_tc(d, T, q_c, q_r, pos, w_uk, q_abs, st);
    dim3 grid(d.n_h, (d.d_c + kAbsorbCols - 1) / kAbsorbCols, (T + kAbsorbTok - 1) / kAbsorbTok);
    size_t smem = sizeof(float) * kAbsorbTok * d.d_h;
    if (d.act_dtype == MLA_DTYPE_BF16) {
        using T_ = __nv_bfloat16;
        absorb_q_kernel<T_><<<grid, kAbsorbCols, smem, st>>>(
            T, d.n_h, d.d_h, d.d_c, d.d_r, make_rope_freqs((double)d.rope_base, d.d_r), (const T_ *)q_c, (const T_ *)q_r,
            pos, (const T_ *)w_uk, (T_ *)q_abs);
    } else {
        absorb_q_kernel<float><<<grid, kAbsorbCols, smem, st>>>(
            T, d.n_h, d.d_h, d.d_c, d.d_r, make_rope_freqs((double)d.rope_base, d.d_r), (const float *)q_c,
            (const float *)q_r, pos, (const float *)w_uk, (float *)q_abs);
    }
    return cudaGetLastError();
}

cudaError_t launch_out_proj(const mla_dims_t &d, int T, const float *o_lat, const void *w_uv,
                            void *o, mla_dtype_t out_dtype, cudaStream_t st) {
    if (T == 0) return cudaSuccess;
    if (!(d.flags & MLA_FLAG_SIMT_PROJ) && proj_tc_supported(d) && aligned16(o_lat) && aligned16(w_uv))
        return launch_out_proj_tc(d, T, o_lat, w_uv, o, out_dtype, st);
    dim3 grid(d.n_h, (d.d_h + kOutRowsPerBlock - 1) / kOutRowsPerBlock, (T + kOutTok - 1) / kOutTok);
    dim3 block(kOutRowsPerBlock * 32);
    const bool wb = d.act_dtype == MLA_DTYPE_BF16;
    const bool ob = out_dtype == MLA_DTYPE_BF16;
    using B16 = __nv_bfloat16;
    if (wb && ob)
        out_proj_kernel<B16, B16><<<grid, block, 0, st>>>(T, d.n_h, d.d_h, d.d_c, o_lat, (const B16 *)w_uv, (B16 *)o);
    else if (wb)
        out_proj_kernel<B16, float><<<grid, block, 0, st>>>(T, d.n_h, d.d_h, d.d_c, o_lat, (const B16 *)w_uv, (float *)o);
    else if (ob)
        out_proj_kernel<float, B16><<<grid, block, 0, st>>>(T, d.n_h, d.d_h, d.d_c, o_lat, (const float *)w_uv, (B16 *)o);
    else
        out_proj_kernel<float, float><<<grid, block, 0, st>>>(T, d.n_h, d.d_h, d.d_c, o_lat, (const float *)w_uv, (float *)o);
    return cudaGetLastError();
}

}  // namespace mla
