// Exact merge of decode results computed over disjoint token ranges of the same sequences
// (sequence split across GPUs).
//
// MLA article, section 한계 (limitations): tensor parallelism over heads cannot shard the
// latent cache, since every head reads all of it.  Splitting the context instead is exact:
// for one query row and head, a rank that attended over its tokens J_r returns
//     o_r = sum_{j in J_r} e^{s_j} c_j / l_r,   lse_r = ln l_r,   l_r = sum_{j in J_r} e^{s_j},
// and the result over all tokens is
//     M = max_r lse_r,   w_r = e^{lse_r - M},   o = sum_r w_r o_r / sum_r w_r,
//     lse = M + ln sum_r w_r.
// The sums over ranks are one all-reduce of (w_r o_r, w_r) after one all-reduce of the max;
// the two kernels here are the per-rank steps before and after the sum.
#include <math.h>

#include "mla_internal.cuh"

namespace mla {
namespace {

// acc[r, h, :d_c] = w o_lat[r, h, :],  acc_l[r, h] = w,  w = e^{lse - M} (0 where lse = -inf)
__global__ void lse_merge_prepare_kernel(int rows, int n_h, int d_c, const float *__restrict__ o_lat,
                                         const float *__restrict__ lse, const float *__restrict__ lse_max,
                                         float *__restrict__ acc) {
    const size_t rh = blockIdx.x;
    if (rh >= (size_t)rows * n_h) return;
    const float m = lse_max[rh], x = lse[rh];
    const float w = (x == -INFINITY || m == -INFINITY) ? 0.f : expf(x - m);
    const float *src = o_lat + rh * d_c;
    float *dst = acc + rh * d_c;
    for (int c = threadIdx.x; c < d_c; c += blockDim.x) dst[c] = w * src[c];
    if (threadIdx.x == 0) acc[(size_t)rows * n_h * d_c + rh] = w;
}

// o_lat[r, h, :] = acc[r, h, :] / acc_l[r, h],  lse[r, h] = M + ln acc_l[r, h]
// (0 and -inf where no rank saw a token)
__global__ void lse_merge_finish_kernel(int rows, int n_h, int d_c, const float *__restrict__ acc,
                                        const float *__restrict__ lse_max, float *__restrict__ o_lat,
                                        float *__restrict__ lse) {
    const size_t rh = blockIdx.x;
    if (rh >= (size_t)rows * n_h) return;
    const float l = acc[(size_t)rows * n_h * d_c + rh];
    const float inv = l > 0.f ? 1.f / l : 0.f;
    const float *src = acc + rh * d_c;
    float *dst = o_lat + rh * d_c;
    for (int c = threadIdx.x; c < d_c; c += blockDim.x) dst[c] = src[c] * inv;
    if (lse && threadIdx.x == 0) lse[rh] = l > 0.f ? lse_max[rh] + logf(l) : -INFINITY;
}

int merge_threads(int d_c) { return d_c >= 256 ? 256 : (d_c >= 128 ? 128 : 64); }

}  // namespace

cudaError_t launch_lse_merge_prepare(int rows, int n_h, int d_c, const float *o_lat, const float *lse,
                                     const float *lse_max, float *acc, cudaStream_t st) {
    const size_t blocks = (size_t)rows * n_h;
    if (blocks == 0) return cudaSuccess;
    lse_merge_prepare_kernel<<<(unsigned)blocks, merge_threads(d_c), 0, st>>>(rows, n_h, d_c, o_lat, lse, lse_max,
                                                                              acc);
    return cudaGetLastError();
}

cudaError_t launch_lse_merge_finish(int rows, int n_h, int d_c, const float *acc, const float *lse_max,
                                    float *o_lat, float *lse, cudaStream_t st) {
    const size_t blocks = (size_t)rows * n_h;
    if (blocks == 0) return cudaSuccess;
    lse_merge_finish_kernel<<<(unsigned)blocks, merge_threads(d_c), 0, st>>>(rows, n_h, d_c, acc, lse_max, o_lat,
                                                                             lse);
    return cudaGetLastError();
}

}  // namespace mla
