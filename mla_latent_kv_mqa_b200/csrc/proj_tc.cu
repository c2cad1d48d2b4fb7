// Tensor-core (tcgen05) versions of the per-head projections around the absorbed attention,
// for d_h = 128, d_c = 512, bf16 weights.
//
// MLA article (itwiki "멀티 헤드 잠재 어텐션"), section 행렬 흡수 (matrix absorption):
//   absorb:   q_lat[t,h,:] = W^UK_h^T q^C[t,h,:]     (d_c <- d_h)
//   out_proj: o[t,h,:]     = W^UV_h o_lat[t,h,:]     (d_h <- d_c)
// with W^UK, W^UV = [n_h*d_h, d_c] row-major (section 구조), head h owning rows h*d_h...
//
// Both are small GEMMs per head with the weight rows as M (swap-AB: a decode batch has only
// T = 16..256 tokens, far below the M = 128 the tensor core wants):
//   absorb:   D[c, t] = sum_k W_h[k, c] q_c[t, k]     M = 512 (4 tiles), N = tokens, K = 128;
//             A = W_h read MN-major straight from its row-major layout.
//   out_proj: D[d, t] = sum_c W_h[d, c] o_lat[t, c]   M = 128, N = tokens, K = 512;
//             o_lat is fp32, so B is split into bf16 hi + lo (two MMAs per k-step) to keep
//             ~16 mantissa bits.
// One CTA per (head, 128-token tile): TMA streams the head's 128 KB weight slice (the dominant
// traffic, 2 x 16.8 MB per layer), the tokens come in through registers, the accumulator sits
// in TMEM, and the epilogue writes straight from tcgen05.ld.
#include <math.h>

#include "append_body.cuh"
#include "mla_internal.cuh"
#include "sm100.cuh"
#include "tmap.cuh"

namespace mla {
namespace {

using namespace sm100;

constexpr int DH = 128, DCL = 512, DR = 64;
constexpr int TN = 128;            // tokens per CTA
constexpr int WBOX = 64 * 128 * 2;  // one [128 rows x 64 cols] bf16 box of a weight slice: 16 KB
constexpr int NWB = DCL / 64;       // 8 boxes per head

struct __align__(8) ProjCtrl {
    uint64_t a_full[NWB];
    uint64_t b_done[2];
    uint64_t b_full;  // fused combine: every column block of the B tile has arrived
    uint64_t d_full;
    uint32_t tmem_base;
    uint32_t abort;
};

// ------------------------------------------------------------------------------------------
// out_proj: smem = W_h (8 x 16 KB, K-major) + the CTA's o_lat tokens as bf16 hi + lo, one
// [hi: TNO rows x 128 B][lo: TNO rows x 128 B] pair per 64-column block of d_c.
// All of the tile's o_lat is requested at once (one round trip to memory, not one per block):
// an 8-float group (token r, columns 8g..8g+7) is copied as two 16-byte halves into the hi and lo
// slots it will finally occupy, and the thread that copied it splits it there, so no other
// thread touches those bytes and the split needs no barrier.
// ------------------------------------------------------------------------------------------
constexpr int TNO = 32;                           // tokens per out_proj CTA
constexpr int OP_A = 0;
constexpr int OP_B = NWB * WBOX;                  // 131072
constexpr int OP_BBLK = 2 * TNO * 128;            // hi + lo of one column block: 8 KB
constexpr int OP_DATA = OP_B + NWB * OP_BBLK;     // 196608
constexpr int OP_SMEM = 1024 + OP_DATA + 256;

template <typename To>
__global__ void __launch_bounds__(128, 1)
out_proj_tc_kernel(const __grid_constant__ CUtensorMap tm_w, int T, int n_h, const float *__restrict__ o_lat,
                   To *__restrict__ o, unsigned *err) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_s = smem_u32(smem_raw);
    const uint32_t data_s = (raw_s + 1023u) & ~1023u;
    ProjCtrl *ctrl = reinterpret_cast<ProjCtrl *>(smem_raw + (data_s - raw_s) + OP_DATA);
    volatile uint32_t *abort_flag = &ctrl->abort;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int h = blockIdx.x, t0 = blockIdx.y * TNO;
    const int nt = min(TNO, T - t0);
    const int npad = (nt + 15) & ~15;

    if (tid == 0) {
        for (int i = 0; i < NWB; ++i) mbar_init(smem_u32(&ctrl->a_full[i]), 1);
        mbar_init(smem_u32(&ctrl->d_full), 1);
        ctrl->abort = 0;
        fence_mbarrier_init_cluster();
        // The weights are constants of the layer: their load starts first and overlaps the end
        // of the kernel ahead of this one on the stream.
        prefetch_tensormap(&tm_w);
        for (int kb = 0; kb < NWB; ++kb) {
            mbar_arrive_expect_tx(smem_u32(&ctrl->a_full[kb]), WBOX);
            tma_load_2d(data_s + OP_A + kb * WBOX, &tm_w, kb * 64, h * DH, smem_u32(&ctrl->a_full[kb]));
        }
    }
    if (warp == 0) {
        __syncwarp();
        tmem_alloc(smem_u32(&ctrl->tmem_base), TNO);
        tmem_relinquish();
    }
    pdl_trigger();
    pdl_wait();  // o_lat is the previous kernel's output
    const uint32_t bs = data_s + OP_B;
    for (int idx = tid; idx < npad * 64; idx += 128) {
        const int r = idx >> 6, g = idx & 63, c = g & 7;
        const uint32_t hs = bs + (g >> 3) * OP_BBLK + r * 128 + ((c ^ (r & 7)) << 4);
        if (r < nt) {
            const float *src = o_lat + ((size_t)(t0 + r) * n_h + h) * DCL + g * 8;
            cp_async16(hs, src);
            cp_async16(hs + TNO * 128, src + 4);
        } else {
            st_shared_v4(hs, 0u, 0u, 0u, 0u);
            st_shared_v4(hs + TNO * 128, 0u, 0u, 0u, 0u);
        }
    }
    cp_async_wait_all();
    for (int idx = tid; idx < npad * 64; idx += 128) {
        const int r = idx >> 6, g = idx & 63, c = g & 7;
        const uint32_t hs = bs + (g >> 3) * OP_BBLK + r * 128 + ((c ^ (r & 7)) << 4);
        float x[8];
        ld_shared_f4(hs, x);
        ld_shared_f4(hs + TNO * 128, x + 4);
        uint32_t hw[4], lw[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const __nv_bfloat162 hv = __floats2bfloat162_rn(x[2 * i], x[2 * i + 1]);
            const float2 hf = __bfloat1622float2(hv);
            const __nv_bfloat162 lv = __floats2bfloat162_rn(x[2 * i] - hf.x, x[2 * i + 1] - hf.y);
            hw[i] = *reinterpret_cast<const uint32_t *>(&hv);
            lw[i] = *reinterpret_cast<const uint32_t *>(&lv);
        }
        st_shared_v4(hs, hw[0], hw[1], hw[2], hw[3]);
        st_shared_v4(hs + TNO * 128, lw[0], lw[1], lw[2], lw[3]);
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = ctrl->tmem_base;
    if (tid == 0) {
        const uint32_t idesc = idesc_bf16(128, npad, false, false);
        bool good = true;
        for (int kb = 0; kb < NWB; ++kb) {
            if (!wait(smem_u32(&ctrl->a_full[kb]), 0, abort_flag)) {
                good = false;
                break;
            }
            tc_fence_after();
            const uint32_t bhi = bs + kb * OP_BBLK, blo = bhi + TNO * 128;
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const uint64_t a = sdesc_sw128(data_s + OP_A + kb * WBOX + k * 32, 16, 1024);
                mma_ss(tmem, a, sdesc_sw128(bhi + k * 32, 16, 1024), idesc, (kb | k) != 0 ? 1u : 0u);
                mma_ss(tmem, a, sdesc_sw128(blo + k * 32, 16, 1024), idesc, 1u);
            }
        }
        if (good) mma_commit(smem_u32(&ctrl->d_full));
        else *abort_flag = 1;
    }
    bool ok = __syncthreads_and(*abort_flag == 0);
    if (ok) ok = __syncthreads_and(wait(smem_u32(&ctrl->d_full), 0, abort_flag));
    if (ok) {
        tc_fence_after();
        const int d = warp * 32 + lane;
        uint32_t v[32];
        tmem_ld32(tmem + ((uint32_t)(warp * 32) << 16), v);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 32; ++j)
            if (j < nt) o[((size_t)(t0 + j) * n_h + h) * DH + d] = from_f32<To>(__uint_as_float(v[j]));
    } else if (tid == 0) {
        record_error(err, kErrTimeout);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, TNO);
    }
}

// ------------------------------------------------------------------------------------------
// combine + out_proj in one kernel, after the tensor-core decode.
// The decode leaves, per split slot s of a query row, the unnormalised partial O_s as bf16
// pairs of columns laid out [slot][d_c / 2][n_h] words, with its log2-domain max m_s and sum
// l_s per head.  The merge is the combine kernel's, term for term (same order, same fused
// multiply-adds), so o_lat and lse come out bit-identical to it:
//     M = max_s m_s,  w_s = 2^(m_s - M),  L = sum_s w_s l_s,
//     o_lat = sum_s w_s O_s / L,  lse = (M + log2 L) ln 2.
// Grid (n_h, tiles of TNO rows) in clusters of 4 CTAs along the heads (clusters of 8 would
// not all fit on the GPU at once with one CTA per SM).  CTA q of the cluster that owns heads
// 4g..4g+3 merges latent columns [128 q, 128 q + 128) for all 4 heads and all rows of its
// tile: a warp's loads then read 4 heads x 4 bytes = half a 32-byte sector per column pair,
// where a CTA merging only its own head would use 4 bytes of every sector it reads.  The merged values go, split into bf16 hi + lo exactly as out_proj splits o_lat,
// straight into the B tile of the CTA that owns the head (st.async into a peer's shared
// memory, completing on its b_full barrier; a plain store for the CTA's own head); o_lat and
// lse are also written out.  Then every CTA runs
// the out_proj MMAs of its head as out_proj_tc_kernel does.
// ------------------------------------------------------------------------------------------
constexpr int CO_CLUSTER = 4;
constexpr int CO_COLS = DCL / CO_CLUSTER;   // latent columns merged per CTA: 128 = 2 column blocks
constexpr int CO_THREADS = 256;
constexpr int CO_FAST = 8;  // rows split over at most this many slots take the all-loads-first path

template <typename To>
__global__ void __cluster_dims__(CO_CLUSTER, 1, 1) __launch_bounds__(CO_THREADS, 1)
combine_out_proj_tc_kernel(const __grid_constant__ CUtensorMap tm_w, int T, int n_h,
                           const int32_t *__restrict__ seg_range, const uint32_t *__restrict__ o_part,
                           const float *__restrict__ m_part, const float *__restrict__ l_part,
                           float *__restrict__ o_lat, float *__restrict__ lse, To *__restrict__ o,
                           unsigned *err) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_s = smem_u32(smem_raw);
    const uint32_t data_s = (raw_s + 1023u) & ~1023u;
    ProjCtrl *ctrl = reinterpret_cast<ProjCtrl *>(smem_raw + (data_s - raw_s) + OP_DATA);
    volatile uint32_t *abort_flag = &ctrl->abort;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int h = blockIdx.x, t0 = blockIdx.y * TNO;
    const int nt = min(TNO, T - t0);
    const int npad = (nt + 15) & ~15;
    const uint32_t q = cluster_ctarank();  // merges latent columns [128 q, 128 q + 128); == h % 4
    const int hg = h - (int)q;             // first head of the cluster

    if (tid == 0) {
        for (int i = 0; i < NWB; ++i) mbar_init(smem_u32(&ctrl->a_full[i]), 1);
        mbar_init(smem_u32(&ctrl->b_full), 1);
        mbar_init(smem_u32(&ctrl->d_full), 1);
        ctrl->abort = 0;
        // the column blocks merged by the other CTAs of the cluster: 2 blocks per CTA, nt rows,
        // hi + lo, 128 B each
        mbar_arrive_expect_tx(smem_u32(&ctrl->b_full), (uint32_t)((CO_CLUSTER - 1) * nt * 512));
        fence_mbarrier_init_cluster();
        prefetch_tensormap(&tm_w);
        for (int kb = 0; kb < NWB; ++kb) {
            mbar_arrive_expect_tx(smem_u32(&ctrl->a_full[kb]), WBOX);
            tma_load_2d(data_s + OP_A + kb * WBOX, &tm_w, kb * 64, h * DH, smem_u32(&ctrl->a_full[kb]));
        }
    }
    if (warp == 0) {
        __syncwarp();
        tmem_alloc(smem_u32(&ctrl->tmem_base), TNO);
        tmem_relinquish();
    }
    cluster_sync();  // every b_full of the cluster is initialised and armed before any st.async
    pdl_trigger();
    pdl_wait();      // the partials and the slot ranges are the decode's output
    const uint32_t bs = data_s + OP_B;

    // ---- merge: thread = (head i of the cluster, 8-column chunk c of this CTA's 128, row r = rq mod 4) ----
    // Every load a row needs is requested before any is used (up to CO_FAST slots), and the
    // next row's slot range is requested before this row is merged, so a row costs about one
    // round trip to L2.
    {
        const int i = tid & 3, c = (tid >> 2) & 15, rq = tid >> 6;
        const int hh = hg + i;
        const size_t slot_words = (size_t)(DCL / 2) * n_h;
        const uint32_t *src = o_part + (size_t)(q * (CO_COLS / 2) + c * 4) * n_h + hh;
        const uint32_t dst_bar = mapa(smem_u32(&ctrl->b_full), (uint32_t)i);
        int s0 = 0, s1 = 0;
        if (rq < nt) {
            s0 = __ldcg(seg_range + 2 * (t0 + rq));
            s1 = __ldcg(seg_range + 2 * (t0 + rq) + 1);
        }
        for (int r = rq; r < nt; r += CO_THREADS / 64) {
            const int row = t0 + r;
            int n0 = 0, n1 = 0;
            if (r + CO_THREADS / 64 < nt) {
                n0 = __ldcg(seg_range + 2 * (row + CO_THREADS / 64));
                n1 = __ldcg(seg_range + 2 * (row + CO_THREADS / 64) + 1);
            }
            float M = -INFINITY, L = 0.f, acc[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) acc[j] = 0.f;
            if (s1 - s0 <= CO_FAST) {
                float ms[CO_FAST], ls[CO_FAST];
                uint32_t v[CO_FAST][4];
#pragma unroll
                for (int j = 0; j < CO_FAST; ++j) {
                    const int s = s0 + j;
                    ms[j] = -INFINITY;
                    ls[j] = 0.f;
                    if (s < s1) {
                        ms[j] = __ldcg(m_part + (size_t)s * n_h + hh);
                        ls[j] = __ldcg(l_part + (size_t)s * n_h + hh);
#pragma unroll
                        for (int k = 0; k < 4; ++k) v[j][k] = __ldcg(src + (size_t)s * slot_words + (size_t)k * n_h);
                    }
                }
#pragma unroll
                for (int j = 0; j < CO_FAST; ++j) M = fmaxf(M, ms[j]);
#pragma unroll
                for (int j = 0; j < CO_FAST; ++j) {
                    if (ms[j] == -INFINITY) continue;  // empty or past the range: weight 0, never read
                    const float w = exp2f(ms[j] - M);
                    L = fmaf(w, ls[j], L);
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        acc[2 * k] = fmaf(w, __uint_as_float(v[j][k] << 16), acc[2 * k]);
                        acc[2 * k + 1] = fmaf(w, __uint_as_float(v[j][k] & 0xffff0000u), acc[2 * k + 1]);
                    }
                }
            } else {
                for (int s = s0; s < s1; ++s) M = fmaxf(M, __ldcg(m_part + (size_t)s * n_h + hh));
                for (int s = s0; s < s1; ++s) {
                    const float ms = __ldcg(m_part + (size_t)s * n_h + hh);
                    if (ms == -INFINITY) continue;
                    const float w = exp2f(ms - M);
                    L = fmaf(w, __ldcg(l_part + (size_t)s * n_h + hh), L);
                    uint32_t v[4];
#pragma unroll
                    for (int k = 0; k < 4; ++k) v[k] = __ldcg(src + (size_t)s * slot_words + (size_t)k * n_h);
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        acc[2 * k] = fmaf(w, __uint_as_float(v[k] << 16), acc[2 * k]);
                        acc[2 * k + 1] = fmaf(w, __uint_as_float(v[k] & 0xffff0000u), acc[2 * k + 1]);
                    }
                }
            }
            s0 = n0;
            s1 = n1;
            const float inv = L > 0.f ? 1.f / L : 0.f;
            float x[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) x[j] = acc[j] * inv;
            if (o_lat) {
                float4 *dst = reinterpret_cast<float4 *>(o_lat + ((size_t)row * n_h + hh) * DCL + q * CO_COLS + c * 8);
                dst[0] = make_float4(x[0], x[1], x[2], x[3]);
                dst[1] = make_float4(x[4], x[5], x[6], x[7]);
            }
            if (lse && q == 0 && c == 0)
                lse[(size_t)row * n_h + hh] = L > 0.f ? (M + log2f(L)) * 0.69314718055994531f : -INFINITY;
            uint32_t hw[4], lw[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const __nv_bfloat162 hv = __floats2bfloat162_rn(x[2 * k], x[2 * k + 1]);
                const float2 hf = __bfloat1622float2(hv);
                const __nv_bfloat162 lv = __floats2bfloat162_rn(x[2 * k] - hf.x, x[2 * k + 1] - hf.y);
                hw[k] = *reinterpret_cast<const uint32_t *>(&hv);
                lw[k] = *reinterpret_cast<const uint32_t *>(&lv);
            }
            const uint32_t loc = bs + (2 * q + (c >> 3)) * OP_BBLK + r * 128 + (((c & 7) ^ (r & 7)) << 4);
            if (i == (int)q) {  // this CTA's own head: a plain shared-memory store
                st_shared_v4(loc, hw[0], hw[1], hw[2], hw[3]);
                st_shared_v4(loc + TNO * 128, lw[0], lw[1], lw[2], lw[3]);
            } else {
                const uint32_t dst = mapa(loc, (uint32_t)i);
                st_async_v4(dst, hw[0], hw[1], hw[2], hw[3], dst_bar);
                st_async_v4(dst + TNO * 128, lw[0], lw[1], lw[2], lw[3], dst_bar);
            }
        }
    }
    // rows nt..npad-1 of the MMA's N are zero (only rows < nt are merged)
    for (int idx = tid; idx < (npad - nt) * 64; idx += CO_THREADS) {
        const int r = nt + (idx >> 6), g = idx & 63, c = g & 7;
        const uint32_t hs = bs + (g >> 3) * OP_BBLK + r * 128 + ((c ^ (r & 7)) << 4);
        st_shared_v4(hs, 0u, 0u, 0u, 0u);
        st_shared_v4(hs + TNO * 128, 0u, 0u, 0u, 0u);
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = ctrl->tmem_base;
    if (tid == 0) {
        const uint32_t idesc = idesc_bf16(128, npad, false, false);
        bool good = wait<true>(smem_u32(&ctrl->b_full), 0, abort_flag);
        tc_fence_after();
        for (int kb = 0; good && kb < NWB; ++kb) {
            if (!wait(smem_u32(&ctrl->a_full[kb]), 0, abort_flag)) {
                good = false;
                break;
            }
            tc_fence_after();
            const uint32_t bhi = bs + kb * OP_BBLK, blo = bhi + TNO * 128;
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const uint64_t a = sdesc_sw128(data_s + OP_A + kb * WBOX + k * 32, 16, 1024);
                mma_ss(tmem, a, sdesc_sw128(bhi + k * 32, 16, 1024), idesc, (kb | k) != 0 ? 1u : 0u);
                mma_ss(tmem, a, sdesc_sw128(blo + k * 32, 16, 1024), idesc, 1u);
            }
        }
        if (good) mma_commit(smem_u32(&ctrl->d_full));
        else *abort_flag = 1;
    }
    bool ok = __syncthreads_and(*abort_flag == 0);
    if (ok) ok = __syncthreads_and(wait(smem_u32(&ctrl->d_full), 0, abort_flag));
    if (ok) {
        if (warp < 4) {  // the accumulator's 128 lanes = the head's 128 output rows
            tc_fence_after();
            const int d = warp * 32 + lane;
            uint32_t v[32];
            tmem_ld32(tmem + ((uint32_t)(warp * 32) << 16), v);
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 32; ++j)
                if (j < nt) o[((size_t)(t0 + j) * n_h + h) * DH + d] = from_f32<To>(__uint_as_float(v[j]));
        }
    } else if (tid == 0) {
        record_error(err, kErrTimeout);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, TNO);
    }
    // No CTA leaves while a peer may still be sending into its shared memory: every CTA has
    // issued its sends and waited for its own tile before it reaches this barrier.
    cluster_sync();
}

// ------------------------------------------------------------------------------------------
// absorb: smem = W_h (8 x 16 KB boxes [128 k-rows x 64 c], read MN-major) + q tile (2 x TN x 128 B).
// After the MMAs the weight region holds the bf16 result [token][d_c] for coalesced stores.
// ------------------------------------------------------------------------------------------
constexpr int AB_A = 0;
constexpr int AB_B = NWB * WBOX;                  // 131072
constexpr int AB_DATA = AB_B + 2 * TN * 128;      // + 32 KB
constexpr int AB_SMEM = 1024 + AB_DATA + 256;
static_assert(TN * DCL * 2 <= NWB * WBOX, "the result tile reuses the weight region");

// KV >= 0: the same launch also appends job.T new tokens to the cache (mla_cache_append's
// work, KV as in append_token: 1 = bf16 cache, 2 = fp8 content cache) in extra CTAs
// blockIdx.x >= n_h of the first token tile, one warp per token; their work is independent
// of the absorption, so it overlaps the absorption's weight fetch instead of preceding it.
template <int KV>
__global__ void __launch_bounds__(128, 1)
absorb_tc_kernel(const __grid_constant__ CUtensorMap tm_w, int T, int n_h, const __grid_constant__ RopeFreqs rope,
                 const __nv_bfloat16 *__restrict__ q_c, const __nv_bfloat16 *__restrict__ q_r,
                 const int32_t *__restrict__ pos, __nv_bfloat16 *__restrict__ q_abs, unsigned *err,
                 const __grid_constant__ AppendArgs job) {
    pdl_trigger();  // the decode that follows may set itself up (it waits for q_abs on the device)
    if (KV >= 0 && (int)blockIdx.x >= n_h) {  // an append CTA
        if (blockIdx.y != 0) return;
        pdl_wait();  // the new tokens may be the previous kernel's output
        const int t = ((int)blockIdx.x - n_h) * 4 + (threadIdx.x >> 5);
        if (t < job.T) append_token<__nv_bfloat16, (KV < 0 ? 1 : KV)>(job, rope, t, threadIdx.x & 31, err);
        return;
    }
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_s = smem_u32(smem_raw);
    const uint32_t data_s = (raw_s + 1023u) & ~1023u;
    ProjCtrl *ctrl = reinterpret_cast<ProjCtrl *>(smem_raw + (data_s - raw_s) + AB_DATA);
    volatile uint32_t *abort_flag = &ctrl->abort;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int h = blockIdx.x, t0 = blockIdx.y * TN;
    const int nt = min(TN, T - t0);
    const int npad = (nt + 15) & ~15;
    constexpr int ROWQ = DCL + DR;

    if (tid == 0) {
        for (int i = 0; i < NWB; ++i) mbar_init(smem_u32(&ctrl->a_full[i]), 1);
        mbar_init(smem_u32(&ctrl->d_full), 1);
        ctrl->abort = 0;
        fence_mbarrier_init_cluster();
        // The weights are constants of the layer: their load starts first and overlaps the end
        // of the kernel ahead of this one on the stream.
        prefetch_tensormap(&tm_w);
        for (int kb = 0; kb < NWB; ++kb) {
            mbar_arrive_expect_tx(smem_u32(&ctrl->a_full[kb]), WBOX);
            tma_load_2d(data_s + AB_A + kb * WBOX, &tm_w, kb * 64, h * DH, smem_u32(&ctrl->a_full[kb]));
        }
    }
    if (warp == 0) {
        __syncwarp();
        tmem_alloc(smem_u32(&ctrl->tmem_base), 512);
        tmem_relinquish();
    }
    pdl_wait();  // the queries may be the previous kernel's output
    // q_c rows of this head for the tile's tokens -> two K-major column blocks (k 0-63, 64-127),
    // copied asynchronously so that the RoPE loads below go out at the same time.
    const uint32_t bq = data_s + AB_B;
    for (int idx = tid; idx < npad * 16; idx += 128) {
        const int r = idx >> 4, c = idx & 15;
        const int cb = c >> 3, cc = c & 7;
        const uint32_t dst = bq + cb * TN * 128 + r * 128 + ((cc ^ (r & 7)) << 4);
        if (r < nt) cp_async16(dst, q_c + ((size_t)(t0 + r) * n_h + h) * DH + c * 8);
        else st_shared_v4(dst, 0u, 0u, 0u, 0u);
    }
    // RoPE part of the query (분리 RoPE section): pairs (k, k + 32), eight pairs per item.
    for (int idx = tid; idx < nt * (DR / 16); idx += 128) {
        const int t = t0 + (idx >> 2), kg = (idx & 3) * 8;
        const int p = pos[t];
        const __nv_bfloat16 *x = q_r + ((size_t)t * n_h + h) * DR;
        const uint4 u0 = *reinterpret_cast<const uint4 *>(x + kg);
        const uint4 u1 = *reinterpret_cast<const uint4 *>(x + DR / 2 + kg);
        const __nv_bfloat16 *x0 = reinterpret_cast<const __nv_bfloat16 *>(&u0);
        const __nv_bfloat16 *x1 = reinterpret_cast<const __nv_bfloat16 *>(&u1);
        __align__(16) __nv_bfloat16 y0[8], y1[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            float cs, sn;
            rope_cos_sin(rope, kg + e, p, &cs, &sn);
            const float a = __bfloat162float(x0[e]), b = __bfloat162float(x1[e]);
            y0[e] = __float2bfloat16_rn(a * cs - b * sn);
            y1[e] = __float2bfloat16_rn(b * cs + a * sn);
        }
        __nv_bfloat16 *y = q_abs + ((size_t)t * n_h + h) * ROWQ + DCL;
        *reinterpret_cast<uint4 *>(y + kg) = *reinterpret_cast<const uint4 *>(y0);
        *reinterpret_cast<uint4 *>(y + DR / 2 + kg) = *reinterpret_cast<const uint4 *>(y1);
    }
    cp_async_wait_all();
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = ctrl->tmem_base;
    if (tid == 0) {
        const uint32_t idesc = idesc_bf16(128, npad, true, false);
        bool good = true;
        for (int mt = 0; mt < 4 && good; ++mt) {
            good = wait(smem_u32(&ctrl->a_full[2 * mt]), 0, abort_flag) &&
                   wait(smem_u32(&ctrl->a_full[2 * mt + 1]), 0, abort_flag);
            if (!good) break;
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < DH / 16; ++kk) {
                const uint64_t a = sdesc_sw128(data_s + AB_A + 2 * mt * WBOX + kk * 2048, WBOX, 1024);
                const uint64_t b = sdesc_sw128(bq + (kk >> 2) * TN * 128 + (kk & 3) * 32, 16, 1024);
                mma_ss(tmem + mt * npad, a, b, idesc, kk > 0 ? 1u : 0u);
            }
        }
        if (good) mma_commit(smem_u32(&ctrl->d_full));
        else *abort_flag = 1;
    }
    bool ok = __syncthreads_and(*abort_flag == 0);
    if (ok) ok = __syncthreads_and(wait(smem_u32(&ctrl->d_full), 0, abort_flag));
    if (ok) {
        // D[c, t] (lane = latent column) -> bf16 rows [t][d_c] in the (now free) weight region,
        // then whole-row 16-byte stores.
        tc_fence_after();
        const uint32_t stage = data_s + AB_A;
        const int cl = warp * 32 + lane;
        for (int mt = 0; mt < 4; ++mt) {
            for (int c0 = 0; c0 < npad; c0 += 32) {
                uint32_t v[32];
                tmem_ld32(tmem + ((uint32_t)(warp * 32) << 16) + mt * npad + c0, v);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    const int t = c0 + j;
                    if (t < nt) {
                        const __nv_bfloat16 b = __float2bfloat16_rn(__uint_as_float(v[j]));
                        asm volatile("st.shared.b16 [%0], %1;" ::"r"(stage + t * (DCL * 2) + (mt * 128 + cl) * 2),
                                     "h"(*reinterpret_cast<const unsigned short *>(&b)) : "memory");
                    }
                }
            }
        }
        __syncthreads();
        for (int idx = tid; idx < nt * (DCL / 8); idx += 128) {
            const int t = idx >> 6, q = idx & 63;
            uint32_t w0, w1, w2, w3;
            asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                         : "=r"(w0), "=r"(w1), "=r"(w2), "=r"(w3) : "r"(stage + t * (DCL * 2) + q * 16) : "memory");
            *reinterpret_cast<uint4 *>(q_abs + ((size_t)(t0 + t) * n_h + h) * ROWQ + q * 8) = make_uint4(w0, w1, w2, w3);
        }
    } else if (tid == 0) {
        record_error(err, kErrTimeout);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

}  // namespace

bool proj_tc_supported(const mla_dims_t &d) {
    return d.d_h == DH && d.d_c == DCL && d.d_r == DR && d.act_dtype == MLA_DTYPE_BF16;
}

namespace {
// Both projections are launched as programmatic dependents of the kernel before them on the
// stream: their blocks start (and fetch the constant weights) while that kernel drains, and wait
// for it on the device before they read an activation or write an output.
template <typename... Exp, typename... Act>
cudaError_t launch_dependent_n(void (*kernel)(Exp...), dim3 grid, int threads, int smem, cudaStream_t st,
                               Act &&...args) {
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    cudaLaunchAttribute pdl;
    pdl.id = cudaLaunchAttributeProgrammaticStreamSerialization;
    pdl.val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(threads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cfg.attrs = &pdl;
#ifdef MLA_NO_PDL
    cfg.numAttrs = 0;
#else
    cfg.numAttrs = 1;
#endif
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<Act &&>(args)...);
}
template <typename... Exp, typename... Act>
cudaError_t launch_dependent(void (*kernel)(Exp...), dim3 grid, int smem, cudaStream_t st, Act &&...args) {
    return launch_dependent_n(kernel, grid, 128, smem, st, static_cast<Act &&>(args)...);
}
}  // namespace

cudaError_t launch_absorb_q_tc(const mla_dims_t &d, int T, const void *q_c, const void *q_r,
                               const int32_t *pos, const void *w_uk, void *q_abs, cudaStream_t st) {
    CUtensorMap tm;
    if (!tmap_bf16_2d(&tm, w_uk, DCL, (uint64_t)d.n_h * DH, DCL * 2, 64, 128)) return cudaErrorInvalidValue;
    AppendArgs none = {};
    return launch_dependent(absorb_tc_kernel<-1>, dim3(d.n_h, (T + TN - 1) / TN), AB_SMEM, st, tm, T, d.n_h,
                            make_rope_freqs((double)d.rope_base, d.d_r), reinterpret_cast<const __nv_bfloat16 *>(q_c),
                            reinterpret_cast<const __nv_bfloat16 *>(q_r), pos,
                            reinterpret_cast<__nv_bfloat16 *>(q_abs), device_error_word(), none);
}

bool append_absorb_tc_supported(const mla_dims_t &d) {
    return proj_tc_supported(d) && (d.kv_dtype == MLA_DTYPE_BF16 || d.kv_dtype == MLA_DTYPE_FP8_E4M3);
}

cudaError_t launch_append_absorb_tc(const mla_dims_t &d, const AppendArgs &job, int T, const void *q_c,
                                    const void *q_r, const int32_t *pos, const void *w_uk, void *q_abs,
                                    cudaStream_t st) {
    CUtensorMap tm;
    if (!tmap_bf16_2d(&tm, w_uk, DCL, (uint64_t)d.n_h * DH, DCL * 2, 64, 128)) return cudaErrorInvalidValue;
    const dim3 grid(d.n_h + (job.T + 3) / 4, (T + TN - 1) / TN);
    const RopeFreqs rope = make_rope_freqs((double)d.rope_base, d.d_r);
    auto qc = reinterpret_cast<const __nv_bfloat16 *>(q_c);
    auto qr = reinterpret_cast<const __nv_bfloat16 *>(q_r);
    auto qa = reinterpret_cast<__nv_bfloat16 *>(q_abs);
    if (d.kv_dtype == MLA_DTYPE_FP8_E4M3)
        return launch_dependent(absorb_tc_kernel<2>, grid, AB_SMEM, st, tm, T, d.n_h, rope, qc, qr, pos, qa,
                                device_error_word(), job);
    return launch_dependent(absorb_tc_kernel<1>, grid, AB_SMEM, st, tm, T, d.n_h, rope, qc, qr, pos, qa,
                            device_error_word(), job);
}

cudaError_t launch_out_proj_tc(const mla_dims_t &d, int T, const float *o_lat, const void *w_uv, void *o,
                               mla_dtype_t out_dtype, cudaStream_t st) {
    CUtensorMap tm;
    if (!tmap_bf16_2d(&tm, w_uv, DCL, (uint64_t)d.n_h * DH, DCL * 2, 64, 128)) return cudaErrorInvalidValue;
    const dim3 grid(d.n_h, (T + TNO - 1) / TNO);
    if (out_dtype == MLA_DTYPE_BF16)
        return launch_dependent(out_proj_tc_kernel<__nv_bfloat16>, grid, OP_SMEM, st, tm, T, d.n_h, o_lat,
                                reinterpret_cast<__nv_bfloat16 *>(o), device_error_word());
    return launch_dependent(out_proj_tc_kernel<float>, grid, OP_SMEM, st, tm, T, d.n_h, o_lat,
                            reinterpret_cast<float *>(o), device_error_word());
}

cudaError_t launch_combine_out_proj_tc(const mla_dims_t &d, int T, const int32_t *seg_range,
                                       const uint32_t *o_part, const float *m_part, const float *l_part,
                                       float *o_lat, float *lse, const void *w_uv, void *o,
                                       mla_dtype_t out_dtype, cudaStream_t st) {
    if (d.n_h % CO_CLUSTER != 0) return cudaErrorInvalidValue;
    CUtensorMap tm;
    if (!tmap_bf16_2d(&tm, w_uv, DCL, (uint64_t)d.n_h * DH, DCL * 2, 64, 128)) return cudaErrorInvalidValue;
    const dim3 grid(d.n_h, (T + TNO - 1) / TNO);
    if (out_dtype == MLA_DTYPE_BF16)
        return launch_dependent_n(combine_out_proj_tc_kernel<__nv_bfloat16>, grid, CO_THREADS, OP_SMEM, st, tm, T,
                                  d.n_h, seg_range, o_part, m_part, l_part, o_lat, lse,
                                  reinterpret_cast<__nv_bfloat16 *>(o), device_error_word());
    return launch_dependent_n(combine_out_proj_tc_kernel<float>, grid, CO_THREADS, OP_SMEM, st, tm, T, d.n_h,
                              seg_range, o_part, m_part, l_part, o_lat, lse, reinterpret_cast<float *>(o),
                              device_error_word());
}

}  // namespace mla
