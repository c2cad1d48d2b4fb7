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
    uint64_t d_full;
    uint32_t tmem_base;
    uint32_t abort;
};

#ifdef MLA_PROF
// Development instrumentation: per CTA of the last launch of each kernel (0 = absorb,
// 1 = out_proj), globaltimer at entry and exit and clock64 offsets from entry at marks 1..13.
__device__ unsigned long long g_proj_prof[2][512][16];
#define PPROF_DECL(kid) const long long pp_c0 = clock64(); const int pp_k = (kid); \
    unsigned long long *pp_row = g_proj_prof[pp_k][min(blockIdx.x + blockIdx.y * gridDim.x, 511u)]; \
    if (threadIdx.x == 0) pp_row[0] = globaltimer();
#define PPROF_MARK(i) do { if (threadIdx.x == 0) pp_row[i] = clock64() - pp_c0; } while (0)
#define PPROF_END() do { if (threadIdx.x == 0) { pp_row[15] = globaltimer(); pp_row[14] = clock64() - pp_c0; } } while (0)
#else
#define PPROF_DECL(kid)
#define PPROF_MARK(i)
#define PPROF_END()
#endif

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
    PPROF_DECL(1)
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
    PPROF_MARK(1);
    pdl_trigger();
    pdl_wait();  // o_lat is the previous kernel's output
    PPROF_MARK(2);
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
    PPROF_MARK(3);
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
    PPROF_MARK(4);
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
        PPROF_MARK(5);
    }
    bool ok = __syncthreads_and(*abort_flag == 0);
    if (ok) ok = __syncthreads_and(wait(smem_u32(&ctrl->d_full), 0, abort_flag));
    PPROF_MARK(6);
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
    PPROF_MARK(7);
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, TNO);
    }
    PPROF_END();
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

__global__ void __launch_bounds__(128, 1)
absorb_tc_kernel(const __grid_constant__ CUtensorMap tm_w, int T, int n_h, const __grid_constant__ RopeFreqs rope,
                 const __nv_bfloat16 *__restrict__ q_c, const __nv_bfloat16 *__restrict__ q_r,
                 const int32_t *__restrict__ pos, __nv_bfloat16 *__restrict__ q_abs, unsigned *err) {
    PPROF_DECL(0)
    pdl_trigger();  // the decode that follows may set itself up (it waits for q_abs on the device)
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
    PPROF_MARK(1);
    pdl_wait();  // the queries may be the previous kernel's output
    PPROF_MARK(2);
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
    PPROF_MARK(3);
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
        PPROF_MARK(4);
    }
    bool ok = __syncthreads_and(*abort_flag == 0);
    if (ok) ok = __syncthreads_and(wait(smem_u32(&ctrl->d_full), 0, abort_flag));
    PPROF_MARK(6);
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
    PPROF_MARK(7);
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
    PPROF_END();
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
cudaError_t launch_dependent(void (*kernel)(Exp...), dim3 grid, int smem, cudaStream_t st, Act &&...args) {
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    cudaLaunchAttribute pdl;
    pdl.id = cudaLaunchAttributeProgrammaticStreamSerialization;
    pdl.val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(128);
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
}  // namespace

cudaError_t launch_absorb_q_tc(const mla_dims_t &d, int T, const void *q_c, const void *q_r,
                               const int32_t *pos, const void *w_uk, void *q_abs, cudaStream_t st) {
    CUtensorMap tm;
    if (!tmap_bf16_2d(&tm, w_uk, DCL, (uint64_t)d.n_h * DH, DCL * 2, 64, 128)) return cudaErrorInvalidValue;
    return launch_dependent(absorb_tc_kernel, dim3(d.n_h, (T + TN - 1) / TN), AB_SMEM, st, tm, T, d.n_h,
                            make_rope_freqs((double)d.rope_base, d.d_r), reinterpret_cast<const __nv_bfloat16 *>(q_c),
                            reinterpret_cast<const __nv_bfloat16 *>(q_r), pos,
                            reinterpret_cast<__nv_bfloat16 *>(q_abs), device_error_word());
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

#ifdef MLA_PROF
// Copies the per-CTA timelines (2 x 512 x 16 u64) of the projection kernels and clears them.
extern "C" int mla_proj_prof_dump(unsigned long long *host) {
    if (cudaDeviceSynchronize() != cudaSuccess) return -1;
    cudaMemcpyFromSymbol(host, g_proj_prof, sizeof(g_proj_prof));
    static unsigned long long zeros[2 * 512 * 16];
    cudaMemcpyToSymbol(g_proj_prof, zeros, sizeof(zeros));
    return 0;
}
#endif

}  // namespace mla
