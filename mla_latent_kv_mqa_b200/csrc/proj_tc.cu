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

// ------------------------------------------------------------------------------------------
// out_proj: smem = W_h (8 x 16 KB, K-major) + 2 stages x (B_hi, B_lo) of TN x 64 bf16.
// ------------------------------------------------------------------------------------------
constexpr int OP_A = 0;
constexpr int OP_B = NWB * WBOX;                  // 131072
constexpr int OP_BSTAGE = 2 * TN * 128;           // hi + lo: 32 KB
constexpr int OP_DATA = OP_B + 2 * OP_BSTAGE;     // 196608
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
    const int h = blockIdx.x, t0 = blockIdx.y * TN;
    const int nt = min(TN, T - t0);
    const int npad = (nt + 15) & ~15;

    if (tid == 0) {
        for (int i = 0; i < NWB; ++i) mbar_init(smem_u32(&ctrl->a_full[i]), 1);
        for (int i = 0; i < 2; ++i) mbar_init(smem_u32(&ctrl->b_done[i]), 1);
        mbar_init(smem_u32(&ctrl->d_full), 1);
        ctrl->abort = 0;
        fence_mbarrier_init_cluster();
    }
    if (warp == 0) {
        tmem_alloc(smem_u32(&ctrl->tmem_base), TN);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = ctrl->tmem_base;
    if (tid == 0) {
        prefetch_tensormap(&tm_w);
        for (int kb = 0; kb < NWB; ++kb) {
            mbar_arrive_expect_tx(smem_u32(&ctrl->a_full[kb]), WBOX);
            tma_load_2d(data_s + OP_A + kb * WBOX, &tm_w, kb * 64, h * DH, smem_u32(&ctrl->a_full[kb]));
        }
    }
    const uint32_t idesc = idesc_bf16(128, npad, false, false);
    bool ok = true;
    for (int kb = 0; kb < NWB && ok; ++kb) {
        const int s = kb & 1;
        if (kb >= 2) ok = __syncthreads_and(wait(smem_u32(&ctrl->b_done[s]), ((kb - 2) >> 1) & 1, abort_flag));
        if (!ok) break;
        const uint32_t bhi = data_s + OP_B + s * OP_BSTAGE, blo = bhi + TN * 128;
        for (int idx = tid; idx < npad * 8; idx += 128) {
            const int r = idx >> 3, c = idx & 7;
            float x[8];
            if (r < nt) {
                const float4 *src = reinterpret_cast<const float4 *>(o_lat + ((size_t)(t0 + r) * n_h + h) * DCL + kb * 64 + c * 8);
                const float4 u0 = src[0], u1 = src[1];
                x[0] = u0.x; x[1] = u0.y; x[2] = u0.z; x[3] = u0.w;
                x[4] = u1.x; x[5] = u1.y; x[6] = u1.z; x[7] = u1.w;
            } else {
#pragma unroll
                for (int i = 0; i < 8; ++i) x[i] = 0.f;
            }
            uint32_t hw[4], lw[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const __nv_bfloat162 hv = __floats2bfloat162_rn(x[2 * i], x[2 * i + 1]);
                const float2 hf = __bfloat1622float2(hv);
                const __nv_bfloat162 lv = __floats2bfloat162_rn(x[2 * i] - hf.x, x[2 * i + 1] - hf.y);
                hw[i] = *reinterpret_cast<const uint32_t *>(&hv);
                lw[i] = *reinterpret_cast<const uint32_t *>(&lv);
            }
            const uint32_t off = r * 128 + ((c ^ (r & 7)) << 4);
            asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(bhi + off), "r"(hw[0]), "r"(hw[1]), "r"(hw[2]), "r"(hw[3]) : "memory");
            asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(blo + off), "r"(lw[0]), "r"(lw[1]), "r"(lw[2]), "r"(lw[3]) : "memory");
        }
        fence_proxy_async_smem();
        __syncthreads();
        if (tid == 0) {
            if (!wait(smem_u32(&ctrl->a_full[kb]), 0, abort_flag)) {
                *abort_flag = 1;
            } else {
                tc_fence_after();
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const uint64_t a = sdesc_sw128(data_s + OP_A + kb * WBOX + k * 32, 16, 1024);
                    mma_ss(tmem, a, sdesc_sw128(bhi + k * 32, 16, 1024), idesc, (kb | k) != 0 ? 1u : 0u);
                    mma_ss(tmem, a, sdesc_sw128(blo + k * 32, 16, 1024), idesc, 1u);
                }
                mma_commit(smem_u32(&ctrl->b_done[s]));
                if (kb == NWB - 1) mma_commit(smem_u32(&ctrl->d_full));
            }
        }
        ok = __syncthreads_and(*abort_flag == 0);
    }
    if (ok) ok = __syncthreads_and(wait(smem_u32(&ctrl->d_full), 0, abort_flag));
    if (ok) {
        tc_fence_after();
        const int d = warp * 32 + lane;
        for (int c0 = 0; c0 < npad; c0 += 32) {
            uint32_t v[32];
            tmem_ld32(tmem + ((uint32_t)(warp * 32) << 16) + c0, v);
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                const int t = c0 + j;
                if (t < nt) o[((size_t)(t0 + t) * n_h + h) * DH + d] = from_f32<To>(__uint_as_float(v[j]));
            }
        }
    } else if (tid == 0) {
        record_error(err, kErrTimeout);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, TN);
    }
}

// ------------------------------------------------------------------------------------------
// absorb: smem = W_h (8 x 16 KB boxes [128 k-rows x 64 c], read MN-major) + q tile (2 x TN x 128 B).
// ------------------------------------------------------------------------------------------
constexpr int AB_A = 0;
constexpr int AB_B = NWB * WBOX;                  // 131072
constexpr int AB_DATA = AB_B + 2 * TN * 128;      // + 32 KB
constexpr int AB_SMEM = 1024 + AB_DATA + 256;

__global__ void __launch_bounds__(128, 1)
absorb_tc_kernel(const __grid_constant__ CUtensorMap tm_w, int T, int n_h, double rope_base,
                 const __nv_bfloat16 *__restrict__ q_c, const __nv_bfloat16 *__restrict__ q_r,
                 const int32_t *__restrict__ pos, __nv_bfloat16 *__restrict__ q_abs, unsigned *err) {
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
    }
    if (warp == 0) {
        tmem_alloc(smem_u32(&ctrl->tmem_base), 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = ctrl->tmem_base;
    if (tid == 0) {
        prefetch_tensormap(&tm_w);
        for (int kb = 0; kb < NWB; ++kb) {
            mbar_arrive_expect_tx(smem_u32(&ctrl->a_full[kb]), WBOX);
            tma_load_2d(data_s + AB_A + kb * WBOX, &tm_w, kb * 64, h * DH, smem_u32(&ctrl->a_full[kb]));
        }
    }
    // q_c rows of this head for the tile's tokens -> two K-major column blocks (k 0-63, 64-127)
    const uint32_t bq = data_s + AB_B;
    for (int idx = tid; idx < npad * 16; idx += 128) {
        const int r = idx >> 4, c = idx & 15;
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (r < nt) v = *reinterpret_cast<const uint4 *>(q_c + ((size_t)(t0 + r) * n_h + h) * DH + c * 8);
        const int cb = c >> 3, cc = c & 7;
        asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(bq + cb * TN * 128 + r * 128 + ((cc ^ (r & 7)) << 4)),
                     "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w) : "memory");
    }
    fence_proxy_async_smem();
    __syncthreads();
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
        tc_fence_after();
        const int cl = warp * 32 + lane;  // latent column within the 128-wide tile
        for (int mt = 0; mt < 4; ++mt) {
            for (int c0 = 0; c0 < npad; c0 += 32) {
                uint32_t v[32];
                tmem_ld32(tmem + ((uint32_t)(warp * 32) << 16) + mt * npad + c0, v);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    const int t = c0 + j;
                    if (t < nt)
                        q_abs[((size_t)(t0 + t) * n_h + h) * ROWQ + mt * 128 + cl] = __float2bfloat16_rn(__uint_as_float(v[j]));
                }
            }
        }
    } else if (tid == 0) {
        record_error(err, kErrTimeout);
    }
    // RoPE part of the query (분리 RoPE section), pairs (k, k + 32), angle in fp64.
    for (int i = tid; i < nt * (DR / 2); i += 128) {
        const int tt = i / (DR / 2), k = i % (DR / 2);
        const int t = t0 + tt;
        float cs, sn;
        rope_cos_sin(k, DR, rope_base, pos[t], &cs, &sn);
        const __nv_bfloat16 *x = q_r + ((size_t)t * n_h + h) * DR;
        const float x0 = __bfloat162float(x[k]), x1 = __bfloat162float(x[k + DR / 2]);
        __nv_bfloat16 *y = q_abs + ((size_t)t * n_h + h) * ROWQ + DCL;
        y[k] = __float2bfloat16_rn(x0 * cs - x1 * sn);
        y[k + DR / 2] = __float2bfloat16_rn(x1 * cs + x0 * sn);
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

cudaError_t launch_absorb_q_tc(const mla_dims_t &d, int T, const void *q_c, const void *q_r,
                               const int32_t *pos, const void *w_uk, void *q_abs, cudaStream_t st) {
    CUtensorMap tm;
    if (!tmap_bf16_2d(&tm, w_uk, DCL, (uint64_t)d.n_h * DH, DCL * 2, 64, 128)) return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(absorb_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, AB_SMEM);
    if (e != cudaSuccess) return e;
    dim3 grid(d.n_h, (T + TN - 1) / TN);
    absorb_tc_kernel<<<grid, 128, AB_SMEM, st>>>(tm, T, d.n_h, (double)d.rope_base,
                                                 reinterpret_cast<const __nv_bfloat16 *>(q_c),
                                                 reinterpret_cast<const __nv_bfloat16 *>(q_r), pos,
                                                 reinterpret_cast<__nv_bfloat16 *>(q_abs), device_error_word());
    return cudaGetLastError();
}

cudaError_t launch_out_proj_tc(const mla_dims_t &d, int T, const float *o_lat, const void *w_uv, void *o,
                               mla_dtype_t out_dtype, cudaStream_t st) {
    CUtensorMap tm;
    if (!tmap_bf16_2d(&tm, w_uv, DCL, (uint64_t)d.n_h * DH, DCL * 2, 64, 128)) return cudaErrorInvalidValue;
    dim3 grid(d.n_h, (T + TN - 1) / TN);
    if (out_dtype == MLA_DTYPE_BF16) {
        cudaError_t e = cudaFuncSetAttribute(out_proj_tc_kernel<__nv_bfloat16>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, OP_SMEM);
        if (e != cudaSuccess) return e;
        out_proj_tc_kernel<__nv_bfloat16><<<grid, 128, OP_SMEM, st>>>(tm, T, d.n_h, o_lat,
                                                                      reinterpret_cast<__nv_bfloat16 *>(o),
                                                                      device_error_word());
    } else {
        cudaError_t e = cudaFuncSetAttribute(out_proj_tc_kernel<float>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, OP_SMEM);
        if (e != cudaSuccess) return e;
        out_proj_tc_kernel<float><<<grid, 128, OP_SMEM, st>>>(tm, T, d.n_h, o_lat, reinterpret_cast<float *>(o),
                                                              device_error_word());
    }
    return cudaGetLastError();
}

}  // namespace mla
