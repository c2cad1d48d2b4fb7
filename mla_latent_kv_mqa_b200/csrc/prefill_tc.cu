// MHA-mode (naive-mode) prefill for the DeepSeek-V3 head shape on tcgen05.
//
// MLA article, sections 구조 (structure) and 분리 RoPE (decoupled RoPE): for a prompt of L
// tokens, head h attends with
//     q_{t,h} = [q^C_{t,h} ; RoPE(q^R_{t,h}, t)]                    (d_h + d_R = 192 wide)
//     k_{j,h} = [W^UK_h c^KV_j ; RoPE(k^R_j, j)]                    (the RoPE key is shared)
//     v_{j,h} = W^UV_h c^KV_j                                       (d_h = 128 wide)
//     o_{t,h} = sum_{j <= t} softmax_j(q_{t,h} . k_{j,h} / sqrt(d_h + d_R)) v_{j,h}
// The 한계 section and the remarks of the 행렬 흡수 section on choosing the mode: prefill has
// as many queries as keys, so reconstructing K and V once (MHA mode) does less work than
// running every query in the 576-wide latent space (MQA mode), which pays off only in decode.
//
// Three kernels, all in this file:
//   1. prefill_prep_kernel: the cos / sin table cs[t][k] of each token's position and
//      kr[t] = RoPE(k^R_t), positions t - cu_seqlens[b] (token index within its prompt), rows up
//      to the padded length zeroed.
//   2. prefill_kv_up_kernel: Kh[h][t] = W^UK_h c_t and Vh[h][t] = W^UV_h c_t, a tcgen05 GEMM
//      (tile 128 tokens x 256 output columns = 2 heads, K = d_c = 512), bf16 out through TMA.
//   3. prefill_attn_kernel: causal flash attention per (head, prompt, 128-query tile): Q = q^C
//      (read in place from the token-major input by a 4-D TMA map) next to RoPE(q^R) (rotated
//      by the softmax warps from q^R and the table on the way into shared memory); S = Q K^T into
//      TMEM (three buffers), softmax by 8 warps (two per query row), P written back over S in
//      TMEM as bf16 and used as the A operand of O += P V (O in TMEM), lazy rescale of O.
// Intermediate layouts (workspace, head-major so a (head, 128-token) tile is 128 consecutive
// rows): Kh, Vh [n_h][T_pad][128], kr [T_pad][64], all bf16, and cs [T_pad][32] float2;
// T_pad = T rounded up to 128.
#include <math.h>

#include "mla_internal.cuh"
#include "sm100.cuh"
#include "tmap.cuh"

namespace mla {
namespace {

using namespace sm100;

constexpr int PDH = 128, PDC = 512, PDR = 64;
constexpr int PT = 128;                                       // query / key / token tile

// 2^x by the hardware's approximation (relative error about 2^-22, flushes denormals): the
// probabilities are rounded to bf16 right after.
__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// ---- packed fp32 pairs (Blackwell f32x2 arithmetic: two lanes of work per instruction) ----
__device__ __forceinline__ uint64_t f2pack(float lo, float hi) {
    return (uint64_t)__float_as_uint(lo) | ((uint64_t)__float_as_uint(hi) << 32);
}
__device__ __forceinline__ float f2lo(uint64_t a) { return __uint_as_float((uint32_t)a); }
__device__ __forceinline__ float f2hi(uint64_t a) { return __uint_as_float((uint32_t)(a >> 32)); }
__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
__device__ __forceinline__ uint64_t add2(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ uint64_t sub2(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}

// 2^x for a pair, on the FMA pipe instead of the MUFU unit (whose 16 results per clock per SM
// otherwise bound the softmax).  Cody-Waite style: x = j + f with j = rint(x), taken by adding
// 1.5 * 2^23 (j then sits in the low mantissa bits of t), f in [-1/2, 1/2]; 2^f by a degree-3
// polynomial whose coefficients are the minimax fit of the relative error on [-1/2, 1/2]
// (Remez exchange, rounded to fp32; max relative error 7.5e-5, 1/26 of the bf16 rounding that P
// gets next); 2^j enters as j added to the exponent field.  x is clamped to >= -126 first, so
// the result stays a non-negative finite number (2^-126 or less where x was lower).
constexpr float kEx2C0 = 0.9999280571937561f, kEx2C1 = 0.6932609677314758f;
constexpr float kEx2C2 = 0.2426111251115799f, kEx2C3 = 0.0551716685295105f;
__device__ __forceinline__ uint64_t ex2_poly2(uint64_t x) {
    constexpr float kRound = 12582912.f;  // 1.5 * 2^23
    x = f2pack(fmaxf(f2lo(x), -126.f), fmaxf(f2hi(x), -126.f));
    const uint64_t t = add2(x, f2pack(kRound, kRound));
    const uint64_t f = sub2(x, sub2(t, f2pack(kRound, kRound)));
    uint64_t p = fma2(f2pack(kEx2C3, kEx2C3), f, f2pack(kEx2C2, kEx2C2));
    p = fma2(p, f, f2pack(kEx2C1, kEx2C1));
    p = fma2(p, f, f2pack(kEx2C0, kEx2C0));
    const uint32_t lo = (uint32_t)p + ((uint32_t)t << 23), hi = (uint32_t)(p >> 32) + ((uint32_t)(t >> 32) << 23);
    return (uint64_t)lo | ((uint64_t)hi << 32);
}

// P = 2^(S scale_log2 - m) for this warp's 64 keys of a row: packed bf16 pairs into pk, the fp32
// sum returned.  With POLY, the pairs c with c % 4 == 3 take ex2_poly2 (a quarter of the
// exponentials); only for tiles without masked keys, whose scores are all finite.
template <bool POLY>
__device__ __forceinline__ float softmax_exp(const uint32_t (&v)[64], float scale_log2, float nm, uint32_t (&pk)[32]) {
    const uint64_t sl2 = f2pack(scale_log2, scale_log2), nm2 = f2pack(nm, nm);
    uint64_t acc[2] = {0ull, 0ull};
#pragma unroll
    for (int c = 0; c < 32; ++c) {
        const uint64_t x = fma2(f2pack(__uint_as_float(v[2 * c]), __uint_as_float(v[2 * c + 1])), sl2, nm2);
        uint64_t p;
        if (POLY && (c & 3) == 3)
            p = ex2_poly2(x);
        else
            p = f2pack(ex2(f2lo(x)), ex2(f2hi(x)));
        acc[c & 1] = add2(acc[c & 1], p);
        pk[c] = pack_bf16x2(f2lo(p), f2hi(p));
    }
    const uint64_t a = add2(acc[0], acc[1]);
    return f2lo(a) + f2hi(a);
}

__device__ __forceinline__ float2 bf16x2_to_float2(uint32_t v) {
    return make_float2(__uint_as_float(v << 16), __uint_as_float(v & 0xffff0000u));
}

__device__ __forceinline__ int seq_of(const int32_t *cu, int B, int t) {
    int lo = 0, hi = B;  // largest b with cu[b] <= t
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (__ldg(cu + mid) <= t) lo = mid;
        else hi = mid;
    }
    return lo;
}

// ---- 1. prep ----------------------------------------------------------------------------------
// Block = 8 tokens of [0, T_pad), a warp per token, lane k = frequency pair k: the token's
// cos / sin table row (cs[t][k] = (cos, sin)(pos_t * theta_k), read by the attention kernel to
// rotate q^R) and kr[t] = RoPE(k^R_t); rows t >= T are written as zeros.  Also checks the prompt
// table once (block 0): cu[0] = 0, non-decreasing, cu[B] = T, every length <= max_len.
constexpr int PREP_TOKENS = 8;
__global__ void __launch_bounds__(32 * PREP_TOKENS)
prefill_prep_kernel(int B, const int32_t *__restrict__ cu, int T, int max_len, const __grid_constant__ RopeFreqs rope,
                    const __nv_bfloat16 *__restrict__ k_r, float2 *__restrict__ cs, __nv_bfloat16 *__restrict__ kr,
                    unsigned *err) {
    const int t = blockIdx.x * PREP_TOKENS + (threadIdx.x >> 5), k = threadIdx.x & 31;
    pdl_trigger();
    pdl_wait();  // the activations may be the previous kernel's output
    if (blockIdx.x == 0 && threadIdx.x == 0) {
        bool ok = __ldg(cu) == 0 && __ldg(cu + B) == T;
        for (int b = 0; b < B && ok; ++b) {
            const int len = __ldg(cu + b + 1) - __ldg(cu + b);
            ok = len >= 0 && len <= max_len;
        }
        if (!ok) record_error(err, kErrBadSeqLen);
    }
    float c = 0.f, s = 0.f, a = 0.f, b = 0.f;
    if (t < T) {
        const int pos = t - __ldg(cu + seq_of(cu, B, t));
        rope_cos_sin(rope, k, pos, &c, &s);
        // RoPE pair k = (x_k, x_{k+32})
        const float x0 = __bfloat162float(k_r[(size_t)t * PDR + k]);
        const float x1 = __bfloat162float(k_r[(size_t)t * PDR + k + PDR / 2]);
        a = x0 * c - x1 * s;
        b = x1 * c + x0 * s;
    }
    cs[(size_t)t * (PDR / 2) + k] = make_float2(c, s);
    kr[(size_t)t * PDR + k] = __float2bfloat16_rn(a);
    kr[(size_t)t * PDR + k + PDR / 2] = __float2bfloat16_rn(b);
}

// ---- 2. K / V reconstruction GEMM -----------------------------------------------------------
// CTA = (pair of heads, 128-token tile, K or V).  D[t, n] = sum_c c[t, c] W[n0 + n, c]:
// M = 128 tokens, N = 256 (two heads), K = 512 in 8 chunks of 64 through a 2-stage TMA ring;
// one thread issues loads and MMAs; the 4 warps move D (TMEM) to a bf16 staging tile in shared
// memory that one TMA store writes per head.  ~98 KB of shared memory and 256 TMEM columns,
// so two CTAs share an SM and one's epilogue overlaps the other's MMAs (measured ~5% fewer
// cycles per call than one CTA per SM with a 4-stage ring).
constexpr int UP_STAGES = 2;
constexpr int UP_A = PT * 128;            // [128 tokens x 64 cols] bf16: 16 KB
constexpr int UP_B = 256 * 128;           // [256 rows x 64 cols]: 32 KB
constexpr int UP_STAGE = UP_A + UP_B;     // 48 KB
constexpr int UP_DATA = UP_STAGES * UP_STAGE;
constexpr int UP_SMEM = 1024 + UP_DATA + 256;
static_assert(2 * 2 * PT * 128 <= UP_DATA, "the staging tile reuses the ring");

struct __align__(8) UpCtrl {
    uint64_t full[UP_STAGES], empty[UP_STAGES], d_full;
    uint32_t tmem_base, abort;
    uint32_t never;  // stays 0: the abort word of drain waits, which must not give up early
};

__global__ void __launch_bounds__(128, 2)
prefill_kv_up_kernel(const __grid_constant__ CUtensorMap tm_c, const __grid_constant__ CUtensorMap tm_wk,
                     const __grid_constant__ CUtensorMap tm_wv, const __grid_constant__ CUtensorMap tm_kh,
                     const __grid_constant__ CUtensorMap tm_vh, int T_pad, unsigned *err) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_s = smem_u32(smem_raw);
    const uint32_t data_s = (raw_s + 1023u) & ~1023u;
    UpCtrl *ctrl = reinterpret_cast<UpCtrl *>(smem_raw + (data_s - raw_s) + UP_DATA);
    volatile uint32_t *abort_flag = &ctrl->abort;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int hp = blockIdx.x, t0 = blockIdx.y * PT;
    const bool is_v = blockIdx.z != 0;
    const CUtensorMap *tm_w = is_v ? &tm_wv : &tm_wk;
    auto bar = [&](uint64_t &b) { return smem_u32(&b); };

    if (tid == 0) {
        for (int i = 0; i < UP_STAGES; ++i) {
            mbar_init(bar(ctrl->full[i]), 1);
            mbar_init(bar(ctrl->empty[i]), 1);
        }
        mbar_init(bar(ctrl->d_full), 1);
        ctrl->abort = 0;
        ctrl->never = 0;
        fence_mbarrier_init_cluster();
    }
    if (warp == 0) {
        __syncwarp();
        tmem_alloc(smem_u32(&ctrl->tmem_base), 256);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = ctrl->tmem_base;
    pdl_trigger();
    pdl_wait();  // c_kv and the weights may be the previous kernels' output

    if (tid == 0) {
        constexpr uint32_t idesc = idesc_bf16(128, 256, false, false);
        bool ok = true;
        int issued = 0;
        auto load = [&](int kc) {
            const int s = kc % UP_STAGES;
            const uint32_t a = data_s + s * UP_STAGE;
            mbar_arrive_expect_tx(bar(ctrl->full[s]), UP_STAGE);
            tma_load_3d(a, &tm_c, 0, t0, kc, bar(ctrl->full[s]));
            tma_load_3d(a + UP_A, tm_w, 0, hp * 256, kc, bar(ctrl->full[s]));
        };
        for (; issued < UP_STAGES; ++issued) load(issued);
        for (int kc = 0; kc < PDC / 64; ++kc) {
            const int s = kc % UP_STAGES;
            if (!(ok = wait(bar(ctrl->full[s]), (kc / UP_STAGES) & 1u, abort_flag))) break;
            tc_fence_after();
            const uint32_t a = data_s + s * UP_STAGE, b = a + UP_A;
#pragma unroll
            for (int k = 0; k < 4; ++k)
                mma_ss(tmem, sdesc_sw128(a + k * 32, 16, 1024), sdesc_sw128(b + k * 32, 16, 1024), idesc,
                       (kc | k) != 0 ? 1u : 0u);
            mma_commit(bar(ctrl->empty[s]));
            // refill the stage of the previous chunk (its MMAs are queued before this chunk's, so
            // waiting for them keeps this chunk's MMAs in the tensor pipe meanwhile)
            if (kc >= 1 && issued < PDC / 64) {
                const int ps = (kc - 1) % UP_STAGES;
                if (!(ok = wait(bar(ctrl->empty[ps]), ((kc - 1) / UP_STAGES) & 1u, abort_flag))) break;
                load(issued++);
            }
        }
        if (ok) {
            mma_commit(bar(ctrl->d_full));
        } else {
            *abort_flag = 1;
            record_error(err, kErrTimeout);
            // drain: the loads still in flight (the last one of each stage) land before the
            // CTA can leave
            for (int kc = max(0, issued - UP_STAGES); kc < issued; ++kc)
                wait(bar(ctrl->full[kc % UP_STAGES]), (kc / UP_STAGES) & 1u, &ctrl->never, 1000000000ull);
        }
    }
    bool ok = __syncthreads_and(*abort_flag == 0);
    if (ok) ok = __syncthreads_and(wait(bar(ctrl->d_full), 0, abort_flag));
    if (ok) {
        tc_fence_after();
        // staging: [head (2)][column block (2)][128 rows x 128 B], 128-byte swizzle
        const int r = warp * 32 + lane;
        const uint32_t stg = data_s;
#pragma unroll 1
        for (int ch = 0; ch < 8; ++ch) {
            uint32_t v[32];
            tmem_ld32(tmem + ((uint32_t)(warp * 32) << 16) + ch * 32, v);
            tmem_wait_ld();
            const int n = ch * 32, hl = n >> 7, cb = (n & 127) >> 6;
            const uint32_t base = stg + (hl * 2 + cb) * (PT * 128) + r * 128;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int c16 = ((n & 63) >> 3) + q;
                st_shared_v4(base + ((c16 ^ (r & 7)) << 4),
                             pack_bf16x2(__uint_as_float(v[8 * q + 0]), __uint_as_float(v[8 * q + 1])),
                             pack_bf16x2(__uint_as_float(v[8 * q + 2]), __uint_as_float(v[8 * q + 3])),
                             pack_bf16x2(__uint_as_float(v[8 * q + 4]), __uint_as_float(v[8 * q + 5])),
                             pack_bf16x2(__uint_as_float(v[8 * q + 6]), __uint_as_float(v[8 * q + 7])));
            }
        }
        fence_proxy_async_smem();
        __syncthreads();
        if (tid == 0) {
            const CUtensorMap *out = is_v ? &tm_vh : &tm_kh;
            for (int hl = 0; hl < 2; ++hl)
                tma_store_3d(out, stg + hl * 2 * (PT * 128), 0, (2 * hp + hl) * T_pad + t0, 0);
            bulk_wait_group_all();
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 256);
    }
}

// ---- 3. causal attention ------------------------------------------------------------------
// CTA = (query tile qt, head h, prompt b), 352 threads: warp 0 loads (TMA; lane 0 Q and K,
// lane 1 V), warp 1 issues the QK MMAs and warp 10 the PV MMAs, warps 2-9 run the softmax, two
// warps per TMEM lane quarter (warp w reads lanes 32 (w % 4) ...), each on 64 of the tile's
// 128 keys; the two exchange their row maxima through shared memory once per tile.  (Reading the whole row in
// both warps instead, to skip the exchange, measured slower.)
// Shared: Q [3 blocks x 128 rows x 128 B] 48 KB; K ring 2 x (Kh 2 blocks + kr 1 block) 48 KB;
// V ring 2 x (2 blocks of [128 keys x 64 d]) 32 KB.  TMEM: S buffers [0,128), [128,256),
// [256,384), O [384,512).  Pipeline: QK_j runs up to NSB tiles ahead of the softmax; P_j
// overwrites S_j's first 64 columns (bf16 pairs), and QK_{j+NSB} reuses that buffer only after
// PV_j has completed.
constexpr int AT_Q = 0;
constexpr int AT_QB = PT * 128;                 // one [128 x 64] bf16 block: 16 KB
constexpr int AT_K = 3 * AT_QB;                 // 48 KB
constexpr int AT_KS = 3 * AT_QB;                // K stage: 48 KB
constexpr int AT_V = AT_K + 2 * AT_KS;          // 144 KB
constexpr int AT_VS = 2 * AT_QB;                // V stage: 32 KB
constexpr int AT_DATA = AT_V + 2 * AT_VS;       // 208 KB
constexpr int AT_SMEM = 1024 + AT_DATA + 5120;
constexpr int AT_THREADS = 352;  // 11 warps
constexpr int NSB = 3;                             // S buffers in TMEM
constexpr uint32_t S_COL0 = 0, O_COL = NSB * 128;  // S: [0, 384), O: [384, 512)
constexpr float kRescaleLog2 = 8.f;  // O is rescaled only when the running max grows by > 2^8

struct __align__(8) AtCtrl {
    uint64_t q_full, qr_full, k_full[2], k_empty[2], v_full[2], v_empty[2], s_full[NSB], p_ready[NSB], pv_done[NSB], idle[2];
    uint64_t xbar[4][1 + NSB];  // the two softmax warps of a lane quarter meet here: [0] the final row
                                // sums, [1 + s] the row maxima of S buffer s
    float xmax[NSB][2][128];  // [S buffer][half][row]: row max of each half's raw scores
    uint32_t tmem_base, abort;
    uint32_t never;           // stays 0: the abort word of drain waits
    float xsum[2][128];       // [half][row]: the final row sums
};
static_assert(sizeof(AtCtrl) <= 5120, "control block");

__global__ void __launch_bounds__(AT_THREADS, 1)
prefill_attn_kernel(const __grid_constant__ CUtensorMap tm_qc, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_kr, const __grid_constant__ CUtensorMap tm_v, int B,
                    const __nv_bfloat16 *__restrict__ q_r, const float2 *__restrict__ rope_cs,
                    const int32_t *__restrict__ cu, int T, int T_pad, int n_h, int q_tiles, float scale_log2,
                    __nv_bfloat16 *__restrict__ o, float *__restrict__ lse, unsigned *err) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_s = smem_u32(smem_raw);
    const uint32_t data_s = (raw_s + 1023u) & ~1023u;
    AtCtrl *ctrl = reinterpret_cast<AtCtrl *>(smem_raw + (data_s - raw_s) + AT_DATA);
    volatile uint32_t *abort_flag = &ctrl->abort;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // x = query tile (longest first), so the CTAs that run together share one (head, prompt)
    // and read its K and V from L2 rather than each from memory
    const int qt = q_tiles - 1 - (int)blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    auto bar = [&](uint64_t &x) { return smem_u32(&x); };

    pdl_trigger();
    pdl_wait();  // Kh, Vh, kr, cs are the previous kernels' output (q^C, q^R perhaps too)
    // the prompt (clamped to [0, T] so that a bad table cannot move a load or store out of range)
    const int start = min(max(__ldg(cu + b), 0), T);
    const int L = min(max(__ldg(cu + b + 1), start), T) - start;
    const int q0 = qt * PT;
    if (q0 >= L) return;  // whole CTA: this tile lies beyond the prompt
    const int n_kt = qt + 1;

    if (tid == 0) {
        mbar_init(bar(ctrl->q_full), 1);   // the loader: q^C's bytes
        mbar_init(bar(ctrl->qr_full), 8);  // the 8 softmax warps: RoPE(q^R)
        for (int i = 0; i < 2; ++i) {
            mbar_init(bar(ctrl->k_full[i]), 1);
            mbar_init(bar(ctrl->k_empty[i]), 1);
            mbar_init(bar(ctrl->v_full[i]), 1);
            mbar_init(bar(ctrl->v_empty[i]), 1);
        }
        for (int i = 0; i < NSB; ++i) {
            mbar_init(bar(ctrl->s_full[i]), 1);
            mbar_init(bar(ctrl->p_ready[i]), 8);
            mbar_init(bar(ctrl->pv_done[i]), 1);
        }
        mbar_init(bar(ctrl->idle[0]), 1);
        mbar_init(bar(ctrl->idle[1]), 1);
        for (int qq = 0; qq < 4; ++qq)
            for (int i = 0; i < 1 + NSB; ++i) mbar_init(bar(ctrl->xbar[qq][i]), 2);
        ctrl->abort = 0;
        ctrl->never = 0;
        fence_mbarrier_init_cluster();
    }
    if (warp == 0) {
        __syncwarp();
        tmem_alloc(smem_u32(&ctrl->tmem_base), 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = ctrl->tmem_base;
    const int qrow = h * T_pad + start;  // Kh / Vh row of the prompt's token 0 for this head

    if (warp == 0) {
        if (lane == 0) {  // ---- loads: Q, then the K ring (refilled as soon as a QK is done) ----
            bool ok = true;
            int issued = 0;
            mbar_arrive_expect_tx(bar(ctrl->q_full), 2 * AT_QB);
            tma_load_4d(data_s + AT_Q, &tm_qc, 0, start + q0, 0, h, bar(ctrl->q_full));  // q^C: blocks 0, 1
            for (int j = 0; j < n_kt; ++j) {
                const int s = j & 1;
                if (!(ok = wait(bar(ctrl->k_empty[s]), ((uint32_t)(j >> 1) & 1u) ^ 1u, abort_flag))) break;
                mbar_arrive_expect_tx(bar(ctrl->k_full[s]), AT_KS);
                tma_load_3d(data_s + AT_K + s * AT_KS, &tm_k, 0, qrow + j * PT, 0, bar(ctrl->k_full[s]));
                tma_load_3d(data_s + AT_K + s * AT_KS + 2 * AT_QB, &tm_kr, 0, start + j * PT, 0,
                            bar(ctrl->k_full[s]));
                ++issued;
            }
            if (!ok) *abort_flag = 1;
            // drain: loads in flight land before the CTA leaves
            wait(bar(ctrl->q_full), 0u, &ctrl->never, 1000000000ull);
            for (int j = max(0, issued - 2); j < issued; ++j)
                wait(bar(ctrl->k_full[j & 1]), (uint32_t)(j >> 1) & 1u, &ctrl->never, 1000000000ull);
        } else if (lane == 1) {  // ---- the V ring (refilled as soon as a PV is done) ----
            bool ok = true;
            int issued = 0;
            for (int j = 0; j < n_kt; ++j) {
                const int s = j & 1;
                if (!(ok = wait(bar(ctrl->v_empty[s]), ((uint32_t)(j >> 1) & 1u) ^ 1u, abort_flag))) break;
                mbar_arrive_expect_tx(bar(ctrl->v_full[s]), AT_VS);
                tma_load_3d(data_s + AT_V + s * AT_VS, &tm_v, 0, qrow + j * PT, 0, bar(ctrl->v_full[s]));
                ++issued;
            }
            if (!ok) *abort_flag = 1;
            for (int j = max(0, issued - 2); j < issued; ++j)
                wait(bar(ctrl->v_full[j & 1]), (uint32_t)(j >> 1) & 1u, &ctrl->never, 1000000000ull);
        }
    } else if (warp == 1) {
        if (lane == 0) {  // ---- QK issue: S_j = Q K_j^T into S buffer j % NSB ----
            constexpr uint32_t idesc_qk = idesc_bf16(128, 128, false, false);
            bool ok = wait(bar(ctrl->q_full), 0u, abort_flag);
            bool qr_in = false;  // the first tile's q^C MMAs go ahead while q^R is being rotated
            for (int j = 0; ok && j < n_kt; ++j) {
                const int s = j & 1, sb = j % NSB;  // K stage; S buffer
                if (!(ok = wait(bar(ctrl->k_full[s]), (uint32_t)(j >> 1) & 1u, abort_flag))) break;
                if (j >= NSB) {  // the PV that read P_{j-NSB} from this S buffer has completed
                    const int pj = j - NSB;
                    if (!(ok = wait(bar(ctrl->pv_done[sb]), (uint32_t)(pj / NSB) & 1u, abort_flag))) break;
                }
                tc_fence_after();
                const uint32_t kb = data_s + AT_K + s * AT_KS, d = tmem + S_COL0 + sb * 128;
#pragma unroll
                for (int cb = 0; cb < 3; ++cb) {
                    if (cb == 2 && !qr_in) {
                        if (!(ok = wait(bar(ctrl->qr_full), 0u, abort_flag))) break;
                        tc_fence_after();
                        qr_in = true;
                    }
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        mma_ss(d, sdesc_sw128(data_s + AT_Q + cb * AT_QB + k * 32, 16, 1024),
                               sdesc_sw128(kb + cb * AT_QB + k * 32, 16, 1024), idesc_qk, (cb | k) != 0 ? 1u : 0u);
                }
                if (!ok) break;
                mma_commit(bar(ctrl->k_empty[s]));
                mma_commit(bar(ctrl->s_full[sb]));
            }
            if (!ok) *abort_flag = 1;
            // no MMA of this thread may still run when TMEM is released
            mma_commit(bar(ctrl->idle[0]));
            wait(bar(ctrl->idle[0]), 0u, &ctrl->never, 1000000000ull);
        }
    } else if (warp == 10) {
        if (lane == 0) {  // ---- PV issue: O += P_j V_j ----
            // (A second issuing thread: one thread issues a tcgen05.mma about every 100 clocks,
            // and the 20 MMAs of a key tile from one thread took longer than the tensor core.)
            constexpr uint32_t idesc_pv = idesc_bf16(128, 128, false, true);
            bool ok = true;
            for (int j = 0; ok && j < n_kt; ++j) {
                const int s = j & 1, sb = j % NSB;
                if (!(ok = wait(bar(ctrl->p_ready[sb]), (uint32_t)(j / NSB) & 1u, abort_flag))) break;
                if (!(ok = wait(bar(ctrl->v_full[s]), (uint32_t)(j >> 1) & 1u, abort_flag))) break;
                tc_fence_after();
                const uint32_t vb = data_s + AT_V + s * AT_VS, p = tmem + S_COL0 + sb * 128;
#pragma unroll
                for (int kk = 0; kk < PT / 16; ++kk)
                    mma_ts(tmem + O_COL, p + kk * 8, sdesc_sw128(vb + kk * 2048, AT_QB, 1024), idesc_pv,
                           (j | kk) != 0 ? 1u : 0u);
                mma_commit(bar(ctrl->v_empty[s]));
                mma_commit(bar(ctrl->pv_done[sb]));
            }
            if (!ok) *abort_flag = 1;
            mma_commit(bar(ctrl->idle[1]));
            wait(bar(ctrl->idle[1]), 0u, &ctrl->never, 1000000000ull);
        }
    } else if (warp >= 2 && warp < 10) {  // ---- softmax: two warps per TMEM lane quarter, 64 keys each ----
        const int quarter = warp & 3, half = (warp - 2) >> 2;
        const int row = quarter * 32 + lane;  // query row of the tile = TMEM lane
        const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
        const int qi = q0 + row;              // query index within the prompt
        const int cbase = half * 64;          // this warp's key columns of the tile
        const uint32_t xbar0 = bar(ctrl->xbar[quarter][0]);
        {  // RoPE(q^R) of the tile's rows into Q's column block 2 (rows of 128 B, 128-byte swizzle):
           // thread = (row r, pairs k0 .. k0 + 15), pair k = (x_k, x_{k+32}) at position q0 + r
            const int st = tid - 64, r = st >> 1, k0 = (st & 1) * 16;
            uint32_t ya[8] = {}, yb[8] = {};  // bf16 pairs: elements k0 .. k0+15 and k0+32 .. k0+47
            if (q0 + r < L) {
                const size_t t = (size_t)(start + q0 + r);
                const uint4 *x = reinterpret_cast<const uint4 *>(q_r + (t * n_h + h) * PDR);
                const float4 *cs = reinterpret_cast<const float4 *>(rope_cs + t * (PDR / 2) + k0);
                uint32_t xa[8], xb[8];
                *reinterpret_cast<uint4 *>(xa) = __ldg(x + k0 / 8);
                *reinterpret_cast<uint4 *>(xa + 4) = __ldg(x + k0 / 8 + 1);
                *reinterpret_cast<uint4 *>(xb) = __ldg(x + (k0 + 32) / 8);
                *reinterpret_cast<uint4 *>(xb + 4) = __ldg(x + (k0 + 32) / 8 + 1);
#pragma unroll
                for (int i = 0; i < 8; ++i) {  // pairs k0 + 2i, k0 + 2i + 1
                    const float4 q = __ldg(cs + i);  // (cos, sin) of both
                    const float2 x0 = bf16x2_to_float2(xa[i]), x1 = bf16x2_to_float2(xb[i]);
                    ya[i] = pack_bf16x2(x0.x * q.x - x1.x * q.y, x0.y * q.z - x1.y * q.w);
                    yb[i] = pack_bf16x2(x1.x * q.x + x0.x * q.y, x1.y * q.z + x0.y * q.w);
                }
            }
            const uint32_t rowp = data_s + AT_Q + 2 * AT_QB + r * 128;
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                const int ca = k0 / 8 + c, cb = (k0 + 32) / 8 + c;  // 16-byte chunks of the row
                st_shared_v4(rowp + ((ca ^ (r & 7)) << 4), ya[4 * c], ya[4 * c + 1], ya[4 * c + 2], ya[4 * c + 3]);
                st_shared_v4(rowp + ((cb ^ (r & 7)) << 4), yb[4 * c], yb[4 * c + 1], yb[4 * c + 2], yb[4 * c + 3]);
            }
            fence_proxy_async_smem();  // visible to the tensor core's reads
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(ctrl->qr_full));
        }
        float m_run = -INFINITY, l_run = 0.f;  // l_run: the sum over this warp's keys
        bool ok = true;
        int j = 0;
        for (; j < n_kt; ++j) {
            const int s = j % NSB;
            const uint32_t ph = (uint32_t)(j / NSB) & 1u;
            if (!(ok = __all_sync(0xffffffffu, wait(bar(ctrl->s_full[s]), ph, abort_flag)))) break;
            tc_fence_after();
            uint32_t v[64];
            tmem_ld32(lane_base + S_COL0 + s * 128 + cbase, *reinterpret_cast<uint32_t(*)[32]>(v + 0));
            tmem_ld32(lane_base + S_COL0 + s * 128 + cbase + 32, *reinterpret_cast<uint32_t(*)[32]>(v + 32));
            tmem_wait_ld();
            // keys j*128 + cbase + c with c <= lim are visible (causal, and inside the prompt)
            const int lim = min(qi, L - 1) - j * PT - cbase;
            float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};  // row max of this warp's raw scores
            const bool unmasked = __all_sync(0xffffffffu, lim >= 63);
            if (unmasked) {
#pragma unroll
                for (int c = 0; c < 64; ++c) mx[c & 3] = fmaxf(mx[c & 3], __uint_as_float(v[c]));
            } else {
#pragma unroll
                for (int c = 0; c < 64; ++c) {
                    const float x = c <= lim ? __uint_as_float(v[c]) : -INFINITY;
                    v[c] = __float_as_uint(x);
                    mx[c & 3] = fmaxf(mx[c & 3], x);
                }
            }
            const float pm = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
            // the row max over both halves: exchange with the partner warp of this quarter
            ctrl->xmax[s][half][row] = pm;
            __syncwarp();
            if (lane == 0) mbar_arrive(xbar0 + (1 + s) * 8);
            if (!(ok = __all_sync(0xffffffffu, wait(xbar0 + (1 + s) * 8, ph, abort_flag)))) break;
            const float mt = fmaxf(pm, ctrl->xmax[s][half ^ 1][row]) * scale_log2;
            float fac = 1.f;
            if (mt > m_run + kRescaleLog2) {  // also the first visible key (m_run = -inf)
                fac = ex2(m_run - mt);        // 0 when m_run = -inf
                m_run = mt;
                l_run *= fac;
            }
            // O rows whose max moved: wait for the previous PV, then scale them (this warp: its
            // half of the 128 value columns)
            if (j > 0 && __any_sync(0xffffffffu, fac != 1.f)) {
                const int pj = j - 1;
                if (!(ok = __all_sync(0xffffffffu, wait(bar(ctrl->pv_done[pj % NSB]), (uint32_t)(pj / NSB) & 1u,
                                                        abort_flag))))
                    break;
                tc_fence_after();
#pragma unroll 1
                for (int ch = 0; ch < 2; ++ch) {
                    uint32_t w[32];
                    tmem_ld32(lane_base + O_COL + cbase + ch * 32, w);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 32; ++i) w[i] = __float_as_uint(__uint_as_float(w[i]) * fac);
                    tmem_st32(lane_base + O_COL + cbase + ch * 32, w);
                }
                tmem_wait_st();
            }
            const bool live = m_run != -INFINITY;  // false only for a row with no visible key yet
            const float nm = live ? -m_run : 0.f;
            uint32_t pk[32];
            float psum = unmasked ? softmax_exp<true>(v, scale_log2, nm, pk) : softmax_exp<false>(v, scale_log2, nm, pk);
            if (!live) {
                psum = 0.f;
#pragma unroll
                for (int c = 0; c < 32; ++c) pk[c] = 0u;
            }
            l_run += psum;
            // P over the first 64 columns of this S buffer: keys 2c, 2c+1 in column c
            tmem_st32(lane_base + S_COL0 + s * 128 + half * 32, pk);
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(ctrl->p_ready[s]));
        }
        if (ok) {
            const int lj = n_kt - 1;
            ok = __all_sync(0xffffffffu, wait(bar(ctrl->pv_done[lj % NSB]), (uint32_t)(lj / NSB) & 1u, abort_flag));
        }
        if (ok) {  // the row sum over both halves (one more exchange, tile index n_kt)
            ctrl->xsum[half][row] = l_run;
            __syncwarp();
            if (lane == 0) mbar_arrive(xbar0);  // the barrier's only use: phase 0
            ok = __all_sync(0xffffffffu, wait(xbar0, 0u, abort_flag));
        }
        if (ok) {
            tc_fence_after();
            const float l = l_run + ctrl->xsum[half ^ 1][row];
            const float inv = l > 0.f ? 1.f / l : 0.f;
            __nv_bfloat16 *dst = o + ((size_t)(start + qi) * n_h + h) * PDH + cbase;
#pragma unroll 1
            for (int ch = 0; ch < 2; ++ch) {
                uint32_t w[32];
                tmem_ld32(lane_base + O_COL + cbase + ch * 32, w);
                tmem_wait_ld();
                if (qi < L) {
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        *reinterpret_cast<uint4 *>(dst + ch * 32 + q * 8) =
                            make_uint4(pack_bf16x2(__uint_as_float(w[8 * q + 0]) * inv, __uint_as_float(w[8 * q + 1]) * inv),
                                       pack_bf16x2(__uint_as_float(w[8 * q + 2]) * inv, __uint_as_float(w[8 * q + 3]) * inv),
                                       pack_bf16x2(__uint_as_float(w[8 * q + 4]) * inv, __uint_as_float(w[8 * q + 5]) * inv),
                                       pack_bf16x2(__uint_as_float(w[8 * q + 6]) * inv, __uint_as_float(w[8 * q + 7]) * inv));
                }
            }
            if (lse && half == 0 && qi < L)
                lse[(size_t)(start + qi) * n_h + h] = l > 0.f ? (m_run + log2f(l)) * 0.69314718055994531f : -INFINITY;
        } else {
            *abort_flag = 1;
            if (lane == 0) record_error(err, kErrTimeout);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

template <typename... Exp, typename... Act>
cudaError_t launch_pdl(void (*kernel)(Exp...), dim3 grid, int threads, int smem, cudaStream_t st, Act &&...args) {
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
    }
    cudaLaunchAttribute pdl;
    pdl.id = cudaLaunchAttributeProgrammaticStreamSerialization;
    pdl.val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(threads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cfg.attrs = &pdl;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<Act &&>(args)...);
}

struct PrefillWs {
    float2 *cs;
    __nv_bfloat16 *kh, *vh, *kr;
};

size_t prefill_layout(int n_h, int T_pad, char *base, PrefillWs *w) {
    size_t off = 0;
    auto take = [&](size_t bytes) {
        char *p = base ? base + off : nullptr;
        off += align_up(bytes, 256);
        return p;
    };
    float2 *cs = reinterpret_cast<float2 *>(take((size_t)T_pad * (PDR / 2) * sizeof(float2)));
    __nv_bfloat16 *kh = reinterpret_cast<__nv_bfloat16 *>(take((size_t)n_h * T_pad * PDH * 2));
    __nv_bfloat16 *vh = reinterpret_cast<__nv_bfloat16 *>(take((size_t)n_h * T_pad * PDH * 2));
    __nv_bfloat16 *kr = reinterpret_cast<__nv_bfloat16 *>(take((size_t)T_pad * PDR * 2));
    if (w) *w = PrefillWs{cs, kh, vh, kr};
    return off;
}

}  // namespace

bool prefill_supported(const mla_dims_t &d) {
    return d.d_h == PDH && d.d_c == PDC && d.d_r == PDR && d.n_h % 2 == 0 && d.act_dtype == MLA_DTYPE_BF16;
}

size_t prefill_workspace_bytes(const mla_dims_t &d, int T) {
    const int T_pad = (T + PT - 1) / PT * PT;
    return prefill_layout(d.n_h, T_pad, nullptr, nullptr);
}

cudaError_t launch_prefill(const mla_dims_t &d, int B, const int32_t *cu_seqlens, int T, int max_seq_len,
                           const void *q_c, const void *q_r, const void *c_kv, const void *k_r, const void *w_uk,
                           const void *w_uv, void *ws, size_t ws_bytes, void *o, float *lse, cudaStream_t st) {
    const int T_pad = (T + PT - 1) / PT * PT;
    PrefillWs w;
    if (prefill_layout(d.n_h, T_pad, reinterpret_cast<char *>(ws), &w) > ws_bytes) return cudaErrorInvalidValue;
    const uint64_t hrows = (uint64_t)d.n_h * T_pad;
    CUtensorMap tm_c, tm_wk, tm_wv, tm_kh, tm_vh, tm_qc, tm_k, tm_kr, tm_v;
    const bool maps = tmap_bf16_colblocks(&tm_c, c_kv, (uint64_t)T, PDC, PDC * 2, PT, 1) &&
                      tmap_bf16_colblocks(&tm_wk, w_uk, (uint64_t)d.n_h * PDH, PDC, PDC * 2, 256, 1) &&
                      tmap_bf16_colblocks(&tm_wv, w_uv, (uint64_t)d.n_h * PDH, PDC, PDC * 2, 256, 1) &&
                      tmap_bf16_colblocks(&tm_kh, w.kh, hrows, PDH, PDH * 2, PT, 2) &&
                      tmap_bf16_colblocks(&tm_vh, w.vh, hrows, PDH, PDH * 2, PT, 2) &&
                      tmap_bf16_head_colblocks(&tm_qc, q_c, (uint64_t)T, (uint64_t)d.n_h, PDH, PT, 2) &&
                      tmap_bf16_colblocks(&tm_k, w.kh, hrows, PDH, PDH * 2, PT, 2) &&
                      tmap_bf16_colblocks(&tm_kr, w.kr, (uint64_t)T_pad, PDR, PDR * 2, PT, 1) &&
                      tmap_bf16_colblocks(&tm_v, w.vh, hrows, PDH, PDH * 2, PT, 2);
    if (!maps) return cudaErrorInvalidValue;
    unsigned *err = device_error_word();
    cudaError_t e = launch_pdl(prefill_prep_kernel, dim3(T_pad / PREP_TOKENS), 32 * PREP_TOKENS, 0, st, B, cu_seqlens,
                               T, max_seq_len, make_rope_freqs((double)d.rope_base, d.d_r),
                               reinterpret_cast<const __nv_bfloat16 *>(k_r), w.cs, w.kr, err);
    if (e != cudaSuccess) return e;
    cudaFuncSetAttribute(prefill_kv_up_kernel, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    e = launch_pdl(prefill_kv_up_kernel, dim3(d.n_h / 2, T_pad / PT, 2), 128, UP_SMEM, st, tm_c, tm_wk, tm_wv, tm_kh,
                   tm_vh, T_pad, err);
    if (e != cudaSuccess) return e;
    const int q_tiles = (max_seq_len + PT - 1) / PT;
    const float scale_log2 = (float)(1.4426950408889634 / sqrt((double)(d.d_h + d.d_r)));
    return launch_pdl(prefill_attn_kernel, dim3(q_tiles, d.n_h, B), AT_THREADS, AT_SMEM, st, tm_qc, tm_k, tm_kr,
                      tm_v, B, reinterpret_cast<const __nv_bfloat16 *>(q_r), static_cast<const float2 *>(w.cs), cu_seqlens, T, T_pad, d.n_h, q_tiles, scale_log2, reinterpret_cast<__nv_bfloat16 *>(o), lse,
                      err);
}

}  // namespace mla
