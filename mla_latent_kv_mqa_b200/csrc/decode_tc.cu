// Tensor-core (tcgen05 / TMEM / TMA) absorbed-MLA decode for the DeepSeek-V3 shape
// (n_h = 128, d_c = 512, d_R = 64, 64-token pages, bf16 cache).
//
// What it computes -- MLA article (itwiki "멀티 헤드 잠재 어텐션"), section 분리 RoPE output
// equation in the absorbed form of section 행렬 흡수: for query row t and head h,
//     s_j   = q_abs[t,h,:] . [c_j ; kR_j] / sqrt(d_h + d_R)     (576-wide dot product)
//     o_lat = sum_j softmax(s)_j c_j                             (all heads share c_j)
// The 128 heads are the M dimension of two dense contractions per 64-token page:
//     S[128 x 64]  = Q[128 x 576] . KV[64 x 576]^T      (QK, K = 576)
//     O[128 x 512] += P[128 x 64] . V[64 x 512]         (PV, V = the c_j part of KV)
//
// Decomposition.  O in fp32 is 128 lanes x 512 columns: all of one SM's tensor memory.  A
// 2-CTA cluster therefore splits the two contractions between two SMs instead of splitting
// either one:
//   CTA 0 ("QK"): Q (576 bf16 per head) lives in TMEM columns [0,288); three S buffers of 64
//     columns follow.  A TMA warp streams each page's 576-wide rows (9 column blocks of 64,
//     128-byte swizzle) into a 3-stage ring; one thread issues 36 tcgen05.mma (M=128, N=64,
//     K=16, A from TMEM); 4 softmax warps (one head per thread) run the online softmax in fp32
//     and ship bf16 P (16 KB) plus per-head rescale factors to CTA 1 with st.async.
//   CTA 1 ("PV"): O lives in all 512 TMEM columns.  A TMA warp streams the same page's 512
//     content columns (mostly L2 hits) into a 2-stage ring; one thread issues 8 tcgen05.mma
//     (M=128, N=256, K=16, A = P, B = V read MN-major); 4 warps zero the rows of ragged last
//     pages, apply the (rare) lazy rescale of O rows, release P slots and write each segment's
//     partial O.
// QK : PV work is 576 : 512, so the two tensor pipes are nearly balanced and no FLOP or byte
// is done twice (the second read of a page is an L2 hit).
//
// Split-KV.  A tiny scheduler kernel spreads all (query row, page) units evenly over the
// clusters; a cluster's contiguous range may cover parts of several query rows, each part a
// segment whose (O, m, l) partial is merged exactly by the log-sum-exp combine kernel.
//
// Lazy rescaling (log2 units): a row's running max only moves when a page's max exceeds it by
// more than 8, so P stays <= 256 and O rows are rescaled only on those (rare) pages.
//
// Every mbarrier wait is bounded (2 s); on give-up a CTA raises an abort flag in itself and its
// peer, records MLA_ERR_DEVICE_TIMEOUT and leaves through the normal teardown.
#include <cudaTypedefs.h>
#include <math.h>

#include "mla_internal.cuh"
#include "sm100.cuh"
#include "tmap.cuh"

namespace mla {
namespace {

using namespace sm100;

constexpr int NH = 128, DC = 512, ROW = 576, PG = 64;
constexpr int CB = PG * 128;                // one 64-row x 64-column bf16 box, 128-byte swizzle
constexpr int NCB = ROW / 64;               // 9 column blocks per cache row
// ---- QK CTA shared memory ----
// A page (64 tokens x 576) is one TMA operation (a 3-D box {64, 64, 9} over the cache viewed as
// column blocks), so one issuing thread streams whole pages: TMA operations of one thread are
// served one after another, and 8 KB operations would cap a thread at ~24 GB/s.
constexpr int KV_STAGES = 2;
constexpr int KV_STAGE = NCB * CB;          // 73728
constexpr int QC_BYTES = 8 * CB;            // Q content of 64 heads (8 column blocks): 65536
constexpr int QROPE_OFF = KV_STAGES * KV_STAGE;  // 147456: Q RoPE part, [128 heads x 64] bf16
constexpr int STAGE_OFF = QROPE_OFF + 2 * CB;
constexpr int P_TILE = NH * PG * 2;         // 16384: P[128 heads][64 tokens] bf16, SW128 K-major
constexpr int P_FACT = P_TILE;              // 128 fp32 rescale factors
constexpr int P_FLAG = P_TILE + NH * 4;     // one u32: any factor != 1
constexpr int P_SLOT = 17408;               // message slot, padded to 1 KB
constexpr uint32_t MSG_BYTES = P_TILE + NH * 4 + 16;  // bulk-copy size (multiple of 16)
constexpr int STAGE_SLOTS = 2;              // local P staging slots
constexpr int DATA_A = STAGE_OFF + STAGE_SLOTS * P_SLOT;
// ---- PV CTA shared memory ----
constexpr int V_STAGES = 2;
constexpr int V_STAGE = (DC / 64) * CB;     // 65536: the content columns of one page
constexpr int V_OFF = 0;
constexpr int P_OFF = V_STAGES * V_STAGE;
constexpr int P_SLOTS = 3;                  // P receive slots
constexpr int EPI_OFF = P_OFF + P_SLOTS * P_SLOT;  // 2 x 16 KB staging of O chunks for TMA stores
constexpr int EPI_CHUNK = NH * 128;         // [128 heads x 32 fp32] with 128-byte swizzle
constexpr int DATA_B = EPI_OFF + 2 * EPI_CHUNK;
constexpr int DATA = DATA_A > DATA_B ? DATA_A : DATA_B;
static_assert(P_SLOT % 1024 == 0 && P_OFF % 1024 == 0 && STAGE_OFF % 1024 == 0 &&
              QROPE_OFF % 1024 == 0 && EPI_OFF % 1024 == 0, "swizzled tiles need 1 KB alignment");
static_assert(MSG_BYTES <= (uint32_t)P_SLOT, "message slot");
// ---- QK CTA tensor memory: Q content, then 2 sets x 2 partial S accumulators ----
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t Q_COL = 0, S_COL = DC / 2;  // 256
constexpr int S_SETS = 2;
static_assert(S_COL + S_SETS * 2 * PG <= TMEM_COLS, "QK-CTA TMEM budget");
// The 36 k-steps of QK are split between two issuing warps (one issuer cannot keep the
// tensor pipe busy at N = 64): warp 1 takes column blocks 0..4, warp 2 blocks 5..8 (block 8
// is the RoPE part, with A read from shared memory).
constexpr int SPLIT_CB = 5;
constexpr int THREADS = 256;                // 8 warps
// Each stage is filled by two producer warps (warp 0: column blocks 0..4, warp 7: 5..8; PV CTA:
// 0..3 and 4..7), i.e. two TMA streams that the copy engine serves in parallel.
constexpr int PROD2_WARP = 7;
constexpr int SPLIT_LOAD = 5;
constexpr int SM_THREAD0 = 96;              // first softmax thread (warps 3..6)
constexpr float RESCALE_LOG2 = 8.0f;

struct __align__(8) Ctrl {
    uint64_t kv_full[KV_STAGES], kv_empty[KV_STAGES];
    uint64_t s_full[S_SETS], s_free[S_SETS];
    uint64_t q_ready, rope_full, rope_free;
    uint64_t pfree[P_SLOTS];
    uint64_t v_full[V_STAGES], v_empty[V_STAGES], v_ready[V_STAGES];
    uint64_t p_full[P_SLOTS], pv_done[P_SLOTS];
    uint64_t corr_done, o_free;
    uint32_t tmem_base;
    uint32_t abort;
};
constexpr int SMEM_BYTES = 1024 + DATA + (int)((sizeof(Ctrl) + 127) / 128 * 128);

struct Params {
    const int32_t *bt;
    int max_blocks, num_blocks;
    const int32_t *seq_lens;
    int s_q, rows, max_seq_len;
    const int32_t *work;  // [pairs][4]: first row, first page, number of pages
    float *o_part, *m_part, *l_part;
    float scale_log2;
    unsigned *err;
};

__device__ __forceinline__ int row_tokens(const Params &P, int r) {
    if (r < 0 || r >= P.rows) return 0;
    const int b = r / P.s_q, i = r - b * P.s_q;
    const int L = P.seq_lens[b];
    if (L < P.s_q || L > P.max_seq_len || L > P.max_blocks * PG) return 0;
    return L - P.s_q + i + 1;
}

// Walks one cluster's pages in order; every role of both CTAs walks the same sequence.
struct PageIt {
    int r, pg, left, nv, np;
    bool first;
    __device__ void init(const Params &P, int pair) {
        r = P.work[4 * pair];
        pg = P.work[4 * pair + 1];
        left = P.work[4 * pair + 2];
        nv = row_tokens(P, r);
        np = (nv + PG - 1) / PG;
        if (np == 0 || pg >= np) left = 0;
        first = true;
    }
    __device__ bool done() const { return left <= 0; }
    __device__ int valid() const { return min(PG, nv - pg * PG); }
    __device__ bool last() const { return left == 1 || pg == np - 1; }
    __device__ void next(const Params &P) {
        const bool was_last = last();
        --left;
        ++pg;
        if (pg >= np) {
            pg = 0;
            do {
                ++r;
                nv = row_tokens(P, r);
                np = (nv + PG - 1) / PG;
            } while (left > 0 && np == 0 && r < P.rows);
            if (r >= P.rows) left = 0;
        }
        first = was_last;
    }
};

// Position in a ring of n buffers: index and phase parity.
struct Ring {
    int i;
    uint32_t ph;
    __device__ void adv(int n, int by = 1) {
        i += by;
        while (i >= n) { i -= n; ph ^= 1u; }
    }
};

__device__ __forceinline__ int block_of(const Params &P, int r, int pg) {
    const int b = r / P.s_q;
    int blk = P.bt[(size_t)b * P.max_blocks + pg];
    if (blk < 0 || blk >= P.num_blocks) {
        record_error(P.err, kErrBadBlock);
        blk = 0;  // keep the copy in bounds; the result is flagged as invalid
    }
    return blk;
}

__device__ __forceinline__ uint4 ld_shared_v4(uint32_t a) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(a));
    return v;
}
__device__ __forceinline__ uint32_t ld_shared_u32(uint32_t a) {
    uint32_t v;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(a));
    return v;
}
__device__ __forceinline__ void st_shared_v4(uint32_t a, uint32_t x, uint32_t y, uint32_t z, uint32_t w) {
    asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(x), "r"(y), "r"(z), "r"(w)
                 : "memory");
}
__device__ __forceinline__ void st_shared_u32(uint32_t a, uint32_t x) {
    asm volatile("st.shared.u32 [%0], %1;" ::"r"(a), "r"(x) : "memory");
}
__device__ __forceinline__ void named_sync(int id, int n) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}
__device__ __forceinline__ bool named_red_or(bool v, int id, int n) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\t"
        "barrier.cta.red.or.pred q, %2, %3, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)v), "r"(id), "r"(n)
        : "memory");
    return r != 0;
}
__device__ __forceinline__ bool named_red_and(bool v, int id, int n) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\t"
        "barrier.cta.red.and.pred q, %2, %3, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)v), "r"(id), "r"(n)
        : "memory");
    return r != 0;
}
// 2^x on the SFU (ex2.approx, flush-to-zero): P only needs bf16 precision.
__device__ __forceinline__ float fast_exp2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
// Bulk copy of `bytes` from this CTA's shared memory to another CTA's (TMA engine), completing
// `bytes` on the destination's mbarrier.
__device__ __forceinline__ void bulk_copy_to_peer(uint32_t dst_remote, uint32_t src_local, uint32_t bytes,
                                                  uint32_t bar_remote) {
    asm volatile(
        "cp.async.bulk.shared::cluster.shared::cta.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            dst_remote),
        "r"(src_local), "r"(bytes), "r"(bar_remote)
        : "memory");
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait_read_le1() {
    asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

#ifdef MLA_TRACE
// Development instrumentation: globaltimer stamps of pipeline events of one cluster.  Each warp
// of each CTA writes its own 4096-entry region (no atomics on the traced path).
constexpr int kTraceMax = 1 << 16;
constexpr int kTraceRegion = 4096;
__device__ uint32_t g_trace[2 * kTraceMax];
__device__ uint32_t g_trace_n;
__device__ __forceinline__ void trace_event(int pair, uint32_t code, uint32_t unit, uint32_t &n) {
    if (pair != MLA_TRACE) return;
    const uint32_t region = cluster_ctarank() * 8 + (threadIdx.x >> 5);
    if (n < kTraceRegion) {
        const uint32_t i = region * kTraceRegion + n++;
        g_trace[2 * i] = code | (unit << 8);
        g_trace[2 * i + 1] = (uint32_t)globaltimer();
    }
}
#define TRACE(code, unit) trace_event(pair, (code), (uint32_t)(unit), tr_n)
#else
#define TRACE(code, unit) ((void)0)
#endif

// Named barriers of the 4 softmax warps (QK CTA) and of the 4 epilogue warps (PV CTA).
constexpr int BAR_Q = 1, BAR_FLAG = 2, BAR_OK = 3, BAR_EPI = 4;

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(THREADS, 1)
decode_tc_kernel(const __grid_constant__ CUtensorMap tm_kv5, const __grid_constant__ CUtensorMap tm_kv4,
                 const __grid_constant__ CUtensorMap tm_q4, const __grid_constant__ CUtensorMap tm_qr,
                 const __grid_constant__ CUtensorMap tm_o, const Params P) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_s = smem_u32(smem_raw);
    const uint32_t data_s = (raw_s + 1023u) & ~1023u;
    Ctrl *ctrl = reinterpret_cast<Ctrl *>(smem_raw + (data_s - raw_s) + DATA);
    volatile uint32_t *abort_flag = &ctrl->abort;
    auto bar = [&](uint64_t &b) { return smem_u32(&b); };

    const uint32_t rank = cluster_ctarank();
    const int pair = blockIdx.x >> 1;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
#ifdef MLA_TRACE
    uint32_t tr_n = 0;
#endif

    if (threadIdx.x == 0) {
        for (int i = 0; i < KV_STAGES; ++i) {
            mbar_init(bar(ctrl->kv_full[i]), 2);    // two producer warps
            mbar_init(bar(ctrl->kv_empty[i]), 2);  // both QK issuers (or the Q copy) release a stage
        }
        for (int i = 0; i < S_SETS; ++i) {
            mbar_init(bar(ctrl->s_full[i]), 2);
            mbar_init(bar(ctrl->s_free[i]), 4);
        }
        mbar_init(bar(ctrl->q_ready), 1);
        mbar_init(bar(ctrl->rope_full), 1);
        mbar_init(bar(ctrl->rope_free), 1);
        for (int i = 0; i < P_SLOTS; ++i) {
            mbar_init(bar(ctrl->pfree[i]), 1);
            mbar_init(bar(ctrl->p_full[i]), 1);
            mbar_init(bar(ctrl->pv_done[i]), 1);
        }
        for (int i = 0; i < V_STAGES; ++i) {
            mbar_init(bar(ctrl->v_full[i]), 2);     // two producer warps
            mbar_init(bar(ctrl->v_empty[i]), 1);
            mbar_init(bar(ctrl->v_ready[i]), 4);
        }
        mbar_init(bar(ctrl->corr_done), 4);
        mbar_init(bar(ctrl->o_free), 4);
        ctrl->abort = 0;
        if (rank == 1)
            for (int i = 0; i < P_SLOTS; ++i) mbar_arrive_expect_tx(bar(ctrl->p_full[i]), MSG_BYTES);
        fence_mbarrier_init_cluster();
    }
    if (warp == 0) {
        tmem_alloc(smem_u32(&ctrl->tmem_base), TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    cluster_sync();
    const uint32_t tmem = ctrl->tmem_base;
    const uint32_t peer = rank ^ 1u;
    if (threadIdx.x == 0) TRACE(20 + rank, (uint32_t)clock64() >> 8);
    auto fail = [&]() {
        if (*abort_flag == 0) {
            *abort_flag = 1;
            st_shared_cluster_u32(mapa(smem_u32(&ctrl->abort), peer), 1u);
            record_error(P.err, kErrTimeout);
        }
    };

    if (rank == 0) {
        // ===================================== QK CTA =====================================
        if ((warp == 0 || warp == PROD2_WARP) && lane == 0) {  // TMA producers (two streams)
            const int half = warp == 0 ? 0 : 1;
            prefetch_tensormap(half ? &tm_kv4 : &tm_kv5);
            prefetch_tensormap(&tm_q4);
            if (!half) prefetch_tensormap(&tm_qr);
            PageIt it;
            it.init(P, pair);
            Ring st{0, 0};
            uint32_t nseg = 0;
            int u = 0;
            bool ok = true;
            while (ok && !it.done()) {
                if (it.first) {
                    if (!half) {
                        if (!(ok = wait(bar(ctrl->rope_free), (nseg & 1u) ^ 1u, abort_flag))) break;
                        mbar_arrive_expect_tx(bar(ctrl->rope_full), 2 * CB);
                        tma_load_2d(data_s + QROPE_OFF, &tm_qr, DC, it.r * NH, bar(ctrl->rope_full));
                    }
                    // Q content: stage s <- heads 0-63, stage s+1 <- heads 64-127; this stream
                    // loads column blocks 4*half .. 4*half+3 of each
                    for (int hh = 0; hh < 2 && ok; ++hh) {
                        if (!(ok = wait(bar(ctrl->kv_empty[st.i]), st.ph ^ 1u, abort_flag))) break;
                        mbar_arrive_expect_tx(bar(ctrl->kv_full[st.i]), QC_BYTES / 2);
                        tma_load_3d(data_s + st.i * KV_STAGE + half * 4 * CB, &tm_q4, 0, it.r * NH + hh * 64,
                                    half * 4, bar(ctrl->kv_full[st.i]));
                        st.adv(KV_STAGES);
                    }
                    if (!ok) break;
                    ++nseg;
                    if (!half) TRACE(1, u);
                }
                if (!(ok = wait(bar(ctrl->kv_empty[st.i]), st.ph ^ 1u, abort_flag))) break;
                const int blk = block_of(P, it.r, it.pg);
                const int cbs = half ? NCB - SPLIT_LOAD : SPLIT_LOAD;
                mbar_arrive_expect_tx(bar(ctrl->kv_full[st.i]), cbs * CB);
                tma_load_3d(data_s + st.i * KV_STAGE + half * SPLIT_LOAD * CB, half ? &tm_kv4 : &tm_kv5, 0,
                            blk * PG, half * SPLIT_LOAD, bar(ctrl->kv_full[st.i]));
                st.adv(KV_STAGES);
                if (!half) TRACE(2, u);
                ++u;
                it.next(P);
            }
            if (!ok) fail();
        } else if ((warp == 1 || warp == 2) && lane == 0) {  // MMA issuers: partial S = Q . KV^T
            constexpr uint32_t idesc = idesc_bf16(128, PG, false, false);
            const int part = warp - 1;                  // 0: blocks 0..4, 1: blocks 5..8
            const int cb0 = part ? SPLIT_CB : 0, cb1 = part ? NCB : SPLIT_CB;
            PageIt it;
            it.init(P, pair);
            Ring st{0, 0}, sb{0, 0};
            uint32_t qn = 0;
            int u = 0;
            bool ok = true;
            while (ok && !it.done()) {
                if (it.first) {
                    st.adv(KV_STAGES, 2);  // the segment's Q stages (copied to TMEM by the softmax warps)
                    if (!(ok = wait(bar(ctrl->q_ready), qn & 1u, abort_flag))) break;
                    if (part && !(ok = wait(bar(ctrl->rope_full), qn & 1u, abort_flag))) break;
                    ++qn;
                }
                if (!(ok = wait(bar(ctrl->s_free[sb.i]), sb.ph ^ 1u, abort_flag))) break;
                tc_fence_after();  // orders our S writes after the softmax's TMEM reads
                // TMA-filled shared memory needs no tcgen05 fence: the mbarrier completion already
                // makes it visible to the MMAs issued after the wait.
                if (!(ok = wait(bar(ctrl->kv_full[st.i]), st.ph, abort_flag))) break;
                const uint32_t d = tmem + S_COL + sb.i * 2 * PG + part * PG;
                const uint32_t kvb = data_s + st.i * KV_STAGE;
                for (int cb = cb0; cb < cb1; ++cb) {
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const uint64_t b = sdesc_sw128(kvb + cb * CB + k * 32, 16, 1024);
                        const uint32_t acc = (cb == cb0 && k == 0) ? 0u : 1u;
                        if (cb < NCB - 1)
                            mma_ts(d, tmem + Q_COL + (cb * 4 + k) * 8, b, idesc, acc);
                        else
                            mma_ss(d, sdesc_sw128(data_s + QROPE_OFF + k * 32, 16, 1024), b, idesc, acc);
                    }
                }
                mma_commit(bar(ctrl->kv_empty[st.i]));
                mma_commit(bar(ctrl->s_full[sb.i]));
                if (part && it.last()) mma_commit(bar(ctrl->rope_free));
                TRACE(3 + part, u);
                ++u;
                st.adv(KV_STAGES);
                sb.adv(S_SETS);
                it.next(P);
            }
            if (!ok) fail();
        } else if (warp >= 3 && warp <= 6) {  // softmax warps: thread = head
            const int t = threadIdx.x - SM_THREAD0;
            const int sub = warp & 3;
            const int h = sub * 32 + lane;
            const uint32_t lane_base = (uint32_t)(sub * 32) << 16;
            uint32_t p_slot_r[P_SLOTS], p_full_r[P_SLOTS];
            for (int i = 0; i < P_SLOTS; ++i) {
                p_slot_r[i] = mapa(data_s + P_OFF + i * P_SLOT, 1);
                p_full_r[i] = mapa(bar(ctrl->p_full[i]), 1);
            }
            PageIt it;
            it.init(P, pair);
            Ring st{0, 0}, sb{0, 0}, ps{0, 0}, sg{0, 0};  // sg: local P staging slot
            float m_used = -INFINITY, l = 0.f;
            int u = 0;
            bool ok = true, pfail = false;  // pfail: thread 0 gave up waiting for a P slot

            // Q content of a segment (2 stages: heads 0-63, 64-127) -> this thread's TMEM lane.
            auto load_q = [&]() -> bool {
                const Ring q0 = st;
                st.adv(KV_STAGES);
                const Ring q1 = st;
                st.adv(KV_STAGES);
                bool w = wait(bar(ctrl->kv_full[q0.i]), q0.ph, abort_flag) &&
                         wait(bar(ctrl->kv_full[q1.i]), q1.ph, abort_flag);
                if (!named_red_and(w, BAR_OK, 128)) return false;
                const int rr = h & 63;
                const uint32_t rowa = data_s + ((h >> 6) ? q1.i : q0.i) * KV_STAGE + rr * 128;
#pragma unroll 1
                for (int cb = 0; cb < 8; ++cb) {
                    uint32_t v[32];
#pragma unroll
                    for (int c = 0; c < 8; ++c) {
                        const uint4 x = ld_shared_v4(rowa + cb * CB + ((c ^ (rr & 7)) << 4));
                        v[4 * c + 0] = x.x;
                        v[4 * c + 1] = x.y;
                        v[4 * c + 2] = x.z;
                        v[4 * c + 3] = x.w;
                    }
                    tmem_st32(tmem + lane_base + Q_COL + cb * 32, v);
                }
                tmem_wait_st();
                tc_fence_before();
                named_sync(BAR_Q, 128);
                if (t == 0) {
                    for (int k = 0; k < 2; ++k) {
                        mbar_arrive(bar(ctrl->kv_empty[q0.i]));
                        mbar_arrive(bar(ctrl->kv_empty[q1.i]));
                    }
                    mbar_arrive(bar(ctrl->q_ready));
                }
                return true;
            };

            if (!it.done()) ok = load_q();
            while (ok && !it.done()) {
                if (t == 0) bulk_wait_read_le1();  // staging slot sg was read by its copy
                bool w = !pfail && wait(bar(ctrl->s_full[sb.i]), sb.ph, abort_flag);
                if (!(ok = named_red_and(w, BAR_OK, 128))) break;
                if (t == 0) TRACE(5, u);
                tc_fence_after();
                float x[64];
                {
                    uint32_t a0[32], a1[32], b0[32], b1[32];
                    const uint32_t sa = tmem + lane_base + S_COL + sb.i * 2 * PG;
                    tmem_ld32(sa, a0);
                    tmem_ld32(sa + 32, a1);
                    tmem_ld32(sa + PG, b0);
                    tmem_ld32(sa + PG + 32, b1);
                    tmem_wait_ld();
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        x[j] = __uint_as_float(a0[j]) + __uint_as_float(b0[j]);
                        x[32 + j] = __uint_as_float(a1[j]) + __uint_as_float(b1[j]);
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(ctrl->s_free[sb.i]));
                if (t == 0) TRACE(24, u);
                sb.adv(S_SETS);
                st.adv(KV_STAGES);  // this page's stage

                const bool first = it.first, last = it.last();
                const int valid = it.valid();
                const int r = it.r;
                // The last page's S is complete, so every QK of this segment has finished and
                // the next segment's Q may overwrite TMEM now.
                if (last && it.left > 1) {
                    if (!(ok = load_q())) break;
                }

                // ---- online softmax (log2 units; scale folded into one FFMA) ----
                float mraw = -INFINITY;
                if (valid < PG) {
#pragma unroll
                    for (int j = 0; j < 64; ++j)
                        if (j >= valid) x[j] = -INFINITY;
                }
#pragma unroll
                for (int j = 0; j < 64; ++j) mraw = fmaxf(mraw, x[j]);
                const float mx = mraw * P.scale_log2;
                float m_new = m_used, fac = 1.f;
                bool need = false;
                if (first) {
                    m_new = mx;
                    l = 0.f;
                } else if (mx > m_used + RESCALE_LOG2) {
                    m_new = mx;
                    fac = fast_exp2(m_used - m_new);
                    need = true;
                }
                float sum = 0.f;
                uint32_t pk[32];
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    const float p0 = fast_exp2(fmaf(x[2 * j], P.scale_log2, -m_new));
                    const float p1 = fast_exp2(fmaf(x[2 * j + 1], P.scale_log2, -m_new));
                    sum += p0 + p1;
                    pk[j] = pack_bf16x2(p0, p1);
                }
                l = l * fac + sum;
                m_used = m_new;
                if (t == 0) TRACE(25, u);

                // ---- stage P, factors and flag locally; one bulk copy to the PV CTA ----
                const uint32_t sbase = data_s + STAGE_OFF + sg.i * P_SLOT;
                const uint32_t rowa = sbase + h * 128;
#pragma unroll
                for (int c = 0; c < 8; ++c)
                    st_shared_v4(rowa + ((c ^ (h & 7)) << 4), pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
                st_shared_u32(sbase + P_FACT + h * 4, __float_as_uint(need ? fac : 1.f));
                fence_proxy_async_smem();
                const bool any = named_red_or(need, BAR_FLAG, 128);
                if (t == 0) {
                    st_shared_u32(sbase + P_FLAG, any ? 1u : 0u);
                    fence_proxy_async_smem();
                    TRACE(9, u);
                    if (!wait<true>(bar(ctrl->pfree[ps.i]), ps.ph ^ 1u, abort_flag)) {
                        pfail = true;  // joins the next page's barrier vote, so all threads leave
                    } else {
                        bulk_copy_to_peer(p_slot_r[ps.i], sbase, MSG_BYTES, p_full_r[ps.i]);
                        TRACE(8, u);
                    }
                }
                ps.adv(P_SLOTS);
                sg.adv(STAGE_SLOTS);
                ++u;

                if (last) {
                    const size_t slot = (size_t)pair + r;
                    P.m_part[slot * NH + h] = m_used;
                    P.l_part[slot * NH + h] = l;
                    m_used = -INFINITY;
                    l = 0.f;
                }
                it.next(P);
            }
            if (t == 0) bulk_wait_all();
            if (!ok || pfail) fail();
        }
    } else {
        // ===================================== PV CTA =====================================
        if ((warp == 0 || warp == PROD2_WARP) && lane == 0) {  // TMA producers: content columns
            const int half = warp == 0 ? 0 : 1;                    // column blocks 4*half .. +3
            prefetch_tensormap(&tm_kv4);
            PageIt it;
            it.init(P, pair);
            Ring vs{0, 0};
            int u = 0;
            bool ok = true;
            while (!it.done()) {
                if (!(ok = wait(bar(ctrl->v_empty[vs.i]), vs.ph ^ 1u, abort_flag))) break;
                const int blk = block_of(P, it.r, it.pg);
                mbar_arrive_expect_tx(bar(ctrl->v_full[vs.i]), V_STAGE / 2);
                tma_load_3d(data_s + V_OFF + vs.i * V_STAGE + half * 4 * CB, &tm_kv4, 0, blk * PG, half * 4,
                            bar(ctrl->v_full[vs.i]));
                if (!half) TRACE(11, u);
                ++u;
                vs.adv(V_STAGES);
                it.next(P);
            }
            if (!ok) fail();
        } else if (warp == 1 && lane == 0) {  // MMA issuer: O += P . V
            constexpr uint32_t idesc = idesc_bf16(128, 256, false, true);
            PageIt it;
            it.init(P, pair);
            Ring vs{0, 0}, ps{0, 0};
            uint32_t ncorr = 0, nseg = 0;
            int u = 0;
            bool ok = true;
            while (!it.done()) {
                if (!(ok = wait(bar(ctrl->v_ready[vs.i]), vs.ph, abort_flag))) break;
                TRACE(12, u);
                if (!(ok = wait<true>(bar(ctrl->p_full[ps.i]), ps.ph, abort_flag))) break;
                TRACE(13, u);
                const uint32_t pa = data_s + P_OFF + ps.i * P_SLOT;
                const uint32_t flag = ld_shared_u32(pa + P_FLAG);
                mbar_arrive_expect_tx(bar(ctrl->p_full[ps.i]), MSG_BYTES);  // arm the slot's next use
                if (flag) {
                    if (!(ok = wait(bar(ctrl->corr_done), ncorr & 1u, abort_flag))) break;
                    ++ncorr;
                }
                const bool first = it.first;
                if (first && nseg > 0) {
                    if (!(ok = wait(bar(ctrl->o_free), (nseg - 1) & 1u, abort_flag))) break;
                }
                tc_fence_after();
                const uint32_t vb = data_s + V_OFF + vs.i * V_STAGE;
#pragma unroll
                for (int kk = 0; kk < PG / 16; ++kk)
#pragma unroll
                    for (int nh = 0; nh < 2; ++nh) {
                        const uint64_t a = sdesc_sw128(pa + kk * 32, 16, 1024);
                        const uint64_t b = sdesc_sw128(vb + nh * 4 * CB + kk * 2048, CB, 1024);
                        mma_ss(tmem + nh * 256, a, b, idesc, (first && kk == 0) ? 0u : 1u);
                    }
                mma_commit(bar(ctrl->v_empty[vs.i]));
                mma_commit(bar(ctrl->pv_done[ps.i]));
                TRACE(14, u);
                ++u;
                if (it.last()) ++nseg;
                vs.adv(V_STAGES);
                ps.adv(P_SLOTS);
                it.next(P);
            }
            if (!ok) fail();
        } else if (warp >= 2 && warp <= 5) {  // ragged-page zeroing, lazy rescale, P release, epilogue
            const int sub = warp & 3;
            const int h = sub * 32 + lane;
            const uint32_t lane_base = (uint32_t)(sub * 32) << 16;
            uint32_t pfree_r[P_SLOTS];
            for (int i = 0; i < P_SLOTS; ++i) pfree_r[i] = mapa(bar(ctrl->pfree[i]), 0);
            PageIt it;
            it.init(P, pair);
            Ring vs{0, 0}, ps{0, 0}, prev{0, 0};
            int u = 0;
            bool ok = true;
            while (!it.done()) {
                // 1. the V stage: zero token rows past the end of a ragged last page
                if (!(ok = __all_sync(0xffffffffu, wait(bar(ctrl->v_full[vs.i]), vs.ph, abort_flag)))) break;
                if (h == 0) TRACE(15, u);
                const int valid = it.valid();
                if (valid < PG) {
                    const int nz = PG - valid;
                    const uint32_t vb = data_s + V_OFF + vs.i * V_STAGE;
                    for (int i = h; i < nz * (DC / 64) * 8; i += 128) {
                        const int c = i & 7, pr = i >> 3;
                        const int cb = pr / nz, row = valid + pr % nz;
                        st_shared_v4(vb + cb * CB + row * 128 + c * 16, 0u, 0u, 0u, 0u);
                    }
                    fence_proxy_async_smem();
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(ctrl->v_ready[vs.i]));
                // 2. the P message of this page
                if (!(ok = __all_sync(0xffffffffu, wait<true>(bar(ctrl->p_full[ps.i]), ps.ph, abort_flag)))) break;
                if (h == 0) TRACE(16, u);
                const uint32_t pa = data_s + P_OFF + ps.i * P_SLOT;
                const float fac = __uint_as_float(ld_shared_u32(pa + P_FACT + h * 4));
                const uint32_t flag = ld_shared_u32(pa + P_FLAG);
                const bool first = it.first, last = it.last();
                // 3. release the previous page's P slot once its PV has completed
                if (!first) {
                    if (!(ok = __all_sync(0xffffffffu, wait(bar(ctrl->pv_done[prev.i]), prev.ph, abort_flag)))) break;
                    if (h == 0) mbar_arrive_remote(pfree_r[prev.i]);
                    if (h == 0) TRACE(17, u);
                }
                // 4. lazy rescale of O rows whose running max moved (PV of the previous page done)
                if (flag) {
                    tc_fence_after();
                    if (__any_sync(0xffffffffu, fac != 1.f)) {
#pragma unroll 1
                        for (int ch = 0; ch < 16; ++ch) {
                            uint32_t v[32];
                            tmem_ld32(tmem + lane_base + ch * 32, v);
                            tmem_wait_ld();
#pragma unroll
                            for (int i = 0; i < 32; ++i) v[i] = __float_as_uint(__uint_as_float(v[i]) * fac);
                            tmem_st32(tmem + lane_base + ch * 32, v);
                        }
                        tmem_wait_st();
                    }
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(bar(ctrl->corr_done));
                }
                // 5. end of segment: write the partial O (not normalised) of this row and head
                if (last) {
                    if (!(ok = __all_sync(0xffffffffu, wait(bar(ctrl->pv_done[ps.i]), ps.ph, abort_flag)))) break;
                    if (h == 0) mbar_arrive_remote(pfree_r[ps.i]);
                    if (h == 0) TRACE(18, u);
                    tc_fence_after();
                    // O rows -> swizzled staging (one 32-column chunk at a time) -> TMA store, so the
                    // global writes are whole 128-byte lines instead of one row per thread.
                    const int orow = (pair + it.r) * NH;
#pragma unroll 1
                    for (int ch = 0; ch < DC / 32; ++ch) {
                        const uint32_t eb = data_s + EPI_OFF + (ch & 1) * EPI_CHUNK;
                        if (h == 0) bulk_wait_group_read_le1();  // this buffer's previous store has read it
                        named_sync(BAR_EPI, 128);
                        uint32_t v[32];
                        tmem_ld32(tmem + lane_base + ch * 32, v);
                        tmem_wait_ld();
#pragma unroll
                        for (int c = 0; c < 8; ++c)
                            st_shared_v4(eb + h * 128 + ((c ^ (h & 7)) << 4), v[4 * c], v[4 * c + 1], v[4 * c + 2],
                                         v[4 * c + 3]);
                        fence_proxy_async_smem();
                        named_sync(BAR_EPI, 128);
                        if (h == 0) tma_store_2d(&tm_o, eb, ch * 32, orow);
                    }
                    if (h == 0) bulk_wait_group_all();
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(bar(ctrl->o_free));
                    if (h == 0) TRACE(19, u);
                }
                ++u;
                prev = ps;
                vs.adv(V_STAGES);
                ps.adv(P_SLOTS);
                it.next(P);
            }
            if (!ok && lane == 0) fail();
        }
    }

    // ---- teardown: both CTAs quiesce before either releases TMEM or exits ----
    __syncwarp();
    if (threadIdx.x == 0) TRACE(22 + rank, (uint32_t)clock64() >> 8);
    tc_fence_before();
    __syncthreads();
    cluster_sync();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}

// ---- scheduler: balanced split of all (query row, page) units over the clusters ----------
__device__ __forceinline__ long long unit_start(int c, long long U, int pairs) {
    return (long long)c * U / pairs;
}

__global__ void __launch_bounds__(1024)
schedule_kernel(int s_q, int rows, const int32_t *__restrict__ seq_lens, int max_seq_len,
                int max_blocks, int pairs, int32_t *prefix, int32_t *work, int32_t *seg_range,
                float *m_part, unsigned *err) {
    __shared__ int warp_tot[32];
    __shared__ int carry_s;
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    if (tid == 0) carry_s = 0;
    __syncthreads();
    for (int base = 0; base < rows; base += 1024) {
        const int r = base + tid;
        int n = 0;
        if (r < rows) {
            const int b = r / s_q, i = r - b * s_q;
            const int L = seq_lens[b];
            if (L < s_q || L > max_seq_len || L > max_blocks * PG) {
                if (i == 0) record_error(err, kErrBadSeqLen);
            } else {
                n = (L - s_q + i + 1 + PG - 1) / PG;
            }
        }
        int x = n;  // inclusive warp scan
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += y;
        }
        if (lane == 31) warp_tot[wid] = x;
        __syncthreads();
        if (wid == 0) {
            int t = warp_tot[lane];
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, t, o);
                if (lane >= o) t += y;
            }
            warp_tot[lane] = t;  // inclusive over warps
        }
        __syncthreads();
        const int incl = x + (wid > 0 ? warp_tot[wid - 1] : 0);
        const int carry = carry_s;
        if (r < rows) prefix[r] = carry + incl - n;
        __syncthreads();
        if (tid == 1023) carry_s = carry + incl;
        __syncthreads();
    }
    if (tid == 0) prefix[rows] = carry_s;
    // Every partial slot starts empty: a row's slot range also spans clusters that got none of
    // its pages (when there are fewer pages than clusters), and the combine must skip those.
    for (size_t i = tid; i < ((size_t)pairs + rows) * NH; i += 1024) m_part[i] = -INFINITY;
    __syncthreads();
    const long long U = carry_s;
    for (int c = tid; c < pairs; c += 1024) {
        const long long s0 = unit_start(c, U, pairs), s1 = unit_start(c + 1, U, pairs);
        int r0 = 0;
        if (s1 > s0) {  // largest r with prefix[r] <= s0
            int lo = 0, hi = rows - 1;
            while (lo < hi) {
                const int mid = (lo + hi + 1) >> 1;
                if (prefix[mid] <= s0) lo = mid; else hi = mid - 1;
            }
            r0 = lo;
        }
        work[4 * c + 0] = r0;
        work[4 * c + 1] = s1 > s0 ? (int)(s0 - prefix[r0]) : 0;
        work[4 * c + 2] = (int)(s1 - s0);
        work[4 * c + 3] = 0;
    }
    for (int r = tid; r < rows; r += 1024) {
        const long long u0 = prefix[r], u1 = prefix[r + 1];
        if (u1 <= u0) {
            seg_range[2 * r] = 0;
            seg_range[2 * r + 1] = 0;
            continue;
        }
        auto pair_of = [&](long long u) {
            int c = (int)(u * pairs / U);
            while (c + 1 < pairs && unit_start(c + 1, U, pairs) <= u) ++c;
            while (c > 0 && unit_start(c, U, pairs) > u) --c;
            return c;
        };
        seg_range[2 * r] = pair_of(u0) + r;
        seg_range[2 * r + 1] = pair_of(u1 - 1) + r + 1;
    }
}

// ---- host side ------------------------------------------------------------------------------
int g_pairs[64] = {};

int tc_pairs() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
    if (g_pairs[dev]) return g_pairs[dev];
    if (cudaFuncSetAttribute(decode_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES) !=
        cudaSuccess)
        return 0;
    int sms = 148;
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * (sms / 2));
    cfg.blockDim = dim3(THREADS);
    cfg.dynamicSmemBytes = SMEM_BYTES;
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeClusterDimension;
    attr.val.clusterDim.x = 2;
    attr.val.clusterDim.y = 1;
    attr.val.clusterDim.z = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, decode_tc_kernel, &cfg) != cudaSuccess || n < 1) {
        cudaGetLastError();
        n = sms / 2;
    }
    g_pairs[dev] = n;
    return n;
}

struct TcWs {
    float *o, *m, *l;
    int32_t *work, *seg_range, *prefix;
};

size_t tc_layout(int pairs, int rows, char *base, TcWs *w) {
    const size_t slots = (size_t)pairs + rows;
    size_t off = 0;
    auto take = [&](size_t bytes) {
        char *p = base ? base + off : nullptr;
        off += align_up(bytes, 256);
        return p;
    };
    char *o = take(slots * NH * DC * sizeof(float));
    char *m = take(slots * NH * sizeof(float));
    char *l = take(slots * NH * sizeof(float));
    char *wk = take((size_t)pairs * 4 * sizeof(int32_t));
    char *sr = take((size_t)rows * 2 * sizeof(int32_t));
    char *pf = take(((size_t)rows + 1) * sizeof(int32_t));
    if (w) {
        w->o = reinterpret_cast<float *>(o);
        w->m = reinterpret_cast<float *>(m);
        w->l = reinterpret_cast<float *>(l);
        w->work = reinterpret_cast<int32_t *>(wk);
        w->seg_range = reinterpret_cast<int32_t *>(sr);
        w->prefix = reinterpret_cast<int32_t *>(pf);
    }
    return off;
}

}  // namespace

#ifdef MLA_TRACE
// Copies the whole trace buffer (kTraceMax entries of {code | unit << 8, time}) and clears it.
extern "C" int mla_trace_dump(uint32_t *host, int max_entries) {
    if (cudaDeviceSynchronize() != cudaSuccess) return -1;
    const int n = max_entries < kTraceMax ? max_entries : kTraceMax;
    cudaMemcpyFromSymbol(host, g_trace, 2 * (size_t)n * sizeof(uint32_t));
    static uint32_t zeros[2 * kTraceMax];
    cudaMemcpyToSymbol(g_trace, zeros, sizeof(zeros));
    return n;
}
#endif

bool tc_supported(const mla_dims_t &d) {
    return d.n_h == NH && d.d_c == DC && d.d_r == ROW - DC && d.page_size == PG &&
           d.act_dtype == MLA_DTYPE_BF16 && d.kv_dtype == MLA_DTYPE_BF16;
}

size_t tc_workspace_bytes(const mla_dims_t &, int B, int s_q, int) {
    const int pairs = tc_pairs();
    if (pairs < 1) return 0;
    return tc_layout(pairs, B * s_q, nullptr, nullptr);
}

cudaError_t launch_decode_tc(const mla_dims_t &d, int B, int s_q, const void *q_abs,
                             const void *kv_pool, const void *, const float *, const int32_t *bt,
                             int max_blocks, int num_blocks, const int32_t *seq_lens, int max_seq_len,
                             void *ws, size_t ws_bytes, float *o_lat, float *lse, cudaStream_t st) {
    const int rows = B * s_q;
    const int pairs = tc_pairs();
    if (pairs < 1) return cudaErrorNotSupported;
    TcWs w;
    if (tc_layout(pairs, rows, reinterpret_cast<char *>(ws), &w) > ws_bytes) return cudaErrorInvalidValue;
    CUtensorMap tm_kv5, tm_kv4, tm_q4, tm_qr, tm_o;
    const uint64_t pool_rows = (uint64_t)num_blocks * PG, q_rows = (uint64_t)rows * NH;
    if (!tmap_bf16_colblocks(&tm_kv5, kv_pool, pool_rows, ROW, ROW * 2, PG, SPLIT_LOAD) ||
        !tmap_bf16_colblocks(&tm_kv4, kv_pool, pool_rows, ROW, ROW * 2, PG, 4) ||
        !tmap_bf16_colblocks(&tm_q4, q_abs, q_rows, ROW, ROW * 2, 64, 4) ||
        !tmap_bf16_2d(&tm_qr, q_abs, ROW, q_rows, ROW * 2, 64, NH) ||
        !tmap_2d(&tm_o, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, w.o, DC, ((uint64_t)pairs + rows) * NH, DC * 4, 32, NH))
        return cudaErrorInvalidValue;
    unsigned *err = device_error_word();
    schedule_kernel<<<1, 1024, 0, st>>>(s_q, rows, seq_lens, max_seq_len, max_blocks, pairs, w.prefix,
                                        w.work, w.seg_range, w.m, err);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    Params P;
    P.bt = bt;
    P.max_blocks = max_blocks;
    P.num_blocks = num_blocks;
    P.seq_lens = seq_lens;
    P.s_q = s_q;
    P.rows = rows;
    P.max_seq_len = max_seq_len;
    P.work = w.work;
    P.o_part = w.o;
    P.m_part = w.m;
    P.l_part = w.l;
    P.scale_log2 = (float)(1.4426950408889634 / sqrt((double)(d.d_h + d.d_r)));
    P.err = err;
    decode_tc_kernel<<<2 * pairs, THREADS, SMEM_BYTES, st>>>(tm_kv5, tm_kv4, tm_q4, tm_qr, tm_o, P);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    Partials part{w.o, w.m, w.l};
    return launch_combine(rows, NH, DC, part, w.seg_range, 0, o_lat, lse, st);
}

}  // namespace mla
