// Tensor-core (tcgen05 / TMEM / TMA) absorbed-MLA decode for the DeepSeek-V3 shape
// (n_h = 128, d_c = 512, d_R = 64, 64-token pages), bf16 or FP8 cache.
//
// What it computes -- MLA article (itwiki "멀티 헤드 잠재 어텐션"), section 분리 RoPE output
// equation in the absorbed form of section 행렬 흡수: for query row t and head h,
//     s_j   = q_abs[t,h,:] . [c_j ; kR_j] / sqrt(d_h + d_R)     (576-wide dot product)
//     o_lat = sum_j softmax(s)_j c_j                             (all heads share c_j)
// The 128 heads are the M dimension of two dense contractions per 64-token page:
//     S[128 x 64]  = Q[128 x 576] . KV[64 x 576]^T      (QK, K = 576)
//     O[128 x 512] += P[128 x 64] . V[64 x 512]         (PV, V = the c_j part of KV)
//
// Decomposition.  O in fp32 is 128 lanes x 512 columns: all of one SM's tensor memory, so a
// 2-CTA cluster splits the two contractions between two SMs:
//   CTA 0 ("QK"): Q (576 bf16 per head, 288 TMEM columns) sits in TMEM next to three 64-column
//     S buffers.  One TMA thread streams whole pages (one 72 KB 3-D box each) into a 3-stage
//     ring; the segment's Q arrives through the same ring.  Two MMA threads split each page's
//     36 tcgen05.mma (M = 128, N = 64, K = 16, A from TMEM) by column blocks (one thread cannot
//     issue N = 64 MMAs as fast as the tensor core runs them).  Eight softmax warps, two per TMEM lane quarter and each
//     owning 32 of a page's 64 columns, run the online softmax in fp32 and put bf16 P into 32
//     spare TMEM columns.  Four sender warps take it from there and store P, per-head rescale
//     factors and a flag into CTA 1's shared memory with st.async.  The distributed-shared-
//     memory link (about 20 GB/s per SM pair) is the slowest step of the page, so the softmax
//     warps hand off and go on to the next page while the senders drain it, and the TMA
//     engine stays free for the page stream.
//   CTA 1 ("PV"): O lives in all 512 TMEM columns.  A TMA thread streams the same page's 512
//     content columns (mostly L2 hits) as two 32 KB halves into a 4-deep ring; one thread
//     issues 8 tcgen05.mma per page (M = 128, N = 256, K = 16, A = P, B = V read MN-major)
//     and, through a multicast commit, hands the P slot back to CTA 0 the moment those MMAs
//     are done.  Four warps zero the rows of ragged last pages, apply the (rare) lazy
//     rescale of O rows, and write each segment's partial O with coalesced stores.
// QK : PV work is 576 : 512, so the two tensor pipes are nearly balanced and no FLOP or byte
// is done twice (the second read of a page is an L2 hit).
//
// FP8 cache (e4m3 content codes, a fp32 scale per token, bf16 RoPE keys; the F8 instantiation):
// each CTA dequantises the pages it needs, bf16(code * scale), into exactly the bf16 page tiles
// the bf16 path loads, so everything after the page ring is shared.  The QK CTA's softmax warps
// convert the next page before each page's softmax (2 page stages + 2 staging slots of raw
// codes); four otherwise idle PV-CTA warps convert its half pages.
//
// Split-KV.  All (query row, page) units are spread evenly over the clusters (each cluster
// works out its own contiguous range in its prologue, see schedule()); a range may cover parts
// of several query rows, each part a segment whose (O, m, l) partial is merged exactly by the
// log-sum-exp combine kernel.
//
// Lazy rescaling (log2 units): a row's running max only moves when a page's max exceeds it by
// more than 8, so P stays <= 256 and O rows are rescaled only on those (rare) pages.
//
// Every wait is bounded (2 s).  On give-up a CTA raises an abort flag in itself and its peer
// and records MLA_ERR_DEVICE_TIMEOUT; before the teardown every thread that started copies or
// MMAs waits (again bounded) for them, so no asynchronous write targets a CTA that has left.
#include <cuda_fp16.h>
#include <cudaTypedefs.h>
#include <float.h>
#include <math.h>

#include <mutex>

#include "mla_internal.cuh"
#include "sm100.cuh"
#include "tmap.cuh"

namespace mla {
namespace {

using namespace sm100;

constexpr int NH = 128, DC = 512, ROW = 576, PG = 64;
constexpr int CB = PG * 128;                // one 64-row x 64-column bf16 tile, 128-byte swizzle
constexpr int NCB = ROW / 64;               // 9 column blocks per cache row
// ---- QK CTA shared memory: a ring of whole pages ----
// A page (64 tokens x 576) is one TMA operation: a 3-D box {64, 64, 9} over the cache viewed as
// column blocks, landing as 9 K-major SW128 tiles.  A segment's Q (128 heads x 576) takes two
// ring stages (heads 0-63, 64-127) through the same box shape over q_abs.
constexpr int KV_STAGES = 3;
constexpr int KV_STAGE = NCB * CB;          // 73728
// ---- PV CTA shared memory ----
constexpr int VH_STAGES = 4;                // ring of half pages: 4 column blocks (256 columns)
constexpr int VH_STAGE = 4 * CB;            // 32768
constexpr int V_OFF = 0;
constexpr int P_OFF = VH_STAGES * VH_STAGE;
constexpr int P_TILE = NH * PG * 2;         // 16384: P[128 heads][64 tokens] bf16, SW128 K-major
constexpr int P_FACT = P_TILE;              // 128 fp32 rescale factors
constexpr int P_FLAG = P_TILE + NH * 4;     // one u32: some factor != 1
constexpr uint32_t MSG_BYTES = P_TILE + NH * 4 + 4;  // bytes st.async delivers per page
constexpr int P_SLOT = 17408;               // slot stride, 1 KB aligned
constexpr int P_SLOTS = 3;
constexpr int DATA_B = P_OFF + P_SLOTS * P_SLOT;
static_assert(P_SLOT % 1024 == 0 && P_OFF % 1024 == 0 && VH_STAGE % 1024 == 0,
              "swizzled tiles need 1 KB alignment");
// ---- FP8 cache: e4m3 content codes [page][64][512], a fp32 scale per token, bf16 RoPE keys ----
// The pages are dequantised on chip, bf16(code * scale), into exactly the bf16 page tiles the
// bf16 path loads, so everything after the page ring is shared by both.  The codes come in raw
// (row-major [token][code]) into staging slots: QK CTA whole pages, PV CTA half pages.
constexpr int STG_CODES = PG * DC;          // 32768: one page's codes
constexpr int STG_SLOT = 33792;             // codes + 64 scales, 1 KB aligned
constexpr int VSTG_CODES = PG * DC / 2;     // 16384: codes of one half page ([64][256])
constexpr int VSTG_SLOT = 17408;
static_assert(STG_CODES + PG * 4 <= STG_SLOT && VSTG_CODES + PG * 4 <= VSTG_SLOT, "staging slot layout");
static_assert(MSG_BYTES <= (uint32_t)P_SLOT, "message slot");
// ---- QK CTA tensor memory: three S buffers, then Q (content and RoPE part) ----
constexpr uint32_t TMEM_COLS = 512;
constexpr int S_SETS = 3;
constexpr uint32_t S_COL = 0;
constexpr uint32_t Q_COL = S_SETS * PG;     // 192; column block c of Q at Q_COL + 32 c
constexpr uint32_t P_COL = Q_COL + NCB * 32;  // 480: P of one page, bf16 pairs (32 columns)
static_assert(P_COL + PG / 2 <= TMEM_COLS, "QK-CTA TMEM budget");
// ---- threads ----
constexpr int THREADS = 480;                // 15 warps
constexpr int SM_WARP0 = 3;                 // QK CTA: softmax warps 3..10
constexpr int SM_THREADS = 256;
constexpr int SD_WARP0 = 11;                // QK CTA: sender warps 11..14 (P -> CTA 1 by st.async)
constexpr int SD_THREADS = 128;
constexpr int EP_WARP0 = 2;                 // PV CTA: correction / epilogue warps 2..5
constexpr int VC_WARP0 = 6;                 // PV CTA, FP8: converter warps 6..9 (codes -> bf16 V)
constexpr int VC_THREADS = 128;
constexpr float RESCALE_LOG2 = 8.0f;

struct __align__(8) Ctrl {
    // QK CTA
    uint64_t kv_full[KV_STAGES], kv_empty[KV_STAGES];
    uint64_t stg_full[2], stg_empty[2];     // FP8: raw page codes landed / converted
    uint64_t conv_full[KV_STAGES];          // FP8: a page stage's content columns dequantised
    uint64_t s_full[S_SETS], s_free[S_SETS];
    uint64_t k0_done[S_SETS];   // MMA thread 0 has issued its part of the page in this S buffer
    uint64_t q_ready;
    uint64_t p_ready, p_taken;  // P in TMEM: written by the softmax / read by the senders
    uint64_t pfree[P_SLOTS];    // P slot of CTA 1 reusable: its PV MMAs done (1) + read by 4 warps
    // PV CTA
    uint64_t v_full[VH_STAGES], v_empty[VH_STAGES], v_ready[VH_STAGES];
    uint64_t p_full[P_SLOTS], pv_done[P_SLOTS];
    uint64_t vstg_full[2], vstg_empty[2];   // FP8: raw half-page codes landed / converted
    uint64_t corr_done, o_free;
    uint64_t mma_idle[2];       // drains: one per MMA-issuing thread
    uint64_t never_done;        // test of the failure path: a barrier that nothing completes
    uint32_t tmem_base;
    uint32_t abort;
    uint32_t never;             // stays 0: the abort word of drain waits, which must not give up early
    int w_r0, w_pg0, w_n;       // this cluster's work: first row, first page of it, number of pages
    int scan[THREADS / 32 + 1]; // scheduling scratch (warp totals)
    float lx[2][NH];            // QK CTA: the second softmax half's row sums, by segment parity
    float fac[2][NH];           // QK CTA: per-head rescale factors of a page, by page parity
};
// FP8 cache with the content scores on the FP8 tensor core (MM): per segment, the per-head
// scale of the e4m3 query and the two halves' max |q_lat|; per page (ring of 3, by page count),
// the tokens' scales times log2(e)/sqrt(d_h + d_R).
struct Q8Extra {
    float qalpha[NH];
    float qamax[2][NH];
    float pscale[3][PG];
};
// Shared-memory plan of the bf16 (F8 = false) and FP8 (F8 = true) kernels.  The FP8 QK CTA
// keeps two page stages, and its staging slots take the third; with MM = true the codes land
// in the stage itself, so all three stages stay, followed by the Q8Extra block.
template <bool F8, bool MM = false>
struct Lay {
    static constexpr int kv_stages = (F8 && !MM) ? 2 : KV_STAGES;
    static constexpr int stg_off = kv_stages * KV_STAGE;
    static constexpr int q8_off = stg_off;
    static constexpr int data_a = stg_off + (F8 ? (MM ? (int)sizeof(Q8Extra) : 2 * STG_SLOT) : 0);
    static constexpr int vstg_off = DATA_B;
    static constexpr int data_b = DATA_B + (F8 ? 2 * VSTG_SLOT : 0);
    static constexpr int data = data_a > data_b ? data_a : data_b;
    static constexpr int smem = 1024 + data + (int)((sizeof(Ctrl) + 127) / 128 * 128);
};
static_assert(Lay<false>::smem <= 232448 && Lay<true>::smem <= 232448 && Lay<true, true>::smem <= 232448,
              "shared memory per block");
static_assert(Lay<true>::stg_off % 1024 == 0 && Lay<true>::vstg_off % 1024 == 0, "staging alignment");
// MM page stage: content codes as 4 K-major SW128 blocks [64 tokens x 128 B] (blocks 0-3), the
// tokens' scales at block 4, the RoPE keys (bf16, divided on chip by the token's scale) at block 8.
constexpr int MM_SCALE_OFF = 4 * CB;

struct Params {
    const int32_t *bt;
    int max_blocks, num_blocks;
    const int32_t *seq_lens;
    int s_q, rows, max_seq_len;
    int pairs;            // clusters of the grid
    int32_t *seg_range;   // [rows][2]: the row's slot range, written by cluster 0
    uint32_t *o_part;  // [slot][d_c / 2][n_h]: bf16 pairs of columns (c = 2k, 2k + 1) per head
    float *m_part, *l_part;
    float scale_log2;
    unsigned *err;
    int test_give_up;         // MLA_FLAG_TEST_GIVE_UP: the QK producer gives up before its second page
    const uint8_t *codes;     // FP8: content codes [num_blocks][64][512]
    const float *kv_scale;    // FP8: per-token scales [num_blocks][64]
};

__device__ __forceinline__ int row_tokens(const Params &P, int r) {
    if (r < 0 || r >= P.rows) return 0;
    const int b = r / P.s_q, i = r - b * P.s_q;
    const int L = P.seq_lens[b];
    if (L < P.s_q || L > P.max_seq_len || L > P.max_blocks * PG) return 0;
    return L - P.s_q + i + 1;
}

// Walks one cluster's pages in order; every role of both CTAs walks the same sequence.
// The next row's length is loaded one row ahead, so a segment change does not wait on memory.
struct PageIt {
    int r, pg, left, nv, np, nv_next;
    bool first;
    __device__ void init(const Params &P, const int *work) {
        r = work[0];
        pg = work[1];
        left = work[2];
        nv = row_tokens(P, r);
        nv_next = row_tokens(P, r + 1);
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
                nv = nv_next;
                nv_next = row_tokens(P, r + 1);
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

// FP8 page tiles: one 8-code group of token row j (codes at src) -> bf16(code * sc), one 16-byte
// chunk of the K-major SW128 tile at dst.  e4m3 codes are exact in fp16 and fp32, so the code *
// scale product is rounded once to fp32 and once to bf16.
// Each group costs 16 conversion instructions.  Variants that build the values with integer and
// bf16x2 arithmetic instead (exact as well) measured slower in the full kernel.
__device__ __forceinline__ void dequant8(uint32_t src, float sc, uint32_t dst) {
    uint32_t w0, w1;
    asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(w0), "=r"(w1) : "r"(src));
    uint32_t o[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const uint32_t w = (k < 2) ? w0 : w1;
        const unsigned short pr = (unsigned short)(w >> ((k & 1) * 16));  // codes 2k, 2k+1 (low byte first)
        uint32_t hh;
        asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(hh) : "h"(pr));
        const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&hh));
        o[k] = pack_bf16x2(f.x * sc, f.y * sc);
    }
    st_shared_v4(dst, o[0], o[1], o[2], o[3]);
}

// bf16 pair (low half first) -> two floats.
__device__ __forceinline__ float2 bf16x2_to_float2(uint32_t w) {
    return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
}
// Two floats -> two e4m3 codes (nearest even, saturating), x in the low byte.
__device__ __forceinline__ uint32_t f32x2_to_e4m3x2(float x, float y) {
    unsigned short r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(y), "f"(x));
    return r;
}
// Two e4m3 codes (low byte first) -> their exact values.
__device__ __forceinline__ float2 e4m3x2_to_float2(uint32_t w) {
    uint32_t hh;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(hh) : "h"((unsigned short)w));
    return __half22float2(*reinterpret_cast<const __half2 *>(&hh));
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
// 2^x on the SFU (ex2.approx, flush-to-zero): P only needs bf16 precision.
__device__ __forceinline__ float fast_exp2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float max32(const float (&x)[32]) {
    float a = fmaxf(x[0], x[1]), b = fmaxf(x[2], x[3]), c = fmaxf(x[4], x[5]), d = fmaxf(x[6], x[7]);
#pragma unroll
    for (int j = 8; j < 32; j += 8) {
        a = fmaxf(a, fmaxf(x[j + 0], x[j + 1]));
        b = fmaxf(b, fmaxf(x[j + 2], x[j + 3]));
        c = fmaxf(c, fmaxf(x[j + 4], x[j + 5]));
        d = fmaxf(d, fmaxf(x[j + 6], x[j + 7]));
    }
    return fmaxf(fmaxf(a, b), fmaxf(c, d));
}

// ---- the cluster's share of the work (every CTA computes it; cluster 0 also writes the
// per-row slot ranges the combine kernel reads) --------------------------------------------
// All (query row, page) units are numbered row by row; cluster c takes units
// [c U / pairs, (c + 1) U / pairs).  A row's partial results go to slots c + r of the clusters c
// that hold its units; a cluster that holds none (possible when there are fewer units than
// clusters) but sits inside a row's slot range marks its slot empty (m = -inf).
__device__ __forceinline__ long long unit_start(long long c, long long U, int pairs) { return c * U / pairs; }
__device__ __forceinline__ int pages_of_row(const Params &P, int r, bool &bad) {
    const int b = r / P.s_q, i = r - b * P.s_q;
    const int L = P.seq_lens[b];
    if (L < P.s_q || L > P.max_seq_len || L > P.max_blocks * PG) {
        bad |= i == 0;
        return 0;
    }
    return (L - P.s_q + i + 1 + PG - 1) / PG;
}
// Block-wide inclusive scan (THREADS threads); returns this thread's inclusive value and sets
// total.  Uses ctrl->scan; ends with a barrier, so it can be called again right away.
__device__ __forceinline__ long long block_scan(int x, Ctrl *ctrl, long long &total) {
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) ctrl->scan[wid] = x;
    __syncthreads();
    long long before = 0, all = 0;
    for (int w = 0; w < THREADS / 32; ++w) {
        const int v = ctrl->scan[w];
        if (w < wid) before += v;
        all += v;
    }
    total = all;
    __syncthreads();
    return before + x;
}
// The cluster holding unit u (the inverse of unit_start).
__device__ __forceinline__ int pair_of_unit(long long u, long long U, int pairs) {
    int c = (int)(u * pairs / U);
    while (c + 1 < pairs && unit_start(c + 1, U, pairs) <= u) ++c;
    while (c > 0 && unit_start(c, U, pairs) > u) --c;
    return c;
}
// Row r has n > 0 units starting at unit u0: record this cluster's work if it starts inside the
// row, mark this cluster's slot empty if the row's slot range covers it but it got no units,
// and (cluster 0) write the row's slot range.
__device__ __forceinline__ void schedule_row(const Params &P, int pair, uint32_t rank, Ctrl *ctrl, int r, int n,
                                             long long u0, long long U, long long s0, long long s1) {
    if (n > 0 && u0 <= s0 && s0 < u0 + n) {  // the row holding unit s0
        if (s1 > s0) {
            ctrl->w_r0 = r;
            ctrl->w_pg0 = (int)(s0 - u0);
        } else if (rank == 0) {
            for (int h = 0; h < NH; ++h) P.m_part[((size_t)pair + r) * NH + h] = -INFINITY;
        }
    }
    if (pair == 0 && rank == 0 && r < P.rows) {
        P.seg_range[2 * r] = n > 0 ? pair_of_unit(u0, U, P.pairs) + r : 0;
        P.seg_range[2 * r + 1] = n > 0 ? pair_of_unit(u0 + n - 1, U, P.pairs) + r + 1 : 0;
    }
}
__device__ __noinline__ void schedule(const Params &P, int pair, uint32_t rank, Ctrl *ctrl) {
    const int tid = threadIdx.x;
    bool bad = false;
    if (tid == 0) {
        ctrl->w_r0 = 0;
        ctrl->w_pg0 = 0;
    }
    if (P.rows <= THREADS) {  // one pass: every row's length is read once, one block-wide scan
        const int r = tid;
        const int n = r < P.rows ? pages_of_row(P, r, bad) : 0;
        long long U;
        const long long u0 = block_scan(n, ctrl, U) - n;  // ends with a barrier (orders tid 0's defaults)
        const long long s0 = unit_start(pair, U, P.pairs), s1 = unit_start(pair + 1, U, P.pairs);
        if (tid == 0) ctrl->w_n = (int)(s1 - s0);
        if (bad && pair == 0 && rank == 0) record_error(P.err, kErrBadSeqLen);
        schedule_row(P, pair, rank, ctrl, r, n, u0, U, s0, s1);
        __syncthreads();
        return;
    }
    long long U = 0;
    for (int base = 0; base < P.rows; base += THREADS) {  // pass 1: all units
        const int r = base + tid;
        long long chunk;
        block_scan(r < P.rows ? pages_of_row(P, r, bad) : 0, ctrl, chunk);
        U += chunk;
    }
    if (bad && pair == 0 && rank == 0) record_error(P.err, kErrBadSeqLen);
    const long long s0 = unit_start(pair, U, P.pairs), s1 = unit_start(pair + 1, U, P.pairs);
    if (tid == 0) ctrl->w_n = (int)(s1 - s0);
    long long carry = 0;
    for (int base = 0; base < P.rows; base += THREADS) {  // pass 2: locate s0, slot ranges
        const int r = base + tid;
        bool b2 = false;
        const int n = r < P.rows ? pages_of_row(P, r, b2) : 0;
        long long chunk;
        const long long u0 = carry + block_scan(n, ctrl, chunk) - n;  // this row's first unit
        schedule_row(P, pair, rank, ctrl, r, n, u0, U, s0, s1);
        carry += chunk;
    }
    __syncthreads();
}

// Warms L2 (and the address translation) for the sequence lengths and the block table, which
// the schedule and the first page loads read through a chain of dependent accesses.  A prefetch
// returns nothing and L2 is coherent, so it may precede the wait for the kernel before this one.
__device__ __noinline__ void warm_tables(const Params &P) {
    const int nb = P.rows / P.s_q;
    const char *sl = reinterpret_cast<const char *>(P.seq_lens);
    for (int off = threadIdx.x * 128; off < nb * 4; off += THREADS * 128) prefetch_l2(sl + off);
    const char *btp = reinterpret_cast<const char *>(P.bt);
    const size_t bt_bytes = (size_t)nb * P.max_blocks * 4;
    for (size_t off = ((size_t)blockIdx.x * THREADS + threadIdx.x) * 128; off < bt_bytes;
         off += (size_t)gridDim.x * THREADS * 128)
        prefetch_l2(btp + off);
}

// Named barriers: the 256 softmax threads and the 128 sender threads (QK CTA).
constexpr int BAR_FAIL = 1, BAR_Q = 2, BAR_SFAIL = 3, BAR_SFLAG = 4, BAR_CONV = 5;
constexpr int BAR_VCONV = 5;  // PV CTA: the FP8 converter warps

// F8 = false: bf16 cache; tm_kv9 loads whole pages {64, 64, 9}, tm_kv4 half pages {64, 64, 4}.
// F8 = true: FP8 cache; tm_kv9 loads a page's RoPE keys as one {64, 64} tile, tm_kv4 a half
// page of raw codes {256, 64}; the codes of whole pages and the scales come by bulk copy.
template <bool F8, bool MM = false>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(THREADS, 1)
decode_tc_kernel(const __grid_constant__ CUtensorMap tm_kv9, const __grid_constant__ CUtensorMap tm_kv4,
                 const __grid_constant__ CUtensorMap tm_q9, const __grid_constant__ CUtensorMap tm_c8,
                 const __grid_constant__ Params P) {
    constexpr bool QF8 = F8 && MM;  // content scores on the FP8 tensor core
    using L = Lay<F8, MM>;
    constexpr int KVS = L::kv_stages;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_s = smem_u32(smem_raw);
    const uint32_t data_s = (raw_s + 1023u) & ~1023u;
    Ctrl *ctrl = reinterpret_cast<Ctrl *>(smem_raw + (data_s - raw_s) + L::data);
    volatile uint32_t *abort_flag = &ctrl->abort;
    auto bar = [&](uint64_t &b) { return smem_u32(&b); };

    const uint32_t rank = cluster_ctarank();
    const int pair = blockIdx.x >> 1;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    warm_tables(P);

    if (threadIdx.x == 0) {
        for (int i = 0; i < KV_STAGES; ++i) {
            mbar_init(bar(ctrl->kv_full[i]), 1);
            mbar_init(bar(ctrl->kv_empty[i]), 2);  // both MMA threads (or the Q copy, twice)
            mbar_init(bar(ctrl->conv_full[i]), SM_THREADS / 32);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(bar(ctrl->stg_full[i]), 1);
            mbar_init(bar(ctrl->stg_empty[i]), SM_THREADS / 32);
            mbar_init(bar(ctrl->vstg_full[i]), 1);
            mbar_init(bar(ctrl->vstg_empty[i]), VC_THREADS / 32);
        }
        for (int i = 0; i < S_SETS; ++i) {
            mbar_init(bar(ctrl->s_full[i]), 2);
            mbar_init(bar(ctrl->k0_done[i]), 1);
            mbar_init(bar(ctrl->s_free[i]), SM_THREADS / 32);
        }
        mbar_init(bar(ctrl->q_ready), 1);
        mbar_init(bar(ctrl->p_ready), SM_THREADS / 32);
        mbar_init(bar(ctrl->p_taken), SD_THREADS / 32);
        for (int i = 0; i < P_SLOTS; ++i) {
            mbar_init(bar(ctrl->pfree[i]), 1 + 4);
            mbar_init(bar(ctrl->p_full[i]), 1);
            mbar_init(bar(ctrl->pv_done[i]), 1);
        }
        for (int i = 0; i < VH_STAGES; ++i) {
            mbar_init(bar(ctrl->v_full[i]), F8 ? VC_THREADS / 32 : 1);  // TMA, or the FP8 converters
            mbar_init(bar(ctrl->v_empty[i]), 1);
            mbar_init(bar(ctrl->v_ready[i]), 4);
        }
        mbar_init(bar(ctrl->corr_done), 4);
        mbar_init(bar(ctrl->o_free), 4);
        mbar_init(bar(ctrl->mma_idle[0]), 1);
        mbar_init(bar(ctrl->mma_idle[1]), 1);
        mbar_init(bar(ctrl->never_done), 1);
        ctrl->abort = 0;
        ctrl->never = 0;
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
    // Everything above overlaps the kernel before this one; inputs are read from here on.
    pdl_trigger();
    pdl_wait();
    schedule(P, pair, rank, ctrl);
    const uint32_t tmem = ctrl->tmem_base;
    const uint32_t peer = rank ^ 1u;
    auto fail = [&]() {
        if (*abort_flag == 0) {
            *abort_flag = 1;
            st_shared_cluster_u32(mapa(smem_u32(&ctrl->abort), peer), 1u);
            record_error(P.err, kErrTimeout);
        }
    };
    // Drain waits ignore the abort flag: they wait for hardware that is already running.
    volatile uint32_t *never = &ctrl->never;
    Q8Extra *q8 = reinterpret_cast<Q8Extra *>(smem_raw + (data_s - raw_s) + L::q8_off);  // QF8 only

    if (rank == 0) {
        // ===================================== QK CTA =====================================
        if (warp == 0 && lane == 0) {  // TMA producer: per segment 2 Q stages, then its pages
            prefetch_tensormap(&tm_kv9);
            prefetch_tensormap(&tm_q9);
            PageIt it;
            it.init(P, &ctrl->w_r0);
            Ring st{0, 0};
            int issued[KV_STAGES];           // phase + 1 of the last copy into each stage (0: none)
            for (int i = 0; i < KV_STAGES; ++i) issued[i] = 0;
            uint32_t nph[KV_STAGES] = {};
            int u = 0;
            bool ok = true;
            auto load = [&](const CUtensorMap *map, int y) -> bool {
                if (!wait(bar(ctrl->kv_empty[st.i]), st.ph ^ 1u, abort_flag)) return false;
                mbar_arrive_expect_tx(bar(ctrl->kv_full[st.i]), KV_STAGE);
                tma_load_3d(data_s + st.i * KV_STAGE, map, 0, y, 0, bar(ctrl->kv_full[st.i]));
                issued[st.i] = 1;
                nph[st.i] = st.ph;
                st.adv(KVS);
                return true;
            };
            // FP8: a page's raw codes and scales go to a staging slot (the softmax warps dequantise
            // them into the page stage); its RoPE keys go straight to the stage's last column block.
            Ring g{0, 0};
            int g_issued[2] = {0, 0};
            uint32_t g_nph[2] = {0u, 0u};
            auto load_f8 = [&](int blk) -> bool {
                if (!wait(bar(ctrl->stg_empty[g.i]), g.ph ^ 1u, abort_flag)) return false;
                const uint32_t sdst = data_s + L::stg_off + g.i * STG_SLOT;
                mbar_arrive_expect_tx(bar(ctrl->stg_full[g.i]), STG_CODES + PG * 4);
                bulk_load(sdst, P.codes + (size_t)blk * STG_CODES, STG_CODES, bar(ctrl->stg_full[g.i]));
                bulk_load(sdst + STG_CODES, P.kv_scale + (size_t)blk * PG, PG * 4, bar(ctrl->stg_full[g.i]));
                g_issued[g.i] = 1;
                g_nph[g.i] = g.ph;
                g.adv(2);
                if (!wait(bar(ctrl->kv_empty[st.i]), st.ph ^ 1u, abort_flag)) return false;
                mbar_arrive_expect_tx(bar(ctrl->kv_full[st.i]), CB);
                tma_load_2d(data_s + st.i * KV_STAGE + (NCB - 1) * CB, &tm_kv9, 0, blk * PG, bar(ctrl->kv_full[st.i]));
                issued[st.i] = 1;
                nph[st.i] = st.ph;
                st.adv(KVS);
                return true;
            };
            // FP8 with the content scores on the tensor core: codes (4 swizzled blocks), scales and
            // RoPE keys straight into the page stage.
            auto load_mm = [&](int blk) -> bool {
                if (!wait(bar(ctrl->kv_empty[st.i]), st.ph ^ 1u, abort_flag)) return false;
                const uint32_t dst = data_s + st.i * KV_STAGE;
                mbar_arrive_expect_tx(bar(ctrl->kv_full[st.i]), 5 * CB + PG * 4);
                tma_load_3d(dst, &tm_c8, 0, blk * PG, 0, bar(ctrl->kv_full[st.i]));
                tma_load_2d(dst + (NCB - 1) * CB, &tm_kv9, 0, blk * PG, bar(ctrl->kv_full[st.i]));
                bulk_load(dst + MM_SCALE_OFF, P.kv_scale + (size_t)blk * PG, PG * 4, bar(ctrl->kv_full[st.i]));
                issued[st.i] = 1;
                nph[st.i] = st.ph;
                st.adv(KVS);
                return true;
            };
            if (QF8) prefetch_tensormap(&tm_c8);
            while (ok && !it.done()) {
                if (it.first) {
                    if (!(ok = load(&tm_q9, it.r * NH) && load(&tm_q9, it.r * NH + 64))) break;
                }
                const int blk = block_of(P, it.r, it.pg);
                // Test of the failure path: with copies (and soon MMAs) of the first page in flight,
                // wait a short while on a barrier that nothing completes, and give up like any
                // timed-out wait: abort flags in both CTAs, error word, bounded drains, exit.
                if (P.test_give_up && u == 1 && !(ok = wait(bar(ctrl->never_done), 0u, abort_flag, 20000ull)))
                    break;
                if (!(ok = QF8 ? load_mm(blk) : (F8 ? load_f8(blk) : load(&tm_kv9, blk * PG)))) break;
                ++u;
                it.next(P);
            }
            if (!ok) fail();
            for (int i = 0; i < KV_STAGES; ++i)  // drain: every copy this thread started has landed
                if (issued[i]) wait(bar(ctrl->kv_full[i]), nph[i], never);
            for (int i = 0; i < 2; ++i)
                if (g_issued[i]) wait(bar(ctrl->stg_full[i]), g_nph[i], never);
        } else if ((warp == 1 || warp == 2) && lane == 0) {  // MMA issuers: S += Q . KV^T, split K
            // Both threads work on every page: thread 0 column blocks 0-4, thread 1 blocks 5-8 (the
            // RoPE part).  One thread cannot issue N = 64 MMAs as fast as the tensor core runs them,
            // and splitting the page (not alternating pages) keeps each stage busy for the shortest
            // time.  All MMAs accumulate: the softmax zeroes an S buffer when it has read it.
            // Thread 1 issues a page's part only after thread 0 has issued its own (k0_done, with
            // the tcgen05 thread-sync fences on both sides), so every page sums in the same order
            // and results are bitwise reproducible; thread 0 meanwhile goes on to the next page.
            // (Splitting by tokens instead -- N = 32 per thread over the whole K, into separate
            // columns -- needs no ordering but doubles each thread's MMA count; measured slower.)
            const int part = warp - 1;
            constexpr uint32_t idesc = idesc_bf16(128, PG, false, false);
            const int cb0 = part ? 5 : 0, cb1 = part ? NCB : 5;
            PageIt it;
            it.init(P, &ctrl->w_r0);
            Ring st{0, 0}, sb{0, 0};
            uint32_t qn = 0;
            uint32_t cv_ph = 0;  // FP8: phase bit of conv_full[i] (it completes on page uses only)
            int u = 0;
            bool ok = true, any = false;
            while (ok && !it.done()) {
                if (it.first) {
                    st.adv(KVS, 2);  // the segment's Q stages (copied to TMEM by the softmax warps)
                    if (!(ok = wait(bar(ctrl->q_ready), qn & 1u, abort_flag))) break;
                    ++qn;
                }
                if (!(ok = wait(bar(ctrl->s_free[sb.i]), sb.ph ^ 1u, abort_flag))) break;
                if (part && !(ok = wait(bar(ctrl->k0_done[sb.i]), sb.ph, abort_flag))) break;
                tc_fence_after();  // orders the MMAs after the softmax's TMEM zeroing / thread 0's MMAs
                // TMA-filled shared memory needs no tcgen05 fence: the mbarrier completion already
                // makes it visible to MMAs issued after the wait.
                if (!(ok = wait(bar(ctrl->kv_full[st.i]), st.ph, abort_flag))) break;
                if (F8) {  // the content columns are written by the softmax warps' dequantisation
                    if (!(ok = wait(bar(ctrl->conv_full[st.i]), (cv_ph >> st.i) & 1u, abort_flag))) break;
                    cv_ph ^= 1u << st.i;
                }
                const uint32_t d = tmem + S_COL + sb.i * PG;
                const uint32_t kvb = data_s + st.i * KV_STAGE;
                if (QF8) {
                    // e4m3 content: thread 0 the query's high part, thread 1 its low part (TMEM
                    // columns Q_COL and Q_COL + 128: 4 codes per column, 8 columns per K = 32),
                    // then thread 1 the RoPE part in bf16 (TMEM Q_COL + 256, the stage's block 8)
                    constexpr uint32_t idesc8 = idesc_e4m3(128, PG);
                    const uint32_t qa = tmem + Q_COL + (part ? 128u : 0u);
#pragma unroll 1
                    for (int kb = 0; kb < 4; ++kb) {
#pragma unroll
                        for (int k = 0; k < 4; ++k)
                            mma_ts_f8(d, qa + (kb * 4 + k) * 8, sdesc_sw128(kvb + kb * CB + k * 32, 16, 1024), idesc8,
                                      1u);
                    }
                    if (part) {
#pragma unroll
                        for (int k = 0; k < 4; ++k)
                            mma_ts(d, tmem + Q_COL + 256 + k * 8,
                                   sdesc_sw128(kvb + (NCB - 1) * CB + k * 32, 16, 1024), idesc, 1u);
                    }
                } else {
#pragma unroll 1
                    for (int cb = cb0; cb < cb1; ++cb) {
#pragma unroll
                        for (int k = 0; k < 4; ++k)
                            mma_ts(d, tmem + Q_COL + (cb * 4 + k) * 8, sdesc_sw128(kvb + cb * CB + k * 32, 16, 1024),
                                   idesc, 1u);
                    }
                }
                if (!part) {
                    tc_fence_before();
                    mbar_arrive(bar(ctrl->k0_done[sb.i]));
                }
                mma_commit(bar(ctrl->kv_empty[st.i]));
                mma_commit(bar(ctrl->s_full[sb.i]));
                any = true;
                ++u;
                st.adv(KVS);
                sb.adv(S_SETS);
                it.next(P);
            }
            if (!ok) fail();
            if (any) {  // drain: the MMAs this thread issued are complete before TMEM is released
                mma_commit(bar(ctrl->mma_idle[part]));
                wait(bar(ctrl->mma_idle[part]), 0u, never);
            }
        } else if (warp >= SM_WARP0 && warp < SM_WARP0 + 8) {  // softmax: 2 warps per lane quarter
            const int t = threadIdx.x - SM_WARP0 * 32;          // 0..255
            const int quarter = warp & 3;
            const int half = (warp - SM_WARP0) >> 2;            // which 32 of the 64 columns
            const int h = quarter * 32 + lane;                  // head = TMEM lane
            const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
            PageIt it;
            it.init(P, &ctrl->w_r0);
            Ring st{0, 0}, sb{0, 0};
            float m_used = -INFINITY, l = 0.f;
            int u = 0, seg = 0;
            bool ok = true;

            // Q of a segment (2 stages: heads 0-63, 64-127) -> TMEM lane h; this half copies
            // column blocks 0-4 (half 0) or 5-8 (half 1).  Uniform across the 256 threads.
            auto load_q = [&]() -> bool {
                const Ring q0 = st;
                st.adv(KVS);
                const Ring q1 = st;
                st.adv(KVS);
                const bool w = wait(bar(ctrl->kv_full[q0.i]), q0.ph, abort_flag) &&
                               wait(bar(ctrl->kv_full[q1.i]), q1.ph, abort_flag);
                if (named_red_or(!w, BAR_Q, SM_THREADS)) return false;
                const int rr = h & 63;
                const uint32_t rowa = data_s + ((h >> 6) ? q1.i : q0.i) * KV_STAGE + rr * 128;
                const int cb0 = half ? 5 : 0, cb1 = half ? NCB : 5;
                if (QF8) {
                    // e4m3 query, per head: alpha = max|q_lat| / 448 (both halves' columns),
                    // hi = e4m3(q / alpha), lo = e4m3(q / alpha - hi), so q ~ alpha (hi + lo) with
                    // about 7 significant bits.  Codes into TMEM (4 per column): hi at Q_COL + c / 4,
                    // lo at Q_COL + 128 + c / 4; the RoPE part as bf16(q_rope / alpha) at Q_COL + 256.
                    const int ce = half ? NCB - 1 : 5;  // content blocks of this half: [cb0, ce)
                    float am = 0.f;
#pragma unroll 1
                    for (int cb = cb0; cb < ce; ++cb)
#pragma unroll
                        for (int c = 0; c < 8; ++c) {
                            const uint4 x = ld_shared_v4(rowa + cb * CB + ((c ^ (rr & 7)) << 4));
                            const uint32_t xw[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const float2 f = bf16x2_to_float2(xw[e]);
                                am = fmaxf(am, fmaxf(fabsf(f.x), fabsf(f.y)));
                            }
                        }
                    q8->qamax[half][h] = am;
                    named_sync(BAR_Q, SM_THREADS);
                    const float alpha = fmaxf(fmaxf(q8->qamax[0][h], q8->qamax[1][h]) / 448.f, FLT_MIN);
                    const float ia = 1.f / alpha;
                    if (!half) q8->qalpha[h] = alpha;
#pragma unroll 1
                    for (int cb = cb0; cb < ce; ++cb) {
                        uint32_t hw[16], lw[16];
#pragma unroll
                        for (int c = 0; c < 8; ++c) {
                            const uint4 x = ld_shared_v4(rowa + cb * CB + ((c ^ (rr & 7)) << 4));
                            const uint32_t xw[4] = {x.x, x.y, x.z, x.w};
                            uint32_t hc[4], lc[4];
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const float2 f = bf16x2_to_float2(xw[e]);
                                const float y0 = f.x * ia, y1 = f.y * ia;
                                const uint32_t h2 = f32x2_to_e4m3x2(y0, y1);
                                const float2 b = e4m3x2_to_float2(h2);
                                hc[e] = h2;
                                lc[e] = f32x2_to_e4m3x2(y0 - b.x, y1 - b.y);
                            }
                            hw[2 * c] = hc[0] | (hc[1] << 16);
                            hw[2 * c + 1] = hc[2] | (hc[3] << 16);
                            lw[2 * c] = lc[0] | (lc[1] << 16);
                            lw[2 * c + 1] = lc[2] | (lc[3] << 16);
                        }
                        tmem_st16(tmem + lane_base + Q_COL + cb * 16, hw);
                        tmem_st16(tmem + lane_base + Q_COL + 128 + cb * 16, lw);
                    }
                    if (half) {  // the RoPE part
                        uint32_t v[32];
#pragma unroll
                        for (int c = 0; c < 8; ++c) {
                            const uint4 x = ld_shared_v4(rowa + (NCB - 1) * CB + ((c ^ (rr & 7)) << 4));
                            const uint32_t xw[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const float2 f = bf16x2_to_float2(xw[e]);
                                v[4 * c + e] = pack_bf16x2(f.x * ia, f.y * ia);
                            }
                        }
                        tmem_st32(tmem + lane_base + Q_COL + 256, v);
                    }
                }
#pragma unroll 1
                for (int cb = cb0; cb < (QF8 ? cb0 : cb1); ++cb) {
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
                named_sync(BAR_Q, SM_THREADS);
                if (t == 0) {
                    for (int k = 0; k < 2; ++k) {
                        mbar_arrive(bar(ctrl->kv_empty[q0.i]));
                        mbar_arrive(bar(ctrl->kv_empty[q1.i]));
                    }
                    mbar_arrive(bar(ctrl->q_ready));
                }
                return true;
            };

            // FP8: dequantise the page whose raw codes are in staging slot cg into page stage c
            // (sixteen 8-code groups per thread), then release the slot and report the stage.
            // Pages are converted one ahead of the softmax: the next page of the segment before
            // this page's softmax, a segment's first page right after its Q copy.
            Ring cg{0, 0};
            int uc = 0;  // FP8 tensor-core QK: pages prepared so far (index of the scale ring)
            auto convert = [&](Ring c) -> bool {
                if (QF8) {
                    // The page's RoPE keys divided by the token's scale (in place, 16 values per
                    // thread), so that S = alpha_h s_j (hi + lo).c8_j + (q_rope / alpha_h).(k_j / s_j)
                    // needs one per-column factor; the factors go to the scale ring for the softmax.
                    const bool w = wait(bar(ctrl->kv_full[c.i]), c.ph, abort_flag);
                    if (named_red_or(!w, BAR_CONV, SM_THREADS)) return false;
                    const uint32_t stage = data_s + c.i * KV_STAGE;
                    const float *scl = reinterpret_cast<const float *>(smem_raw + (stage - raw_s) + MM_SCALE_OFF);
#pragma unroll
                    for (int q = t; q < PG * 8; q += SM_THREADS) {  // 512 chunks of 8 keys
                        const int j = q >> 3, cc = q & 7;
                        const uint32_t a = stage + (NCB - 1) * CB + j * 128 + ((cc ^ (j & 7)) << 4);
                        const uint4 x = ld_shared_v4(a);
                        const float inv = 1.f / scl[j];
                        const uint32_t xw[4] = {x.x, x.y, x.z, x.w};
                        uint32_t o[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float2 f = bf16x2_to_float2(xw[e]);
                            o[e] = pack_bf16x2(f.x * inv, f.y * inv);
                        }
                        st_shared_v4(a, o[0], o[1], o[2], o[3]);
                    }
                    if (t < PG) q8->pscale[uc % 3][t] = scl[t] * P.scale_log2;
                    ++uc;
                    fence_proxy_async_smem();
                    named_sync(BAR_CONV, SM_THREADS);  // the factors are visible to every softmax thread
                    if (lane == 0) mbar_arrive(bar(ctrl->conv_full[c.i]));
                    return true;
                }
                const bool w = wait(bar(ctrl->stg_full[cg.i]), cg.ph, abort_flag) &&
                               wait(bar(ctrl->kv_empty[c.i]), c.ph ^ 1u, abort_flag);
                if (named_red_or(!w, BAR_CONV, SM_THREADS)) return false;
                const uint32_t src = data_s + L::stg_off + cg.i * STG_SLOT;
                const float *scl = reinterpret_cast<const float *>(smem_raw + (src - raw_s) + STG_CODES);
                const uint32_t dst = data_s + c.i * KV_STAGE;
#pragma unroll 4
                for (int q = t; q < PG * (DC / 8); q += SM_THREADS) {  // 4096 groups, 16 per thread
                    const int j = q >> 6, cc = q & 63;
                    dequant8(src + j * DC + cc * 8, scl[j], dst + (cc >> 3) * CB + j * 128 + (((cc & 7) ^ (j & 7)) << 4));
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(bar(ctrl->conv_full[c.i]));
                    mbar_arrive(bar(ctrl->stg_empty[cg.i]));
                }
                cg.adv(2);
                return true;
            };
            auto first_page = [&]() -> bool { return !F8 || convert(st); };

            {   // the MMAs only accumulate into S: start from zero
                uint32_t z[32];
#pragma unroll
                for (int j = 0; j < 32; ++j) z[j] = 0u;
                for (int i = 0; i < S_SETS; ++i) tmem_st32(tmem + lane_base + S_COL + i * PG + half * 32, z);
                tmem_wait_st();
            }
            if (!it.done()) ok = load_q() && first_page();  // load_q's barrier also orders the zeroing before q_ready
            while (ok && !it.done()) {
                if (F8 && !it.last()) {  // the next page of this segment (its stage follows this page's)
                    Ring c = st;
                    c.adv(KVS);
                    if (!(ok = convert(c))) break;
                }
                bool good = wait(bar(ctrl->s_full[sb.i]), sb.ph, abort_flag);
                float mine[32], other[32];
                {
                    uint32_t a[32], b[32];
                    const uint32_t sa = tmem + lane_base + S_COL + sb.i * PG;
                    tc_fence_after();
                    tmem_ld32(sa + half * 32, a);
                    tmem_ld32(sa + (half ^ 1) * 32, b);
                    tmem_wait_ld();
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        mine[j] = __uint_as_float(a[j]);
                        other[j] = __uint_as_float(b[j]);
                    }
                }
                const uint32_t s_buf = sb.i;  // zeroed and released after the vote (all warps have read it)
                sb.adv(S_SETS);
                st.adv(KVS);  // this page's stage

                const bool first = it.first, last = it.last();
                const int valid = it.valid();
                const int r = it.r;
                // ---- online softmax (log2 units; scale folded into one FFMA) ----
                float sl2 = P.scale_log2;
                if (QF8) {  // per-column factors alpha_h s_j log2(e)/sqrt(d): scale first, then one
                    const float al = q8->qalpha[h];
                    const float *ps = q8->pscale[u % 3];
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        mine[j] *= al * ps[half * 32 + j];
                        other[j] *= al * ps[(half ^ 1) * 32 + j];
                    }
                    sl2 = 1.f;
                }
                if (valid < PG) {
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        if (half * 32 + j >= valid) mine[j] = -INFINITY;
                        if ((half ^ 1) * 32 + j >= valid) other[j] = -INFINITY;
                    }
                }
                const float mx = fmaxf(max32(mine), max32(other)) * sl2;
                float m_new = m_used, fac = 1.f;
                if (first) {
                    m_new = mx;
                    l = 0.f;
                } else if (mx > m_used + RESCALE_LOG2) {
                    m_new = mx;
                    fac = fast_exp2(m_used - m_new);
                }
                float s0 = 0.f, s1 = 0.f;
                uint32_t pk[16];
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const float p0 = fast_exp2(fmaf(mine[2 * j], sl2, -m_new));
                    const float p1 = fast_exp2(fmaf(mine[2 * j + 1], sl2, -m_new));
                    s0 += p0;
                    s1 += p1;
                    pk[j] = pack_bf16x2(p0, p1);
                }
                l = l * fac + (s0 + s1);
                m_used = m_new;
                if (last && half) ctrl->lx[seg & 1][h] = l;  // read by the other half after the vote

                // ---- hand P to the senders through TMEM (one buffer: the senders took the last) ----
                good = good && wait(bar(ctrl->p_taken), (uint32_t)(u & 1) ^ 1u, abort_flag);
                if (named_red_or(!good, BAR_FAIL, SM_THREADS)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                {   // every softmax warp has read this S buffer: zero my half for its next page
                    uint32_t z[32];
#pragma unroll
                    for (int j = 0; j < 32; ++j) z[j] = 0u;
                    tmem_st32(tmem + lane_base + S_COL + s_buf * PG + half * 32, z);
                }
                tmem_st16(tmem + lane_base + P_COL + half * 16, pk);
                if (!half) ctrl->fac[u & 1][h] = fac;
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(bar(ctrl->s_free[s_buf]));
                    mbar_arrive(bar(ctrl->p_ready));
                }
                ++u;

                if (last) {
                    if (!half) {
                        const size_t sl = (size_t)pair + r;
                        P.m_part[sl * NH + h] = m_used;
                        P.l_part[sl * NH + h] = l + ctrl->lx[seg & 1][h];
                    }
                    m_used = -INFINITY;
                    l = 0.f;
                    ++seg;
                    // The last page's S is complete, so every QK MMA of this segment has finished
                    // and the next segment's Q may overwrite TMEM now.
                    if (it.left > 1 && !(ok = load_q() && first_page())) break;
                }
                it.next(P);
            }
            if (!ok) fail();
        } else if (warp >= SD_WARP0 && warp < SD_WARP0 + 4) {  // senders: P in TMEM -> CTA 1 slot
            const int t = threadIdx.x - SD_WARP0 * 32;          // 0..127
            const int quarter = warp & 3;
            const int h = quarter * 32 + lane;
            const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
            const uint32_t slot_r = mapa(data_s + P_OFF, 1), p_full_r = mapa(bar(ctrl->p_full[0]), 1);
            PageIt it;
            it.init(P, &ctrl->w_r0);
            Ring ps{0, 0};
            int u = 0;
            bool ok = true;
            uint32_t sent = 0, sent_ph = 0;  // slots with a message out, and its phase
            while (ok && !it.done()) {
                bool good = wait(bar(ctrl->p_ready), (uint32_t)(u & 1), abort_flag);
                good = good && wait<true>(bar(ctrl->pfree[ps.i]), ps.ph ^ 1u, abort_flag);
                if (named_red_or(!good, BAR_SFAIL, SD_THREADS)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                uint32_t pv[32];
                tmem_ld32(tmem + lane_base + P_COL, pv);
                tmem_wait_ld();
                const float fac = ctrl->fac[u & 1][h];
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(ctrl->p_taken));
                const uint32_t slot = slot_r + ps.i * P_SLOT, fb = p_full_r + ps.i * 8;
#pragma unroll
                for (int c = 0; c < 8; ++c)
                    st_async_v4(slot + h * 128 + ((c ^ (h & 7)) << 4), pv[4 * c], pv[4 * c + 1], pv[4 * c + 2],
                                pv[4 * c + 3], fb);
                st_async_b32(slot + P_FACT + h * 4, __float_as_uint(fac), fb);
                const bool any = named_red_or(fac != 1.f, BAR_SFLAG, SD_THREADS);
                if (t == 0) {
                    st_async_b32(slot + P_FLAG, any ? 1u : 0u, fb);
                    sent |= 1u << ps.i;
                    sent_ph = (sent_ph & ~(1u << ps.i)) | (ps.ph << ps.i);
                }
                ps.adv(P_SLOTS);
                ++u;
                it.next(P);
            }
            if (!ok) fail();
            // drain: CTA 1's arrivals on our slot barriers (its MMA commits, its readers) for the
            // messages still out have landed before this CTA can leave
            if (t == 0)
                for (int i = 0; i < P_SLOTS; ++i)
                    if (sent & (1u << i)) wait<true>(bar(ctrl->pfree[i]), (sent_ph >> i) & 1u, never, 10000000ull);
        }
    } else {
        // ===================================== PV CTA =====================================
        if (warp == 0 && lane == 0) {  // TMA producer: content columns as two half pages
            prefetch_tensormap(&tm_kv4);
            PageIt it;
            it.init(P, &ctrl->w_r0);
            Ring vs{0, 0};
            int issued[VH_STAGES];
            uint32_t nph[VH_STAGES] = {};
            for (int i = 0; i < VH_STAGES; ++i) issued[i] = 0;
            int u = 0;
            bool ok = true;
            Ring vg{0, 0};  // FP8: staging slot of the next half page of raw codes
            int g_issued[2] = {0, 0};
            uint32_t g_nph[2] = {0u, 0u};
            while (ok && !it.done()) {
                const int blk = block_of(P, it.r, it.pg);
                for (int hh = 0; F8 && hh < 2; ++hh) {  // FP8: codes [64][256] + scales -> staging
                    if (!(ok = wait(bar(ctrl->vstg_empty[vg.i]), vg.ph ^ 1u, abort_flag))) break;
                    const uint32_t sdst = data_s + L::vstg_off + vg.i * VSTG_SLOT;
                    mbar_arrive_expect_tx(bar(ctrl->vstg_full[vg.i]), VSTG_CODES + PG * 4);
                    tma_load_2d(sdst, &tm_kv4, hh * (DC / 2), blk * PG, bar(ctrl->vstg_full[vg.i]));
                    bulk_load(sdst + VSTG_CODES, P.kv_scale + (size_t)blk * PG, PG * 4, bar(ctrl->vstg_full[vg.i]));
                    g_issued[vg.i] = 1;
                    g_nph[vg.i] = vg.ph;
                    vg.adv(2);
                }
                for (int hh = 0; !F8 && hh < 2; ++hh) {
                    if (!(ok = wait(bar(ctrl->v_empty[vs.i]), vs.ph ^ 1u, abort_flag))) break;
                    mbar_arrive_expect_tx(bar(ctrl->v_full[vs.i]), VH_STAGE);
                    tma_load_3d(data_s + V_OFF + vs.i * VH_STAGE, &tm_kv4, 0, blk * PG, hh * 4,
                                bar(ctrl->v_full[vs.i]));
                    issued[vs.i] = 1;
                    nph[vs.i] = vs.ph;
                    vs.adv(VH_STAGES);
                }
                if (!ok) break;
                ++u;
                it.next(P);
            }
            if (!ok) fail();
            for (int i = 0; i < VH_STAGES; ++i)
                if (issued[i]) wait(bar(ctrl->v_full[i]), nph[i], never);
            for (int i = 0; i < 2; ++i)
                if (g_issued[i]) wait(bar(ctrl->vstg_full[i]), g_nph[i], never);
        } else if (warp == 1 && lane == 0) {  // MMA issuer: O += P . V
            constexpr uint32_t idesc = idesc_bf16(128, 256, false, true);
            PageIt it;
            it.init(P, &ctrl->w_r0);
            Ring vs{0, 0}, ps{0, 0};
            uint32_t ncorr = 0, nseg = 0;
            uint32_t vr_ph = 0;  // phase bit of v_ready[i]: it completes only on ragged pages
            int u = 0;
            bool ok = true, any = false;
            while (ok && !it.done()) {
                if (!(ok = wait<true>(bar(ctrl->p_full[ps.i]), ps.ph, abort_flag))) break;
                const uint32_t pa = data_s + P_OFF + ps.i * P_SLOT;
                const uint32_t flag = ld_shared_u32(pa + P_FLAG);
                mbar_arrive_expect_tx(bar(ctrl->p_full[ps.i]), MSG_BYTES);  // arm the slot's next use
                if (flag) {
                    if (!(ok = wait(bar(ctrl->corr_done), ncorr & 1u, abort_flag))) break;
                    ++ncorr;
                }
                const bool first = it.first, ragged = it.valid() < PG;
                if (first && nseg > 0) {
                    if (!(ok = wait(bar(ctrl->o_free), (nseg - 1) & 1u, abort_flag))) break;
                }
                for (int nh = 0; nh < 2; ++nh) {
                    if (ragged) {
                        ok = wait(bar(ctrl->v_ready[vs.i]), (vr_ph >> vs.i) & 1u, abort_flag);
                        vr_ph ^= 1u << vs.i;
                    } else {
                        ok = wait(bar(ctrl->v_full[vs.i]), vs.ph, abort_flag);
                    }
                    if (!ok) break;
                    tc_fence_after();
                    const uint32_t vb = data_s + V_OFF + vs.i * VH_STAGE;
#pragma unroll
                    for (int kk = 0; kk < PG / 16; ++kk) {
                        const uint64_t a = sdesc_sw128(pa + kk * 32, 16, 1024);
                        const uint64_t b = sdesc_sw128(vb + kk * 2048, CB, 1024);
                        mma_ss(tmem + nh * 256, a, b, idesc, (first && kk == 0) ? 0u : 1u);
                    }
                    mma_commit(bar(ctrl->v_empty[vs.i]));
                    vs.adv(VH_STAGES);
                }
                if (!ok) break;
                mma_commit(bar(ctrl->pv_done[ps.i]));
                mma_commit_mc(bar(ctrl->pfree[ps.i]), (uint16_t)1u);  // CTA 0's slot barrier
                any = true;
                ++u;
                if (it.last()) ++nseg;
                ps.adv(P_SLOTS);
                it.next(P);
            }
            if (!ok) fail();
            if (any) {
                mma_commit(bar(ctrl->mma_idle[0]));
                wait(bar(ctrl->mma_idle[0]), 0u, never);
            }
            // drain: messages CTA 0 may already have sent land before this CTA can leave
            if (!ok)
                for (int i = 0; i < P_SLOTS; ++i) {
                    wait<true>(bar(ctrl->p_full[ps.i]), ps.ph, never, 1000000ull);
                    ps.adv(P_SLOTS);
                }
        } else if (F8 && warp >= VC_WARP0 && warp < VC_WARP0 + 4) {  // FP8: codes -> bf16 V stages
            const int t = threadIdx.x - VC_WARP0 * 32;  // 0..127
            PageIt it;
            it.init(P, &ctrl->w_r0);
            Ring vs{0, 0}, vg{0, 0};
            bool ok = true;
            while (ok && !it.done()) {
                for (int hh = 0; hh < 2; ++hh) {
                    bool w = wait(bar(ctrl->vstg_full[vg.i]), vg.ph, abort_flag);
                    w = w && wait(bar(ctrl->v_empty[vs.i]), vs.ph ^ 1u, abort_flag);
                    if (named_red_or(!w, BAR_VCONV, VC_THREADS)) {
                        ok = false;
                        break;
                    }
                    const uint32_t src = data_s + L::vstg_off + vg.i * VSTG_SLOT;
                    const float *scl = reinterpret_cast<const float *>(smem_raw + (src - raw_s) + VSTG_CODES);
                    const uint32_t dst = data_s + V_OFF + vs.i * VH_STAGE;
#pragma unroll 4
                    for (int q = t; q < PG * (DC / 16); q += VC_THREADS) {  // 64 tokens x 32 groups
                        const int j = q >> 5, cc = q & 31;
                        dequant8(src + j * (DC / 2) + cc * 8, scl[j],
                                 dst + (cc >> 3) * CB + j * 128 + (((cc & 7) ^ (j & 7)) << 4));
                    }
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) {
                        mbar_arrive(bar(ctrl->v_full[vs.i]));
                        mbar_arrive(bar(ctrl->vstg_empty[vg.i]));
                    }
                    vs.adv(VH_STAGES);
                    vg.adv(2);
                }
                it.next(P);
            }
            if (!ok && lane == 0) fail();
        } else if (warp >= EP_WARP0 && warp < EP_WARP0 + 4) {  // ragged zeroing, rescale, epilogue
            const int quarter = warp & 3;
            const int h = quarter * 32 + lane;
            const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
            const uint32_t pfree_r = mapa(bar(ctrl->pfree[0]), 0);
            PageIt it;
            it.init(P, &ctrl->w_r0);
            Ring vs{0, 0}, ps{0, 0}, prev{0, 0};
            int u = 0;
            bool ok = true;
            while (ok && !it.done()) {
                const int valid = it.valid();
                // 1. ragged last page: zero token rows [valid, 64) of both V halves
                if (valid < PG) {
                    Ring v2 = vs;
                    for (int hh = 0; hh < 2; ++hh) {
                        if (!(ok = __all_sync(0xffffffffu, wait(bar(ctrl->v_full[v2.i]), v2.ph, abort_flag)))) break;
                        const int nz = PG - valid;
                        const uint32_t vb = data_s + V_OFF + v2.i * VH_STAGE;
                        for (int i = h; i < nz * 4 * 8; i += 128) {  // 4 tiles x nz rows x 8 chunks
                            const int c = i & 7, pr = i >> 3;
                            const int cb = pr / nz, row = valid + pr % nz;
                            st_shared_v4(vb + cb * CB + row * 128 + c * 16, 0u, 0u, 0u, 0u);
                        }
                        fence_proxy_async_smem();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(bar(ctrl->v_ready[v2.i]));
                        v2.adv(VH_STAGES);
                    }
                    if (!ok) break;
                }
                // 2. the P message: this head's factor and the flag; then free the slot for reading
                if (!(ok = __all_sync(0xffffffffu, wait<true>(bar(ctrl->p_full[ps.i]), ps.ph, abort_flag)))) break;
                const uint32_t pa = data_s + P_OFF + ps.i * P_SLOT;
                const float fac = __uint_as_float(ld_shared_u32(pa + P_FACT + h * 4));
                const uint32_t flag = ld_shared_u32(pa + P_FLAG);
                __syncwarp();
                if (lane == 0) mbar_arrive_remote(pfree_r + ps.i * 8);
                const bool last = it.last();
                // 3. lazy rescale of O rows whose running max moved (the previous page's PV done)
                if (flag) {
                    if (!(ok = __all_sync(0xffffffffu, wait(bar(ctrl->pv_done[prev.i]), prev.ph, abort_flag)))) break;
                    tc_fence_after();
                    if (__any_sync(0xffffffffu, fac != 1.f)) {
#pragma unroll 1
                        for (int ch = 0; ch < DC / 32; ++ch) {
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
                // 4. end of segment: this warp writes its 32 heads of the partial O (not normalised)
                // as bf16 pairs of columns, [slot][d_c / 2][n_h] words, so that each store
                // instruction of the warp covers one whole 128-byte line (32 heads, one pair).
                if (last) {
                    if (!(ok = __all_sync(0xffffffffu, wait(bar(ctrl->pv_done[ps.i]), ps.ph, abort_flag)))) break;
                    tc_fence_after();
                    uint32_t *dst = P.o_part + (size_t)(pair + it.r) * (DC / 2) * NH + h;
#pragma unroll 1
                    for (int ch = 0; ch < DC / 32; ++ch) {
                        uint32_t v[32];
                        tmem_ld32(tmem + lane_base + ch * 32, v);
                        tmem_wait_ld();
#pragma unroll
                        for (int j = 0; j < 16; ++j)
                            __stcg(dst + (size_t)(ch * 16 + j) * NH,
                                   pack_bf16x2(__uint_as_float(v[2 * j]), __uint_as_float(v[2 * j + 1])));
                    }
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(bar(ctrl->o_free));
                }
                ++u;
                prev = ps;
                vs.adv(VH_STAGES, 2);
                ps.adv(P_SLOTS);
                it.next(P);
            }
            if (!ok && lane == 0) fail();
        }
    }

    // ---- teardown: both CTAs quiesce before either releases TMEM or exits ----
    __syncwarp();
    tc_fence_before();
    __syncthreads();
    cluster_sync();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}

// ---- combine: exact log-sum-exp merge of a row's segment partials --------------------------
// Block (row r, 16-column chunk); thread = head.  For head h with segments s of the row,
//     M = max_s m_s,  w_s = 2^(m_s - M),  L = sum_s w_s l_s,
//     o_lat[r,h,c] = sum_s w_s O_s[c,h] / L,   lse[r,h] = (M + log2 L) ln 2.
// Partials are bf16 pairs of columns, [slot][d_c / 2][n_h] words, so every load instruction of a
// warp reads one 128-byte line.  Empty slots (m = -inf: a cluster that got none of the row's
// pages) have weight 0 and are not read.
constexpr int CMB_COLS = 16;
constexpr int CMB_FAST = 8;  // rows split over at most this many slots take the fast path
__global__ void __launch_bounds__(NH)
combine_tc_kernel(const int32_t *__restrict__ seg_range, const uint32_t *__restrict__ o_part,
                  const float *__restrict__ m_part, const float *__restrict__ l_part,
                  float *__restrict__ o_lat, float *__restrict__ lse, int vec_out) {
    const int r = blockIdx.x, cc = blockIdx.y, h = threadIdx.x;
    pdl_trigger();  // the output projection may start fetching its weights
    pdl_wait();     // the partials of the main kernel
    const int s0 = seg_range[2 * r], s1 = seg_range[2 * r + 1];
    float M = -INFINITY, L = 0.f, acc[CMB_COLS];
#pragma unroll
    for (int j = 0; j < CMB_COLS; ++j) acc[j] = 0.f;
    if (s1 - s0 <= CMB_FAST) {
        // Common case: all loads of the row's slots are issued before any is used.
        float ms[CMB_FAST], ls[CMB_FAST];
        uint32_t v[CMB_FAST][CMB_COLS / 2];
#pragma unroll
        for (int i = 0; i < CMB_FAST; ++i) {
            const int s = s0 + i;
            ms[i] = -INFINITY;
            ls[i] = 0.f;
            if (s < s1) {
                ms[i] = __ldcg(m_part + (size_t)s * NH + h);
                ls[i] = __ldcg(l_part + (size_t)s * NH + h);
                const uint32_t *src = o_part + ((size_t)s * (DC / 2) + cc * (CMB_COLS / 2)) * NH + h;
#pragma unroll
                for (int k = 0; k < CMB_COLS / 2; ++k) v[i][k] = __ldcg(src + (size_t)k * NH);
            }
        }
#pragma unroll
        for (int i = 0; i < CMB_FAST; ++i) M = fmaxf(M, ms[i]);
#pragma unroll
        for (int i = 0; i < CMB_FAST; ++i) {
            // empty slots (m = -inf) and slots past the row's range have weight 0: their (never
            // written) partials must not enter the sums, not even as 0 * NaN
            if (ms[i] == -INFINITY) continue;
            const float w = exp2f(ms[i] - M);
            L = fmaf(w, ls[i], L);
#pragma unroll
            for (int k = 0; k < CMB_COLS / 2; ++k) {
                acc[2 * k] = fmaf(w, __uint_as_float(v[i][k] << 16), acc[2 * k]);
                acc[2 * k + 1] = fmaf(w, __uint_as_float(v[i][k] & 0xffff0000u), acc[2 * k + 1]);
            }
        }
    } else {
        for (int s = s0; s < s1; ++s) M = fmaxf(M, __ldcg(m_part + (size_t)s * NH + h));
#pragma unroll 2
        for (int s = s0; s < s1; ++s) {
            const float ms = __ldcg(m_part + (size_t)s * NH + h);
            if (ms == -INFINITY) continue;  // empty slot (uniform across the block)
            const float w = exp2f(ms - M);
            L = fmaf(w, __ldcg(l_part + (size_t)s * NH + h), L);
            const uint32_t *src = o_part + ((size_t)s * (DC / 2) + cc * (CMB_COLS / 2)) * NH + h;
            uint32_t v[CMB_COLS / 2];
#pragma unroll
            for (int k = 0; k < CMB_COLS / 2; ++k) v[k] = __ldcg(src + (size_t)k * NH);
#pragma unroll
            for (int k = 0; k < CMB_COLS / 2; ++k) {
                acc[2 * k] = fmaf(w, __uint_as_float(v[k] << 16), acc[2 * k]);
                acc[2 * k + 1] = fmaf(w, __uint_as_float(v[k] & 0xffff0000u), acc[2 * k + 1]);
            }
        }
    }
    const float inv = L > 0.f ? 1.f / L : 0.f;
    float *out = o_lat + ((size_t)r * NH + h) * DC + cc * CMB_COLS;
    if (vec_out) {  // o_lat 16-byte aligned
        float4 *dst = reinterpret_cast<float4 *>(out);
#pragma unroll
        for (int j = 0; j < CMB_COLS / 4; ++j)
            dst[j] = make_float4(acc[4 * j] * inv, acc[4 * j + 1] * inv, acc[4 * j + 2] * inv, acc[4 * j + 3] * inv);
    } else {
#pragma unroll
        for (int j = 0; j < CMB_COLS; ++j) out[j] = acc[j] * inv;
    }
    if (lse && cc == 0) lse[(size_t)r * NH + h] = L > 0.f ? (M + log2f(L)) * 0.69314718055994531f : -INFINITY;
}

// ---- host side ------------------------------------------------------------------------------
int g_pairs[3][64] = {};  // [bf16 | FP8 | FP8 with the content scores on the FP8 tensor core][device]
std::mutex g_pairs_mu;

// Co-resident clusters of the kernel on the current device (cached per device; the first call
// on a device sets the kernel's shared-memory attribute and queries the occupancy, under a lock
// so that concurrent first calls from several host threads do it once).
template <bool F8, bool MM = false>
int tc_pairs() {
    constexpr int K = F8 ? (MM ? 2 : 1) : 0;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
    std::lock_guard<std::mutex> lk(g_pairs_mu);
    if (g_pairs[K][dev]) return g_pairs[K][dev];
    if (cudaFuncSetAttribute(decode_tc_kernel<F8, MM>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             Lay<F8, MM>::smem) !=
        cudaSuccess)
        return 0;
    int sms = 148;
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * (sms / 2));
    cfg.blockDim = dim3(THREADS);
    cfg.dynamicSmemBytes = Lay<F8, MM>::smem;
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeClusterDimension;
    attr.val.clusterDim.x = 2;
    attr.val.clusterDim.y = 1;
    attr.val.clusterDim.z = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, decode_tc_kernel<F8, MM>, &cfg) != cudaSuccess || n < 1) {
        cudaGetLastError();
        n = sms / 2;
    }
    g_pairs[K][dev] = n;
    return n;
}
int tc_pairs(const mla_dims_t &d) {
    if (d.kv_dtype != MLA_DTYPE_FP8_E4M3) return tc_pairs<false>();
    return (d.flags & MLA_FLAG_FP8_MMA) ? tc_pairs<true, true>() : tc_pairs<true>();
}

struct TcWs {
    uint32_t *o;  // bf16 pairs
    float *m, *l;
    int32_t *seg_range;
};

size_t tc_layout(int pairs, int rows, char *base, TcWs *w) {
    const size_t slots = (size_t)pairs + rows;
    size_t off = 0;
    auto take = [&](size_t bytes) {
        char *p = base ? base + off : nullptr;
        off += align_up(bytes, 256);
        return p;
    };
    char *o = take(slots * NH * (DC / 2) * sizeof(uint32_t));
    char *m = take(slots * NH * sizeof(float));
    char *l = take(slots * NH * sizeof(float));
    char *sr = take((size_t)rows * 2 * sizeof(int32_t));
    if (w) {
        w->o = reinterpret_cast<uint32_t *>(o);
        w->m = reinterpret_cast<float *>(m);
        w->l = reinterpret_cast<float *>(l);
        w->seg_range = reinterpret_cast<int32_t *>(sr);
    }
    return off;
}

}  // namespace

bool tc_supported(const mla_dims_t &d) {
    return d.n_h == NH && d.d_c == DC && d.d_r == ROW - DC && d.page_size == PG &&
           d.act_dtype == MLA_DTYPE_BF16 && (d.kv_dtype == MLA_DTYPE_BF16 || d.kv_dtype == MLA_DTYPE_FP8_E4M3);
}

size_t tc_workspace_bytes(const mla_dims_t &d, int B, int s_q, int) {
    const int pairs = tc_pairs(d);
    if (pairs < 1) return 0;
    return tc_layout(pairs, B * s_q, nullptr, nullptr);
}

cudaError_t launch_decode_tc(const mla_dims_t &d, int B, int s_q, const void *q_abs,
                             const void *kv_pool, const void *kr_pool, const float *kv_scale, const int32_t *bt,
                             int max_blocks, int num_blocks, const int32_t *seq_lens, int max_seq_len,
                             void *ws, size_t ws_bytes, float *o_lat, float *lse, cudaStream_t st,
                             const FusedOutProj *fuse) {
    const int rows = B * s_q;
    const bool f8 = d.kv_dtype == MLA_DTYPE_FP8_E4M3;
    const int pairs = tc_pairs(d);
    if (pairs < 1) return cudaErrorNotSupported;
    TcWs w;
    if (tc_layout(pairs, rows, reinterpret_cast<char *>(ws), &w) > ws_bytes) return cudaErrorInvalidValue;
    CUtensorMap tm_kv9, tm_kv4, tm_q9, tm_c8;
    const bool mm = f8 && (d.flags & MLA_FLAG_FP8_MMA);
    const uint64_t pool_rows = (uint64_t)num_blocks * PG, q_rows = (uint64_t)rows * NH;
    const bool maps =
        f8 ? (tmap_bf16_2d(&tm_kv9, kr_pool, ROW - DC, pool_rows, (ROW - DC) * 2, 64, PG) &&
              tmap_u8_rows(&tm_kv4, kv_pool, DC, pool_rows, DC, DC / 2, PG))
           : (tmap_bf16_colblocks(&tm_kv9, kv_pool, pool_rows, ROW, ROW * 2, PG, NCB) &&
              tmap_bf16_colblocks(&tm_kv4, kv_pool, pool_rows, ROW, ROW * 2, PG, 4));
    if (!maps || !tmap_bf16_colblocks(&tm_q9, q_abs, q_rows, ROW, ROW * 2, 64, NCB)) return cudaErrorInvalidValue;
    // FP8 with the content scores on the tensor core: the codes as 4 K-major 128-byte blocks
    // per page (the map is passed, unused, to the other instantiations)
    if (mm ? !tmap_u8_colblocks(&tm_c8, kv_pool, pool_rows, DC, DC, PG, 4) : false) return cudaErrorInvalidValue;
    if (!mm) tm_c8 = tm_q9;
    unsigned *err = device_error_word();
    cudaError_t e;
    Params P;
    P.bt = bt;
    P.max_blocks = max_blocks;
    P.num_blocks = num_blocks;
    P.seq_lens = seq_lens;
    P.s_q = s_q;
    P.rows = rows;
    P.max_seq_len = max_seq_len;
    P.pairs = pairs;
    P.seg_range = w.seg_range;
    P.o_part = w.o;
    P.m_part = w.m;
    P.l_part = w.l;
    P.scale_log2 = (float)(1.4426950408889634 / sqrt((double)(d.d_h + d.d_r)));
    P.err = err;
    P.test_give_up = (d.flags & MLA_FLAG_TEST_GIVE_UP) ? 1 : 0;
    P.codes = f8 ? reinterpret_cast<const uint8_t *>(kv_pool) : nullptr;
    P.kv_scale = f8 ? kv_scale : nullptr;
    // The main and combine kernels are launched as programmatic dependents of the kernel before
    // them: their blocks may start while it drains, and they wait for its results on the device
    // before reading any input.
    cudaLaunchAttribute pdl;
    pdl.id = cudaLaunchAttributeProgrammaticStreamSerialization;
    pdl.val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * pairs);
    cfg.blockDim = dim3(THREADS);
    cfg.dynamicSmemBytes = mm ? Lay<true, true>::smem : (f8 ? Lay<true>::smem : Lay<false>::smem);
    cfg.stream = st;
    cfg.attrs = &pdl;
#ifdef MLA_NO_PDL
    cfg.numAttrs = 0;
#else
    cfg.numAttrs = 1;
#endif
    e = mm   ? cudaLaunchKernelEx(&cfg, decode_tc_kernel<true, true>, tm_kv9, tm_kv4, tm_q9, tm_c8, P)
        : f8 ? cudaLaunchKernelEx(&cfg, decode_tc_kernel<true>, tm_kv9, tm_kv4, tm_q9, tm_c8, P)
             : cudaLaunchKernelEx(&cfg, decode_tc_kernel<false>, tm_kv9, tm_kv4, tm_q9, tm_c8, P);
    if (e != cudaSuccess) return e;
    if (fuse)
        return launch_combine_out_proj_tc(d, rows, w.seg_range, w.o, w.m, w.l, o_lat, lse, fuse->w_uv, fuse->o,
                                          fuse->out_dtype, st);
    const int vec_out = (reinterpret_cast<uintptr_t>(o_lat) & 15) == 0;
    cfg.gridDim = dim3(rows, DC / CMB_COLS);
    cfg.blockDim = dim3(NH);
    cfg.dynamicSmemBytes = 0;
    return cudaLaunchKernelEx(&cfg, combine_tc_kernel, (const int32_t *)w.seg_range, (const uint32_t *)w.o,
                              (const float *)w.m, (const float *)w.l, o_lat, lse, vec_out);
}

}  // namespace mla
