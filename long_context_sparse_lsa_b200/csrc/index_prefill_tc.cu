// index_prefill_tc.cu — fine indexer scores of a causal prefill chunk as one
// dense int8 contraction on the 5th-generation tensor cores.
//
// The method: the same score as the decode indexer, score_t = sum_h w_h *
// ReLU(q_h . k_t), for every middle token of every query row of the chunk
// ("LongCat-2.0 (molayo1419.me)", section "1M 토큰에서의 Sparse Attention 문제":
// LSA keeps DSA's lightning indexer, which scores every cached token; with HI
// off every middle token is a candidate). Each query token i of a chunk
// appended to a cache of C tokens sees C + i + 1 tokens.
//
// Design (B200): D[token, (row, head)] = K . Q^T on tcgen05.mma kind::i8 with
// int32 accumulators in tensor memory (TMEM).
//  * A = 128 cached tokens: one TMA tile of 128 key rows (128 bytes each),
//    128-byte swizzle, through a ring of stages. B = 256 query-head rows
//    (256 / H_I query rows x H_I heads) of the CTA, loaded once and resident.
//    K = d_I = 128 in four 32-byte MMA steps.
//  * Tokens are the MMA's M dimension so that the head reduction is a
//    per-thread loop in the epilogue: a thread owns one TMEM lane (one token),
//    reads its row of accumulators, applies ReLU and the query row's weights,
//    sums each row's heads into the key (score + 1) of that (row, token), and
//    keeps the key as a candidate only if it passes the row's running
//    threshold (the filter below), so the selection reads a few percent of
//    the keys instead of all of them.
//  * Warp roles: warp 0 issues the TMA loads, one thread of warp 1 issues the
//    MMAs, warps 2..17 drain the accumulators (four warps per TMEM lane
//    quarter, each taking a quarter of the columns: four query rows, read 16
//    columns at a time). TMEM holds two 256-column accumulators so the MMAs of
//    tile j+1 overlap the epilogue of tile j.
//  * Every mbarrier wait is bounded; on expiry the kernel flags
//    LSA_DEV_TIMEOUT, stops issuing work, waits (bounded) for what it issued,
//    frees its TMEM and returns.
#include <cuda.h>

#include <cstddef>
#include <cstring>
#include <type_traits>

#include "common.cuh"
#include "internal.h"

namespace lsa {
namespace {

constexpr int kTcTokens = LSA_TC_TOKENS;             // M: cached tokens per tile
constexpr int kTcCols = 256;                         // N: query-head rows per CTA
constexpr int kTcK = 128;                            // d_I bytes per key row
constexpr int kTcStages = 6;                         // A-tile ring
constexpr int kTcEpiWarps = 16;  // four per TMEM lane quarter, each a quarter of the columns
constexpr int kTcThreads = (2 + kTcEpiWarps) * kWarp;
constexpr uint32_t kATileBytes = kTcTokens * kTcK;   // 16 KB
constexpr uint32_t kBTileBytes = kTcCols * kTcK;     // 32 KB
constexpr uint32_t kTmemCols = 2 * kTcCols;          // two accumulators

// Instruction descriptor of tcgen05.mma kind::i8: s32 accumulate, s8 A and B,
// both K-major, N = 256, M = 128.
constexpr uint32_t kIdesc = (2u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(kTcCols >> 3) << 17) |
                            ((uint32_t)(kTcTokens >> 4) << 24);

struct TcArgs {
    CUtensorMap tmap_k;  // key cache [total_tokens, 128] int8, box 128 x 128, 128-byte swizzle
    CUtensorMap tmap_q;  // queries [n_q * H_I, 128] int8, box 256 x 128, 128-byte swizzle
    const int32_t* w;
    const int32_t* q_seq;
    const int32_t* q_len;
    const int64_t* kv_offset;
    const int32_t* seq_lens;
    uint64_t* cand;        // [n_q][fine_cap] candidates: key << 32 | position
    int32_t* cand_seg;     // [n_q][kTcMaxSplits][4][2] (first slot, count) per token split and lane quarter
    uint32_t* ghist;       // [n_q][kTcBins] the row's counts over every split (zeroed before the launch)
    int32_t* dev_status;
    int64_t total_tokens;
    int32_t n_q, max_len, w_max, sink, window, fine_cap, topk;
};

// Candidate filter. A row's kept keys (those at or above its threshold) are
// counted in a histogram of kTcBins bins on a logarithmic scale (bit length
// and the 4 bits after the leading one). Every kTcUpdate tiles each CTA adds
// its counts into the row's histogram in global memory, shared by the CTAs
// of every token split, and reads it back; the lower edge of the highest bin
// whose count from the top reaches topk becomes the row's threshold. Every
// counted key is a distinct token of the row, so at least topk of the row's
// keys lie at or above the threshold: it never exceeds the row's k-th largest
// key, and every key of the final top-k, being at least the threshold in
// force when it is scored, is kept as a candidate.
constexpr int kTcBins = LSA_TC_BINS;
constexpr int kTcMaxSplits = LSA_TC_MAX_SPLITS;
static_assert(LSA_TC_SEGS == 4, "one candidate segment per TMEM lane quarter");
constexpr int kTcUpdate = 8;
constexpr int kTcBinsPerLane = kTcBins / 32;  // a warp scans a row's histogram, lane l bins l*this..
static_assert(kTcBins == 512, "bit length (5 bits) x 16 sub-bins");
__device__ __forceinline__ uint32_t tc_bin(uint32_t key) {
    if (key < 16u) return key;
    const int nb = 32 - __clz((int)key);  // 5..32
    return ((uint32_t)(nb - 4) << 4) | ((key >> (nb - 5)) & 15u);
}
__device__ __forceinline__ uint32_t tc_bin_floor(uint32_t b) {
    if (b < 16u) return b;
    return (16u | (b & 15u)) << ((b >> 4) - 1u);
}

struct TcShared {
    uint64_t full[kTcStages];
    uint64_t empty[kTcStages];
    uint64_t bfull;
    uint64_t tfull[2];
    uint64_t tempty[2];
    uint64_t drain;  // completion of every MMA issued, before TMEM is freed
    uint32_t tmem_base;
    int32_t abort;
    int32_t row_s[kTcCols];   // per query row of the CTA: middle start,
    int32_t row_ws[kTcCols];  // window start (= middle end),
    int32_t row_ok[kTcCols];  // and validity
    alignas(16) int32_t w[kTcCols];  // weight of each query-head row (read as 16-byte vectors)
    uint32_t thr[kTcCols / 16];             // per query row of the CTA: candidate threshold
    uint32_t hist[kTcCols / 16][kTcBins];   // per query row: kept keys here not yet added to ghist
};
static_assert(offsetof(TcShared, w) % 16 == 0, "weights are read with 16-byte shared loads");
static_assert(sizeof(TcShared) % 16 == 0, "TcShared follows 1024-byte aligned tiles");

constexpr size_t kTcSmem = 1024 + (size_t)kTcStages * kATileBytes + kBTileBytes + sizeof(TcShared);

// Shared-memory matrix descriptor: K-major, 128-byte swizzle, rows of 128
// bytes, 8-row groups 1024 bytes apart (the layout a 128-byte-swizzled TMA
// tile of 128-byte rows has).
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
    uint64_t d = (uint64_t)((saddr & 0x3FFFFu) >> 4);
    d |= (uint64_t)1 << 16;             // leading byte offset (unused with this swizzle)
    d |= (uint64_t)(1024 >> 4) << 32;   // stride byte offset: 8 rows x 128 B
    d |= (uint64_t)1 << 46;             // descriptor version
    d |= (uint64_t)2 << 61;             // 128-byte swizzle
    return d;
}

__device__ __forceinline__ void umma_i8(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t accumulate) {
    asm volatile(
        "{\n .reg .pred p;\n setp.ne.b32 p, %3, 0;\n"
        " tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %4, p;\n}\n" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(accumulate), "r"(kIdesc)
        : "memory");
}
__device__ __forceinline__ void umma_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
                 : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }


// 32 consecutive accumulator columns of this warp's 32 TMEM lanes. The load
// is asynchronous: its registers are valid only after tmem_wait(v), which
// names them as operands so that no use can be scheduled before the wait.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&v)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];\n"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
          "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15]),
          "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]),
          "=r"(v[24]), "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
        : "r"(taddr));
}
__device__ __forceinline__ void tmem_wait(uint32_t (&v)[32]) {
    asm volatile("tcgen05.wait::ld.sync.aligned;"
                 : "+r"(v[0]), "+r"(v[1]), "+r"(v[2]), "+r"(v[3]), "+r"(v[4]), "+r"(v[5]), "+r"(v[6]), "+r"(v[7]),
                   "+r"(v[8]), "+r"(v[9]), "+r"(v[10]), "+r"(v[11]), "+r"(v[12]), "+r"(v[13]), "+r"(v[14]),
                   "+r"(v[15]), "+r"(v[16]), "+r"(v[17]), "+r"(v[18]), "+r"(v[19]), "+r"(v[20]), "+r"(v[21]),
                   "+r"(v[22]), "+r"(v[23]), "+r"(v[24]), "+r"(v[25]), "+r"(v[26]), "+r"(v[27]), "+r"(v[28]),
                   "+r"(v[29]), "+r"(v[30]), "+r"(v[31])
                 :
                 : "memory");
}

// 16 consecutive accumulator columns of this warp's 32 TMEM lanes (as tmem_ld32).
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&v)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15}, [%16];\n"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
          "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
        : "r"(taddr));
}
__device__ __forceinline__ void tmem_wait(uint32_t (&v)[16]) {
    asm volatile("tcgen05.wait::ld.sync.aligned;"
                 : "+r"(v[0]), "+r"(v[1]), "+r"(v[2]), "+r"(v[3]), "+r"(v[4]), "+r"(v[5]), "+r"(v[6]), "+r"(v[7]),
                   "+r"(v[8]), "+r"(v[9]), "+r"(v[10]), "+r"(v[11]), "+r"(v[12]), "+r"(v[13]), "+r"(v[14]),
                   "+r"(v[15])
                 :
                 : "memory");
}

// Bounded wait shared by every role: on expiry flags the timeout and raises
// the CTA's abort flag.
__device__ __forceinline__ bool tc_wait(TcShared& sh, uint32_t bar, uint32_t parity, int32_t* status) {
    if (mbar_wait_bounded(bar, parity, kWaitLimitNs)) return true;
    flag(status, LSA_DEV_TIMEOUT);
    atomicExch(&sh.abort, 1);
    return false;
}
__device__ __forceinline__ bool tc_aborted(const TcShared& sh) {
    return *reinterpret_cast<const volatile int32_t*>(&sh.abort) != 0;
}

template <int H_I>
__global__ void __launch_bounds__(kTcThreads, 1) fine_score_tc_kernel(const __grid_constant__ TcArgs a) {
    pdl_enter();
    constexpr int R = kTcCols / H_I;  // query rows per CTA
    extern __shared__ __align__(16) uint8_t dyn_raw[];
    const uint32_t raw = smem_u32(dyn_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;  // 1024-byte aligned tiles (128-byte swizzle atoms)
    uint8_t* dyn = dyn_raw + (base - raw);
    const uint32_t sA = base;                                  // kTcStages x 16 KB
    const uint32_t sB = base + kTcStages * kATileBytes;        // 32 KB
    TcShared& sh = *reinterpret_cast<TcShared*>(dyn + kTcStages * kATileBytes + kBTileBytes);
    const int warp = warp_id(), lane = lane_id(), tid = threadIdx.x;
    const int row0 = blockIdx.y * R;

    // ---- setup: barriers, TMEM, the CTA's query rows -----------------------
    if (tid == 0) {
        for (int i = 0; i < kTcStages; ++i) {
            mbar_init(smem_u32(&sh.full[i]), 1);
            mbar_init(smem_u32(&sh.empty[i]), 1);
        }
        mbar_init(smem_u32(&sh.bfull), 1);
        mbar_init(smem_u32(&sh.drain), 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(smem_u32(&sh.tfull[i]), 1);
            mbar_init(smem_u32(&sh.tempty[i]), kTcEpiWarps);
        }
        sh.abort = 0;
        mbar_fence_init();
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&sh.tmem_base)),
                     "r"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    bool bad_w = false;
    for (int n = tid; n < kTcCols; n += kTcThreads) {
        const int r = row0 + n / H_I;
        int32_t wv = 0;
        if (r < a.n_q) {
            wv = a.w[(int64_t)r * H_I + n % H_I];
            if (wv < 0 || wv > a.w_max) {
                bad_w = true;
                wv = 0;
            }
        }
        sh.w[n] = wv;
    }
    if (bad_w) flag(a.dev_status, LSA_DEV_BAD_WEIGHT);
    const int64_t off = a.kv_offset[0];
    const int slen = a.seq_lens[0];
    for (int i = tid; i < R; i += kTcThreads) {
        const int r = row0 + i;
        int ok = 0, s = 0, ws = 0;
        if (r < a.n_q) {
            const int L = a.q_len[r];
            ok = a.q_seq[r] == 0 && L >= 1 && L <= a.max_len && L <= slen && off >= 0 &&
                 off + slen <= a.total_tokens;
            s = min(a.sink, L);
            ws = max(s, L - a.window);
        }
        sh.row_ok[i] = ok;
        sh.row_s[i] = s;
        sh.row_ws[i] = ws;
        sh.thr[i] = 1u;  // every key (score + 1 >= 1) until the histogram holds topk keys
    }
    for (int i = tid; i < R * kTcBins; i += kTcThreads) (&sh.hist[0][0])[i] = 0u;
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sh.tmem_base;

    // token range: the union of the rows' middles, split over gridDim.x
    int t_lo = 0x7fffffff, t_hi = 0;
    for (int i = 0; i < R; ++i) {
        if (sh.row_ok[i] && sh.row_ws[i] > sh.row_s[i]) {
            t_lo = min(t_lo, sh.row_s[i]);
            t_hi = max(t_hi, sh.row_ws[i]);
        }
    }
    const int nt_all = t_hi > t_lo ? (t_hi - t_lo + kTcTokens - 1) / kTcTokens : 0;
    const int j_lo = (int)((int64_t)nt_all * blockIdx.x / gridDim.x);
    const int j_hi = (int)((int64_t)nt_all * (blockIdx.x + 1) / gridDim.x);
    const int nt = j_hi - j_lo;


    if (warp == 0) {
        // ---- TMA producer ---------------------------------------------------
        if (lane == 0 && nt > 0) {
            mbar_arrive_expect_tx(smem_u32(&sh.bfull), kBTileBytes);
            tma_load_2d(sB, &a.tmap_q, 0, row0 * H_I, smem_u32(&sh.bfull));
            int issued = 0;
            for (int j = 0; j < nt; ++j) {
                const int st = j % kTcStages;
                if (j >= kTcStages && !tc_wait(sh, smem_u32(&sh.empty[st]), ((j / kTcStages) + 1) & 1, a.dev_status))
                    break;
                if (tc_aborted(sh)) break;
                mbar_arrive_expect_tx(smem_u32(&sh.full[st]), kATileBytes);
                tma_load_2d(sA + st * kATileBytes, &a.tmap_k, 0, (int)(off + t_lo + (j_lo + j) * kTcTokens),
                            smem_u32(&sh.full[st]));
                ++issued;
            }
            // wait (bounded) until every issued copy has landed before the CTA can exit
            for (int j = (issued > kTcStages ? issued - kTcStages : 0); j < issued; ++j)
                mbar_wait_bounded(smem_u32(&sh.full[j % kTcStages]), (j / kTcStages) & 1, kWaitLimitNs);
            mbar_wait_bounded(smem_u32(&sh.bfull), 0, kWaitLimitNs);
        }
    } else if (warp == 1) {
        // ---- MMA issuer -----------------------------------------------------
        if (lane == 0 && nt > 0) {
            bool ok = tc_wait(sh, smem_u32(&sh.bfull), 0, a.dev_status);
            const uint64_t bdesc = sw128_desc(sB);
            for (int j = 0; ok && j < nt; ++j) {
                const int st = j % kTcStages, buf = j & 1, use = j >> 1;
                if (!tc_wait(sh, smem_u32(&sh.full[st]), (j / kTcStages) & 1, a.dev_status)) break;
                if (use >= 1 && !tc_wait(sh, smem_u32(&sh.tempty[buf]), (use - 1) & 1, a.dev_status)) break;
                if (tc_aborted(sh)) break;
                tc_fence_after();
                const uint64_t adesc = sw128_desc(sA + st * kATileBytes);
                const uint32_t d = tmem + (uint32_t)(buf * kTcCols);
#pragma unroll
                for (int k = 0; k < kTcK / 32; ++k)  // 32-byte K steps: +2 in the 16-byte address units
                    umma_i8(d, adesc + (uint64_t)(2 * k), bdesc + (uint64_t)(2 * k), k > 0 ? 1u : 0u);
                umma_commit(smem_u32(&sh.empty[st]));
                umma_commit(smem_u32(&sh.tfull[buf]));
            }
        }
    } else {
        // ---- epilogue: TMEM -> keys ---------------------------------------------
        static_assert(H_I == 16, "one 16-column TMEM load per query row");
        constexpr int kParts = kTcEpiWarps / 4;        // warps per TMEM lane quarter
        constexpr int kCols = kTcCols / kParts;        // accumulator columns of a warp
        constexpr int kRows = kCols / H_I;             // its query rows
        const int quarter = warp & 3;                  // TMEM lanes 32*quarter .. +31
        const int part = (warp - 2) >> 2;              // accumulator columns kCols*part ..
        const int lane_tok = 32 * quarter + lane;
        // the warp's row bounds stay in registers for every tile; its weights
        // are re-read per row with warp-wide broadcast 16-byte loads (volatile,
        // so they are not hoisted out of the tile loop)
        const uint32_t wsh = smem_u32(&sh.w[kCols * part]);
        const int rl0 = kRows * part;  // first query row (of the CTA) of this warp's columns
        int32_t rs[kRows], rws[kRows];
#pragma unroll
        for (int i = 0; i < kRows; ++i) {
            rs[i] = sh.row_ok[rl0 + i] ? sh.row_s[rl0 + i] : 0x7fffffff;  // invalid row: no token qualifies
            rws[i] = sh.row_ws[rl0 + i];
        }
        int rs_max = 0, rws_min = 0x7fffffff;
#pragma unroll
        for (int i = 0; i < kRows; ++i) {
            rs_max = max(rs_max, rs[i]);
            rws_min = min(rws_min, rws[i]);
        }
        // This warp's candidates of each of its rows go to its own slots: the
        // slots of the CTA's tokens (from the union's first middle token; splits
        // are disjoint and the union spans at most fine_cap slots), quarter q of
        // them for lane quarter q: one slot per token the warp scores, so the
        // count lives in a register and no slot is reserved atomically.
        const int64_t seg_q = (int64_t)j_lo * kTcTokens + (int64_t)quarter * nt * kWarp;
        const int64_t room = (int64_t)a.fine_cap - seg_q;
        uint64_t* cand0 = a.cand + (int64_t)(row0 + rl0) * a.fine_cap + seg_q;
        const uint32_t lt_mask = (1u << lane) - 1u;
        uint32_t cnt[kRows], thr[kRows];
#pragma unroll
        for (int i = 0; i < kRows; ++i) {
            cnt[i] = 0u;
            thr[i] = 1u;
        }
        // one query row's 16 accumulator columns -> its key, kept if it passes
        auto row_of = [&](const uint32_t (&v)[16], int i, int t, auto all_in) {
            int32_t w[16];
#pragma unroll
            for (int q = 0; q < 4; ++q)
                asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                             : "=r"(w[4 * q]), "=r"(w[4 * q + 1]), "=r"(w[4 * q + 2]), "=r"(w[4 * q + 3])
                             : "r"(wsh + 4u * (uint32_t)(H_I * i + 4 * q)));
            // four independent partial sums: a 16-long chain of dependent
            // multiply-adds would stall on its own latency
            int32_t acc4[4] = {0, 0, 0, 0};
#pragma unroll
            for (int h = 0; h < H_I; ++h) acc4[h & 3] += max((int32_t)v[h], 0) * w[h];
            const int32_t acc = (acc4[0] + acc4[1]) + (acc4[2] + acc4[3]);
            const uint32_t key = (uint32_t)acc + 1u;
            const bool emit = key >= thr[i] && (decltype(all_in)::value || (t >= rs[i] && t < rws[i]));
            const uint32_t m = __ballot_sync(0xffffffffu, emit);
            if (m != 0u) {  // warp-uniform: most rows of a tile keep nothing once their threshold has risen
                if (emit) {
                    atomicAdd(&sh.hist[rl0 + i][tc_bin(key)], 1u);
                    const uint32_t slot = cnt[i] + __popc(m & lt_mask);
                    if ((int64_t)slot < room)
                        cand0[(int64_t)i * a.fine_cap + slot] = ((uint64_t)key << 32) | (uint32_t)t;
                }
                cnt[i] += __popc(m);
            }
        };
        // Threshold updates of this warp's query row (row w' of the CTA, w'
        // the epilogue warp index), spread over three tiles so that the global
        // round trip overlaps the tiles' work: flush() adds the CTA's new
        // counts into the row's global histogram (reductions, no value
        // returned) and loads its totals (lane l: its kTcBinsPerLane bins, the
        // loads in flight while the next tiles are scored); settle() turns them
        // into the threshold two tiles later; the warps of the row read it back
        // a tile after that. A load may miss other CTAs' latest counts: fewer
        // counted keys only lower the threshold.
        const int urow = warp - 2;
        const bool ulive = row0 + urow < a.n_q;
        uint32_t gc[kTcBinsPerLane];
        // Only the bins at or above the row's threshold bin are touched: no
        // key below the threshold is counted, and the threshold only rises.
        auto flush = [&]() {
            const uint32_t tb = tc_bin(*reinterpret_cast<volatile uint32_t*>(&sh.thr[urow]));
            uint32_t* g = a.ghist + (int64_t)(ulive ? row0 + urow : 0) * kTcBins + kTcBinsPerLane * lane;
#pragma unroll
            for (int j = 0; j < kTcBinsPerLane; ++j) {
                const uint32_t b = (uint32_t)(kTcBinsPerLane * lane + j);
                uint32_t c = 0u;
                if (ulive && b >= tb) {
                    const uint32_t d = atomicExch(&sh.hist[urow][b], 0u);
                    if (d != 0u) atomicAdd(g + j, d);  // result unused: a reduction
                    c = __ldcg(g + j);
                }
                gc[j] = c;
            }
        };
        auto settle = [&]() {
            uint32_t own = 0;
#pragma unroll
            for (int j = 0; j < kTcBinsPerLane; ++j) own += gc[j];
            uint32_t x = own;  // keys in bins >= kTcBinsPerLane * lane
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const uint32_t y = __shfl_down_sync(0xffffffffu, x, o);
                if (lane + o < 32) x += y;
            }
            const uint32_t k = (uint32_t)a.topk;
            uint32_t best = 0u;  // the highest bin whose suffix count reaches k, + 1 (0: none)
            if (k > 0u && x >= k) {
                uint32_t run = x - own;
#pragma unroll
                for (int j = kTcBinsPerLane - 1; j >= 0; --j) {
                    run += gc[j];
                    if (run >= k && best == 0u) best = (uint32_t)(kTcBinsPerLane * lane + j) + 1u;
                }
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) best = max(best, __shfl_xor_sync(0xffffffffu, best, o));
            if (lane == 0 && best > 0u) {
                const uint32_t th = tc_bin_floor(best - 1u);
                volatile uint32_t* st = &sh.thr[urow];
                if (th > *st) *st = th;
            }
        };
        auto refresh = [&]() {
#pragma unroll
            for (int i = 0; i < kRows; ++i) thr[i] = max(thr[i], *reinterpret_cast<volatile uint32_t*>(&sh.thr[rl0 + i]));
        };
        for (int j = 0; j < nt; ++j) {
            const int buf = j & 1, use = j >> 1;
            if (!tc_wait(sh, smem_u32(&sh.tfull[buf]), use & 1, a.dev_status)) break;
            tc_fence_after();
            const int tt0 = t_lo + (j_lo + j) * kTcTokens;  // the tile's first token
            const int t = tt0 + lane_tok;
            const uint32_t tbase = tmem + ((uint32_t)(32 * quarter) << 16) + (uint32_t)(buf * kTcCols + kCols * part);
            // two register buffers: the load of row i+1 is in flight while row i is reduced
            auto drain = [&](auto all_in) {
                static_assert(kRows == 4, "the drain below walks four rows");
                uint32_t va[16], vb[16];
                tmem_ld16(tbase, va);
                tmem_wait(va);
                tmem_ld16(tbase + 16u, vb);
                row_of(va, 0, t, all_in);
                tmem_wait(vb);
                tmem_ld16(tbase + 32u, va);
                row_of(vb, 1, t, all_in);
                tmem_wait(va);
                tmem_ld16(tbase + 48u, vb);
                row_of(va, 2, t, all_in);
                tmem_wait(vb);
                row_of(vb, 3, t, all_in);
            };
            // a tile inside the middle of every row of the warp needs no
            // per-token range test (most tiles of a chunk)
            if (tt0 >= rs_max && tt0 + kTcTokens <= rws_min) drain(std::true_type{});
            else drain(std::false_type{});
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&sh.tempty[buf]));
            const int ph = j % kTcUpdate;
            if (ph == kTcUpdate - 3) flush();
            else if (ph == kTcUpdate - 1) settle();
            else if (ph == 0 && j > 0) refresh();
        }
        // this warp's segment of each of its rows
        if (lane == 0) {
#pragma unroll
            for (int i = 0; i < kRows; ++i) {
                const int r = row0 + rl0 + i;
                if (r < a.n_q)
                    reinterpret_cast<int2*>(a.cand_seg)[((int64_t)r * kTcMaxSplits + blockIdx.x) * 4 + quarter] =
                        make_int2((int)seg_q, (int)min((int64_t)cnt[i], max(room, (int64_t)0)));
            }
        }
    }

    // ---- teardown: wait for every issued MMA, then free TMEM -----------------
    tc_fence_before();
    __syncthreads();
    if (warp == 1 && lane == 0) {
        umma_commit(smem_u32(&sh.drain));  // arrives once all MMAs of this thread are complete
        mbar_wait_bounded(smem_u32(&sh.drain), 0, kWaitLimitNs);
    }
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
    }
}

}  // namespace

int prefill_tc_splits(int n_q) {
    constexpr int R = kTcCols / 16;
    const int row_tiles = (n_q + R - 1) / R;
    // token splits per row tile: the fewest that fill the last wave of
    // one-CTA-per-SM launches to >= 95% (or the best of 1..kTcMaxSplits)
    const int sms = device_sm_count();
    int splits = 1;
    double best = 0.0;
    for (int sp = 1; sp <= kTcMaxSplits; ++sp) {
        const long ctas = (long)row_tiles * sp;
        const long waves = (ctas + sms - 1) / sms;
        const double eff = (double)ctas / (double)(waves * sms);
        if (eff > best + 1e-9) {
            best = eff;
            splits = sp;
        }
        if (eff >= 0.95) break;
    }
    return splits;
}

bool prefill_tc_supported(int H_I, int d_I, int n_seq, int64_t total_tokens) {
    return d_I == kTcK && H_I == 16 && n_seq == 1 && total_tokens + kTcTokens < (int64_t)0x7fffffff &&
           tensor_maps_available();
}

cudaError_t launch_fine_scores_tc(const IndexArgs& ia, cudaStream_t stream) {
    TcArgs a;
    std::memset(&a, 0, sizeof a);
    if (!tensor_map_rows128(&a.tmap_k, ia.k_idx, (uint64_t)ia.total_tokens, kTcTokens)) return cudaErrorInvalidValue;
    if (!tensor_map_rows128(&a.tmap_q, ia.q_idx, (uint64_t)ia.n_q * ia.H_I, kTcCols)) return cudaErrorInvalidValue;
    a.w = ia.w;
    a.q_seq = ia.q_seq;
    a.q_len = ia.q_len;
    a.kv_offset = ia.kv_offset;
    a.seq_lens = ia.seq_lens;
    a.cand = ia.cand;
    a.cand_seg = ia.cand_seg;
    a.ghist = ia.ghist;
    a.topk = ia.topk;
    a.dev_status = ia.dev_status;
    a.total_tokens = ia.total_tokens;
    a.n_q = ia.n_q;
    a.max_len = ia.max_len;
    a.w_max = ia.w_max;
    a.sink = ia.sink;
    a.window = ia.window;
    a.fine_cap = ia.fine_cap;
    constexpr int R = kTcCols / 16;
    const int row_tiles = (ia.n_q + R - 1) / R;
    const int splits = ia.tc_splits;
    if (splits < 1 || splits > kTcMaxSplits) return cudaErrorInvalidValue;
    // every split of a row writes its segment; the segments of splits that do
    // not exist read as empty (the selection reads `splits` of them)
    cudaError_t e = cudaFuncSetAttribute(fine_score_tc_kernel<16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)kTcSmem);
    if (e != cudaSuccess) return e;
    e = cudaMemsetAsync(a.ghist, 0, (size_t)ia.n_q * kTcBins * sizeof(uint32_t), stream);
    if (e != cudaSuccess) return e;
    return launch_pdl(fine_score_tc_kernel<16>, dim3((unsigned)splits, (unsigned)row_tiles), dim3(kTcThreads),
                      kTcSmem, stream, 0, a);
}

}  // namespace lsa
