// index_score.cu — the streaming half of the LSA indexer: HI coarse scores of
// candidate blocks and fine scores of candidate tokens.
//
// The method ("LongCat-2.0 (molayo1419.me)", section "1M 토큰에서의 Sparse
// Attention 문제"; "LongCat-Flash-Lite-Sparse (aitrends.kr)", section
// "기술적 특징"): a DSA-style indexer scores cached tokens; HI first scores
// whole blocks on their key sums and scores fine tokens only inside the kept
// blocks.
//
// Design (B200): both kernels are bandwidth kernels. Each CTA scores one
// chunk of one query's candidates (128 blocks, or 256 token slots) with plain
// 16-byte vector loads straight into MMA fragments; small CTAs and modest
// register use keep several CTAs — and thus many loads in flight — on every
// SM. Scores are written as keys (score + 1; 0 = not a candidate) to an
// L2-resident workspace for the selection kernels.
#include <cstring>

#include "index_common.cuh"

namespace lsa {
namespace {

constexpr int kScThreads = 256;
constexpr int kScWarps = kScThreads / kWarp;
constexpr int kCoarseChunk = kScWarps * 16;     // 128 blocks per CTA

// Validates query row r; on success sets the row's cache offset and visible
// length. Uniform over a CTA; flags nothing (the selection kernel reports).
__device__ __forceinline__ bool row_ok(const IndexArgs& a, int r, int64_t& off, int& L, int& slen) {
    const int seq = a.q_seq[r];
    L = a.q_len[r];
    if (seq < 0 || seq >= a.n_seq) return false;
    off = a.kv_offset[seq];
    slen = a.seq_lens[seq];
    if (L < 1 || L > a.max_len || L > slen || off < 0 || off + slen > a.total_tokens) return false;
    if (a.hi_block > 0) {
        const int64_t bo = a.blk_offset[seq];
        if (bo < 0 || bo + (L + a.hi_block - 1) / a.hi_block > a.block_rows) return false;
    }
    return true;
}
__device__ __forceinline__ bool row_ok(const IndexArgs& a, int r, int64_t& off, int& L) {
    int slen;
    return row_ok(a, r, off, L, slen);
}

template <int D_I, int NT>
__global__ void __launch_bounds__(kScThreads) coarse_score_kernel(const __grid_constant__ IndexArgs a) {
    const int r = blockIdx.y;
    int64_t off;
    int L, slen;
    // the row's metadata is the caller's, never written by a kernel of this
    // library: it is checked before the wait for the preceding kernel (which
    // may write the block sums)
    const bool ok = row_ok(a, r, off, L, slen);
    pdl_enter();
    if (!ok) return;
    const int s = min(a.sink, L);
    const int ws = max(s, L - a.window);
    if (ws <= s) return;
    const int B = a.hi_block;
    const int b_lo = s / B, b_hi = (ws + B - 1) / B;
    const int c0 = b_lo + blockIdx.x * kCoarseChunk;
    if (c0 >= b_hi) return;
    // the block holding the row's last visible token, summed over what the
    // row sees when the stored sum also counts later cached tokens (uniform)
    __shared__ int32_t s_sum[D_I];
    __shared__ long long s_fix;
    int b_p;
    const bool fix = partial_block_fix(L, slen, B, ws, b_p) && b_p >= c0 &&
                     b_p < min(c0 + kCoarseChunk, b_hi);
    long long fixed = 0;
    if (fix) fixed = partial_block_score<D_I, kScThreads>(a, r, a.k_idx + off * D_I, b_p * B, L - b_p * B, s_sum, &s_fix);
    const int lane = lane_id(), warp = warp_id(), g = lane >> 2, t4 = lane & 3;
    const int j0 = c0 + warp * 16 + g, j1 = j0 + 8;  // block indices of rows g and g+8
    if (c0 + warp * 16 >= b_hi) return;                // warp-uniform
    const bool v0 = j0 < b_hi, v1 = j1 < b_hi;
    const int8_t* rows = a.block_sums + a.blk_offset[a.q_seq[r]] * (2 * D_I);  // (cached by row_ok)
    RowFrag<D_I> hg, lg, hg8, lg8;
    hg.load(rows + (int64_t)j0 * (2 * D_I), t4, v0);
    lg.load(rows + (int64_t)j0 * (2 * D_I) + D_I, t4, v0);
    hg8.load(rows + (int64_t)j1 * (2 * D_I), t4, v1);
    lg8.load(rows + (int64_t)j1 * (2 * D_I) + D_I, t4, v1);
    QueryFrag<D_I, NT> qf;
    load_query<D_I, NT>(qf, a, r);
    long long x, y;
    coarse_tile<D_I, NT>(qf, hg, lg, hg8, lg8, x, y);
    pdl_trigger();  // only the stores are left
    if (fix && j0 == b_p) x = fixed;
    if (fix && j1 == b_p) y = fixed;
    uint64_t* keys = a.coarse_keys + (int64_t)r * a.coarse_cap;
    if (t4 == 0 && v0) keys[j0 - b_lo] = (unsigned long long)x + 1ull;
    if (t4 == 1 && v1) keys[j1 - b_lo] = (unsigned long long)y + 1ull;
}

// Fine scores: a persistent grid of kFineCtasPerSm CTAs per SM. With n_q <=
// warps, each row gets warps / n_q warps and each warp streams a contiguous
// range of the row's 16-slot tiles; with more rows, warps take whole rows in
// turn. Per warp the tile loop is software-pipelined: the key rows of tile
// j+1 (and the kept-block ids of tile j+2) are in flight while tile j is
// scored, so the dependent chain (row metadata, kept ids, key rows) is paid
// once per warp range rather than once per CTA.
constexpr int kFineCtasPerSm = 2;

template <int D_I>
struct FineTile {
    RowFrag<D_I> ra, rb;  // key rows of slots 16j + g and 16j + g + 8
    bool va, vb;          // slot holds a candidate token
};

template <int D_I, int NT>
__global__ void __launch_bounds__(kScThreads, kFineCtasPerSm) fine_score_kernel(const __grid_constant__ IndexArgs a) {
    pdl_enter();
    const int lane = lane_id(), g = lane >> 2, t4 = lane & 3;
    const int W = gridDim.x * kScWarps;
    const int gw = blockIdx.x * kScWarps + warp_id();
    const bool few_rows = a.n_q <= W;
    const int wpr = few_rows ? W / a.n_q : 1;  // warps per row
    const int seg = few_rows ? gw % wpr : 0;
    const int r0 = few_rows ? gw / wpr : gw;
    const int rstep = few_rows ? a.n_q : W;
    const bool hi = a.hi_block > 0;
    const int B = a.hi_block;
    const int lgB = (hi && (B & (B - 1)) == 0) ? __ffs(B) - 1 : -1;  // power-of-two block: shift, not divide
    for (int r = r0; r < a.n_q; r += rstep) {  // warp-uniform
        int64_t off;
        int L;
        if (!row_ok(a, r, off, L)) continue;
        const int s = min(a.sink, L);
        const int ws = max(s, L - a.window);
        const int n_slots = hi ? a.n_kept[r] * B : ws - s;
        const int nt = (n_slots + 15) / 16;
        const int j_lo = (int)((int64_t)nt * seg / wpr), j_hi = (int)((int64_t)nt * (seg + 1) / wpr);
        if (j_lo >= j_hi) continue;
        const int8_t* kseq = a.k_idx + off * D_I;
        const int32_t* kept = a.kept + (int64_t)r * a.hi_topblocks;
        uint32_t* keys = a.fine_keys + (int64_t)r * a.fine_cap;
        // kept-block ids of this lane's two slots of tile j (HI), or unused
        auto kept_ids = [&](int j, int& ka, int& kb) {
            ka = kb = 0;
            if (!hi) return;
            const int sa = 16 * j + g, sb = sa + 8;
            if (sa < n_slots) ka = __ldg(kept + (lgB >= 0 ? sa >> lgB : sa / B));
            if (sb < n_slots) kb = __ldg(kept + (lgB >= 0 ? sb >> lgB : sb / B));
        };
        auto token_of = [&](int slot, int kid, bool& valid) -> int {
            if (slot >= n_slots) {
                valid = false;
                return 0;
            }
            if (!hi) {
                valid = true;
                return s + slot;
            }
            const int kb = lgB >= 0 ? slot >> lgB : slot / B;
            const int tok = kid * B + (slot - kb * B);
            valid = tok >= s && tok < ws;
            return tok;
        };
        auto issue = [&](FineTile<D_I>& t, int j, int ka, int kb) {
            const int sa = 16 * j + g;
            const int ta = token_of(sa, ka, t.va);
            const int tb = token_of(sa + 8, kb, t.vb);
            t.ra.load(kseq + (int64_t)ta * D_I, t4, t.va);
            t.rb.load(kseq + (int64_t)tb * D_I, t4, t.vb);
        };
        QueryFrag<D_I, NT> qf;
        load_query<D_I, NT>(qf, a, r);
        auto score = [&](const FineTile<D_I>& t, int j) {
            const int2 sc = fine_tile<D_I, NT>(qf, t.ra, t.rb);
            const int sa = 16 * j + g, sb = sa + 8;
            if (t4 == 0 && sa < n_slots) keys[sa] = t.va ? (uint32_t)sc.x + 1u : 0u;
            if (t4 == 1 && sb < n_slots) keys[sb] = t.vb ? (uint32_t)sc.y + 1u : 0u;
        };
        FineTile<D_I> t0, t1;
        int ka0, kb0, ka1 = 0, kb1 = 0;
        kept_ids(j_lo, ka0, kb0);
        issue(t0, j_lo, ka0, kb0);
        if (j_lo + 1 < j_hi) kept_ids(j_lo + 1, ka1, kb1);
        for (int j = j_lo; j < j_hi; j += 2) {
            // tile j is in t0; the kept ids of tile j+1 are in (ka1, kb1)
            if (j + 1 < j_hi) issue(t1, j + 1, ka1, kb1);
            if (j + 2 < j_hi) kept_ids(j + 2, ka0, kb0);
            score(t0, j);
            if (j + 1 >= j_hi) break;
            if (j + 2 < j_hi) issue(t0, j + 2, ka0, kb0);
            if (j + 3 < j_hi) kept_ids(j + 3, ka1, kb1);
            score(t1, j + 1);
        }
    }
}

// ---------------------------------------------------------------------------
// Fine scores with HI on, d_I = 128, hi_block a multiple of 16: the kept
// blocks are contiguous runs of key rows, so each one (or each 64-row part)
// arrives as one TMA tensor copy (128-byte swizzle) instead of per-lane
// gathers. Two persistent CTAs per SM each take a contiguous range of (row,
// kept block, part) items. The producer warp looks up 32 items' kept-block
// ids at once, then one lane issues their copies into a ring of kFtStages
// stages; item k goes to stage k mod kFtStages and consumer warp k mod
// kFtConsumers, which scores its 16-row tiles from shared memory (the swizzle
// spreads the 8 rows a load reads over all banks) and releases the stage.
constexpr int kFtConsumers = 6;
constexpr int kFtThreads = (kFtConsumers + 1) * kWarp;
constexpr int kFtCtasPerSm = 2;
constexpr int kFtStages = 12;
// Stage k mod S always goes to consumer k mod C, so every use of a stage has
// the same consumer, which has seen the stage's previous phase complete
// before it waits on the next one (a parity wait cannot tell them apart).
static_assert(kFtStages % kFtConsumers == 0, "each stage needs a single consumer warp");
constexpr int kFtRows = 64;                   // key rows per item (box rows)
constexpr int kFtStageBytes = kFtRows * 128;  // 8 KB

struct FineTmaArgs {
    CUtensorMap tmap;  // key cache [total_tokens, 128], box kFtRows x 128
    IndexArgs a;
    int32_t sb;        // rows per item: min(hi_block, kFtRows)
};

struct FtItem {
    int32_t row;      // query row, -1: no more items for this warp
    int32_t slot0;    // first slot of the item in the row's key list
    int32_t tok0;     // first token of the item (in its sequence)
    int32_t s, ws;    // the row's middle
    int32_t pad;
    int64_t key_row;  // first key row of the copy in the whole cache
};

struct FtShared {
    uint64_t full[kFtStages];
    uint64_t empty[kFtStages];
    FtItem item[kFtStages];
    FtItem batch[32];  // the producer warp's next 32 items
    int32_t fail;
};

constexpr size_t kFtSmem = 1024 + (size_t)kFtStages * kFtStageBytes + sizeof(FtShared);

template <int NT>
__global__ void __launch_bounds__(kFtThreads, kFtCtasPerSm) fine_score_tma_kernel(const __grid_constant__ FineTmaArgs p) {
    // Before the wait for the block selection: only the caller's inputs (row
    // metadata, queries, weights), which no kernel of this library writes.
    const IndexArgs& a = p.a;
    extern __shared__ __align__(16) uint8_t ft_raw[];
    const uint32_t raw = smem_u32(ft_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;  // 128-byte swizzle atoms are 1024-byte aligned
    FtShared& sh = *reinterpret_cast<FtShared*>(ft_raw + (base - raw) + kFtStages * kFtStageBytes);
    const int warp = warp_id(), lane = lane_id(), g = lane >> 2, t4 = lane & 3;
    const int SB = p.sb;
    const int B = a.hi_block;
    const int parts = B / SB;
    const int64_t per_row = (int64_t)a.hi_topblocks * parts;
    const int64_t total = (int64_t)a.n_q * per_row;
    const int64_t i_lo = total * blockIdx.x / gridDim.x, i_hi = total * (blockIdx.x + 1) / gridDim.x;
    if (threadIdx.x == 0) {
        for (int st = 0; st < kFtStages; ++st) {
            mbar_init(smem_u32(&sh.full[st]), 1);
            mbar_init(smem_u32(&sh.empty[st]), 1);
        }
        sh.fail = 0;
        mbar_fence_init();
    }
    __syncthreads();

    if (warp == kFtConsumers) {
        // ------------------------------ producer ------------------------------
        // the CTA's first and last rows (a range spans at most two rows when
        // there are fewer rows than CTAs) are checked before the wait
        const int r_first = i_lo < i_hi ? (int)(i_lo / per_row) : 0;
        const int r_last = i_lo < i_hi ? (int)((i_hi - 1) / per_row) : 0;
        int64_t c_off = 0;
        int c_L = 0;
        const bool c_ok = lane < 2 && row_ok(a, lane == 0 ? r_first : r_last, c_off, c_L);
        const bool ok_first = __shfl_sync(0xffffffffu, c_ok, 0), ok_last = __shfl_sync(0xffffffffu, c_ok, 1);
        const int64_t off_first = __shfl_sync(0xffffffffu, c_off, 0), off_last = __shfl_sync(0xffffffffu, c_off, 1);
        const int L_first = __shfl_sync(0xffffffffu, c_L, 0), L_last = __shfl_sync(0xffffffffu, c_L, 1);
        pdl_enter();
        int k = 0;  // items issued
        auto next_stage = [&](int kk) -> bool {  // lane 0: wait until stage kk % S is free
            const int st = kk % kFtStages;
            if (kk >= kFtStages &&
                !mbar_wait_bounded(smem_u32(&sh.empty[st]), (uint32_t)(((kk / kFtStages) + 1) & 1), kWaitLimitNs)) {
                sh.fail = 1;
                return false;
            }
            return true;
        };
        bool ok = true;
        for (int64_t c0 = i_lo; ok && c0 < i_hi; c0 += kWarp) {
            // every lane looks up one item of the next 32 (three L2 round trips for all of them)
            const int64_t i = c0 + lane;
            FtItem it;
            it.row = -1;
            if (i < i_hi) {
                const int r = (int)(i / per_row);
                const int rem = (int)(i - (int64_t)r * per_row);
                const int q = rem / parts, part = rem - q * parts;
                // the kept count and id are fetched together with the row check
                const int nk = a.n_kept[r];
                const int kid = a.kept[(int64_t)r * a.hi_topblocks + q];
                int64_t off = r == r_first ? off_first : off_last;
                int L = r == r_first ? L_first : L_last;
                bool ok = r == r_first ? ok_first : ok_last;
                if (r != r_first && r != r_last) ok = row_ok(a, r, off, L);
                if (ok && q < min(max(nk, 0), a.hi_topblocks)) {
                    it.row = r;
                    it.slot0 = q * B + part * SB;
                    it.tok0 = kid * B + part * SB;
                    it.s = min(a.sink, L);
                    it.ws = max(it.s, L - a.window);
                    it.pad = 0;
                    it.key_row = off + it.tok0;
                }
            }
            sh.batch[lane] = it;
            __syncwarp();
            if (lane == 0) {
                const int n = (int)min((int64_t)kWarp, i_hi - c0);
                for (int j = 0; j < n; ++j) {
                    const FtItem b = sh.batch[j];
                    if (b.row < 0) continue;
                    if (!next_stage(k)) {
                        ok = false;
                        break;
                    }
                    const int st = k % kFtStages;
                    sh.item[st] = b;
                    mbar_arrive_expect_tx(smem_u32(&sh.full[st]), (uint32_t)(SB * 128));
                    tma_load_2d(base + (uint32_t)(st * kFtStageBytes), &p.tmap, 0, (int)b.key_row,
                                smem_u32(&sh.full[st]));
                    ++k;
                }
            }
            ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
            __syncwarp();
        }
        pdl_trigger();  // every copy is issued
        // one end marker per consumer warp
        if (lane == 0) {
            for (int w = 0; w < kFtConsumers; ++w) {
                if (!next_stage(k)) break;
                const int st = k % kFtStages;
                sh.item[st].row = -1;
                mbar_arrive(smem_u32(&sh.full[st]));
                ++k;
            }
            // every issued copy lands before the CTA may exit
            for (int kk = max(0, k - kFtStages); kk < k; ++kk)
                mbar_wait_bounded(smem_u32(&sh.full[kk % kFtStages]), (uint32_t)((kk / kFtStages) & 1), kWaitLimitNs);
        }
    } else {
        // ------------------------------ consumers -----------------------------
        // the first item's row is known before any copy lands: fetch its query now
        int qrow = i_lo < i_hi ? (int)(i_lo / per_row) : -1;
        QueryFrag<128, NT> qf;
        if (qrow >= 0) load_query<128, NT>(qf, a, qrow);
        pdl_enter();
        uint32_t* keys = qrow >= 0 ? a.fine_keys + (int64_t)qrow * a.fine_cap : nullptr;
        for (int k = warp;; k += kFtConsumers) {
            const int st = k % kFtStages;
            if (!mbar_wait_bounded(smem_u32(&sh.full[st]), (uint32_t)((k / kFtStages) & 1), kWaitLimitNs)) {
                if (lane == 0) sh.fail = 1;
                break;
            }
            const FtItem it = sh.item[st];
            if (it.row < 0) break;
            if (it.row != qrow) {
                load_query<128, NT>(qf, a, it.row);
                qrow = it.row;
                keys = a.fine_keys + (int64_t)it.row * a.fine_cap;
            }
            const uint32_t sbase = base + (uint32_t)(st * kFtStageBytes);
            for (int t = 0; t < SB / 16; ++t) {
                RowFrag<128> fa, fb;
                const int ra = 16 * t + g, rb = ra + 8;
                // logical 16-byte chunk c of row rr sits at chunk c ^ (rr & 7)
                const uint4 a0 = ld_shared_v4(sbase + (uint32_t)(ra * 128 + 16 * (t4 ^ (ra & 7))));
                const uint4 a1 = ld_shared_v4(sbase + (uint32_t)(ra * 128 + 16 * ((4 + t4) ^ (ra & 7))));
                const uint4 b0 = ld_shared_v4(sbase + (uint32_t)(rb * 128 + 16 * (t4 ^ (rb & 7))));
                const uint4 b1 = ld_shared_v4(sbase + (uint32_t)(rb * 128 + 16 * ((4 + t4) ^ (rb & 7))));
                fa.w[0] = a0.x; fa.w[1] = a0.y; fa.w[2] = a0.z; fa.w[3] = a0.w;
                fa.w[4] = a1.x; fa.w[5] = a1.y; fa.w[6] = a1.z; fa.w[7] = a1.w;
                fb.w[0] = b0.x; fb.w[1] = b0.y; fb.w[2] = b0.z; fb.w[3] = b0.w;
                fb.w[4] = b1.x; fb.w[5] = b1.y; fb.w[6] = b1.z; fb.w[7] = b1.w;
                const int2 sc = fine_tile<128, NT>(qf, fa, fb);
                const int ta = it.tok0 + ra, tb = it.tok0 + rb;
                if (t4 == 0) keys[it.slot0 + ra] = (ta >= it.s && ta < it.ws) ? (uint32_t)sc.x + 1u : 0u;
                if (t4 == 1) keys[it.slot0 + rb] = (tb >= it.s && tb < it.ws) ? (uint32_t)sc.y + 1u : 0u;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&sh.empty[st]));
        }
    }
    __syncthreads();
    if (threadIdx.x == 0 && sh.fail) flag(a.dev_status, LSA_DEV_TIMEOUT);
}

template <int D_I, int NT>
cudaError_t launch_scores_t(const IndexArgs& a, bool coarse, cudaStream_t st) {
    if (coarse) {
        dim3 grid((unsigned)((a.coarse_cap + kCoarseChunk - 1) / kCoarseChunk), (unsigned)a.n_q);
        return launch_pdl(coarse_score_kernel<D_I, NT>, grid, dim3(kScThreads), 0, st, 0, a);
    } else {
        dim3 grid((unsigned)(kFineCtasPerSm * device_sm_count()));
        return launch_pdl(fine_score_kernel<D_I, NT>, grid, dim3(kScThreads), 0, st, 0, a);
    }
}

template <int NT>
cudaError_t launch_fine_tma(const IndexArgs& a, cudaStream_t st) {
    FineTmaArgs p;
    std::memset(&p, 0, sizeof p);
    p.a = a;
    p.sb = a.hi_block < kFtRows ? a.hi_block : kFtRows;
    if (!tensor_map_rows128(&p.tmap, a.k_idx, (uint64_t)a.total_tokens, (uint32_t)p.sb)) return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(fine_score_tma_kernel<NT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)kFtSmem);
    if (e != cudaSuccess) return e;
    return launch_pdl(fine_score_tma_kernel<NT>, dim3((unsigned)(kFtCtasPerSm * device_sm_count())), dim3(kFtThreads),
                      kFtSmem, st, 0,
                      p);
}

// Kept blocks as whole TMA boxes: HI on, 128-byte keys, blocks of a multiple
// of 16 rows that split into equal boxes of at most kFtRows rows.
bool fine_tma_ok(const IndexArgs& a, int d_I) {
    const int B = a.hi_block;
    return B > 0 && d_I == 128 && B % 16 == 0 && (B <= kFtRows || B % kFtRows == 0) &&
           a.total_tokens + kFtRows < (int64_t)0x7fffffff && tensor_maps_available();
}

template <int D_I>
cudaError_t launch_scores_d(const IndexArgs& a, bool coarse, cudaStream_t st) {
    const int nt = (a.H_I + 7) / 8;
    if constexpr (D_I == 128) {
        if (!coarse && fine_tma_ok(a, D_I)) {
            if (nt <= 1) return launch_fine_tma<1>(a, st);
            if (nt <= 2) return launch_fine_tma<2>(a, st);
            if (nt <= 4) return launch_fine_tma<4>(a, st);
            return launch_fine_tma<8>(a, st);
        }
    }
    if (nt <= 1) return launch_scores_t<D_I, 1>(a, coarse, st);
    if (nt <= 2) return launch_scores_t<D_I, 2>(a, coarse, st);
    if (nt <= 4) return launch_scores_t<D_I, 4>(a, coarse, st);
    return launch_scores_t<D_I, 8>(a, coarse, st);
}

}  // namespace

cudaError_t launch_index_scores(const IndexArgs& a, int d_I, bool coarse, cudaStream_t stream) {
    switch (d_I) {
        case 32: return launch_scores_d<32>(a, coarse, stream);
        case 64: return launch_scores_d<64>(a, coarse, stream);
        case 128: return launch_scores_d<128>(a, coarse, stream);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace lsa
