// index_decode.cu — fused LSA indexer: HI coarse pass, block selection, fine
// scoring, token top-k and SI assembly in one launch.
//
// The method ("LongCat-2.0 (molayo1419.me)", section "1M 토큰에서의 Sparse
// Attention 문제"; "LongCat-Flash-Lite-Sparse (aitrends.kr)", section
// "기술적 특징"): a DSA-style indexer scores cached tokens and keeps a
// top-k; SI always keeps a sink run and a local window; HI first keeps the
// best coarse blocks and scores fine tokens only inside them.
//
// Design (B200):
//  * One thread-block cluster per query row. The cluster's CTAs split the
//    query's candidate blocks and tokens into contiguous ranges, so the
//    candidate order (ascending position) is the CTA order.
//  * Scores are exact int8 dot products on the tensor cores
//    (mma.m16n8k32.s8): 16 key rows form the A tile, the query's indexer heads
//    (padded to multiples of 8) the B tile. Because a dot product is a sum,
//    each lane may own any consistent subset of the 128 dims: lane t loads
//    16-byte chunks t and 4+t of a key row, and the query fragment is loaded
//    with the same permutation — so a warp reads 8 rows x 64 contiguous bytes
//    per load instruction, straight from HBM into registers.
//  * HI block sums are stored as int8 high / uint8 low byte planes; the coarse
//    dot is 256 * (q . hi) + (q . lo) from one s8 x s8 and one u8 x s8 MMA.
//  * Keys (score + 1, 0 = not a candidate) stay in the CTA's shared memory.
//    Selection is an MSD radix select (8-bit digits from the highest set bit
//    of the cluster-wide maximum): per pass every CTA builds a local
//    histogram, the cluster barrier publishes it, and every CTA sums the
//    cluster's histograms over distributed shared memory and derives the same
//    digit. The result is the exact k-th largest key T and the number of keys
//    equal to T to keep; compaction keeps key > T plus the lowest-position
//    ties, ranked by a warp-ballot prefix in position order. No CTA waits on
//    a flag: every cross-CTA step is a hardware cluster barrier.
#include <cooperative_groups.h>

#include "common.cuh"
#include "internal.h"

namespace cg = cooperative_groups;

namespace lsa {
namespace {

constexpr int kIxThreads = 256;
constexpr int kIxWarps = kIxThreads / kWarp;
constexpr int kBins = 256;

// ----------------------------------------------------------------------------
// Row fragments: the bytes of a D_I-byte row that lane t (= lane % 4) owns.
// ----------------------------------------------------------------------------
template <int D_I>
struct RowFrag {
    static constexpr int kWords = D_I / 16;  // 32-bit words per lane
    uint32_t w[kWords];

    __device__ __forceinline__ void load(const int8_t* row, int t, bool valid) {
        if constexpr (D_I == 128) {
            uint4 x = make_uint4(0, 0, 0, 0), y = make_uint4(0, 0, 0, 0);
            if (valid) {
                x = ldg16(row + 16 * t);
                y = ldg16(row + 64 + 16 * t);
            }
            w[0] = x.x; w[1] = x.y; w[2] = x.z; w[3] = x.w;
            w[4] = y.x; w[5] = y.y; w[6] = y.z; w[7] = y.w;
        } else if constexpr (D_I == 64) {
            uint4 x = make_uint4(0, 0, 0, 0);
            if (valid) x = ldg16(row + 16 * t);
            w[0] = x.x; w[1] = x.y; w[2] = x.z; w[3] = x.w;
        } else {
            uint2 x = make_uint2(0, 0);
            if (valid) x = ldg8(row + 8 * t);
            w[0] = x.x; w[1] = x.y;
        }
    }
};

// The query's indexer heads as MMA B fragments, plus the per-lane weights.
template <int D_I, int NT>
struct QueryFrag {
    uint32_t b[NT][D_I / 32][2];
    int32_t wlo[NT], whi[NT];  // weights of heads 8n + 2t and 8n + 2t + 1
};

template <int D_I, int NT>
__device__ __forceinline__ void load_query(QueryFrag<D_I, NT>& qf, const IndexArgs& a, int r) {
    const int lane = lane_id(), g = lane >> 2, t = lane & 3;
    bool bad_w = false;
#pragma unroll
    for (int n = 0; n < NT; ++n) {
        const int head = 8 * n + g;
        RowFrag<D_I> f;
        f.load(a.q_idx + ((int64_t)r * a.H_I + head) * D_I, t, head < a.H_I);
#pragma unroll
        for (int s = 0; s < D_I / 32; ++s) {
            qf.b[n][s][0] = f.w[2 * s];
            qf.b[n][s][1] = f.w[2 * s + 1];
        }
        const int h0 = 8 * n + 2 * t, h1 = h0 + 1;
        int32_t w0 = h0 < a.H_I ? a.w[(int64_t)r * a.H_I + h0] : 0;
        int32_t w1 = h1 < a.H_I ? a.w[(int64_t)r * a.H_I + h1] : 0;
        if (w0 < 0 || w0 > a.w_max) { bad_w = true; w0 = 0; }
        if (w1 < 0 || w1 > a.w_max) { bad_w = true; w1 = 0; }
        qf.wlo[n] = w0;
        qf.whi[n] = w1;
    }
    if (bad_w) flag(a.dev_status, LSA_DEV_BAD_WEIGHT);
}

// Fine scores of 16 key rows (rows g and g+8 of this lane). Returns the
// weighted-ReLU sums for rows g (x) and g + 8 (y), reduced over the 4 lanes of
// the row group.
template <int D_I, int NT>
__device__ __forceinline__ int2 fine_tile(const QueryFrag<D_I, NT>& qf, const RowFrag<D_I>& rg,
                                          const RowFrag<D_I>& rg8) {
    int32_t acc[NT][4];
#pragma unroll
    for (int n = 0; n < NT; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0;
#pragma unroll
    for (int s = 0; s < D_I / 32; ++s) {
        const uint32_t a[4] = {rg.w[2 * s], rg8.w[2 * s], rg.w[2 * s + 1], rg8.w[2 * s + 1]};
#pragma unroll
        for (int n = 0; n < NT; ++n) mma_s8s8(acc[n], a, qf.b[n][s][0], qf.b[n][s][1]);
    }
    int32_t x = 0, y = 0;
#pragma unroll
    for (int n = 0; n < NT; ++n) {
        x += qf.wlo[n] * max(acc[n][0], 0) + qf.whi[n] * max(acc[n][1], 0);
        y += qf.wlo[n] * max(acc[n][2], 0) + qf.whi[n] * max(acc[n][3], 0);
    }
    x += __shfl_xor_sync(0xffffffffu, x, 1);
    y += __shfl_xor_sync(0xffffffffu, y, 1);
    x += __shfl_xor_sync(0xffffffffu, x, 2);
    y += __shfl_xor_sync(0xffffffffu, y, 2);
    return make_int2(x, y);
}

// Coarse scores of 16 block-sum rows (two byte planes each).
template <int D_I, int NT>
__device__ __forceinline__ void coarse_tile(const QueryFrag<D_I, NT>& qf, const RowFrag<D_I>& hg,
                                            const RowFrag<D_I>& lg, const RowFrag<D_I>& hg8,
                                            const RowFrag<D_I>& lg8, long long& x, long long& y) {
    int32_t ah[NT][4], al[NT][4];
#pragma unroll
    for (int n = 0; n < NT; ++n) {
        ah[n][0] = ah[n][1] = ah[n][2] = ah[n][3] = 0;
        al[n][0] = al[n][1] = al[n][2] = al[n][3] = 0;
    }
#pragma unroll
    for (int s = 0; s < D_I / 32; ++s) {
        const uint32_t a_hi[4] = {hg.w[2 * s], hg8.w[2 * s], hg.w[2 * s + 1], hg8.w[2 * s + 1]};
        const uint32_t a_lo[4] = {lg.w[2 * s], lg8.w[2 * s], lg.w[2 * s + 1], lg8.w[2 * s + 1]};
#pragma unroll
        for (int n = 0; n < NT; ++n) {
            mma_s8s8(ah[n], a_hi, qf.b[n][s][0], qf.b[n][s][1]);
            mma_u8s8(al[n], a_lo, qf.b[n][s][0], qf.b[n][s][1]);
        }
    }
    x = 0;
    y = 0;
#pragma unroll
    for (int n = 0; n < NT; ++n) {
        const int32_t d0 = ah[n][0] * 256 + al[n][0], d1 = ah[n][1] * 256 + al[n][1];
        const int32_t d2 = ah[n][2] * 256 + al[n][2], d3 = ah[n][3] * 256 + al[n][3];
        x += (long long)qf.wlo[n] * max(d0, 0) + (long long)qf.whi[n] * max(d1, 0);
        y += (long long)qf.wlo[n] * max(d2, 0) + (long long)qf.whi[n] * max(d3, 0);
    }
    x += __shfl_xor_sync(0xffffffffu, x, 1);
    y += __shfl_xor_sync(0xffffffffu, y, 1);
    x += __shfl_xor_sync(0xffffffffu, x, 2);
    y += __shfl_xor_sync(0xffffffffu, y, 2);
}

// ----------------------------------------------------------------------------
// Cluster-wide selection
// ----------------------------------------------------------------------------
struct SelectShared {
    uint32_t hist[2][kBins];
    uint32_t warp_scan[kIxWarps];
    unsigned long long local_max;
    uint32_t local_count;
    uint32_t digit, above;
    uint32_t warp_gt[kIxWarps], warp_eq[kIxWarps];
    uint32_t cta_gt, cta_eq;
};

template <typename K>
__device__ __forceinline__ int key_bits(K v) {
    if constexpr (sizeof(K) == 8) return 64 - __clzll((long long)v);
    else return 32 - __clz((int)v);
}

// Cluster maximum of the CTAs' local_max and sum of their local_count.
__device__ void cluster_max_count(cg::cluster_group& cl, SelectShared& sh, unsigned long long& gmax,
                                  uint32_t& gcount) {
    cl.sync();
    unsigned long long m = 0;
    uint32_t c = 0;
    const uint32_t C = cl.num_blocks();
    for (uint32_t i = 0; i < C; ++i) {
        SelectShared* rs = cl.map_shared_rank(&sh, i);
        m = max(m, rs->local_max);
        c += rs->local_count;
    }
    gmax = m;
    gcount = c;
}

// Exact k-th largest key over the cluster: keys > thresh plus the first
// `quota` keys == thresh (in position order) are the k_target largest.
template <typename K>
__device__ void cluster_select(cg::cluster_group& cl, SelectShared& sh, int& parity, const K* keys, int n,
                               uint32_t k_target, unsigned long long gmax, K& thresh, uint32_t& quota) {
    if (k_target == 0) {
        thresh = ~K(0);
        quota = 0;
        return;
    }
    constexpr int kKeyBits = 8 * sizeof(K);
    const int tid = threadIdx.x;
    const uint32_t C = cl.num_blocks();
    int nbits = key_bits<K>((K)gmax);
    if (nbits < 1) nbits = 1;
    int shift = ((nbits - 1) / 8) * 8;
    K prefix = 0;
    uint32_t krem = k_target;
    for (;;) {
        uint32_t* h = sh.hist[parity];
        for (int i = tid; i < n; i += kIxThreads) {
            const K key = keys[i];
            const K hi = (shift + 8 >= kKeyBits) ? K(0) : (K)(key >> (shift + 8));
            if (hi == prefix) atomicAdd(&h[(uint32_t)(key >> shift) & 0xFFu], 1u);
        }
        cl.sync();
        // The other buffer was read by every CTA before this barrier: clear it
        // for the next pass.
        sh.hist[parity ^ 1][tid] = 0;
        // Cluster-wide count of this bin (thread tid owns bin tid).
        uint32_t tot = 0;
        for (uint32_t c = 0; c < C; ++c) tot += cl.map_shared_rank(h, c)[tid];
        // Suffix sums over bins: S(d) = sum of counts of bins >= d.
        uint32_t x = tot;
        const int lane = lane_id(), wid = warp_id();
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            uint32_t v = __shfl_down_sync(0xffffffffu, x, o);
            if (lane + o < 32) x += v;
        }
        if (lane == 0) sh.warp_scan[wid] = x;
        __syncthreads();
        uint32_t later = 0;
        for (int w2 = wid + 1; w2 < kIxWarps; ++w2) later += sh.warp_scan[w2];
        const uint32_t S = x + later;  // count of keys (matching prefix) with digit >= tid
        const uint32_t above = S - tot;
        if (S >= krem && above < krem) {
            sh.digit = tid;
            sh.above = above;
        }
        __syncthreads();
        prefix = (K)((prefix << 8) | (K)sh.digit);
        krem -= sh.above;
        parity ^= 1;
        __syncthreads();  // digit/above are rewritten by the next pass
        if (shift == 0) break;
        shift -= 8;
    }
    thresh = prefix;
    quota = krem;
}

// Calls emit(slot, rank) for every kept key, rank = its position among the
// kept keys in slot order across the cluster.
template <typename K, typename Emit>
__device__ void cluster_compact(cg::cluster_group& cl, SelectShared& sh, const K* keys, int n, K thresh,
                                uint32_t quota, Emit emit) {
    const int lane = lane_id(), wid = warp_id();
    const int per_warp = ((n + kIxWarps * 32 - 1) / (kIxWarps * 32)) * 32;
    const int b0 = wid * per_warp;
    const int b1 = min(n, b0 + per_warp);
    uint32_t gt = 0, eq = 0;
    for (int base = b0; base < b1; base += 32) {
        const int i = base + lane;
        const K key = i < b1 ? keys[i] : K(0);
        const bool is_gt = i < b1 && key > thresh;
        const bool is_eq = i < b1 && key == thresh;
        gt += __popc(__ballot_sync(0xffffffffu, is_gt));
        eq += __popc(__ballot_sync(0xffffffffu, is_eq));
    }
    if (lane == 0) {
        sh.warp_gt[wid] = gt;
        sh.warp_eq[wid] = eq;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        uint32_t tg = 0, te = 0;
        for (int w2 = 0; w2 < kIxWarps; ++w2) {
            tg += sh.warp_gt[w2];
            te += sh.warp_eq[w2];
        }
        sh.cta_gt = tg;
        sh.cta_eq = te;
    }
    cl.sync();
    uint32_t gt_b = 0, eq_b = 0;
    const uint32_t me = cl.block_rank();
    for (uint32_t c = 0; c < me; ++c) {
        SelectShared* rs = cl.map_shared_rank(&sh, c);
        gt_b += rs->cta_gt;
        eq_b += rs->cta_eq;
    }
    for (int w2 = 0; w2 < wid; ++w2) {
        gt_b += sh.warp_gt[w2];
        eq_b += sh.warp_eq[w2];
    }
    const uint32_t lt = lanemask_lt();
    for (int base = b0; base < b1; base += 32) {
        const int i = base + lane;
        const K key = i < b1 ? keys[i] : K(0);
        const bool is_gt = i < b1 && key > thresh;
        const bool is_eq = i < b1 && key == thresh;
        const uint32_t mg = __ballot_sync(0xffffffffu, is_gt);
        const uint32_t mq = __ballot_sync(0xffffffffu, is_eq);
        const uint32_t my_gt = gt_b + __popc(mg & lt);
        const uint32_t my_eq = eq_b + __popc(mq & lt);
        if (is_gt) emit(i, my_gt + min(my_eq, quota));
        else if (is_eq && my_eq < quota) emit(i, my_gt + my_eq);
        gt_b += __popc(mg);
        eq_b += __popc(mq);
    }
}

// Balanced contiguous split of [0, n) over C parts.
__device__ __forceinline__ int64_t part_begin(int64_t n, uint32_t c, uint32_t C) { return (n * c) / C; }

// ----------------------------------------------------------------------------
// The kernel
// ----------------------------------------------------------------------------
template <int D_I, int NT>
__global__ void __launch_bounds__(kIxThreads) index_kernel(const __grid_constant__ IndexArgs a) {
    cg::cluster_group cl = cg::this_cluster();
    const uint32_t C = cl.num_blocks();
    const uint32_t crank = cl.block_rank();
    const int r = blockIdx.x / C;
    const int tid = threadIdx.x, lane = lane_id(), wid = warp_id();
    const int g = lane >> 2, t4 = lane & 3;

    __shared__ SelectShared sh;
    extern __shared__ __align__(16) uint8_t dyn[];
    int parity = 0;

    int32_t* out = a.index_sets + (int64_t)r * a.budget;

    // ---- query validation (uniform over the cluster) ----
    const int seq = a.q_seq[r];
    const int L = a.q_len[r];
    bool bad = false;
    int64_t off = 0;
    if (seq < 0 || seq >= a.n_seq) {
        bad = true;
        if (tid == 0 && crank == 0) flag(a.dev_status, LSA_DEV_BAD_SEQ);
    } else {
        off = a.kv_offset[seq];
        const int slen = a.seq_lens[seq];
        if (L < 1 || L > a.max_len || L > slen || off < 0 || off + slen > a.total_tokens) bad = true;
        if (!bad && a.hi_block > 0) {
            const int64_t bo = a.blk_offset[seq];
            if (bo < 0 || bo + (L + a.hi_block - 1) / a.hi_block > a.block_rows) bad = true;
        }
        if (bad && tid == 0 && crank == 0) flag(a.dev_status, LSA_DEV_BAD_LENGTH);
    }
    if (bad) {
        for (int e = crank * kIxThreads + tid; e < a.budget; e += C * kIxThreads) out[e] = -1;
        return;  // uniform across the cluster: no barrier is pending
    }

    const int s = min(a.sink, L);
    const int ws = max(s, L - a.window);
    const int n_mid = ws - s;
    const int8_t* kseq = a.k_idx + off * D_I;

    for (int i = tid; i < 2 * kBins; i += kIxThreads) (&sh.hist[0][0])[i] = 0;
    if (tid == 0) {
        sh.local_max = 0;
        sh.local_count = 0;
    }

    QueryFrag<D_I, NT> qf;
    load_query<D_I, NT>(qf, a, r);
    __syncthreads();

    // ---- candidate slots of this CTA ----
    uint32_t* fine_keys = a.smem_fine >= 0 ? reinterpret_cast<uint32_t*>(dyn + a.smem_fine)
                                            : a.g_fine + ((int64_t)r * C + crank) * a.fine_cap;
    int n_fine = 0;          // slots in this CTA
    int flat_begin = 0;      // HI off: first middle token of this CTA
    int B = a.hi_block;
    int32_t* kept_local = reinterpret_cast<int32_t*>(dyn + a.smem_kept_local);
    int kept_begin = 0, n_kept_local = 0;

    if (a.hi_block > 0 && n_mid > 0) {
        // ---------------- HI coarse pass ----------------
        const int b_lo = s / B;
        const int b_hi = (ws + B - 1) / B;
        const int nb = b_hi - b_lo;
        const int cb0 = b_lo + (int)part_begin(nb, crank, C);
        const int cb1 = b_lo + (int)part_begin(nb, crank + 1, C);
        const int n_coarse = cb1 - cb0;
        uint64_t* coarse_keys = a.smem_coarse >= 0
                                    ? reinterpret_cast<uint64_t*>(dyn + a.smem_coarse)
                                    : a.g_coarse + ((int64_t)r * C + crank) * a.coarse_cap;
        const int8_t* srow0 = a.block_sums + a.blk_offset[seq] * (2 * D_I);
        unsigned long long my_max = 0;
        const int n_tiles = (n_coarse + 15) / 16;
        for (int tile = wid; tile < n_tiles; tile += kIxWarps) {
            const int j0 = tile * 16 + g, j1 = j0 + 8;
            const bool v0 = j0 < n_coarse, v1 = j1 < n_coarse;
            RowFrag<D_I> hg, lg, hg8, lg8;
            const int8_t* p0 = srow0 + (int64_t)(cb0 + j0) * (2 * D_I);
            const int8_t* p1 = srow0 + (int64_t)(cb0 + j1) * (2 * D_I);
            hg.load(p0, t4, v0);
            lg.load(p0 + D_I, t4, v0);
            hg8.load(p1, t4, v1);
            lg8.load(p1 + D_I, t4, v1);
            long long x, y;
            coarse_tile<D_I, NT>(qf, hg, lg, hg8, lg8, x, y);
            const unsigned long long kx = (unsigned long long)x + 1ull, ky = (unsigned long long)y + 1ull;
            if (t4 == 0 && v0) coarse_keys[j0] = kx;
            if (t4 == 1 && v1) coarse_keys[j1] = ky;
            if (v0) my_max = max(my_max, kx);
            if (v1) my_max = max(my_max, ky);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) my_max = max(my_max, __shfl_xor_sync(0xffffffffu, my_max, o));
        if (lane == 0) atomicMax(&sh.local_max, my_max);
        if (tid == 0) sh.local_count = n_coarse;
        __syncthreads();
        unsigned long long gmax;
        uint32_t gcount;
        cluster_max_count(cl, sh, gmax, gcount);
        const uint32_t k_blocks = min((uint32_t)a.hi_topblocks, gcount);
        uint64_t thr;
        uint32_t quota;
        cluster_select<uint64_t>(cl, sh, parity, coarse_keys, n_coarse, k_blocks, gmax, thr, quota);
        int32_t* kept_leader = cl.map_shared_rank(reinterpret_cast<int32_t*>(dyn + a.smem_kept), 0);
        cluster_compact<uint64_t>(cl, sh, coarse_keys, n_coarse, thr, quota,
                                  [&](int slot, uint32_t rank) { kept_leader[rank] = cb0 + slot; });
        cl.sync();  // kept list complete in the leader CTA
        kept_begin = (int)part_begin(k_blocks, crank, C);
        const int kept_end = (int)part_begin(k_blocks, crank + 1, C);
        n_kept_local = kept_end - kept_begin;
        for (int i = tid; i < n_kept_local; i += kIxThreads) kept_local[i] = kept_leader[kept_begin + i];
        n_fine = n_kept_local * B;
        if (tid == 0) {
            sh.local_max = 0;
            sh.local_count = 0;
        }
        __syncthreads();
    } else {
        flat_begin = s + (int)part_begin(n_mid, crank, C);
        n_fine = s + (int)part_begin(n_mid, crank + 1, C) - flat_begin;
        __syncthreads();
    }

    // ---------------- fine scoring ----------------
    {
        const bool hi = a.hi_block > 0;
        unsigned long long my_max = 0;
        uint32_t my_count = 0;
        const int n_tiles = (n_fine + 15) / 16;
        auto token_of = [&](int slot, bool& valid) -> int {
            if (slot >= n_fine) {
                valid = false;
                return 0;
            }
            if (!hi) {
                valid = true;
                return flat_begin + slot;
            }
            const int kb = slot / B;
            const int tok = kept_local[kb] * B + (slot - kb * B);
            valid = tok >= s && tok < ws;
            return tok;
        };
        for (int tile = wid; tile < n_tiles; tile += 2 * kIxWarps) {
            const int tileB = tile + kIxWarps;
            bool va0, va1, vb0, vb1;
            const int ta0 = token_of(tile * 16 + g, va0);
            const int ta1 = token_of(tile * 16 + g + 8, va1);
            const int tb0 = token_of(tileB * 16 + g, vb0);
            const int tb1 = token_of(tileB * 16 + g + 8, vb1);
            RowFrag<D_I> ra0, ra1, rb0, rb1;
            ra0.load(kseq + (int64_t)ta0 * D_I, t4, va0);
            ra1.load(kseq + (int64_t)ta1 * D_I, t4, va1);
            rb0.load(kseq + (int64_t)tb0 * D_I, t4, vb0);
            rb1.load(kseq + (int64_t)tb1 * D_I, t4, vb1);
            {
                const int2 sc = fine_tile<D_I, NT>(qf, ra0, ra1);
                const uint32_t k0 = va0 ? (uint32_t)sc.x + 1u : 0u, k1 = va1 ? (uint32_t)sc.y + 1u : 0u;
                const int s0 = tile * 16 + g, s1 = s0 + 8;
                if (t4 == 0 && s0 < n_fine) fine_keys[s0] = k0;
                if (t4 == 1 && s1 < n_fine) fine_keys[s1] = k1;
                my_max = max(my_max, (unsigned long long)max(k0, k1));
                if (t4 == 0) my_count += (va0 ? 1u : 0u) + (va1 ? 1u : 0u);
            }
            if (tileB < n_tiles) {
                const int2 sc = fine_tile<D_I, NT>(qf, rb0, rb1);
                const uint32_t k0 = vb0 ? (uint32_t)sc.x + 1u : 0u, k1 = vb1 ? (uint32_t)sc.y + 1u : 0u;
                const int s0 = tileB * 16 + g, s1 = s0 + 8;
                if (t4 == 0 && s0 < n_fine) fine_keys[s0] = k0;
                if (t4 == 1 && s1 < n_fine) fine_keys[s1] = k1;
                my_max = max(my_max, (unsigned long long)max(k0, k1));
                if (t4 == 0) my_count += (vb0 ? 1u : 0u) + (vb1 ? 1u : 0u);
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            my_max = max(my_max, __shfl_xor_sync(0xffffffffu, my_max, o));
            my_count += __shfl_xor_sync(0xffffffffu, my_count, o);
        }
        if (lane == 0) {
            atomicMax(&sh.local_max, my_max);
            atomicAdd(&sh.local_count, my_count);
        }
        __syncthreads();
    }

    // ---------------- token top-k and SI assembly ----------------
    unsigned long long gmax;
    uint32_t n_valid;
    cluster_max_count(cl, sh, gmax, n_valid);
    const uint32_t k_tok = min((uint32_t)a.topk, n_valid);
    uint32_t thr;
    uint32_t quota;
    cluster_select<uint32_t>(cl, sh, parity, fine_keys, n_fine, k_tok, gmax, thr, quota);
    {
        const bool hi = a.hi_block > 0;
        cluster_compact<uint32_t>(cl, sh, fine_keys, n_fine, thr, quota, [&](int slot, uint32_t rank) {
            int tok;
            if (hi) {
                const int kb = slot / B;
                tok = kept_local[kb] * B + (slot - kb * B);
            } else {
                tok = flat_begin + slot;
            }
            out[s + rank] = tok;
        });
    }
    // Sink run, window run and the -1 tail.
    const int n_sel = (int)k_tok;
    const int win0 = s + n_sel;
    const int n_win = L - ws;
    for (int e = crank * kIxThreads + tid; e < a.budget; e += C * kIxThreads) {
        if (e < s) out[e] = e;
        else if (e >= win0 && e < win0 + n_win) out[e] = ws + (e - win0);
        else if (e >= win0 + n_win) out[e] = -1;
    }
    cl.sync();  // no CTA may exit while another can still read its shared memory
}

template <int D_I, int NT>
cudaError_t launch_t(const IndexArgs& a, const IndexPlan& plan, cudaStream_t stream) {
    auto kern = index_kernel<D_I, NT>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)plan.dyn_smem);
    if (e != cudaSuccess) return e;
    if (plan.cluster > 8) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
        if (e != cudaSuccess) return e;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(a.n_q * plan.cluster), 1, 1);
    cfg.blockDim = dim3(kIxThreads, 1, 1);
    cfg.dynamicSmemBytes = plan.dyn_smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = plan.cluster;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, a);
}

template <int D_I>
cudaError_t launch_d(const IndexArgs& a, const IndexPlan& plan, cudaStream_t stream) {
    const int nt = (a.H_I + 7) / 8;
    switch (nt) {
        case 1: return launch_t<D_I, 1>(a, plan, stream);
        case 2: return launch_t<D_I, 2>(a, plan, stream);
        case 4: return launch_t<D_I, 4>(a, plan, stream);
        case 8: return launch_t<D_I, 8>(a, plan, stream);
        default: break;
    }
    if (nt == 3) return launch_t<D_I, 4>(a, plan, stream);
    return launch_t<D_I, 8>(a, plan, stream);
}

template <int D_I, int NT>
int max_clusters_t(int cluster, size_t smem) {
    auto kern = index_kernel<D_I, NT>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess) return 0;
    if (cluster > 8 && cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess)
        return 0;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)cluster, 1, 1);
    cfg.blockDim = dim3(kIxThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = cluster;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess) {
        cudaGetLastError();
        return 0;
    }
    return n;
}

template <int D_I>
int max_clusters_d(int H_I, int cluster, size_t smem) {
    const int nt = (H_I + 7) / 8;
    if (nt <= 1) return max_clusters_t<D_I, 1>(cluster, smem);
    if (nt <= 2) return max_clusters_t<D_I, 2>(cluster, smem);
    if (nt <= 4) return max_clusters_t<D_I, 4>(cluster, smem);
    return max_clusters_t<D_I, 8>(cluster, smem);
}

}  // namespace

// Shared-memory budget for the per-CTA key arrays; beyond it they go to the
// global workspace.
constexpr size_t kSmemBudget = 160 * 1024;

IndexPlan plan_index(int cluster, int n_q, int max_len, const lsa_budget_t& b) {
    IndexPlan p;
    p.cluster = cluster;
    const int64_t C = cluster;
    size_t off = 0;
    const bool hi = b.hi_block > 0;
    const int64_t max_mid = max_len;  // middle <= L
    if (hi) {
        const int64_t nb = (max_len + b.hi_block - 1) / b.hi_block + 1;
        p.coarse_cap = (int)((nb + C - 1) / C);
        p.kept_cap = b.hi_topblocks;
        const int64_t kept_local = (b.hi_topblocks + C - 1) / C;
        p.fine_cap = (int)(kept_local * b.hi_block);
        p.smem_kept = 0;
        off = ((size_t)p.kept_cap * 4 + 15) / 16 * 16;
        p.smem_kept_local = (int)off;
        off += ((size_t)kept_local * 4 + 15) / 16 * 16;
    } else {
        p.coarse_cap = 0;
        p.kept_cap = 0;
        p.fine_cap = (int)((max_mid + C - 1) / C);
        p.smem_kept = 0;
        p.smem_kept_local = 0;
    }
    if (hi) {
        const size_t cbytes = (size_t)p.coarse_cap * 8;
        if (off + cbytes <= kSmemBudget) {
            p.smem_coarse = (int)off;
            off += (cbytes + 15) / 16 * 16;
        } else {
            p.smem_coarse = -1;
            p.ws_coarse = (size_t)n_q * C * p.coarse_cap * 8;
        }
    }
    const size_t fbytes = (size_t)p.fine_cap * 4;
    if (off + fbytes <= kSmemBudget) {
        p.smem_fine = (int)off;
        off += (fbytes + 15) / 16 * 16;
    } else {
        p.smem_fine = -1;
        p.ws_fine = (size_t)n_q * C * p.fine_cap * 4;
    }
    p.dyn_smem = off < 16 ? 16 : off;
    return p;
}

cudaError_t choose_index_cluster(int d_I, int H_I, int n_q, int max_len, const lsa_budget_t& b,
                                 IndexPlan* out) {
    static const int kChoices[] = {16, 8, 4, 2};
    for (int C : kChoices) {
        IndexPlan p = plan_index(C, n_q, max_len, b);
        int n = 0;
        switch (d_I) {
            case 32: n = max_clusters_d<32>(H_I, C, p.dyn_smem); break;
            case 64: n = max_clusters_d<64>(H_I, C, p.dyn_smem); break;
            default: n = max_clusters_d<128>(H_I, C, p.dyn_smem); break;
        }
        if (n >= n_q) {
            *out = p;
            return cudaSuccess;
        }
    }
    *out = plan_index(1, n_q, max_len, b);
    return cudaSuccess;
}

cudaError_t launch_index(const IndexArgs& a, const IndexPlan& plan, int d_I, cudaStream_t stream) {
    switch (d_I) {
        case 32: return launch_d<32>(a, plan, stream);
        case 64: return launch_d<64>(a, plan, stream);
        case 128: return launch_d<128>(a, plan, stream);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace lsa
