// index_topk.cu — exact top-k selection of a query row's keys with the keys
// held in registers: one CTA of 1024 threads per row (or a cluster of up to 4
// such CTAs for rows with more keys than a CTA holds).
//
// The method: keep the hi_topblocks best blocks (HI), then the topk best
// middle tokens; ties go to the lower position; the index set is the sink
// run, the selected tokens and the window run in ascending order, padded with
// -1 ("LongCat-Flash-Lite-Sparse (aitrends.kr)", section "기술적 특징", SI and
// HI bullets; "LongCat-2.0 (molayo1419.me)", section "1M 토큰에서의 Sparse
// Attention 문제").
//
// Design (B200). A selection is a chain of dependent steps, so its cost is
// the number of barriers and round trips, not arithmetic. Thread i of CTA c
// holds the KP keys of the row's slots [S*c + KP*i, S*c + KP*(i+1)) in
// registers (S = 1024*KP keys per CTA), so:
//   1. one pass of shared-memory atomics builds the histogram of the keys on
//      the logarithmic scale of key_bin (with a cluster, every CTA adds its
//      nonzero bins into every CTA's copy: one cluster barrier);
//   2. a suffix scan finds the bin holding the k-th largest key; the keys of
//      that bin (few, unless many scores tie) go to a candidate list — with
//      a cluster, to every CTA's list, tagged with their CTA, together with
//      each CTA's count above the bin (one more cluster barrier) — and each
//      candidate's rank among them gives the exact k-th largest key T and how
//      many keys equal to T are kept (a bin too full for the list is refined
//      by radix digits over the registers instead);
//   3. the keys > T, and the first keys == T in position order up to that
//      quota, are kept: one block-wide scan of each thread's two counts gives
//      every kept key its output rank, since a thread's keys are consecutive
//      positions.
// No step reads another CTA's shared memory after the last cluster barrier,
// so CTAs may exit independently.
#include <algorithm>

#include "common.cuh"
#include "index_common.cuh"
#include "internal.h"

namespace lsa {
namespace {

constexpr int kTkThreads = 1024;
constexpr int kTkWarps = kTkThreads / kWarp;
constexpr int kTkBinsPerThread = kHistBins / kTkThreads;  // 4
static_assert(kTkBinsPerThread == 4, "the scan gives each thread one 4-bin vector");
constexpr int kTkMaxCluster = 4;
constexpr int kTkCandCap = 2048;  // keys of the threshold bin held in the candidate list
constexpr int kTkDigitBits = 12;

struct TkShared {
    uint32_t hist[kHistBins];        // the row's histogram (every CTA's keys)
    uint32_t local_hist[kHistBins];  // this CTA's keys (clusters only)
    uint64_t cand[kTkCandCap];       // candidate keys, CTA of origin in the top bits
    uint64_t mine[kTkCandCap];       // this CTA's candidates before the exchange (clusters only)
    uint32_t wsum[kTkWarps];
    uint32_t wsum2[kTkWarps];
    uint32_t cta_above[kTkMaxCluster];  // per CTA: keys in bins above the threshold bin
    uint32_t og_gt[kTkMaxCluster];      // per CTA: candidates > T, == T
    uint32_t og_eq[kTkMaxCluster];
    uint32_t bin, above, in_bin;
    uint32_t push_base[kTkMaxCluster];  // this CTA's first slot in each CTA's candidate list
    uint32_t n_cand;  // candidate list length (remote adds with a cluster)
    uint32_t n_mine;  // this CTA's candidates
};

// Dynamic shared memory: TkShared | the keys (KP x 1024, transposed) | kept-block ids.
__host__ __device__ constexpr size_t tk_keys_off() { return (sizeof(TkShared) + 127) / 128 * 128; }

constexpr int kTkOriginShift = 60;
constexpr uint64_t kTkKeyMask = (1ull << kTkOriginShift) - 1ull;

__device__ __forceinline__ uint32_t tk_warp_sum(uint32_t v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Suffix scan of sh.hist (4 bins per thread). Returns the number of counted
// keys; when 1 <= krem <= total sets sh.bin / sh.above / sh.in_bin to the bin
// holding the krem-th largest key, the count above it and the count in it.
__device__ uint32_t tk_find_bin(TkShared& sh, uint32_t krem) {
    const int tid = threadIdx.x, lane = lane_id(), wid = warp_id();
    const uint4 h = reinterpret_cast<const uint4*>(sh.hist)[tid];  // bins 4*tid .. 4*tid+3
    const uint32_t c[4] = {h.x, h.y, h.z, h.w};
    const uint32_t own = c[0] + c[1] + c[2] + c[3];
    uint32_t x = own;  // keys in bins >= 4*tid within this warp
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t v = __shfl_down_sync(0xffffffffu, x, o);
        if (lane + o < 32) x += v;
    }
    if (lane == 0) sh.wsum[wid] = x;
    __syncthreads();
    const uint32_t wt = sh.wsum[lane];
    const uint32_t later = tk_warp_sum(lane > wid ? wt : 0u);
    const uint32_t total = tk_warp_sum(wt);
    const uint32_t S = x + later;  // keys in bins >= 4*tid
    if (krem >= 1u && S >= krem && S - own < krem) {
        uint32_t run = S - own;
#pragma unroll
        for (int j = 3; j >= 0; --j) {
            if (run + c[j] >= krem) {
                sh.bin = (uint32_t)(4 * tid + j);
                sh.above = run;
                sh.in_bin = c[j];
                break;
            }
            run += c[j];
        }
    }
    __syncthreads();
    return total;
}

// Block-wide exclusive scan of two counters (1024 threads). Returns the
// exclusive prefixes; tot_a / tot_b get the CTA totals.
__device__ __forceinline__ void tk_scan2(TkShared& sh, uint32_t a, uint32_t b, uint32_t& pa, uint32_t& pb,
                                         uint32_t& tot_a, uint32_t& tot_b) {
    const int lane = lane_id(), wid = warp_id();
    uint32_t xa = a, xb = b;  // inclusive within the warp
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t va = __shfl_up_sync(0xffffffffu, xa, o);
        const uint32_t vb = __shfl_up_sync(0xffffffffu, xb, o);
        if (lane >= o) {
            xa += va;
            xb += vb;
        }
    }
    if (lane == 31) {
        sh.wsum[wid] = xa;
        sh.wsum2[wid] = xb;
    }
    __syncthreads();
    const uint32_t ta = sh.wsum[lane], tb = sh.wsum2[lane];
    pa = tk_warp_sum(lane < wid ? ta : 0u) + xa - a;
    pb = tk_warp_sum(lane < wid ? tb : 0u) + xb - b;
    tot_a = tk_warp_sum(ta);
    tot_b = tk_warp_sum(tb);
}

// One row (blockIdx.y) selected by one CTA or a cluster of C CTAs (x).
// kTokens: fine top-k and the SI assembly of the index set (u32 keys);
// otherwise the HI block top-k (u64 keys) into the kept-block list.
template <typename K, bool kTokens, int KP>
__global__ void __launch_bounds__(kTkThreads, 1) topk_kernel(const __grid_constant__ IndexArgs a) {
    extern __shared__ __align__(16) uint8_t tk_dyn[];
    TkShared& sh = *reinterpret_cast<TkShared*>(tk_dyn);
    int32_t* s_kept = reinterpret_cast<int32_t*>(tk_dyn + tk_keys_off() + (size_t)KP * kTkThreads * sizeof(K));
    // (tokens with HI: the row's kept-block ids)
    const int r = blockIdx.y;
    const int tid = threadIdx.x;
    const uint32_t C = cluster_size(), c = cluster_rank();
    // the row's metadata is the caller's, never written by a kernel of this
    // library: it is read before the wait for the preceding kernel
    const int Lq = a.q_len[r];
    const int seq_q = a.q_seq[r];
    const int seq_c = min(max(seq_q, 0), a.n_seq - 1);
    const int64_t off_q = a.kv_offset[seq_c];
    const int slen_q = a.seq_lens[seq_c];
    const int64_t boff_q = a.hi_block > 0 ? a.blk_offset[seq_c] : 0;
    pdl_enter();
    const int n_kept_row = (kTokens && a.hi_block > 0) ? min(max(a.n_kept[r], 0), a.hi_topblocks) : 0;
    const int L = min(max(Lq, 0), a.max_len);
    const int s = min(a.sink, L);
    const int ws = max(s, L - a.window);
    const int B = a.hi_block;
    int n, first;  // keys of the row; first slot's block (blocks) or token (flat tokens)
    if (kTokens) {
        n = B > 0 ? n_kept_row * B : ws - s;
        first = s;
    } else {
        first = s / B;
        n = ws > s ? (ws + B - 1) / B - first : 0;
    }
    const int cap = kTokens ? a.fine_cap : a.coarse_cap;
    n = min(n, cap);
    // the keys of this thread: slots [base, base + KP)
    const int base = (int)c * (kTkThreads * KP) + tid * KP;
    const K* row_keys = kTokens ? reinterpret_cast<const K*>(a.fine_keys + (int64_t)r * a.fine_cap)
                                : reinterpret_cast<const K*>(a.coarse_keys + (int64_t)r * a.coarse_cap);
    // this thread's keys, in shared memory transposed (key j of thread t at
    // j * 1024 + t: every pass reads them without bank conflicts). The loads
    // cover the row's capacity (slots past n hold other calls' keys and are
    // zeroed when stored), so they need not wait for n.
    K* skeys = reinterpret_cast<K*>(tk_dyn + tk_keys_off());
    {
        constexpr int kPer = 16 / (int)sizeof(K);  // keys per 16-byte vector
        static_assert(KP % kPer == 0, "whole vectors per thread");
        constexpr int kVec = KP / kPer;
        constexpr int kBatch = kVec < 8 ? kVec : 8;  // 16-byte loads in flight per thread
#pragma unroll
        for (int v0 = 0; v0 < kVec; v0 += kBatch) {
            uint4 x[kBatch];
#pragma unroll
            for (int u = 0; u < kBatch; ++u) {
                const int s0 = base + (v0 + u) * kPer;
                x[u] = s0 < cap ? __ldcg(reinterpret_cast<const uint4*>(row_keys + s0)) : make_uint4(0u, 0u, 0u, 0u);
            }
#pragma unroll
            for (int u = 0; u < kBatch; ++u) {
                const int s0 = base + (v0 + u) * kPer;
                const K* e = reinterpret_cast<const K*>(&x[u]);
#pragma unroll
                for (int j = 0; j < kPer; ++j)
                    skeys[((v0 + u) * kPer + j) * kTkThreads + tid] = (s0 + j < n) ? e[j] : K(0);
            }
        }
    }
    auto key = [&](int j) -> K { return skeys[j * kTkThreads + tid]; };
    if (kTokens && B > 0)
        for (int i = tid; i < n_kept_row; i += kTkThreads) s_kept[i] = a.kept[(int64_t)r * a.hi_topblocks + i];
    uint32_t* hist = C > 1 ? sh.local_hist : sh.hist;
    for (int i = tid; i < kHistBins; i += kTkThreads) {
        sh.hist[i] = 0u;
        if (C > 1) sh.local_hist[i] = 0u;
    }
    if (tid == 0) {
        sh.n_cand = 0u;
        sh.n_mine = 0u;
    }
    // the row check (as in the scoring kernels), uniform over the cluster
    int32_t bits = 0;
    if (seq_q < 0 || seq_q >= a.n_seq) bits = LSA_DEV_BAD_SEQ;
    else if (Lq < 1 || Lq > a.max_len || Lq > slen_q || off_q < 0 || off_q + slen_q > a.total_tokens ||
             (a.hi_block > 0 && (boff_q < 0 || boff_q + (Lq + a.hi_block - 1) / a.hi_block > a.block_rows)))
        bits = LSA_DEV_BAD_LENGTH;
    int32_t* out = a.index_sets + (int64_t)r * a.budget;
    if (bits != 0) {
        if (kTokens) {
            if (c == 0 && tid == 0) flag(a.dev_status, bits);
            for (int e = (int)(c * kTkThreads) + tid; e < a.budget; e += (int)(C * kTkThreads)) out[e] = -1;
        } else if (c == 0 && tid == 0) {
            a.n_kept[r] = 0;  // the token selection reports the row
        }
        return;  // uniform over the cluster, before any cluster barrier
    }
    __syncthreads();
    if (C > 1) cluster_arrive();  // every CTA's histograms are clear
#pragma unroll 4
    for (int j = 0; j < KP; ++j) {
        const K kk = key(j);
        warp_hist_add(hist, kk != K(0) ? key_bin((unsigned long long)kk) : 0xffffffffu);
    }
    __syncthreads();
    if (C > 1) {
        cluster_wait();
        const uint32_t hb = smem_u32(sh.hist);
#pragma unroll
        for (int j = 0; j < kTkBinsPerThread; ++j) {
            const int b = tid + j * kTkThreads;
            const uint32_t v = sh.local_hist[b];
            if (v != 0u)
                for (uint32_t t = 0; t < C; ++t)
                    red_add_cluster(map_cta(hb + 4u * (uint32_t)b, t), v);
        }
        cluster_sync();
    }
    const uint32_t want = (uint32_t)(kTokens ? a.topk : a.hi_topblocks);
    const uint32_t total = tk_find_bin(sh, want);
    pdl_trigger();  // the threshold and the compaction are left
    const uint32_t k = min(want, total);
    // the index set's sink and window runs and padding (tokens)
    if (kTokens) {
        const int win0 = s + (int)k;
        const int n_win = L - ws;
        for (int e = (int)(c * kTkThreads) + tid; e < a.budget; e += (int)(C * kTkThreads)) {
            if (e < s) out[e] = e;
            else if (e >= win0 && e < win0 + n_win) out[e] = ws + (e - win0);
            else if (e >= win0 + n_win) out[e] = -1;
        }
    }
    K T = K(1);                     // keys >= T with the quota rule below are kept
    uint32_t quota = 0xffffffffu;   // keys == T kept (first in position order)
    uint32_t gbase = 0, ebase = 0;  // kept keys > T / == T of the lower-ranked CTAs
    if (k > 0u && k < total) {
        const uint32_t tb = sh.bin, above = sh.above, in_bin = sh.in_bin;
        const uint32_t krem = k - above;
        if (in_bin <= (uint32_t)kTkCandCap) {
            // this CTA's keys above the bin (from its histogram) and its
            // candidates, published to every CTA
            uint32_t ab = 0;
            if (C > 1) {
#pragma unroll
                for (int j = 0; j < kTkBinsPerThread; ++j) {
                    const uint32_t b = (uint32_t)(tid + j * kTkThreads);
                    if (b > tb) ab += sh.local_hist[b];
                }
                ab = tk_warp_sum(ab);
                if (lane_id() == 0) sh.wsum2[warp_id()] = ab;
            }
            const uint64_t tag = (uint64_t)c << kTkOriginShift;
            uint64_t* list = C > 1 ? sh.mine : sh.cand;
#pragma unroll 4
            for (int j = 0; j < KP; ++j) {
                const K kk = key(j);
                const bool take = kk != K(0) && key_bin((unsigned long long)kk) == tb;
                const uint32_t p = warp_append(&sh.n_mine, take);
                if (take && p < (uint32_t)kTkCandCap) list[p] = (uint64_t)kk | tag;
            }
            __syncthreads();
            if (C > 1) {
                // one slot range per target CTA, then the candidates and this
                // CTA's count above the bin into every CTA
                const uint32_t mc = min(sh.n_mine, (uint32_t)kTkCandCap);
                if (tid < (int)C) {
                    uint32_t above_local = 0;
                    for (int w = 0; w < kTkWarps; ++w) above_local += sh.wsum2[w];
                    sh.push_base[tid] = atom_add_cluster(map_cta(smem_u32(&sh.n_cand), (uint32_t)tid), mc);
                    st_cluster(map_cta(smem_u32(&sh.cta_above[c]), (uint32_t)tid), above_local);
                }
                __syncthreads();
                for (uint32_t i = tid; i < mc; i += kTkThreads)
                    for (uint32_t t = 0; t < C; ++t) {
                        const uint32_t p = sh.push_base[t] + i;
                        if (p < (uint32_t)kTkCandCap) st_cluster_u64(map_cta(smem_u32(&sh.cand[p]), t), sh.mine[i]);
                    }
                cluster_sync();  // after this no CTA touches another CTA's shared memory
            }
            // exact T: radix digits below the bin's leading 7 bits, over the
            // candidate list (identical in every CTA of a cluster)
            const uint32_t nc = min(C > 1 ? sh.n_cand : sh.n_mine, (uint32_t)kTkCandCap);
            if (tid < kTkMaxCluster) {
                sh.og_gt[tid] = 0u;
                sh.og_eq[tid] = 0u;
            }
            if (tb < 64u) {  // small bins hold a single key value
                T = (K)tb;
                quota = krem;
            } else {
                const int nb = (int)(tb >> 6) + 6;  // bit length of the bin's keys
                int shift = nb - 7;
                uint64_t prefix = 64u | (tb & 63u);
                uint32_t kr = krem;
                while (shift > 0) {
                    const int width = shift < kTkDigitBits ? shift : kTkDigitBits;
                    shift -= width;
                    const uint32_t mask = (1u << width) - 1u;
                    reinterpret_cast<uint4*>(sh.hist)[tid] = make_uint4(0u, 0u, 0u, 0u);
                    __syncthreads();
                    for (uint32_t i = tid; i < nc; i += kTkThreads) {
                        const uint64_t v = sh.cand[i] & kTkKeyMask;
                        if ((v >> (shift + width)) == prefix) atomicAdd(&sh.hist[(uint32_t)(v >> shift) & mask], 1u);
                    }
                    __syncthreads();
                    tk_find_bin(sh, kr);
                    prefix = (prefix << width) | sh.bin;
                    kr -= sh.above;
                }
                T = (K)prefix;
                quota = kr;
            }
            if (C > 1) {
                for (uint32_t i = tid; i < nc; i += kTkThreads) {
                    const uint64_t e = sh.cand[i];
                    const K v = (K)(e & kTkKeyMask);
                    const uint32_t o = (uint32_t)(e >> kTkOriginShift);
                    if (v > T) atomicAdd(&sh.og_gt[o], 1u);
                    else if (v == T) atomicAdd(&sh.og_eq[o], 1u);
                }
                __syncthreads();
                for (uint32_t o = 0; o < c; ++o) {
                    gbase += sh.cta_above[o] + sh.og_gt[o];
                    ebase += sh.og_eq[o];
                }
            }
        } else {
            // a bin too full for the list (many equal scores): radix digits
            // over the registers, one histogram (and, with a cluster, one
            // exchange) per digit
            const int nb = (int)(tb >> 6) + 6;  // bit length of the bin's keys
            int shift = tb < 64u ? 0 : nb - 7;   // small bins hold a single key value
            K prefix = tb < 64u ? (K)tb : (K)(64u | (tb & 63u));
            uint32_t kr = krem;
            while (shift > 0) {
                const int width = shift < kTkDigitBits ? shift : kTkDigitBits;
                shift -= width;
                const uint32_t mask = (1u << width) - 1u;
                for (int i = tid; i < kHistBins; i += kTkThreads) {
                    sh.hist[i] = 0u;
                    if (C > 1) sh.local_hist[i] = 0u;
                }
                __syncthreads();
                if (C > 1) cluster_sync();
#pragma unroll 4
                for (int j = 0; j < KP; ++j) {
                    const K kk = key(j);
                    warp_hist_add(hist, kk != K(0) && (K)(kk >> (shift + width)) == prefix
                                            ? (uint32_t)(kk >> shift) & mask : 0xffffffffu);
                }
                __syncthreads();
                if (C > 1) {
                    const uint32_t hb = smem_u32(sh.hist);
                    for (int b = tid; b < kHistBins; b += kTkThreads) {
                        const uint32_t v = sh.local_hist[b];
                        if (v != 0u)
                            for (uint32_t t = 0; t < C; ++t) red_add_cluster(map_cta(hb + 4u * (uint32_t)b, t), v);
                    }
                    cluster_sync();
                }
                tk_find_bin(sh, kr);
                prefix = (K)((prefix << width) | (K)sh.bin);
                kr -= sh.above;
            }
            T = prefix;
            quota = kr;
            if (C > 1) {
                // every CTA's counts of keys > T and == T
                uint32_t g = 0, e = 0;
#pragma unroll
                for (int j = 0; j < KP; ++j) {
                    g += key(j) > T ? 1u : 0u;
                    e += key(j) == T ? 1u : 0u;
                }
                g = tk_warp_sum(g);
                e = tk_warp_sum(e);
                if (lane_id() == 0) {
                    sh.wsum[warp_id()] = g;
                    sh.wsum2[warp_id()] = e;
                }
                __syncthreads();
                if (tid < (int)C) {
                    uint32_t tg = 0, te = 0;
                    for (int w = 0; w < kTkWarps; ++w) {
                        tg += sh.wsum[w];
                        te += sh.wsum2[w];
                    }
                    st_cluster(map_cta(smem_u32(&sh.og_gt[c]), (uint32_t)tid), tg);
                    st_cluster(map_cta(smem_u32(&sh.og_eq[c]), (uint32_t)tid), te);
                }
                cluster_sync();  // after this no CTA touches another CTA's shared memory
                for (uint32_t o = 0; o < c; ++o) {
                    gbase += sh.og_gt[o];
                    ebase += sh.og_eq[o];
                }
            }
        }
    } else if (k > 0u && C > 1) {
        // every key is kept: ranks follow the CTAs' key counts
        uint32_t g = 0;
#pragma unroll
        for (int j = 0; j < KP; ++j) g += key(j) != K(0) ? 1u : 0u;
        g = tk_warp_sum(g);
        if (lane_id() == 0) sh.wsum[warp_id()] = g;
        __syncthreads();
        if (tid < (int)C) {
            uint32_t tg = 0;
            for (int w = 0; w < kTkWarps; ++w) tg += sh.wsum[w];
            st_cluster(map_cta(smem_u32(&sh.og_gt[c]), (uint32_t)tid), tg);
        }
        cluster_sync();
        for (uint32_t o = 0; o < c; ++o) gbase += sh.og_gt[o];
    }
    if (k == 0u) {
        if (!kTokens && c == 0 && tid == 0) a.n_kept[r] = 0;
        return;
    }
    // ranks: this thread's keys > T and == T, scanned over the CTA
    uint32_t ng = 0, ne = 0;
#pragma unroll
    for (int j = 0; j < KP; ++j) {
        ng += key(j) > T ? 1u : 0u;
        ne += key(j) == T ? 1u : 0u;
    }
    uint32_t pg, pe, tg, te;
    tk_scan2(sh, ng, ne, pg, pe, tg, te);
    uint32_t gi = gbase + pg, ei = ebase + pe;
    const int lgB = (B > 0 && (B & (B - 1)) == 0) ? __ffs(B) - 1 : -1;
    int32_t* kept_out = a.kept + (int64_t)r * a.hi_topblocks;
#pragma unroll
    for (int j = 0; j < KP; ++j) {
        uint32_t rank = 0xffffffffu;
        if (key(j) > T) {
            rank = gi + min(ei, quota);
            ++gi;
        } else if (key(j) == T) {
            if (ei < quota) rank = gi + ei;
            ++ei;
        }
        if (rank < k) {
            const int slot = base + j;
            if (kTokens) {
                int tok;
                if (B > 0) {
                    const int kb = lgB >= 0 ? slot >> lgB : slot / B;
                    tok = s_kept[kb] * B + (slot - kb * B);
                } else {
                    tok = first + slot;
                }
                out[s + rank] = tok;
            } else {
                kept_out[rank] = first + slot;
            }
        }
    }
    if (!kTokens && c == 0 && tid == 0) a.n_kept[r] = (int32_t)k;
}

// Prefill rows: the tensor-core scoring kept, per row, the (key, position)
// pairs that passed its running threshold, in no particular order. The row's
// exact top-k by (key desc, position asc) is the top-k of the distinct
// values key << 32 | (2^32 - 1 - position), found over the pairs in global
// memory (histogram pass, then radix digits over the threshold bin's
// candidates or, for a bin too full for the list, over all pairs); the kept
// positions are sorted ascending in shared memory (bitonic) and written with
// the SI sink and window runs. One CTA of 1024 threads per row.
constexpr int kPairSortCap = LSA_MAX_BUDGET;  // topk <= budget

struct PairShared {
    uint32_t hist[kHistBins];
    uint64_t cand[kTkCandCap];
    uint32_t wsum[kTkWarps];
    uint32_t wsum2[kTkWarps];
    uint32_t bin, above, in_bin;
    uint32_t n_cand, n_sel;
};

__device__ __forceinline__ uint64_t pair_value(uint64_t e) {
    return (e & 0xffffffff00000000ull) | (uint64_t)(0xffffffffu - (uint32_t)e);
}

// tk_find_bin over PairShared (same scan as for TkShared)
__device__ uint32_t pair_find_bin(PairShared& sh, uint32_t krem) {
    const int tid = threadIdx.x, lane = lane_id(), wid = warp_id();
    const uint4 h = reinterpret_cast<const uint4*>(sh.hist)[tid];
    const uint32_t c[4] = {h.x, h.y, h.z, h.w};
    const uint32_t own = c[0] + c[1] + c[2] + c[3];
    uint32_t x = own;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t v = __shfl_down_sync(0xffffffffu, x, o);
        if (lane + o < 32) x += v;
    }
    if (lane == 0) sh.wsum[wid] = x;
    __syncthreads();
    const uint32_t wt = sh.wsum[lane];
    const uint32_t later = tk_warp_sum(lane > wid ? wt : 0u);
    const uint32_t total = tk_warp_sum(wt);
    const uint32_t S = x + later;
    if (krem >= 1u && S >= krem && S - own < krem) {
        uint32_t run = S - own;
#pragma unroll
        for (int j = 3; j >= 0; --j) {
            if (run + c[j] >= krem) {
                sh.bin = (uint32_t)(4 * tid + j);
                sh.above = run;
                sh.in_bin = c[j];
                break;
            }
            run += c[j];
        }
    }
    __syncthreads();
    return total;
}

__global__ void __launch_bounds__(kTkThreads, 1) topk_pairs_kernel(const __grid_constant__ IndexArgs a) {
    extern __shared__ __align__(16) uint8_t pr_dyn[];
    PairShared& sh = *reinterpret_cast<PairShared*>(pr_dyn);
    int32_t* sel = reinterpret_cast<int32_t*>(pr_dyn + (sizeof(PairShared) + 15) / 16 * 16);
    const int r = blockIdx.x;
    const int tid = threadIdx.x;
    // the row's metadata (the caller's) before the wait for the scoring kernel
    const int Lq = a.q_len[r];
    const int seq_q = a.q_seq[r];
    const int seq_c = min(max(seq_q, 0), a.n_seq - 1);
    const int64_t off_q = a.kv_offset[seq_c];
    const int slen_q = a.seq_lens[seq_c];
    pdl_enter();
    const int L = min(max(Lq, 0), a.max_len);
    const int s = min(a.sink, L);
    const int ws = max(s, L - a.window);
    int32_t* out = a.index_sets + (int64_t)r * a.budget;
    int32_t bits = 0;
    if (seq_q < 0 || seq_q >= a.n_seq) bits = LSA_DEV_BAD_SEQ;
    else if (Lq < 1 || Lq > a.max_len || Lq > slen_q || off_q < 0 || off_q + slen_q > a.total_tokens)
        bits = LSA_DEV_BAD_LENGTH;
    if (bits != 0) {
        if (tid == 0) flag(a.dev_status, bits);
        for (int e = tid; e < a.budget; e += kTkThreads) out[e] = -1;
        return;
    }
    // the row's candidates: one segment per token split of the scoring
    const uint64_t* pairs = a.cand + (int64_t)r * a.fine_cap;
    __shared__ int32_t seg_lo[LSA_TC_MAX_SPLITS], seg_n[LSA_TC_MAX_SPLITS];
    if (tid < a.tc_splits) {
        const int2 sg = reinterpret_cast<const int2*>(a.cand_seg)[(int64_t)r * LSA_TC_MAX_SPLITS + tid];
        const int lo = min(max(sg.x, 0), a.fine_cap);
        seg_lo[tid] = lo;
        seg_n[tid] = min(max(sg.y, 0), a.fine_cap - lo);
    }
    __syncthreads();
    uint32_t n = 0;
    for (int sp = 0; sp < a.tc_splits; ++sp) n += (uint32_t)seg_n[sp];
    // every candidate pair once: f(pair)
    // (every lane of a warp calls f the same number of times: f(pair, ok))
    auto for_each_pair = [&](auto&& f) {
        for (int sp = 0; sp < a.tc_splits; ++sp) {
            const uint64_t* seg = pairs + seg_lo[sp];
            const int cnt = seg_n[sp];
            for (int i0 = tid - (tid & 31); i0 < cnt; i0 += kTkThreads) {
                const int i = i0 + (tid & 31);
                const bool ok = i < cnt;
                f(ok ? __ldcg(seg + i) : 0ull, ok);
            }
        }
    };
    const uint32_t k = min((uint32_t)a.topk, (uint32_t)(ws - s));  // every middle token is a candidate
    // the index set's sink and window runs and padding
    {
        const int win0 = s + (int)k;
        const int n_win = L - ws;
        for (int e = tid; e < a.budget; e += kTkThreads) {
            if (e < s) out[e] = e;
            else if (e >= win0 && e < win0 + n_win) out[e] = ws + (e - win0);
            else if (e >= win0 + n_win) out[e] = -1;
        }
    }
    if (k == 0u) return;
    // the k largest values: value >= T
    uint64_t T = 0ull;
    if (n > k) {
        for (int i = tid; i < kHistBins; i += kTkThreads) sh.hist[i] = 0u;
        if (tid == 0) sh.n_cand = 0u;
        __syncthreads();
        for_each_pair([&](uint64_t e, bool ok) { warp_hist_add(sh.hist, ok ? key_bin(pair_value(e)) : 0xffffffffu); });
        __syncthreads();
        pair_find_bin(sh, k);
        const uint32_t tb = sh.bin, in_bin = sh.in_bin;
        uint32_t kr = k - sh.above;
        const int nb = (int)(tb >> 6) + 6;
        int shift = tb < 64u ? 0 : nb - 7;
        uint64_t prefix = tb < 64u ? (uint64_t)tb : (uint64_t)(64u | (tb & 63u));
        const bool listed = in_bin <= (uint32_t)kTkCandCap;
        if (listed) {
            __syncthreads();
            for_each_pair([&](uint64_t e, bool ok) {
                const uint64_t v = pair_value(e);
                const bool take = ok && key_bin(v) == tb;
                const uint32_t p = warp_append(&sh.n_cand, take);
                if (take && p < (uint32_t)kTkCandCap) sh.cand[p] = v;
            });
            __syncthreads();
        }
        const uint32_t nc = min(sh.n_cand, (uint32_t)kTkCandCap);
        while (shift > 0) {
            const int width = shift < kTkDigitBits ? shift : kTkDigitBits;
            shift -= width;
            const uint64_t mask = (1ull << width) - 1ull;
            reinterpret_cast<uint4*>(sh.hist)[tid] = make_uint4(0u, 0u, 0u, 0u);
            __syncthreads();
            if (listed) {
                for (uint32_t i = tid; i < nc; i += kTkThreads) {
                    const uint64_t v = sh.cand[i];
                    if ((v >> (shift + width)) == prefix) atomicAdd(&sh.hist[(uint32_t)((v >> shift) & mask)], 1u);
                }
            } else {
                for_each_pair([&](uint64_t e, bool ok) {
                    const uint64_t v = pair_value(e);
                    warp_hist_add(sh.hist, ok && (v >> (shift + width)) == prefix ? (uint32_t)((v >> shift) & mask)
                                                                                  : 0xffffffffu);
                });
            }
            __syncthreads();
            pair_find_bin(sh, kr);
            prefix = (prefix << width) | sh.bin;
            kr -= sh.above;
        }
        T = prefix;  // values are distinct: exactly k are >= T
    }
    // the kept positions, then sorted ascending
    if (tid == 0) sh.n_sel = 0u;
    __syncthreads();
    for_each_pair([&](uint64_t e, bool ok) {
        const bool take = ok && pair_value(e) >= T;
        const uint32_t p = warp_append(&sh.n_sel, take);
        if (take && p < (uint32_t)kPairSortCap) sel[p] = (int32_t)(uint32_t)e;
    });
    __syncthreads();
    const uint32_t m = min(sh.n_sel, k);
    uint32_t P = 1;
    while (P < m) P <<= 1;
    for (uint32_t i = m + tid; i < P; i += kTkThreads) sel[i] = 0x7fffffff;
    __syncthreads();
    for (uint32_t size = 2; size <= P; size <<= 1) {
        for (uint32_t stride = size >> 1; stride > 0; stride >>= 1) {
            for (uint32_t i = tid; i < P / 2; i += kTkThreads) {
                const uint32_t lo = 2 * i - (i & (stride - 1));  // index with bit `stride` clear
                const uint32_t hi = lo + stride;
                const bool up = (lo & size) == 0;
                const int32_t x = sel[lo], y = sel[hi];
                if ((x > y) == up) {
                    sel[lo] = y;
                    sel[hi] = x;
                }
            }
            __syncthreads();
        }
    }
    pdl_trigger();
    for (uint32_t i = tid; i < m; i += kTkThreads) out[s + i] = sel[i];
}

}  // namespace

// Keys per thread and CTAs per row for a row capacity of `cap` keys, or
// false when the register selection does not hold that many.
bool topk_plan(int cap, int key_bytes, int& kp, int& cluster) {
    const int kp_max = key_bytes == 4 ? 32 : 16;  // 128 KB of keys per CTA
    for (int C = 1; C <= kTkMaxCluster; C *= 2) {
        for (int k = key_bytes == 4 ? 4 : 2; k <= kp_max; k *= 2) {
            if ((int64_t)C * kTkThreads * k >= cap) {
                kp = k;
                cluster = C;
                return true;
            }
        }
    }
    return false;
}

size_t topk_smem(bool tokens, int kp, int hi_topblocks) {
    return tk_keys_off() + (size_t)kp * kTkThreads * (tokens ? 4 : 8) + (tokens ? (size_t)hi_topblocks * 4 : 0) + 16;
}

template <typename Kern>
static cudaError_t launch_topk_t(Kern kern, const IndexArgs& a, int cluster, size_t smem, cudaStream_t stream) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    return launch_pdl(kern, dim3((unsigned)cluster, (unsigned)a.n_q, 1), dim3(kTkThreads), smem, stream,
                      cluster > 1 ? cluster : 0, a);
}

size_t topk_pairs_smem() { return (sizeof(PairShared) + 15) / 16 * 16 + (size_t)kPairSortCap * 4; }

cudaError_t launch_topk_pairs(const IndexArgs& a, cudaStream_t stream) {
    const size_t smem = topk_pairs_smem();
    cudaError_t e = cudaFuncSetAttribute(topk_pairs_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    return launch_pdl(topk_pairs_kernel, dim3((unsigned)a.n_q), dim3(kTkThreads), smem, stream, 0, a);
}

cudaError_t launch_topk(const IndexArgs& a, bool blocks, int kp, int cluster, cudaStream_t stream) {
    const size_t smem = topk_smem(!blocks, kp, a.hi_block > 0 ? a.hi_topblocks : 0);
    if (blocks) {
        switch (kp) {
            case 2: return launch_topk_t(topk_kernel<uint64_t, false, 2>, a, cluster, smem, stream);
            case 4: return launch_topk_t(topk_kernel<uint64_t, false, 4>, a, cluster, smem, stream);
            case 8: return launch_topk_t(topk_kernel<uint64_t, false, 8>, a, cluster, smem, stream);
            case 16: return launch_topk_t(topk_kernel<uint64_t, false, 16>, a, cluster, smem, stream);
            default: return cudaErrorInvalidValue;
        }
    }
    switch (kp) {
        case 4: return launch_topk_t(topk_kernel<uint32_t, true, 4>, a, cluster, smem, stream);
        case 8: return launch_topk_t(topk_kernel<uint32_t, true, 8>, a, cluster, smem, stream);
        case 16: return launch_topk_t(topk_kernel<uint32_t, true, 16>, a, cluster, smem, stream);
        case 32: return launch_topk_t(topk_kernel<uint32_t, true, 32>, a, cluster, smem, stream);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace lsa
