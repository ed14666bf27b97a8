// index_select.cu — the latency half of the LSA indexer: exact top-k
// selection of HI blocks and of fine tokens, and the SI assembly of the
// index set.
//
// The method: keep the hi_topblocks best blocks (HI), then the topk best
// middle tokens; ties go to the lower position; the index set is the sink
// run, the selected tokens and the window run in ascending order, padded with
// -1 ("LongCat-Flash-Lite-Sparse (aitrends.kr)", section "기술적 특징", SI and
// HI bullets; "LongCat-2.0 (molayo1419.me)", section "1M 토큰에서의 Sparse
// Attention 문제").
//
// Design (B200): a query row is selected by one thread-block cluster of C
// CTAs, each owning a contiguous slice of the row's keys (score + 1, 0 = not
// a candidate), so a pass over a row costs 1/C of a pass on one SM. The few
// cross-CTA steps go through distributed shared memory and cluster barriers:
//   1. every CTA stages its slice in shared memory and builds the slice's
//      histogram on the logarithmic scale of key_bin, then adds its nonzero
//      bins into every CTA's copy of the row histogram (remote red.add);
//   2. each CTA scans the row histogram for the bin holding the k-th largest
//      key (all CTAs reach the same answer), gathers its keys of that bin and
//      appends them to every CTA's candidate list; 12-bit radix levels over
//      that short list give the exact k-th largest key T and how many keys
//      equal to T are kept (a bin too full for the list is refined by more
//      cluster histograms over the slices instead);
//   3. each CTA counts its kept keys and publishes the count; the counts of
//      lower-ranked CTAs give its first output position, and bitmap ballots
//      with one CTA prefix give every kept key its rank in position order.
#include <algorithm>

#include "append.cuh"
#include "common.cuh"
#include "index_common.cuh"
#include "internal.h"

namespace lsa {
namespace {

constexpr int kSelThreads = 512;
constexpr int kSelWarps = kSelThreads / kWarp;
constexpr int kBinsPerThread = kHistBins / kSelThreads;  // 8
static_assert(kBinsPerThread == 8, "the scan gives each thread two 4-bin vectors");
constexpr int kMaxCluster = 16;
constexpr int kDigitBits = 12;            // refinement digit: 4096 bins
constexpr int kCandCap = 2048;            // keys of the threshold bin held in a list
constexpr int kChunkWords = kSelThreads;  // compaction: one bitmap word per thread per chunk
constexpr int kUnroll = 4;                // independent loads in flight per thread

struct SelShared {
    uint32_t local_hist[kHistBins];  // this CTA's slice
    uint32_t hist[kHistBins];        // the row: every CTA adds its slice into every CTA's copy
    uint32_t gt_words[kChunkWords];
    uint32_t eq_words[kChunkWords];
    uint32_t wsum[kSelWarps];
    uint32_t wsum2[kSelWarps];
    uint32_t cta_gt[kMaxCluster];  // kept keys per CTA slice (each CTA writes its own into all)
    uint32_t cta_eq[kMaxCluster];
    uint32_t push_base[kMaxCluster];
    uint32_t cta_above[kMaxCluster];  // keys above the threshold bin per CTA slice (candidate path)
    uint32_t og_gt[kMaxCluster];      // candidates > T and == T per originating CTA
    uint32_t og_eq[kMaxCluster];
    uint32_t bin, above, in_bin;
    uint32_t count;        // length of the row's candidate list (remote adds)
    uint32_t local_count;  // candidates of this slice
    unsigned long long few[kWarp];  // the last <= 32 candidates of the threshold (few_rank)
    unsigned long long few_T;
    uint32_t few_quota;
};

// Candidate list entries: the key in the low 60 bits (scores stay below 2^40
// under the ABI's bounds), the originating CTA's rank in the top 4.
constexpr int kOriginShift = 60;
constexpr uint64_t kKeyMask = (1ull << kOriginShift) - 1ull;

// Dynamic shared memory: SelShared | candidate list | this slice's candidates
// | staged slice keys | kept-block ids of the slice (tokens only).
struct SelLayout {
    uint32_t off_cand, off_mine, off_stage, off_kept, bytes;
};

__host__ __device__ __forceinline__ uint32_t align16u(uint32_t x) { return (x + 15u) / 16u * 16u; }

__host__ __device__ __forceinline__ SelLayout sel_layout(int key_bytes, int stage_keys, int kept_slots) {
    SelLayout L;
    uint32_t o = align16u((uint32_t)sizeof(SelShared));
    L.off_cand = o;
    o += (uint32_t)(kCandCap * 8);
    L.off_mine = o;
    o += (uint32_t)(kCandCap * key_bytes);
    L.off_stage = o;
    o += align16u((uint32_t)stage_keys * (uint32_t)key_bytes);
    L.off_kept = o;
    o += align16u((uint32_t)kept_slots * 4u);
    L.bytes = o;
    return L;
}

template <typename K>
__device__ __forceinline__ void st_cluster_key(uint32_t addr, K v) {
    if constexpr (sizeof(K) == 4) {
        st_cluster(addr, (uint32_t)v);
    } else {
        st_cluster_u64(addr, (uint64_t)v);
    }
}

__device__ __forceinline__ uint32_t warp_sum(uint32_t v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Keys of this CTA's slice, either staged in shared memory or read from
// global memory; index i is relative to the slice start.
template <typename K>
struct Keys {
    const K* g;  // global copy
    uint32_t s;  // shared-memory address of the staged copy (0 when not staged)
    __device__ __forceinline__ K operator[](int i) const {
        if (s != 0u) {
            if constexpr (sizeof(K) == 4) {
                uint32_t v;
                asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(s + 4u * (uint32_t)i));
                return (K)v;
            } else {
                unsigned long long v;
                asm volatile("ld.shared.u64 %0, [%1];" : "=l"(v) : "r"(s + 8u * (uint32_t)i));
                return (K)v;
            }
        }
        return __ldcg(g + i);
    }
    // 16-byte vector i (keys 16/sizeof(K) * i onwards)
    __device__ __forceinline__ uint4 vec(int i) const {
        if (s != 0u) {
            uint4 v;
            asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                         : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                         : "r"(s + 16u * (uint32_t)i));
            return v;
        }
        return __ldcg(reinterpret_cast<const uint4*>(g) + i);
    }
};

// Suffix scan of the row histogram sh.hist. Returns the number of counted
// keys; when 1 <= krem <= total also gives the bin holding the krem-th
// largest key, the count above it (higher bins) and the count in it.
__device__ uint32_t find_bin(SelShared& sh, uint32_t krem, uint32_t& bin, uint32_t& above, uint32_t& in_bin) {
    const int tid = threadIdx.x, lane = lane_id(), wid = warp_id();
    const uint4 h0 = reinterpret_cast<const uint4*>(sh.hist)[2 * tid];  // bins 8*tid .. 8*tid+7
    const uint4 h1 = reinterpret_cast<const uint4*>(sh.hist)[2 * tid + 1];
    const uint32_t c[8] = {h0.x, h0.y, h0.z, h0.w, h1.x, h1.y, h1.z, h1.w};
    uint32_t own = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) own += c[j];
    uint32_t x = own;  // keys in bins >= 8*tid within this warp
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t v = __shfl_down_sync(0xffffffffu, x, o);
        if (lane + o < 32) x += v;
    }
    if (lane == 0) sh.wsum[wid] = x;
    __syncthreads();
    const uint32_t wt = lane < kSelWarps ? sh.wsum[lane] : 0u;
    const uint32_t later = warp_sum(lane > wid ? wt : 0u);
    const uint32_t total = warp_sum(wt);
    const uint32_t S = x + later;  // keys in bins >= 8*tid
    if (krem >= 1u && S >= krem && S - own < krem) {
        uint32_t run = S - own;
#pragma unroll
        for (int j = 7; j >= 0; --j) {
            if (run + c[j] >= krem) {
                sh.bin = (uint32_t)(8 * tid + j);
                sh.above = run;
                sh.in_bin = c[j];
                break;
            }
            run += c[j];
        }
    }
    __syncthreads();
    bin = sh.bin;
    above = sh.above;
    in_bin = sh.in_bin;
    return total;
}

// Adds this CTA's slice histogram (sh.local_hist) into every CTA's row
// histogram; the caller brackets it with cluster barriers.
__device__ void push_hist(SelShared& sh, uint32_t C) {
    const uint32_t base = smem_u32(sh.hist);
#pragma unroll 1
    for (int j = 0; j < kBinsPerThread; ++j) {
        const int b = threadIdx.x + j * kSelThreads;
        const uint32_t v = sh.local_hist[b];
        if (v != 0u)
            for (uint32_t t = 0; t < C; ++t) red_add_cluster(map_cta(base + 4u * (uint32_t)b, t), v);
    }
}

__device__ __forceinline__ void zero_hists(SelShared& sh) {
    uint4* l = reinterpret_cast<uint4*>(sh.local_hist);
    uint4* h = reinterpret_cast<uint4*>(sh.hist);
    const uint4 z = make_uint4(0u, 0u, 0u, 0u);
    l[threadIdx.x] = z;
    l[threadIdx.x + kSelThreads] = z;
    h[threadIdx.x] = z;
    h[threadIdx.x + kSelThreads] = z;
}

// One pass over the slice's keys in 16-byte vectors: copies them to `stage`
// when given and adds the nonzero ones of the first m to sh.local_hist.
template <typename K>
// m_load >= m keys are loaded (and staged), the first m are counted: the
// loads can be issued before m is known.
__device__ void stage_pass(SelShared& sh, const Keys<K>& src, int m, int m_load, K* stage) {
    constexpr int kPer = 16 / (int)sizeof(K);
    const int nv = (m_load + kPer - 1) / kPer;
    for (int i0 = threadIdx.x; i0 < nv; i0 += kSelThreads * kUnroll) {
        uint4 v[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int i = i0 + u * kSelThreads;
            v[u] = i < nv ? src.vec(i) : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int i = i0 + u * kSelThreads;
            if (i >= nv) break;
            if (stage != nullptr) reinterpret_cast<uint4*>(stage)[i] = v[u];
            const K* e = reinterpret_cast<const K*>(&v[u]);
#pragma unroll
            for (int j = 0; j < kPer; ++j) {
                const K key = (kPer * i + j < m) ? e[j] : K(0);
                if (key != K(0)) atomicAdd(&sh.local_hist[key_bin((unsigned long long)key)], 1u);
            }
        }
    }
}

// Local histogram of the `width`-bit digit at `shift` over the keys whose
// bits above shift+width equal `prefix`.
template <typename K, typename Get>
__device__ void digit_hist(uint32_t* hist, Get get, int m, int shift, int width, K prefix) {
    const uint32_t mask = (1u << width) - 1u;
    for (int i0 = threadIdx.x; i0 < m; i0 += kSelThreads * kUnroll) {
        K kv[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int i = i0 + u * kSelThreads;
            kv[u] = i < m ? get(i) : K(0);
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u)
            if (i0 + u * kSelThreads < m && (K)(kv[u] >> (shift + width)) == prefix)
                atomicAdd(&hist[(uint32_t)(kv[u] >> shift) & mask], 1u);
    }
}

// The krem-th largest of the n <= 32 keys of list[0, mm) whose bits above
// `shift` equal `prefix`, and how many keys equal to it that rank takes
// (quota): one warp gathers them by ballot and ranks them by shuffles, in
// place of further radix levels (each a 4096-bin histogram and four CTA
// barriers). Every thread of the CTA calls it; the result is in every thread.
template <typename K, typename Get>
__device__ void few_rank(SelShared& sh, Get get, int mm, int shift, K prefix, uint32_t n, uint32_t krem, K& T,
                         uint32_t& quota) {
    if (warp_id() == 0) {
        const int lane = lane_id();
        uint32_t got = 0;
        for (int i0 = 0; i0 < mm; i0 += kWarp) {  // warp-uniform trip count
            const int i = i0 + lane;
            const K key = i < mm ? get(i) : K(0);
            const bool match = i < mm && (K)(key >> shift) == prefix;
            const uint32_t bal = __ballot_sync(0xffffffffu, match);
            const uint32_t pos = got + (uint32_t)__popc(bal & ((1u << lane) - 1u));
            if (match && pos < (uint32_t)kWarp) sh.few[pos] = (unsigned long long)key;
            got += (uint32_t)__popc(bal);
        }
        __syncwarp();
        const uint32_t cnt = min(got, min(n, (uint32_t)kWarp));
        const K x = lane < (int)cnt ? (K)sh.few[lane] : K(0);
        uint32_t g = 0, e = 0;
        for (uint32_t j = 0; j < cnt; ++j) {
            const K y = (K)__shfl_sync(0xffffffffu, (unsigned long long)x, (int)j);
            g += y > x ? 1u : 0u;
            e += y == x ? 1u : 0u;
        }
        // the lanes holding the rank's key (equal keys write equal values)
        if (lane < (int)cnt && g < krem && krem <= g + e) {
            sh.few_T = (unsigned long long)x;
            sh.few_quota = krem - g;
        }
    }
    __syncthreads();
    T = (K)sh.few_T;
    quota = sh.few_quota;
}

// A threshold bin too full for the candidate list: the remaining digits are
// resolved by cluster histograms over the slices (one per 12-bit digit). Out
// of line: a rare path, kept away from the common one's instructions.
template <typename K>
__device__ __noinline__ void refine_over_slices(SelShared& sh, const Keys<K>& keys, int m, uint32_t C, int shift,
                                                K& prefix, uint32_t& krem) {
    while (shift > 0) {
        const int width = shift < kDigitBits ? shift : kDigitBits;
        shift -= width;
        zero_hists(sh);
        __syncthreads();
        digit_hist<K>(sh.local_hist, [&](int i) { return keys[i]; }, m, shift, width, prefix);
        __syncthreads();
        cluster_sync();  // every CTA's row histogram is clear and its slice counted
        push_hist(sh, C);
        cluster_sync();
        uint32_t d, ab, ib;
        find_bin(sh, krem, d, ab, ib);
        prefix = (K)((prefix << width) | (K)d);
        krem -= ab;
    }
}

// Exact k-th largest key of the row, 1 <= k < total, given the bin tb that
// holds it (`above` keys in higher bins, in_bin in tb). Keys > thresh plus
// the first `quota` keys == thresh in position order are the k largest.
// On the candidate-list path (`carried` set) it also gives this CTA's first
// output ranks: every candidate carries its CTA of origin and every CTA
// publishes its count above the bin with its candidates, so the kept counts
// of the lower-ranked slices follow without another exchange.
template <typename K>
__device__ void resolve_threshold(SelShared& sh, const Keys<K>& keys, int m, uint64_t* cand, K* mine, uint32_t C,
                                  uint32_t c, uint32_t k, uint32_t tb, uint32_t above, uint32_t in_bin, K& thresh,
                                  uint32_t& quota, bool& carried, uint32_t& carry_g, uint32_t& carry_e) {
    carried = false;
    if (tb < 64u) {  // small bins hold a single key value
        thresh = (K)tb;
        quota = k - above;
        return;
    }
    const int nb = (int)(tb >> 6) + 6;  // bit length of the bin's keys
    int shift = nb - 7;
    K prefix = (K)(64u | (tb & 63u));
    uint32_t krem = k - above;
    if (in_bin <= (uint32_t)kCandCap) {
        // gather this slice's keys of the bin, then append them to every
        // CTA's candidate list
        // (warp-uniform trip count: every lane of a warp takes part in warp_append)
        for (int i0 = threadIdx.x; i0 - lane_id() < m; i0 += kSelThreads * kUnroll) {
            K kv[kUnroll];
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) {
                const int i = i0 + u * kSelThreads;
                kv[u] = i < m ? keys[i] : K(0);
            }
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) {
                const bool take = i0 + u * kSelThreads < m && kv[u] != K(0) && (K)(kv[u] >> shift) == prefix;
                const uint32_t p = warp_append(&sh.local_count, take);  // one atomic per warp
                if (take && p < (uint32_t)kCandCap) mine[p] = kv[u];
            }
        }
        // this slice's keys above the bin
        uint32_t ab = 0;
#pragma unroll
        for (int j = 0; j < kBinsPerThread; ++j) {
            const uint32_t b = threadIdx.x + (uint32_t)(j * kSelThreads);
            if (b > tb) ab += sh.local_hist[b];
        }
        ab = warp_sum(ab);
        if (lane_id() == 0) sh.wsum[warp_id()] = ab;
        __syncthreads();
        const uint32_t mc = min(sh.local_count, (uint32_t)kCandCap);
        if (threadIdx.x < C) {
            uint32_t above_local = 0;
            for (int w = 0; w < kSelWarps; ++w) above_local += sh.wsum[w];
            sh.push_base[threadIdx.x] = atom_add_cluster(map_cta(smem_u32(&sh.count), threadIdx.x), mc);
            st_cluster(map_cta(smem_u32(&sh.cta_above[c]), threadIdx.x), above_local);
        }
        __syncthreads();
        const uint32_t cbase = smem_u32(cand);
        const uint64_t tag = (uint64_t)c << kOriginShift;
        for (uint32_t i = threadIdx.x; i < mc; i += kSelThreads) {
            const uint64_t e = (uint64_t)mine[i] | tag;
            for (uint32_t t = 0; t < C; ++t) {
                const uint32_t p = sh.push_base[t] + i;
                if (p < (uint32_t)kCandCap) st_cluster_key<uint64_t>(map_cta(cbase + 8u * p, t), e);
            }
        }
        cluster_sync();  // after this no CTA touches another CTA's shared memory
        const int mm = (int)min(sh.count, (uint32_t)kCandCap);
        uint32_t n_match = in_bin;  // candidates whose bits above shift equal prefix
        while (shift > 0) {  // identical in every CTA
            if (n_match <= (uint32_t)kWarp) {
                K T;
                uint32_t q;
                few_rank<K>(sh, [&](int i) { return (K)(cand[i] & kKeyMask); }, mm, shift, prefix, n_match, krem, T,
                            q);
                prefix = T;
                krem = q;
                break;
            }
            const int width = shift < kDigitBits ? shift : kDigitBits;
            shift -= width;
            reinterpret_cast<uint4*>(sh.hist)[threadIdx.x] = make_uint4(0u, 0u, 0u, 0u);
            reinterpret_cast<uint4*>(sh.hist)[threadIdx.x + kSelThreads] = make_uint4(0u, 0u, 0u, 0u);
            __syncthreads();
            digit_hist<K>(sh.hist, [&](int i) { return (K)(cand[i] & kKeyMask); }, mm, shift, width, prefix);
            __syncthreads();
            uint32_t d, ab, ib;
            find_bin(sh, krem, d, ab, ib);
            prefix = (K)((prefix << width) | (K)d);
            krem -= ab;
            n_match = ib;
        }
        // kept counts per originating slice: keys above the bin plus its
        // candidates > T, and its candidates == T
        if (threadIdx.x < kMaxCluster) {
            sh.og_gt[threadIdx.x] = 0;
            sh.og_eq[threadIdx.x] = 0;
        }
        __syncthreads();
        const K T = prefix;
        // per CTA of origin, with warp ballots (the list's entries share few counters)
        for (int i0 = threadIdx.x - lane_id(); i0 < mm; i0 += kSelThreads) {
            const int i = i0 + lane_id();
            const uint64_t e = i < mm ? cand[i] : 0ull;
            const K key = (K)(e & kKeyMask);
            const uint32_t o = (uint32_t)(e >> kOriginShift);
            for (uint32_t t = 0; t < C; ++t) {
                const uint32_t g = __ballot_sync(0xffffffffu, i < mm && o == t && key > T);
                const uint32_t q = __ballot_sync(0xffffffffu, i < mm && o == t && key == T);
                if (lane_id() == 0) {
                    if (g) atomicAdd(&sh.og_gt[t], (uint32_t)__popc(g));
                    if (q) atomicAdd(&sh.og_eq[t], (uint32_t)__popc(q));
                }
            }
        }
        __syncthreads();
        carry_g = 0;
        carry_e = 0;
        for (uint32_t o = 0; o < c; ++o) {
            carry_g += sh.cta_above[o] + sh.og_gt[o];
            carry_e += sh.og_eq[o];
        }
        carried = true;
    } else {
        refine_over_slices<K>(sh, keys, m, C, shift, prefix, krem);
    }
    thresh = prefix;
    quota = krem;
}

// Kept keys (key > thresh, plus the first `quota` keys == thresh of the row
// in position order) of this CTA's slice; emit(slot, rank) with slot relative
// to the slice and rank the key's position among the row's kept keys.
// This slice's counts of keys > thresh and == thresh without reading its keys:
// the slice histogram's bins above `bin` hold only keys > thresh; bin `bin`
// holds only keys == thresh (exact bins), or its keys are the slice's own
// candidates `mine` (from_mine). Returns the counts in every thread.
template <typename K>
__device__ void slice_counts(SelShared& sh, uint32_t bin, bool from_mine, const K* mine, K thresh, uint32_t& ng,
                             uint32_t& ne) {
    const int lane = lane_id(), wid = warp_id();
    uint32_t g = 0, e = 0;
#pragma unroll
    for (int j = 0; j < kBinsPerThread; ++j) {
        const uint32_t b = threadIdx.x + (uint32_t)(j * kSelThreads);
        const uint32_t v = sh.local_hist[b];
        if (b > bin) g += v;
        else if (b == bin && !from_mine) e += v;
    }
    if (from_mine) {
        const uint32_t mc = min(sh.local_count, (uint32_t)kCandCap);
        for (uint32_t i = threadIdx.x; i < mc; i += kSelThreads) {
            const K key = mine[i];
            g += key > thresh ? 1u : 0u;
            e += key == thresh ? 1u : 0u;
        }
    }
    g = warp_sum(g);
    e = warp_sum(e);
    if (lane == 0) {
        sh.wsum[wid] = g;
        sh.wsum2[wid] = e;
    }
    __syncthreads();
    ng = 0;
    ne = 0;
    for (int w = 0; w < kSelWarps; ++w) {
        ng += sh.wsum[w];
        ne += sh.wsum2[w];
    }
    __syncthreads();  // the warp sums are rewritten by the compaction
}

// With `counted`, (ng, ne) are this slice's counts of keys > thresh and ==
// thresh (slice_counts); otherwise a pass over the slice counts them.
// With `carried`, (carry_g, carry_e) already give this slice's first ranks
// (the candidate path) and no exchange is needed.
template <typename K, typename Emit>
__device__ void cluster_compact(SelShared& sh, const Keys<K>& keys, int m, uint32_t C, uint32_t c, K thresh,
                                uint32_t quota, bool counted, uint32_t ng_in, uint32_t ne_in, bool carried,
                                uint32_t carry_g_in, uint32_t carry_e_in, Emit emit) {
    const int tid = threadIdx.x, lane = lane_id(), wid = warp_id();
    uint32_t carry_g = carry_g_in, carry_e = carry_e_in;
    if (!carried) {
        // 1. this slice's counts, published to every CTA
        const int nw_all = counted ? 0 : (m + 31) / 32;
        uint32_t ng = 0, ne = 0;
        for (int w0 = wid; w0 < nw_all; w0 += kSelWarps * kUnroll) {
            K kv[kUnroll];
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) {
                const int i = 32 * (w0 + u * kSelWarps) + lane;
                kv[u] = i < m ? keys[i] : K(0);
            }
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) {
                const int i = 32 * (w0 + u * kSelWarps) + lane;
                ng += (uint32_t)__popc(__ballot_sync(0xffffffffu, i < m && kv[u] > thresh));
                ne += (uint32_t)__popc(__ballot_sync(0xffffffffu, i < m && kv[u] == thresh));
            }
        }
        if (!counted) {
            if (lane == 0) {
                sh.wsum[wid] = ng;
                sh.wsum2[wid] = ne;
            }
            __syncthreads();
        }
        if (tid < (int)C) {
            uint32_t tg = ng_in, te = ne_in;
            if (!counted) {
                tg = 0;
                te = 0;
                for (int w = 0; w < kSelWarps; ++w) {
                    tg += sh.wsum[w];
                    te += sh.wsum2[w];
                }
            }
            st_cluster(map_cta(smem_u32(&sh.cta_gt[c]), (uint32_t)tid), tg);
            st_cluster(map_cta(smem_u32(&sh.cta_eq[c]), (uint32_t)tid), te);
        }
        cluster_sync();  // after this no CTA touches another CTA's shared memory
        carry_g = 0;
        carry_e = 0;
        for (uint32_t t = 0; t < c; ++t) {
            carry_g += sh.cta_gt[t];
            carry_e += sh.cta_eq[t];
        }
    }
    // 2. ranks within the slice, one bitmap chunk at a time
    for (int c0 = 0; c0 < m; c0 += kChunkWords * 32) {
        const int nw = min(kChunkWords, (m - c0 + 31) / 32);
        for (int w0 = wid; w0 < nw; w0 += kSelWarps * kUnroll) {
            K kv[kUnroll];
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) {
                const int i = c0 + 32 * (w0 + u * kSelWarps) + lane;
                kv[u] = i < m ? keys[i] : K(0);
            }
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) {
                const int w = w0 + u * kSelWarps;
                const int i = c0 + 32 * w + lane;
                const uint32_t g = __ballot_sync(0xffffffffu, i < m && kv[u] > thresh);
                const uint32_t e = __ballot_sync(0xffffffffu, i < m && kv[u] == thresh);
                if (lane == 0 && w < nw) {
                    sh.gt_words[w] = g;
                    sh.eq_words[w] = e;
                }
            }
        }
        __syncthreads();
        const uint32_t g = tid < nw ? sh.gt_words[tid] : 0u;
        const uint32_t e = tid < nw ? sh.eq_words[tid] : 0u;
        const uint32_t cg = (uint32_t)__popc(g), ce = (uint32_t)__popc(e);
        uint32_t xg = cg, xe = ce;  // inclusive prefix over the warp
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t vg = __shfl_up_sync(0xffffffffu, xg, o);
            const uint32_t ve = __shfl_up_sync(0xffffffffu, xe, o);
            if (lane >= o) {
                xg += vg;
                xe += ve;
            }
        }
        if (lane == 31) {
            sh.wsum[wid] = xg;
            sh.wsum2[wid] = xe;
        }
        __syncthreads();
        const uint32_t tg = lane < kSelWarps ? sh.wsum[lane] : 0u;
        const uint32_t te = lane < kSelWarps ? sh.wsum2[lane] : 0u;
        uint32_t gb = carry_g + warp_sum(lane < wid ? tg : 0u) + xg - cg;
        uint32_t eb = carry_e + warp_sum(lane < wid ? te : 0u) + xe - ce;
        carry_g += warp_sum(tg);
        carry_e += warp_sum(te);
        uint32_t both = g | e;
        while (both) {
            const int b = __ffs(both) - 1;
            both &= both - 1;
            const uint32_t below = (1u << b) - 1u;
            const uint32_t pg = gb + (uint32_t)__popc(g & below), pe = eb + (uint32_t)__popc(e & below);
            const int slot = c0 + 32 * tid + b;
            if ((g >> b) & 1u) emit(slot, pg + min(pe, quota));
            else if (pe < quota) emit(slot, pg + pe);
        }
        __syncthreads();  // the words and warp sums are rewritten by the next chunk
    }
}

// Slice of CTA c of C over n keys, in whole 32-key words: [k_lo, k_lo + m).
__device__ __forceinline__ void slice_of(int n, uint32_t C, uint32_t c, int& k_lo, int& m) {
    const int W = (n + 31) / 32;
    const int w_lo = (int)((int64_t)W * c / C), w_hi = (int)((int64_t)W * (c + 1) / C);
    k_lo = 32 * w_lo;
    m = max(0, min(n, 32 * w_hi) - k_lo);
}

// HI with the coarse scores computed in place: the slice's blocks
// [blk0, blk0 + m) of the row are scored straight into `stage` (keys =
// score + 1) and counted into the slice histogram; one 16-block MMA tile per
// warp and pass (the fragment scheme of the coarse scoring kernel). Block-sum
// rows are read at clamped indices, so an invalid row (checked afterwards,
// before anything is written) reads in bounds.
template <int D_I, int NT>
__device__ void coarse_pass(SelShared& sh, const IndexArgs& a, int r, int64_t boff, int blk0, int m, uint64_t* stage) {
    const int lane = lane_id(), g = lane >> 2, t4 = lane & 3;
    QueryFrag<D_I, NT> qf;
    load_query<D_I, NT>(qf, a, r);
    for (int j = warp_id() * 16; j < m; j += kSelWarps * 16) {  // warp-uniform
        const int j0 = j + g, j1 = j0 + 8;
        const int64_t b0 = boff + blk0 + j0, b1 = boff + blk0 + j1;
        const bool v0 = j0 < m && b0 >= 0 && b0 < a.block_rows;
        const bool v1 = j1 < m && b1 >= 0 && b1 < a.block_rows;
        RowFrag<D_I> hg, lg, hg8, lg8;
        hg.load(a.block_sums + (v0 ? b0 : 0) * (2 * D_I), t4, v0);
        lg.load(a.block_sums + (v0 ? b0 : 0) * (2 * D_I) + D_I, t4, v0);
        hg8.load(a.block_sums + (v1 ? b1 : 0) * (2 * D_I), t4, v1);
        lg8.load(a.block_sums + (v1 ? b1 : 0) * (2 * D_I) + D_I, t4, v1);
        long long x, y;
        coarse_tile<D_I, NT>(qf, hg, lg, hg8, lg8, x, y);
        if (t4 == 0 && j0 < m) {
            const uint64_t key = (unsigned long long)x + 1ull;
            stage[j0] = key;
            atomicAdd(&sh.local_hist[key_bin(key)], 1u);
        }
        if (t4 == 1 && j1 < m) {
            const uint64_t key = (unsigned long long)y + 1ull;
            stage[j1] = key;
            atomicAdd(&sh.local_hist[key_bin(key)], 1u);
        }
    }
}

// The fused decode append's CTAs (grid rows n_q onwards of the block
// selection): one append task per CTA. Out of line, away from the
// selection's instructions.
template <int D_I>
__device__ __noinline__ void fused_append(const IndexArgs& a, int* s_part) {
    pdl_enter();  // the caches may still be read by the preceding kernels
    const int t = (int)((blockIdx.y - (unsigned)a.n_q) * gridDim.x + blockIdx.x);
    if (t >= a.app_tasks) return;
    const int per_role = a.app_per_seq * a.app.bs.n_seq;
    const int role = t / per_role, rem = t - role * per_role;
    const int seq = rem / a.app_per_seq, x = rem - seq * a.app_per_seq;
    if constexpr (D_I > 0) {  // the indexer key width is the kernel's (one copy of the append code)
        append_task<D_I, kSelThreads>(a.app, x, seq, role, s_part);
    } else {
        switch (a.app_dI) {
            case 32: append_task<32, kSelThreads>(a.app, x, seq, role, s_part); break;
            case 64: append_task<64, kSelThreads>(a.app, x, seq, role, s_part); break;
            default: append_task<128, kSelThreads>(a.app, x, seq, role, s_part); break;
        }
    }
}

// Selection of one row by one cluster. kTokens: fine top-k and the SI// Selection of one row by one cluster. kTokens: fine top-k and the SI
// assembly of the index set; otherwise the HI block top-k.
// D_I > 0 (HI blocks only): the coarse scores are computed in place
// (coarse_pass) instead of read from the coarse scoring kernel's workspace.
//
// Block selection only: rows n_q onwards of the grid are a decode step's
// append (append_task), one task per CTA, when the caller fuses it here. The
// block selection and the append then touch disjoint memory (the new tokens'
// blocks lie in the window, never among the candidate blocks), and every
// later kernel of the step waits for this grid, so the append costs no
// kernel boundary of its own.
template <typename K, bool kTokens, int D_I = 0, int NT = 0>
__global__ void __launch_bounds__(kSelThreads, 2) select_kernel(const __grid_constant__ IndexArgs a) {
    extern __shared__ __align__(16) uint8_t dyn[];
    if constexpr (!kTokens) {
        if (blockIdx.y >= (unsigned)a.n_q) {  // uniform over the cluster: no cluster barrier is used
            fused_append<D_I>(a, reinterpret_cast<int*>(dyn));
            return;
        }
    }
    SelShared& sh = *reinterpret_cast<SelShared*>(dyn);
    const int r = blockIdx.y;
    const uint32_t C = cluster_size(), c = cluster_rank();
    const int stage_cap = kTokens ? a.fine_stage : a.coarse_stage;
    const SelLayout lay = sel_layout((int)sizeof(K), stage_cap, kTokens ? a.kept_slots : 0);
    uint64_t* cand = reinterpret_cast<uint64_t*>(dyn + lay.off_cand);
    K* mine = reinterpret_cast<K*>(dyn + lay.off_mine);
    K* stage = stage_cap > 0 ? reinterpret_cast<K*>(dyn + lay.off_stage) : nullptr;
    int32_t* s_kept = reinterpret_cast<int32_t*>(dyn + lay.off_kept);
    int32_t* out = a.index_sets + (int64_t)r * a.budget;
    // Row geometry from q_len alone (clamped so every read below stays in
    // bounds), so that the slice's keys stream in while the row's sequence
    // metadata is checked; nothing is written before the check. The metadata
    // is the caller's, never written by a kernel of this library: it is read
    // before the wait for the preceding kernel.
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
    int k_lo, m, m_load;
    if (kTokens && B > 0) {
        // slices of the row's capacity: the keys load before the kept-block
        // count (written by the block selection) is known
        slice_of(a.fine_cap, C, c, k_lo, m_load);
        m = max(0, min(n - k_lo, m_load));
    } else {
        slice_of(n, C, c, k_lo, m);
        m_load = m;
    }
    const K* row_keys = kTokens ? reinterpret_cast<const K*>(a.fine_keys + (int64_t)r * a.fine_cap)
                                : reinterpret_cast<const K*>(a.coarse_keys + (int64_t)r * a.coarse_cap);
    Keys<K> keys{row_keys + k_lo, 0u};
    // kept blocks that this slice's slots fall in (used by the compaction).
    // With at most one per thread, every id the slice's capacity may hold is
    // loaded into a register here, beside the kept count and the keys, and
    // stored after the staging pass: the three loads share one round trip.
    int kb_lo = 0;
    int32_t kid = 0;
    bool has_kid = false;
    if (kTokens && B > 0) {
        kb_lo = k_lo / B;
        const int32_t* kept = a.kept + (int64_t)r * a.hi_topblocks;
        if (a.kept_slots <= kSelThreads) {
            const int i = threadIdx.x;
            if (m_load > 0 && i <= (k_lo + m_load - 1) / B - kb_lo && i < a.kept_slots && kb_lo + i < a.hi_topblocks) {
                kid = kept[kb_lo + i];
                has_kid = true;
            }
        } else if (m > 0) {
            const int kb_hi = (k_lo + m - 1) / B;
            for (int i = threadIdx.x; i <= kb_hi - kb_lo && i < a.kept_slots; i += kSelThreads)
                s_kept[i] = kept[kb_lo + i];
        }
    }
    zero_hists(sh);
    if (threadIdx.x == 0) {
        sh.count = 0;
        sh.local_count = 0;
    }
    __syncthreads();
    // every CTA's row histogram and counters are clear once all CTAs have
    // arrived here; the wait comes after this CTA's own staging pass
    cluster_arrive();
    if constexpr (!kTokens && D_I > 0) {
        coarse_pass<D_I, NT>(sh, a, r, boff_q, first + k_lo, m, reinterpret_cast<uint64_t*>(stage));
    } else {
        stage_pass<K>(sh, keys, m, m_load, stage);
    }
    if (has_kid) s_kept[threadIdx.x] = kid;
    __syncthreads();
    if (stage != nullptr) keys.s = smem_u32(stage);
    // the row check (as in the scoring kernels): uniform over the cluster, and
    // before the first cluster barrier
    int32_t bits = 0;
    if (seq_q < 0 || seq_q >= a.n_seq) bits = LSA_DEV_BAD_SEQ;
    else if (Lq < 1 || Lq > a.max_len || Lq > slen_q || off_q < 0 || off_q + slen_q > a.total_tokens ||
             (a.hi_block > 0 && (boff_q < 0 || boff_q + (Lq + a.hi_block - 1) / a.hi_block > a.block_rows)))
        bits = LSA_DEV_BAD_LENGTH;
    if constexpr (!kTokens && D_I > 0) {
        // a valid row that sees fewer tokens than its sequence holds: the
        // candidate block holding its last visible token is scored over the
        // tokens the row sees, not from the stored sum (uniform over the CTA)
        int b_p;
        if (bits == 0 && partial_block_fix(L, slen_q, B, ws, b_p) && b_p - first - k_lo >= 0 &&
            b_p - first - k_lo < m) {
            const int j = b_p - first - k_lo;
            const long long sc = partial_block_score<D_I, kSelThreads>(
                a, r, a.k_idx + off_q * D_I, b_p * B, L - b_p * B, reinterpret_cast<int32_t*>(sh.gt_words),
                reinterpret_cast<long long*>(sh.eq_words));
            if (threadIdx.x == 0) {
                uint64_t* st = reinterpret_cast<uint64_t*>(stage);
                const uint64_t old = st[j], key = (unsigned long long)sc + 1ull;
                st[j] = key;
                atomicSub(&sh.local_hist[key_bin(old)], 1u);
                atomicAdd(&sh.local_hist[key_bin(key)], 1u);
            }
            __syncthreads();
        }
    }
    cluster_wait();  // complete the barrier every CTA arrived at (an exiting CTA must too)
    if (bits != 0) {
        if (kTokens) {
            if (c == 0 && threadIdx.x == 0) flag(a.dev_status, bits);
            for (int e = (int)(c * kSelThreads) + threadIdx.x; e < a.budget; e += (int)(C * kSelThreads)) out[e] = -1;
        } else if (c == 0 && threadIdx.x == 0) {
            a.n_kept[r] = 0;  // the token selection reports the row
        }
        return;
    }
    push_hist(sh, C);
    cluster_sync();
    const uint32_t want = (uint32_t)(kTokens ? a.topk : a.hi_topblocks);
    uint32_t tb, above, in_bin;
    const uint32_t total = find_bin(sh, want, tb, above, in_bin);
    pdl_trigger();  // what is left is the threshold and the compaction
    const uint32_t k = min(want, total);
    if (k > 0u) {
        K thr = K(1);
        uint32_t quota = 0xffffffffu;  // k == total: every candidate is kept
        bool carried = false;
        uint32_t carry_g = 0, carry_e = 0;
        if (k < total)
            resolve_threshold<K>(sh, keys, m, cand, mine, C, c, k, tb, above, in_bin, thr, quota, carried, carry_g,
                                 carry_e);
        // otherwise this slice's kept counts come from its histogram (exact
        // bins) or a pass over its keys (bin refined over the slices)
        const bool counted = !carried && (k == total || tb < 64u);
        uint32_t ng = 0, ne = 0;
        if (counted) slice_counts<K>(sh, k == total ? 1u : tb, false, mine, thr, ng, ne);
        if (kTokens) {
            const int lgB = (B > 0 && (B & (B - 1)) == 0) ? __ffs(B) - 1 : -1;  // power-of-two block: shift
            cluster_compact<K>(sh, keys, m, C, c, thr, quota, counted, ng, ne, carried, carry_g, carry_e,
                               [&](int slot, uint32_t rank) {
                const int gs = k_lo + slot;
                int tok;
                if (B > 0) {
                    const int kb = lgB >= 0 ? gs >> lgB : gs / B;
                    tok = s_kept[kb - kb_lo] * B + (gs - kb * B);
                } else {
                    tok = first + gs;
                }
                if (rank < k) out[s + rank] = tok;
            });
        } else {
            int32_t* kept = a.kept + (int64_t)r * a.hi_topblocks;
            cluster_compact<K>(sh, keys, m, C, c, thr, quota, counted, ng, ne, carried, carry_g, carry_e,
                               [&](int slot, uint32_t rank) {
                if (rank < k) kept[rank] = first + k_lo + slot;
            });
        }
    }
    if (kTokens) {
        const int win0 = s + (int)k;
        const int n_win = L - ws;
        for (int e = (int)(c * kSelThreads) + threadIdx.x; e < a.budget; e += (int)(C * kSelThreads)) {
            if (e < s) out[e] = e;
            else if (e >= win0 && e < win0 + n_win) out[e] = ws + (e - win0);
            else if (e >= win0 + n_win) out[e] = -1;
        }
    } else if (c == 0 && threadIdx.x == 0) {
        a.n_kept[r] = (int32_t)k;
    }
}

}  // namespace

static size_t align256(size_t x) { return (x + 255) / 256 * 256; }

// Staged slice keys plus kept-block ids stay within this much shared memory.
constexpr size_t kStageSmem = 144 * 1024;

IndexPlan plan_index(int n_q, int max_len, const lsa_budget_t& b, bool dense) {
    IndexPlan p;
    const bool hi = b.hi_block > 0;
    if (hi) {
        p.coarse_cap = (max_len + b.hi_block - 1) / b.hi_block + 1;
        p.coarse_cap = (p.coarse_cap + 1) / 2 * 2;
        p.fine_cap = b.hi_topblocks * b.hi_block;
    } else if (dense) {
        // the tensor-core scoring's slots span the union of its rows' middles
        // in whole tiles
        p.fine_cap = (max_len + LSA_TC_TOKENS - 1) / LSA_TC_TOKENS * LSA_TC_TOKENS;
    } else {
        p.fine_cap = max_len;
    }
    p.fine_cap = (p.fine_cap + 3) / 4 * 4;
    if (p.fine_cap < 4) p.fine_cap = 4;
    // a few rows (the 1M decode has one): 16 CTAs per row (non-portable
    // cluster size) halve each CTA's slice; otherwise 8
    p.cluster = n_q <= 4 ? 16 : 8;
    // largest slice: whole 32-key words split over the cluster
    auto slice_max = [&](int cap) { return 32 * (((cap + 31) / 32 + p.cluster - 1) / p.cluster); };
    if (hi) {
        const int sm = slice_max(p.coarse_cap);
        p.coarse_stage = (size_t)sm * 8 <= kStageSmem ? sm : 0;
        p.smem_blocks = sel_layout(8, p.coarse_stage, 0).bytes;
    }
    {
        const int sm = slice_max(p.fine_cap);
        p.kept_slots = hi ? std::min(b.hi_topblocks, sm / b.hi_block + 2) : 0;
        p.fine_stage = (size_t)sm * 4 + (size_t)p.kept_slots * 4 <= kStageSmem ? sm : 0;
        p.smem_tokens = sel_layout(4, p.fine_stage, p.kept_slots).bytes;
    }
    size_t off = 0;
    p.off_coarse = off;
    off = align256(off + (size_t)n_q * p.coarse_cap * 8);
    p.off_kept = off;
    off = align256(off + (size_t)n_q * (hi ? b.hi_topblocks : 0) * 4);
    p.off_nkept = off;
    off = align256(off + (size_t)n_q * 4);
    p.off_fine = off;
    if (dense) {
        // candidate pairs (8 bytes) in place of the one-key-per-token array
        p.off_cand = off;
        off = align256(off + (size_t)n_q * p.fine_cap * 8);
        p.off_count = off;
        off = align256(off + (size_t)n_q * LSA_TC_MAX_SPLITS * LSA_TC_SEGS * 8);
        p.off_ghist = off;
        off = align256(off + (size_t)n_q * LSA_TC_BINS * 4);
    } else {
        off = align256(off + (size_t)n_q * p.fine_cap * 4);
    }
    p.ws_bytes = off;
    return p;
}

// extra_rows: grid rows past n_q (the fused append's CTAs, block selection only)
template <typename Kern>
static cudaError_t launch_cluster(Kern kern, const IndexArgs& a, int cluster, size_t smem, cudaStream_t stream,
                                  int extra_rows = 0) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    if (cluster > 8) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
        if (e != cudaSuccess) return e;
    }
    return launch_pdl(kern, dim3((unsigned)cluster, (unsigned)(a.n_q + extra_rows), 1), dim3(kSelThreads), smem,
                      stream, cluster, a);
}

template <int D_I>
static cudaError_t launch_blocks_fused(const IndexArgs& a, int cluster, size_t smem, cudaStream_t stream, int extra) {
    if (a.H_I <= 8) return launch_cluster(select_kernel<uint64_t, false, D_I, 1>, a, cluster, smem, stream, extra);
    return launch_cluster(select_kernel<uint64_t, false, D_I, 2>, a, cluster, smem, stream, extra);  // H_I <= 16
}

int index_select_append_rows(const IndexArgs& a, int cluster) {
    return a.app_tasks > 0 ? (a.app_tasks + cluster - 1) / cluster : 0;
}

cudaError_t launch_index_select(const IndexArgs& a, bool blocks, int d_I, int cluster, size_t smem,
                                cudaStream_t stream) {
    if (cluster < 1 || cluster > kMaxCluster) return cudaErrorInvalidValue;
    if (!blocks) {
        if (a.app_tasks > 0) return cudaErrorInvalidValue;  // the append rides on the block selection only
        return launch_cluster(select_kernel<uint32_t, true>, a, cluster, smem, stream);
    }
    if (a.app_tasks > 0 && (a.app_dI != 32 && a.app_dI != 64 && a.app_dI != 128)) return cudaErrorInvalidValue;
    const int extra = index_select_append_rows(a, cluster);
    if (!coarse_in_select(a))
        return launch_cluster(select_kernel<uint64_t, false>, a, cluster, smem, stream, extra);
    switch (d_I) {
        case 32: return launch_blocks_fused<32>(a, cluster, smem, stream, extra);
        case 64: return launch_blocks_fused<64>(a, cluster, smem, stream, extra);
        case 128: return launch_blocks_fused<128>(a, cluster, smem, stream, extra);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace lsa
