// index_pairs.cu — exact top-k of a prefill chunk's rows from the candidate
// (key, position) pairs the tensor-core scoring kept, and the SI assembly of
// their index sets.
//
// The method: the topk best middle tokens of each row, ties to the lower
// position; the index set is the sink run, the selected tokens and the window
// run in ascending order, padded with -1 ("LongCat-Flash-Lite-Sparse
// (aitrends.kr)", section "기술적 특징", SI bullet; "LongCat-2.0
// (molayo1419.me)", section "1M 토큰에서의 Sparse Attention 문제").
#include "common.cuh"
#include "index_common.cuh"
#include "internal.h"

namespace lsa {
namespace {

// 512 threads and at most 64 registers: two rows' CTAs per SM, so one row's
// barriers and L2 round trips overlap the other's
constexpr int kTkThreads = 512;
constexpr int kTkWarps = kTkThreads / kWarp;
constexpr int kTkBinsPer = kHistBins / kTkThreads;  // histogram bins per thread in a scan
static_assert(kTkBinsPer % 4 == 0, "the scan reads each thread's bins as 4-bin vectors");
constexpr int kTkCandCap = 2048;  // keys of the threshold bin held in the candidate list
constexpr int kTkDigitBits = 12;
constexpr int kPassUnroll = 8;  // pair loads in flight per thread in a pass
constexpr int kMergeIdBits = LSA_MERGE_ID_BITS;  // id field of a merge value
constexpr uint32_t kMergeIdMask = (1u << kMergeIdBits) - 1u;

__device__ __forceinline__ uint32_t tk_warp_sum(uint32_t v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Prefill rows: the tensor-core scoring kept, per row, the (key, position)
// pairs that passed its running threshold, in no particular order. The row's
// exact top-k by (key desc, position asc) is the top-k of the distinct
// values key << 32 | (2^32 - 1 - position), found over the pairs in global
// memory (histogram pass, then radix digits over the threshold bin's
// candidates or, for a bin too full for the list, over all pairs); the kept
// positions are sorted ascending in shared memory (bitonic) and written with
// the SI sink and window runs. One CTA of 512 threads per row.
constexpr int kPairSortCap = LSA_MAX_BUDGET;  // topk <= budget

struct PairShared {
    uint32_t hist[kHistBins];
    uint64_t cand[kTkCandCap];
    uint32_t wsum[kTkWarps];
    uint32_t bin, above, in_bin;
    uint32_t n_cand, n_sel;
};

__device__ __forceinline__ uint64_t pair_value(uint64_t e) {
    return (e & 0xffffffff00000000ull) | (uint64_t)(0xffffffffu - (uint32_t)e);
}

// Suffix scan of sh.hist (kTkBinsPer bins per thread). Returns the number of
// counted keys; when 1 <= krem <= total sets sh.bin / sh.above / sh.in_bin to
// the bin holding the krem-th largest value, the count above it and the count
// in it.
__device__ uint32_t pair_find_bin(PairShared& sh, uint32_t krem) {
    const int tid = threadIdx.x, lane = lane_id(), wid = warp_id();
    uint32_t c[kTkBinsPer];
#pragma unroll
    for (int q = 0; q < kTkBinsPer / 4; ++q) {
        const uint4 h = reinterpret_cast<const uint4*>(sh.hist)[tid * (kTkBinsPer / 4) + q];
        c[4 * q] = h.x;
        c[4 * q + 1] = h.y;
        c[4 * q + 2] = h.z;
        c[4 * q + 3] = h.w;
    }
    uint32_t own = 0;
#pragma unroll
    for (int j = 0; j < kTkBinsPer; ++j) own += c[j];
    uint32_t x = own;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t v = __shfl_down_sync(0xffffffffu, x, o);
        if (lane + o < 32) x += v;
    }
    if (lane == 0) sh.wsum[wid] = x;
    __syncthreads();
    const uint32_t wt = lane < kTkWarps ? sh.wsum[lane] : 0u;
    const uint32_t later = tk_warp_sum(lane > wid ? wt : 0u);
    const uint32_t total = tk_warp_sum(wt);
    const uint32_t S = x + later;
    if (krem >= 1u && S >= krem && S - own < krem) {
        uint32_t run = S - own;
#pragma unroll
        for (int j = kTkBinsPer - 1; j >= 0; --j) {
            if (run + c[j] >= krem) {
                sh.bin = (uint32_t)(kTkBinsPer * tid + j);
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

// The k largest of the distinct values value(e) over the pairs that
// for_each_pair presents (n of them), their ids id(e) left sorted ascending in
// sel[0, m); returns m (= k when n >= k, else n). A histogram pass on the
// logarithmic scale of key_bin, then radix digits over the threshold bin's
// candidates (or, for a bin too full for the list, over all pairs), then a
// pass collecting the kept ids and a bitonic sort in shared memory. Every
// thread of the CTA calls it.
template <typename ForEach, typename Value, typename Id>
__device__ uint32_t select_sorted(PairShared& sh, int32_t* sel, uint32_t n, uint32_t k, ForEach for_each_pair,
                                  Value value, Id id) {
    const int tid = threadIdx.x;
    if (k == 0u) return 0u;
    // the k largest values: value >= T
    uint64_t T = 0ull;
    if (n > k) {
        for (int i = tid; i < kHistBins; i += kTkThreads) sh.hist[i] = 0u;
        if (tid == 0) sh.n_cand = 0u;
        __syncthreads();
        for_each_pair([&](uint64_t e, bool ok) {
            if (ok) atomicAdd(&sh.hist[key_bin(value(e))], 1u);
        });
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
                const uint64_t v = value(e);
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
#pragma unroll
            for (int q = 0; q < kTkBinsPer / 4; ++q)
                reinterpret_cast<uint4*>(sh.hist)[tid * (kTkBinsPer / 4) + q] = make_uint4(0u, 0u, 0u, 0u);
            __syncthreads();
            if (listed) {
                for (uint32_t i = tid; i < nc; i += kTkThreads) {
                    const uint64_t v = sh.cand[i];
                    if ((v >> (shift + width)) == prefix) atomicAdd(&sh.hist[(uint32_t)((v >> shift) & mask)], 1u);
                }
            } else {
                for_each_pair([&](uint64_t e, bool ok) {
                    const uint64_t v = value(e);
                    if (ok && (v >> (shift + width)) == prefix) atomicAdd(&sh.hist[(uint32_t)((v >> shift) & mask)], 1u);
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
        const bool take = ok && value(e) >= T;
        const uint32_t p = warp_append(&sh.n_sel, take);
        if (take && p < (uint32_t)kPairSortCap) sel[p] = id(e);
    });
    __syncthreads();
    const uint32_t m = min(sh.n_sel, k);
    uint32_t P = 1;
    while (P < m) P <<= 1;
    for (uint32_t i = m + tid; i < P; i += kTkThreads) sel[i] = 0x7fffffff;
    __syncthreads();
    // (a stride of at most 32 keeps each warp inside its own 64-element blocks
    // 64 (w + m kTkWarps): a warp barrier suffices between two such steps)
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
            // the next step stays inside the warp's 64 elements too: a stride
            // halved, or (after stride 1) the next size's first stride <= 32
            const bool next_local = stride > 1u || (size < P && size <= 32u);
            if (stride <= 32u && next_local) __syncwarp();
            else __syncthreads();
        }
    }
    return m;
}

__global__ void __launch_bounds__(kTkThreads, 2) topk_pairs_kernel(const __grid_constant__ IndexArgs a) {
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
    // the row's candidates: one segment per token split and lane quarter of the scoring
    const uint64_t* pairs = a.cand + (int64_t)r * a.fine_cap;
    constexpr int kMaxSegs = LSA_TC_MAX_SPLITS * LSA_TC_SEGS;
    __shared__ int32_t seg_lo[kMaxSegs], seg_n[kMaxSegs];
    const int n_segs = a.tc_splits * LSA_TC_SEGS;
    if (tid < n_segs) {
        const int2 sg = reinterpret_cast<const int2*>(a.cand_seg)[(int64_t)r * kMaxSegs + tid];
        const int lo = min(max(sg.x, 0), a.fine_cap);
        seg_lo[tid] = lo;
        seg_n[tid] = min(max(sg.y, 0), a.fine_cap - lo);
    }
    __syncthreads();
    uint32_t n = 0;
    for (int sp = 0; sp < n_segs; ++sp) n += (uint32_t)seg_n[sp];
    // every candidate pair once: f(pair)
    // (every lane of a warp calls f the same number of times: f(pair, ok))
    // (8 loads in flight per thread per round: a pass is a few L2 round trips)
    auto for_each_pair = [&](auto&& f) {
        for (int sp = 0; sp < n_segs; ++sp) {
            const uint64_t* seg = pairs + seg_lo[sp];
            const int cnt = seg_n[sp];
            for (int i0 = tid - (tid & 31); i0 < cnt; i0 += kTkThreads * kPassUnroll) {
                uint64_t e[kPassUnroll];
#pragma unroll
                for (int u = 0; u < kPassUnroll; ++u) {
                    const int i = i0 + u * kTkThreads + (tid & 31);
                    e[u] = i < cnt ? __ldcg(seg + i) : 0ull;
                }
#pragma unroll
                for (int u = 0; u < kPassUnroll; ++u) f(e[u], i0 + u * kTkThreads + (tid & 31) < cnt);
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
    const uint32_t m = select_sorted(sh, sel, n, k, for_each_pair, [](uint64_t e) { return pair_value(e); },
                                     [](uint64_t e) { return (int32_t)(uint32_t)e; });
    pdl_trigger();
    for (uint32_t i = tid; i < m; i += kTkThreads) out[s + i] = sel[i];
}


// Context-parallel merge: row r's pairs [r][0, counts[r]) hold values
// score << kMergeIdBits | (2^kMergeIdBits - 1 - id), distinct per row, or 0
// for an empty slot; the ids of the k largest values (score desc, id asc) are
// written ascending to out[r][0, m), -1 after, and (out_values) their values
// in the same order, 0 after.
__global__ void __launch_bounds__(kTkThreads, 2) merge_pairs_kernel(const uint64_t* __restrict__ pairs,
                                                                    const int32_t* __restrict__ counts, int32_t cap,
                                                                    int32_t k, int32_t* __restrict__ out,
                                                                    uint64_t* __restrict__ out_values,
                                                                    int32_t* dev_status) {
    extern __shared__ __align__(16) uint8_t pr_dyn[];
    PairShared& sh = *reinterpret_cast<PairShared*>(pr_dyn);
    int32_t* sel = reinterpret_cast<int32_t*>(pr_dyn + (sizeof(PairShared) + 15) / 16 * 16);
    const int r = blockIdx.x, tid = threadIdx.x;
    pdl_enter();
    const int cnt_raw = counts[r];
    if (cnt_raw < 0 || cnt_raw > cap) {
        if (tid == 0) flag(dev_status, LSA_DEV_BAD_LENGTH);
    }
    const int cnt = min(max(cnt_raw, 0), cap);
    const uint64_t* row = pairs + (int64_t)r * cap;
    auto for_each_pair = [&](auto&& f) {
        for (int i0 = tid - (tid & 31); i0 < cnt; i0 += kTkThreads * kPassUnroll) {
            uint64_t e[kPassUnroll];
#pragma unroll
            for (int u = 0; u < kPassUnroll; ++u) {
                const int i = i0 + u * kTkThreads + (tid & 31);
                e[u] = i < cnt ? __ldcg(row + i) : 0ull;
            }
#pragma unroll
            for (int u = 0; u < kPassUnroll; ++u) f(e[u], e[u] != 0ull);
        }
    };
    // the row's entries (nonzero values)
    if (tid == 0) sh.n_cand = 0u;
    __syncthreads();
    for_each_pair([&](uint64_t e, bool ok) {
        const uint32_t c = (uint32_t)__popc(__ballot_sync(0xffffffffu, ok));
        if ((tid & 31) == 0 && c) atomicAdd(&sh.n_cand, c);
    });
    __syncthreads();
    const uint32_t n = sh.n_cand;
    __syncthreads();
    const uint32_t m = select_sorted(sh, sel, n, (uint32_t)k, for_each_pair, [](uint64_t e) { return e; },
                                     [](uint64_t e) {
                                         return (int32_t)((kMergeIdMask - (uint32_t)(e & kMergeIdMask)));
                                     });
    pdl_trigger();
    int32_t* o = out + (int64_t)r * k;
    for (int i = tid; i < k; i += kTkThreads) o[i] = i < (int)m ? sel[i] : -1;
    if (out_values != nullptr) {
        // each kept id's value, found again among the row's entries
        uint64_t* ov = out_values + (int64_t)r * k;
        for (int i = tid; i < k; i += kTkThreads)
            if (i >= (int)m) ov[i] = 0ull;
        for_each_pair([&](uint64_t e, bool ok) {
            if (!ok) return;
            const int32_t id = (int32_t)(kMergeIdMask - (uint32_t)(e & kMergeIdMask));
            // binary search of id in the sorted ids
            int lo = 0, hi = (int)m - 1;
            while (lo <= hi) {
                const int mid = (lo + hi) >> 1;
                const int32_t x = sel[mid];
                if (x == id) {
                    ov[mid] = e;
                    break;
                }
                if (x < id) lo = mid + 1;
                else hi = mid - 1;
            }
        });
    }
}

}  // namespace

size_t topk_pairs_smem() { return (sizeof(PairShared) + 15) / 16 * 16 + (size_t)kPairSortCap * 4; }

cudaError_t launch_merge_pairs(const uint64_t* pairs, const int32_t* counts, int n_rows, int cap, int k, int32_t* out,
                               uint64_t* out_values, int32_t* dev_status, cudaStream_t stream) {
    const size_t smem = topk_pairs_smem();
    cudaError_t e = cudaFuncSetAttribute(merge_pairs_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    return launch_pdl(merge_pairs_kernel, dim3((unsigned)n_rows), dim3(kTkThreads), smem, stream, 0, pairs, counts,
                      cap, k, out, out_values, dev_status);
}

cudaError_t launch_topk_pairs(const IndexArgs& a, cudaStream_t stream) {
    const size_t smem = topk_pairs_smem();
    cudaError_t e = cudaFuncSetAttribute(topk_pairs_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    return launch_pdl(topk_pairs_kernel, dim3((unsigned)a.n_q), dim3(kTkThreads), smem, stream, 0, a);
}

}  // namespace lsa
