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
// Design (B200): one 1024-thread CTA per query row, so every synchronisation
// is a CTA barrier. Selection starts from a histogram of the row's keys
// (score + 1, 0 = not a candidate) on the logarithmic scale of key_bin: the
// fine scoring kernel accumulates it in global memory while it writes the
// keys; for HI blocks it is built here while the keys are staged. One suffix
// scan of the histogram gives the bin holding the k-th largest key, one pass
// over the keys (staging them in shared memory when they fit) gathers that
// bin's keys into a short list, and 12-bit radix levels over the list give
// the exact k-th largest key T and how many keys equal to T are kept (a bin
// too full for the list is refined over all keys instead). Compaction is
// bitmap based: warp ballots build "key > T" and "key == T" words, each
// thread counts its word, one CTA prefix ranks them, and every thread emits
// its kept positions in order.
#include "common.cuh"
#include "internal.h"

namespace lsa {
namespace {

constexpr int kSelThreads = 1024;
constexpr int kSelWarps = kSelThreads / kWarp;
static_assert(kHistBins == 4 * kSelThreads, "the scan gives each thread four bins");
constexpr int kDigitBits = 12;            // refinement digit: 4096 bins
constexpr int kCandCap = 2048;            // keys of the threshold bin held in a list
constexpr int kChunkWords = kSelThreads;  // compaction: one bitmap word per thread per chunk
constexpr int kUnroll = 4;                // independent loads in flight per thread

struct SelShared {
    uint32_t hist[kHistBins];
    uint32_t wsum[kSelWarps];
    uint32_t wsum2[kSelWarps];
    uint32_t gt_words[kChunkWords];
    uint32_t eq_words[kChunkWords];
    uint32_t bin, above, in_bin, count;
};

__device__ __forceinline__ uint32_t warp_sum(uint32_t v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Keys of one row, either staged in shared memory or read from global memory.
template <typename K>
struct Keys {
    const K* g;     // global copy
    uint32_t s;     // shared-memory address of the staged copy (0 when not staged)
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

// Suffix scan of sh.hist. Returns the number of counted keys; when
// 1 <= krem <= total also gives the bin d holding the krem-th largest key,
// the count above it (bins > d) and the count in it.
__device__ uint32_t find_bin(SelShared& sh, uint32_t krem, uint32_t& bin, uint32_t& above, uint32_t& in_bin) {
    const int tid = threadIdx.x, lane = lane_id(), wid = warp_id();
    const uint4 h = reinterpret_cast<const uint4*>(sh.hist)[tid];  // bins 4*tid .. 4*tid+3
    const uint32_t own = h.x + h.y + h.z + h.w;
    uint32_t x = own;  // bins >= 4*tid within this warp
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t v = __shfl_down_sync(0xffffffffu, x, o);
        if (lane + o < 32) x += v;
    }
    if (lane == 0) sh.wsum[wid] = x;
    __syncthreads();
    const uint32_t wt = sh.wsum[lane];
    const uint32_t later = warp_sum(lane > wid ? wt : 0u);
    const uint32_t total = warp_sum(wt);
    const uint32_t S = x + later;  // keys in bins >= 4*tid
    if (krem >= 1u && S >= krem && S - own < krem) {
        uint32_t run = S - own, b = 4 * tid + 3, c = h.w;
        if (run + c < krem) {
            run += c;
            b = 4 * tid + 2;
            c = h.z;
            if (run + c < krem) {
                run += c;
                b = 4 * tid + 1;
                c = h.y;
                if (run + c < krem) {
                    run += c;
                    b = 4 * tid;
                    c = h.x;
                }
            }
        }
        sh.bin = b;
        sh.above = run;
        sh.in_bin = c;
    }
    __syncthreads();
    bin = sh.bin;
    above = sh.above;
    in_bin = sh.in_bin;
    return total;
}

// One radix level over m keys: histogram of the `width`-bit digit at `shift`
// of the keys whose bits above shift+width equal `prefix`, then the digit
// holding the krem-th largest of them; prefix grows by that digit and krem
// drops by the count above it.
template <typename K, typename Get>
__device__ void radix_level(SelShared& sh, Get get, int m, int shift, int width, K& prefix, uint32_t& krem) {
    const int tid = threadIdx.x;
    reinterpret_cast<uint4*>(sh.hist)[tid] = make_uint4(0u, 0u, 0u, 0u);
    __syncthreads();
    const uint32_t mask = (1u << width) - 1u;
    for (int i0 = tid; i0 < m; i0 += kSelThreads * kUnroll) {
        K kv[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int i = i0 + u * kSelThreads;
            kv[u] = i < m ? get(i) : K(0);
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u)
            if (i0 + u * kSelThreads < m && (K)(kv[u] >> (shift + width)) == prefix)
                atomicAdd(&sh.hist[(uint32_t)(kv[u] >> shift) & mask], 1u);
    }
    __syncthreads();
    uint32_t d, above, in_bin;
    find_bin(sh, krem, d, above, in_bin);
    prefix = (K)((prefix << width) | (K)d);
    krem -= above;
}

// One pass over the row's n keys in 16-byte vectors: copies them to `stage`
// (shared memory) when given, adds the nonzero ones to sh.hist when
// `add_hist`, and when `gather` appends the keys k with (k >> shift) == prefix
// to cand (at most kCandCap; sh.count ends as the number found).
template <typename K>
__device__ void key_pass(SelShared& sh, const Keys<K>& src, int n, K* stage, bool add_hist, bool gather, int shift,
                         K prefix, K* cand) {
    constexpr int kPer = 16 / (int)sizeof(K);
    const int nv = (n + kPer - 1) / kPer;
    const int lane = lane_id();
    for (int b0 = warp_id() * kWarp; b0 < nv; b0 += kSelThreads * kUnroll) {  // warp-uniform
        uint4 v[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int i = b0 + u * kSelThreads + lane;
            v[u] = i < nv ? src.vec(i) : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int i = b0 + u * kSelThreads + lane;
            if (stage != nullptr && i < nv) reinterpret_cast<uint4*>(stage)[i] = v[u];
            const K* e = reinterpret_cast<const K*>(&v[u]);
#pragma unroll
            for (int j = 0; j < kPer; ++j) {
                const K key = (kPer * i + j < n) ? e[j] : K(0);
                if (add_hist && key != K(0)) atomicAdd(&sh.hist[key_bin((unsigned long long)key)], 1u);
                if (gather) {
                    const bool hit = key != K(0) && (K)(key >> shift) == prefix;
                    const uint32_t bal = __ballot_sync(0xffffffffu, hit);
                    if (bal != 0u) {
                        const int leader = __ffs(bal) - 1;
                        uint32_t base = 0;
                        if (lane == leader) base = atomicAdd(&sh.count, (uint32_t)__popc(bal));
                        base = __shfl_sync(0xffffffffu, base, leader);
                        const uint32_t p = base + (uint32_t)__popc(bal & lanemask_lt());
                        if (hit && p < (uint32_t)kCandCap) cand[p] = key;
                    }
                }
            }
        }
    }
}

// Exact k-th largest key, 1 <= k < total, from the row's log-bin histogram
// (in sh.hist; bin tb holds the k-th largest key, `above` keys lie in higher
// bins, in_bin in tb). Keys > thresh plus the first `quota` keys == thresh in
// position order are the k largest. `stage`, when given, receives the keys
// and `keys` is switched to it.
template <typename K>
__device__ void resolve_threshold(SelShared& sh, Keys<K>& keys, int n, K* stage, bool keys_staged, uint32_t k,
                                  uint32_t tb, uint32_t above, uint32_t in_bin, K* cand, K& thresh,
                                  uint32_t& quota) {
    if (tb < 64u) {  // small bins hold a single key value
        thresh = (K)tb;
        quota = k - above;
        return;
    }
    const int nb = (int)(tb >> 6) + 6;  // bit length of the bin's keys
    int shift = nb - 7;
    K prefix = (K)(64u | (tb & 63u));
    const bool list = in_bin <= (uint32_t)kCandCap;
    if (list || (stage != nullptr && !keys_staged)) {
        key_pass<K>(sh, keys, n, keys_staged ? nullptr : stage, false, list, shift, prefix, cand);
        __syncthreads();
        if (stage != nullptr) keys.s = smem_u32(stage);
    }
    uint32_t krem = k - above;
    const int m = list ? (int)min(sh.count, (uint32_t)kCandCap) : n;
    while (shift > 0) {
        const int width = shift < kDigitBits ? shift : kDigitBits;
        shift -= width;
        if (list) radix_level<K>(sh, [&](int i) { return cand[i]; }, m, shift, width, prefix, krem);
        else radix_level<K>(sh, [&](int i) { return keys[i]; }, m, shift, width, prefix, krem);
    }
    thresh = prefix;
    quota = krem;
}

// emit(slot, rank) for every kept key (key > thresh, plus the first `quota`
// keys == thresh in position order), rank = its position among kept keys.
template <typename K, typename Emit>
__device__ void block_compact(SelShared& sh, const Keys<K>& keys, int n, K thresh, uint32_t quota, Emit emit) {
    const int tid = threadIdx.x, lane = lane_id(), wid = warp_id();
    uint32_t carry_g = 0, carry_e = 0;  // kept keys before this chunk
    for (int c0 = 0; c0 < n; c0 += kChunkWords * 32) {
        const int nw = min(kChunkWords, (n - c0 + 31) / 32);
        // bitmap words of this chunk: word w covers keys c0 + 32w .. c0 + 32w + 31
        for (int w0 = wid; w0 < nw; w0 += kSelWarps * kUnroll) {
            K kv[kUnroll];
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) {
                const int i = c0 + 32 * (w0 + u * kSelWarps) + lane;
                kv[u] = i < n ? keys[i] : K(0);
            }
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) {
                const int w = w0 + u * kSelWarps;
                const int i = c0 + 32 * w + lane;
                const uint32_t g = __ballot_sync(0xffffffffu, i < n && kv[u] > thresh);
                const uint32_t e = __ballot_sync(0xffffffffu, i < n && kv[u] == thresh);
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
        const uint32_t tg = sh.wsum[lane], te = sh.wsum2[lane];
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

__device__ __forceinline__ bool row_ok_sel(const IndexArgs& a, int r, int64_t& off, int& L, int32_t& bits) {
    const int seq = a.q_seq[r];
    L = a.q_len[r];
    if (seq < 0 || seq >= a.n_seq) {
        bits = LSA_DEV_BAD_SEQ;
        return false;
    }
    off = a.kv_offset[seq];
    const int slen = a.seq_lens[seq];
    bits = LSA_DEV_BAD_LENGTH;
    if (L < 1 || L > a.max_len || L > slen || off < 0 || off + slen > a.total_tokens) return false;
    if (a.hi_block > 0) {
        const int64_t bo = a.blk_offset[seq];
        if (bo < 0 || bo + (L + a.hi_block - 1) / a.hi_block > a.block_rows) return false;
    }
    bits = 0;
    return true;
}

__host__ __device__ __forceinline__ size_t kept_smem_bytes(int hi_topblocks) {
    return ((size_t)hi_topblocks * 4 + 15) / 16 * 16;
}

// HI: keep the hi_topblocks best candidate blocks (ascending block index).
__global__ void __launch_bounds__(kSelThreads, 1) select_blocks_kernel(const __grid_constant__ IndexArgs a) {
    extern __shared__ __align__(16) uint8_t dyn[];
    __shared__ SelShared sh;
    __shared__ uint64_t s_cand[kCandCap];
    const int r = blockIdx.x;
    int64_t off;
    int L;
    int32_t bits;
    int32_t* kept = a.kept + (int64_t)r * a.hi_topblocks;
    if (!row_ok_sel(a, r, off, L, bits)) {
        if (threadIdx.x == 0) a.n_kept[r] = 0;
        return;  // the token selection reports the row
    }
    const int s = min(a.sink, L);
    const int ws = max(s, L - a.window);
    const int B = a.hi_block;
    const int b_lo = s / B;
    const int nb = ws > s ? (ws + B - 1) / B - b_lo : 0;
    reinterpret_cast<uint4*>(sh.hist)[threadIdx.x] = make_uint4(0u, 0u, 0u, 0u);
    if (threadIdx.x == 0) sh.count = 0;
    __syncthreads();
    uint64_t* stage = a.coarse_in_smem ? reinterpret_cast<uint64_t*>(dyn) : nullptr;
    Keys<uint64_t> keys{a.coarse_keys + (int64_t)r * a.coarse_cap, 0u};
    key_pass<uint64_t>(sh, keys, nb, stage, true, false, 0, 0ull, s_cand);
    __syncthreads();
    if (stage != nullptr) keys.s = smem_u32(stage);
    uint32_t tb, above, in_bin;
    const uint32_t total = find_bin(sh, (uint32_t)a.hi_topblocks, tb, above, in_bin);
    const uint32_t k = min((uint32_t)a.hi_topblocks, total);
    if (k > 0u) {
        uint64_t thr = 1ull;
        uint32_t quota = 0xffffffffu;  // k == total: every candidate is kept
        if (k < total) resolve_threshold<uint64_t>(sh, keys, nb, stage, true, k, tb, above, in_bin, s_cand, thr, quota);
        block_compact<uint64_t>(sh, keys, nb, thr, quota, [&](int slot, uint32_t rank) {
            if (rank < k) kept[rank] = b_lo + slot;
        });
    }
    if (threadIdx.x == 0) a.n_kept[r] = (int32_t)k;
}

// Fine top-k plus the SI assembly of the index set.
__global__ void __launch_bounds__(kSelThreads, 1) select_tokens_kernel(const __grid_constant__ IndexArgs a) {
    extern __shared__ __align__(16) uint8_t dyn[];
    __shared__ SelShared sh;
    __shared__ uint32_t s_cand[kCandCap];
    const int r = blockIdx.x;
    int64_t off;
    int L;
    int32_t bits;
    int32_t* out = a.index_sets + (int64_t)r * a.budget;
    if (!row_ok_sel(a, r, off, L, bits)) {
        if (threadIdx.x == 0) flag(a.dev_status, bits);
        for (int e = threadIdx.x; e < a.budget; e += kSelThreads) out[e] = -1;
        return;
    }
    const int s = min(a.sink, L);
    const int ws = max(s, L - a.window);
    const bool hi = a.hi_block > 0;
    const int B = a.hi_block;
    int32_t* s_kept = reinterpret_cast<int32_t*>(dyn);
    uint32_t* stage = a.fine_in_smem ? reinterpret_cast<uint32_t*>(dyn + (hi ? kept_smem_bytes(a.hi_topblocks) : 0))
                                     : nullptr;
    int n_kept = 0;
    if (hi) {
        n_kept = a.n_kept[r];
        const int32_t* kept = a.kept + (int64_t)r * a.hi_topblocks;
        for (int i = threadIdx.x; i < n_kept; i += kSelThreads) s_kept[i] = kept[i];
    }
    const int n = hi ? n_kept * B : ws - s;
    // the scoring kernel's histogram of this row's keys
    reinterpret_cast<uint4*>(sh.hist)[threadIdx.x] =
        __ldcg(reinterpret_cast<const uint4*>(a.hist + (int64_t)r * kHistBins) + threadIdx.x);
    if (threadIdx.x == 0) sh.count = 0;
    __syncthreads();
    uint32_t tb, above, in_bin;
    const uint32_t total = find_bin(sh, (uint32_t)a.topk, tb, above, in_bin);
    const uint32_t k = min((uint32_t)a.topk, total);
    if (k > 0u) {
        Keys<uint32_t> keys{a.fine_keys + (int64_t)r * a.fine_cap, 0u};
        uint32_t thr = 1u, quota = 0xffffffffu;  // k == total: every candidate is kept
        if (k < total) resolve_threshold<uint32_t>(sh, keys, n, stage, false, k, tb, above, in_bin, s_cand, thr, quota);
        const int lgB = (hi && (B & (B - 1)) == 0) ? __ffs(B) - 1 : -1;  // power-of-two block: shift, not divide
        block_compact<uint32_t>(sh, keys, n, thr, quota, [&](int slot, uint32_t rank) {
            int tok;
            if (hi) {
                const int kb = lgB >= 0 ? slot >> lgB : slot / B;
                tok = s_kept[kb] * B + (slot - kb * B);
            } else {
                tok = s + slot;
            }
            if (rank < k) out[s + rank] = tok;
        });
    }
    const int win0 = s + (int)k;
    const int n_win = L - ws;
    for (int e = threadIdx.x; e < a.budget; e += kSelThreads) {
        if (e < s) out[e] = e;
        else if (e >= win0 && e < win0 + n_win) out[e] = ws + (e - win0);
        else if (e >= win0 + n_win) out[e] = -1;
    }
}

}  // namespace

static size_t align256(size_t x) { return (x + 255) / 256 * 256; }

// Selection kernels keep the row's keys in shared memory up to these sizes.
constexpr size_t kBlockKeySmem = 160 * 1024;
constexpr size_t kTokenKeySmem = 160 * 1024;

IndexPlan plan_index(int n_q, int max_len, const lsa_budget_t& b) {
    IndexPlan p;
    const bool hi = b.hi_block > 0;
    if (hi) {
        p.coarse_cap = (max_len + b.hi_block - 1) / b.hi_block + 1;
        p.coarse_cap = (p.coarse_cap + 1) / 2 * 2;
        p.fine_cap = b.hi_topblocks * b.hi_block;
    } else {
        p.fine_cap = max_len;
    }
    p.fine_cap = (p.fine_cap + 3) / 4 * 4;
    if (p.fine_cap < 4) p.fine_cap = 4;
    p.coarse_in_smem = hi && (size_t)p.coarse_cap * 8 <= kBlockKeySmem;
    p.fine_in_smem = (size_t)p.fine_cap * 4 <= kTokenKeySmem;
    p.smem_blocks = p.coarse_in_smem ? (size_t)p.coarse_cap * 8 : 0;
    p.smem_tokens = (hi ? kept_smem_bytes(b.hi_topblocks) : 0) + (p.fine_in_smem ? (size_t)p.fine_cap * 4 : 0);
    size_t off = 0;
    p.off_coarse = off;
    off = align256(off + (size_t)n_q * p.coarse_cap * 8);
    p.off_kept = off;
    off = align256(off + (size_t)n_q * (hi ? b.hi_topblocks : 0) * 4);
    p.off_nkept = off;
    off = align256(off + (size_t)n_q * 4);
    p.off_fine = off;
    off = align256(off + (size_t)n_q * p.fine_cap * 4);
    p.off_hist = off;
    off = align256(off + (size_t)n_q * kHistBins * 4);
    p.ws_bytes = off;
    return p;
}

cudaError_t launch_index_select(const IndexArgs& a, bool blocks, size_t smem, cudaStream_t stream) {
    if (blocks) {
        cudaError_t e = cudaFuncSetAttribute(select_blocks_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)smem);
        if (e != cudaSuccess) return e;
        select_blocks_kernel<<<a.n_q, kSelThreads, smem, stream>>>(a);
    } else {
        cudaError_t e = cudaFuncSetAttribute(select_tokens_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)smem);
        if (e != cudaSuccess) return e;
        select_tokens_kernel<<<a.n_q, kSelThreads, smem, stream>>>(a);
    }
    return cudaGetLastError();
}

}  // namespace lsa
