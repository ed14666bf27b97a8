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
// is a CTA barrier. The row's keys (score + 1, 0 = not a candidate) are
// staged in shared memory when they fit (the maximum and the candidate count
// are taken during staging). An MSD radix select finds the exact k-th largest
// key T and the number of keys equal to T to keep: its first 8-bit digit is
// the top 8 bits below the row maximum's leading bit; the keys of the
// threshold bin are then gathered into a short list on which one warp
// resolves the remaining digits. Compaction is bitmap based: warp ballots
// build "key > T" and "key == T" words, each thread counts its words, one CTA
// prefix ranks them, and every thread emits its kept positions in order — a
// fixed number of barriers whatever the row length.
#include "common.cuh"
#include "internal.h"

namespace lsa {
namespace {

constexpr int kSelThreads = 1024;
constexpr int kSelWarps = kSelThreads / kWarp;
constexpr int kBins = 256;
constexpr int kCandCap = 2048;        // keys of the threshold bin resolved by one warp
constexpr int kWordsPerThread = 1;    // compaction: bitmap words per thread per chunk
constexpr int kChunkWords = kSelThreads * kWordsPerThread;  // 1024 words = 32768 keys
constexpr int kUnroll = 4;            // independent key loads in flight per thread

struct SelShared {
    uint32_t hist[kBins];
    uint32_t wsum[kSelWarps];
    uint32_t wsum2[kSelWarps];
    unsigned long long wmax[kSelWarps];
    uint32_t gt_words[kChunkWords];
    uint32_t eq_words[kChunkWords];
    uint32_t digit, above, in_bin, count;
    uint32_t carry_gt, carry_eq;
};

template <typename K>
__device__ __forceinline__ int key_bits(K v) {
    if constexpr (sizeof(K) == 8) return 64 - __clzll((long long)v);
    else return 32 - __clz((int)v);
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
};

// Block sum of two counters and maximum of a 64-bit value.
__device__ void block_reduce(SelShared& sh, uint32_t& a, uint32_t& b, unsigned long long& m) {
    const int lane = lane_id(), wid = warp_id();
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        a += __shfl_xor_sync(0xffffffffu, a, o);
        b += __shfl_xor_sync(0xffffffffu, b, o);
        m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
    }
    if (lane == 0) {
        sh.wsum[wid] = a;
        sh.wsum2[wid] = b;
        sh.wmax[wid] = m;
    }
    __syncthreads();
    a = 0;
    b = 0;
    m = 0;
    for (int w = 0; w < kSelWarps; ++w) {
        a += sh.wsum[w];
        b += sh.wsum2[w];
        m = max(m, sh.wmax[w]);
    }
    __syncthreads();
}

// Stages the row's keys in shared memory (when planned) and returns the
// maximum key and the number of nonzero keys.
template <typename K>
__device__ Keys<K> stage_keys(SelShared& sh, const K* g, int n, uint8_t* dyn, bool in_smem, unsigned long long& kmax,
                              uint32_t& nvalid) {
    Keys<K> k{g, 0u};
    unsigned long long m = 0;
    uint32_t c = 0, unused = 0;
    auto see = [&](K v) {
        m = max(m, (unsigned long long)v);
        c += v != 0 ? 1u : 0u;
    };
    constexpr int kPer16 = 16 / (int)sizeof(K);
    const int n16 = n / kPer16;
    K* st = reinterpret_cast<K*>(dyn);
    for (int i = threadIdx.x; i < n16; i += kSelThreads) {
        const uint4 v = __ldcg(reinterpret_cast<const uint4*>(g) + i);
        if (in_smem) reinterpret_cast<uint4*>(st)[i] = v;
        const K* e = reinterpret_cast<const K*>(&v);
#pragma unroll
        for (int j = 0; j < kPer16; ++j) see(e[j]);
    }
    for (int i = n16 * kPer16 + threadIdx.x; i < n; i += kSelThreads) {
        const K v = __ldcg(g + i);
        if (in_smem) st[i] = v;
        see(v);
    }
    block_reduce(sh, c, unused, m);
    kmax = m;
    nvalid = c;
    if (in_smem) k.s = smem_u32(st);
    return k;
}

// Block-level histogram pass: counts the `width`-bit digit at `shift` of the
// keys whose bits above shift+width equal `prefix`, then finds the digit d*
// where the running count from the top reaches krem.
template <typename K>
__device__ void hist_pass(SelShared& sh, const Keys<K>& keys, int n, int shift, int width, K prefix, uint32_t krem,
                          uint32_t& digit, uint32_t& above, uint32_t& in_bin) {
    constexpr int kKeyBits = 8 * sizeof(K);
    const int tid = threadIdx.x, lane = lane_id(), wid = warp_id();
    if (tid < kBins) sh.hist[tid] = 0;
    __syncthreads();
    for (int i0 = tid; i0 < n; i0 += kSelThreads * kUnroll) {
        K kv[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int i = i0 + u * kSelThreads;
            kv[u] = i < n ? keys[i] : K(0);
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int i = i0 + u * kSelThreads;
            const K key = kv[u];
            const K hi = (shift + width >= kKeyBits) ? K(0) : (K)(key >> (shift + width));
            if (i < n && hi == prefix) atomicAdd(&sh.hist[(uint32_t)(key >> shift) & ((1u << width) - 1u)], 1u);
        }
    }
    __syncthreads();
    uint32_t tot = 0, x = 0;
    if (tid < kBins) {
        tot = sh.hist[tid];
        x = tot;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t v = __shfl_down_sync(0xffffffffu, x, o);
            if (lane + o < 32) x += v;
        }
        if (lane == 0) sh.wsum[wid] = x;
    }
    __syncthreads();
    if (tid < kBins) {
        uint32_t later = 0;
        for (int w2 = wid + 1; w2 < kBins / kWarp; ++w2) later += sh.wsum[w2];
        const uint32_t S = x + later;  // count with digit >= tid
        if (S >= krem && S - tot < krem) {
            sh.digit = tid;
            sh.above = S - tot;
            sh.in_bin = tot;
        }
    }
    __syncthreads();
    digit = sh.digit;
    above = sh.above;
    in_bin = sh.in_bin;
    __syncthreads();
}

// Warp-level histogram pass over a short list (warp 0 only; no CTA barrier).
template <typename K>
__device__ void warp_hist_pass(SelShared& sh, const K* cand, int m, int shift, int width, uint32_t krem,
                               uint32_t& digit, uint32_t& above) {
    const int lane = lane_id();
#pragma unroll
    for (int j = 0; j < kBins / kWarp; ++j) sh.hist[lane * (kBins / kWarp) + j] = 0;
    __syncwarp();
    for (int i = lane; i < m; i += kWarp) atomicAdd(&sh.hist[(uint32_t)(cand[i] >> shift) & ((1u << width) - 1u)], 1u);
    __syncwarp();
    // lane l owns bins [8l, 8l+8); suffix sums across lanes, then within the lane
    uint32_t own = 0;
#pragma unroll
    for (int j = 0; j < kBins / kWarp; ++j) own += sh.hist[lane * (kBins / kWarp) + j];
    uint32_t x = own;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t v = __shfl_down_sync(0xffffffffu, x, o);
        if (lane + o < 32) x += v;
    }
    uint32_t S = x;  // count with digit >= 8*lane
    uint32_t d_found = 0xffffffffu, a_found = 0;
    if (S >= krem && S - own < krem) {
        // the crossing is inside this lane's bins: walk them from the top
        uint32_t run = S - own;
        for (int j = kBins / kWarp - 1; j >= 0; --j) {
            const uint32_t c = sh.hist[lane * (kBins / kWarp) + j];
            if (run + c >= krem) {
                d_found = (uint32_t)(lane * (kBins / kWarp) + j);
                a_found = run;
                break;
            }
            run += c;
        }
    }
    const uint32_t who = __ballot_sync(0xffffffffu, d_found != 0xffffffffu);
    const int src = __ffs(who) - 1;
    digit = __shfl_sync(0xffffffffu, d_found, src);
    above = __shfl_sync(0xffffffffu, a_found, src);
    __syncwarp();
}

// Exact k-th largest key: keys > thresh plus the first `quota` keys equal to
// thresh (in position order) are the k_target largest.
template <typename K>
__device__ void block_select(SelShared& sh, const Keys<K>& keys, int n, uint32_t k_target, unsigned long long kmax,
                             uint32_t nvalid, K* cand, K& thresh, uint32_t& quota) {
    if (k_target == 0) {
        thresh = ~K(0);
        quota = 0;
        return;
    }
    if (k_target >= nvalid) {  // every candidate is kept
        thresh = K(1);
        quota = 0xffffffffu;
        return;
    }
    int nbits = key_bits<K>((K)kmax);
    if (nbits < 1) nbits = 1;
    int width = nbits < 8 ? nbits : 8;
    int shift = nbits - width;
    uint32_t d, above, in_bin;
    hist_pass<K>(sh, keys, n, shift, width, K(0), k_target, d, above, in_bin);
    K prefix = (K)d;
    uint32_t krem = k_target - above;
    if (shift > 0 && (int)in_bin <= kCandCap) {
        // gather the threshold bin's keys; one warp resolves the rest
        if (threadIdx.x == 0) sh.count = 0;
        __syncthreads();
        for (int i0 = threadIdx.x; i0 < n; i0 += kSelThreads * kUnroll) {
            K kv[kUnroll];
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) {
                const int i = i0 + u * kSelThreads;
                kv[u] = i < n ? keys[i] : K(0);
            }
#pragma unroll
            for (int u = 0; u < kUnroll; ++u)
                if (i0 + u * kSelThreads < n && (K)(kv[u] >> shift) == prefix) cand[atomicAdd(&sh.count, 1u)] = kv[u];
        }
        __syncthreads();
        if (warp_id() == 0) {
            while (shift > 0) {
                width = shift < 8 ? shift : 8;
                shift -= width;
                // only keys matching the prefix are in the list at the first
                // refinement; later refinements filter by the grown prefix
                uint32_t dd, aa;
                // compact the list to the keys matching the current prefix
                const int m0 = (int)in_bin;
                int m = 0;
                for (int base = 0; base < m0; base += kWarp) {
                    const int i = base + lane_id();
                    const K key = i < m0 ? cand[i] : K(0);
                    const bool keep = i < m0 && (K)(key >> (shift + width)) == prefix;
                    const uint32_t mk = __ballot_sync(0xffffffffu, keep);
                    const int pos = m + __popc(mk & lanemask_lt());
                    __syncwarp();
                    if (keep) cand[pos] = key;
                    m += __popc(mk);
                    __syncwarp();
                }
                in_bin = (uint32_t)m;
                warp_hist_pass<K>(sh, cand, m, shift, width, krem, dd, aa);
                prefix = (K)((prefix << width) | (K)dd);
                krem -= aa;
            }
            if (lane_id() == 0) {
                sh.digit = (uint32_t)0;
                sh.above = krem;
                *reinterpret_cast<K*>(&sh.hist[0]) = prefix;
            }
        }
        __syncthreads();
        prefix = *reinterpret_cast<const K*>(&sh.hist[0]);
        krem = sh.above;
        __syncthreads();
    } else {
        while (shift > 0) {
            width = shift < 8 ? shift : 8;
            shift -= width;
            hist_pass<K>(sh, keys, n, shift, width, prefix, krem, d, above, in_bin);
            prefix = (K)((prefix << width) | (K)d);
            krem -= above;
        }
    }
    thresh = prefix;
    quota = krem;
}

// emit(slot, rank) for every kept key (key > thresh, plus the first `quota`
// keys == thresh in position order), rank = its position among kept keys.
template <typename K, typename Emit>
__device__ void block_compact(SelShared& sh, const Keys<K>& keys, int n, K thresh, uint32_t quota, Emit emit) {
    const int tid = threadIdx.x, lane = lane_id(), wid = warp_id();
    if (tid == 0) {
        sh.carry_gt = 0;
        sh.carry_eq = 0;
    }
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
        const int w0 = tid * kWordsPerThread;
        uint32_t cg = 0, ce = 0;
#pragma unroll
        for (int j = 0; j < kWordsPerThread; ++j) {
            if (w0 + j < nw) {
                cg += __popc(sh.gt_words[w0 + j]);
                ce += __popc(sh.eq_words[w0 + j]);
            }
        }
        // exclusive prefix of (cg, ce) over threads, in thread order
        uint32_t xg = cg, xe = ce;
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
        uint32_t gb = sh.carry_gt, eb = sh.carry_eq;
        for (int w2 = 0; w2 < wid; ++w2) {
            gb += sh.wsum[w2];
            eb += sh.wsum2[w2];
        }
        gb += xg - cg;
        eb += xe - ce;
        for (int j = 0; j < kWordsPerThread; ++j) {
            if (w0 + j >= nw) break;
            const uint32_t g = sh.gt_words[w0 + j], e = sh.eq_words[w0 + j];
            uint32_t both = g | e;
            while (both) {
                const int b = __ffs(both) - 1;
                both &= both - 1;
                const uint32_t below = (1u << b) - 1u;
                const uint32_t pg = gb + __popc(g & below), pe = eb + __popc(e & below);
                const int slot = c0 + 32 * (w0 + j) + b;
                if ((g >> b) & 1u) emit(slot, pg + min(pe, quota));
                else if (pe < quota) emit(slot, pg + pe);
            }
            gb += __popc(g);
            eb += __popc(e);
        }
        __syncthreads();
        if (tid == kSelThreads - 1) {
            sh.carry_gt = gb;
            sh.carry_eq = eb;
        }
        __syncthreads();
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
    unsigned long long kmax;
    uint32_t nvalid;
    const Keys<uint64_t> keys =
        stage_keys<uint64_t>(sh, a.coarse_keys + (int64_t)r * a.coarse_cap, nb, dyn, a.coarse_in_smem, kmax, nvalid);
    const uint32_t k = min((uint32_t)a.hi_topblocks, nvalid);
    uint64_t thr;
    uint32_t quota;
    block_select<uint64_t>(sh, keys, nb, k, kmax, nvalid, s_cand, thr, quota);
    block_compact<uint64_t>(sh, keys, nb, thr, quota, [&](int slot, uint32_t rank) { kept[rank] = b_lo + slot; });
    if (threadIdx.x == 0) a.n_kept[r] = (int32_t)k;
}

// Fine top-k plus the SI assembly of the index set.
__global__ void __launch_bounds__(kSelThreads, 1) select_tokens_kernel(const __grid_constant__ IndexArgs a) {
    extern __shared__ __align__(16) uint8_t dyn[];
    __shared__ SelShared sh;
    __shared__ int32_t s_kept[LSA_MAX_TOPBLOCKS];
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
    int n_kept = 0;
    if (hi) {
        n_kept = a.n_kept[r];
        const int32_t* kept = a.kept + (int64_t)r * a.hi_topblocks;
        for (int i = threadIdx.x; i < n_kept; i += kSelThreads) s_kept[i] = kept[i];
    }
    const int n = hi ? n_kept * B : ws - s;
    unsigned long long kmax;
    uint32_t nvalid;
    const Keys<uint32_t> keys =
        stage_keys<uint32_t>(sh, a.fine_keys + (int64_t)r * a.fine_cap, n, dyn, a.fine_in_smem, kmax, nvalid);
    const uint32_t k = min((uint32_t)a.topk, nvalid);
    uint32_t thr, quota;
    block_select<uint32_t>(sh, keys, n, k, kmax, nvalid, s_cand, thr, quota);
    const int lgB = (hi && (B & (B - 1)) == 0) ? __ffs(B) - 1 : -1;  // power-of-two block: shift, not divide
    block_compact<uint32_t>(sh, keys, n, thr, quota, [&](int slot, uint32_t rank) {
        int tok;
        if (hi) {
            const int kb = lgB >= 0 ? slot >> lgB : slot / B;
            tok = s_kept[kb] * B + (slot - kb * B);
        } else {
            tok = s + slot;
        }
        out[s + rank] = tok;
    });
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
constexpr size_t kTokenKeySmem = 180 * 1024;

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
    p.smem_tokens = p.fine_in_smem ? (size_t)p.fine_cap * 4 : 0;
    size_t off = 0;
    p.off_coarse = off;
    off = align256(off + (size_t)n_q * p.coarse_cap * 8);
    p.off_kept = off;
    off = align256(off + (size_t)n_q * (hi ? b.hi_topblocks : 0) * 4);
    p.off_nkept = off;
    off = align256(off + (size_t)n_q * 4);
    p.off_fine = off;
    off = align256(off + (size_t)n_q * p.fine_cap * 4);
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
