// draft_union.cu — the union of the index sets of a group of draft rows.
//
// A decode step that verifies several draft tokens of one sequence (the
// multi-token prediction used for speculative decoding, "LongCat-2.0
// (molayo1419.me)", section "1M 토큰에서의 Sparse Attention 문제") has one
// decode row per draft token, each with its own index set. Their sink and
// window runs coincide almost entirely and their selected tokens overlap, so
// the attention reads the union of the group's sets once and lets every row
// attend over its own members. This kernel builds that union: the positions
// held by any row of the group, ascending, each with a mask of the rows that
// hold it.
//
// Design: one 1024-thread CTA per group. The group's sets are staged in
// shared memory (entries outside [0, q_len) of their row are flagged and
// dropped); the position range is swept in chunks of 65536 positions: each
// row's entries in the chunk set bits of a per-row bitmap, then each thread
// takes two 32-position words, ORs the rows' words, and a CTA prefix sum of
// the bit counts places its positions (ascending) and their row masks in the
// output. Duplicate entries of one row count once. Last, a prefix sum of the
// masks' member counts cuts the union into the attention's splits of equal
// work.
#include "common.cuh"
#include "internal.h"

namespace lsa {
namespace {

constexpr int kUnThreads = 1024;
constexpr int kUnWarps = kUnThreads / kWarp;
constexpr int kUnWordsPerThread = 2;
constexpr int kUnChunkWords = kUnThreads * kUnWordsPerThread;  // 2048 words
constexpr int kUnChunk = kUnChunkWords * 32;                   // 65536 positions

__global__ void __launch_bounds__(kUnThreads, 1) union_sets_kernel(const __grid_constant__ UnionArgs u) {
    extern __shared__ __align__(16) uint8_t un_dyn[];
    __shared__ uint32_t s_warp[kUnWarps];
    __shared__ int32_t s_len[kMaxGroupRows];
    __shared__ int32_t s_bad_group;
    const int D = u.group_rows;
    uint32_t* bits = reinterpret_cast<uint32_t*>(un_dyn);          // [D][kUnChunkWords]
    int32_t* lists = reinterpret_cast<int32_t*>(bits + D * kUnChunkWords);  // [D][budget]
    const int grp = blockIdx.x, tid = threadIdx.x, lane = lane_id(), warp = warp_id();
    const int r0 = grp * D;
    // the rows' metadata (the caller's) before the wait for the index sets
    if (tid == 0) s_bad_group = 0;
    __syncthreads();
    if (tid < D) {
        const int r = r0 + tid;
        const int seq = u.q_seq[r];
        const int L = u.q_len[r];
        const int seq_c = min(max(seq, 0), u.n_seq - 1);
        const int64_t off = u.kv_offset[seq_c];
        const int slen = u.seq_lens[seq_c];
        const bool ok = seq >= 0 && seq < u.n_seq && L >= 1 && L <= u.max_len && L <= slen && off >= 0 &&
                        off + slen <= u.total_tokens;
        s_len[tid] = ok ? L : 0;  // an invalid row holds nothing (the attention flags it)
        if (seq != u.q_seq[r0]) s_bad_group = 1;  // the group's rows must share one sequence
    }
    pdl_enter();
    __syncthreads();
    if (s_bad_group) {
        if (tid == 0) {
            flag(u.dev_status, LSA_DEV_BAD_SEQ);
            u.union_len[grp] = 0;
        }
        for (int sp = tid; sp <= u.n_splits; sp += kUnThreads) u.union_split[(int64_t)grp * (u.n_splits + 1) + sp] = 0;
        return;
    }
    int l_max = 0;
    for (int j = 0; j < D; ++j) l_max = max(l_max, s_len[j]);
    // stage the sets, dropping what a row cannot hold
    bool bad_entry = false;
    for (int i = tid; i < D * u.budget; i += kUnThreads) {
        const int j = i / u.budget;
        const int32_t e = u.sets[(int64_t)r0 * u.budget + i];
        const int L = s_len[j];
        const bool keep = e >= 0 && e < L;
        bad_entry |= L > 0 && (e < -1 || e >= L);
        lists[i] = keep ? e : -1;
    }
    if (bad_entry) flag(u.dev_status, LSA_DEV_BAD_INDEX);
    int32_t* out_pos = u.union_pos + (int64_t)grp * u.union_cap;
    uint8_t* out_msk = u.union_msk + (int64_t)grp * u.union_cap;
    uint32_t base = 0;  // union entries written so far (the same in every thread)
    for (int c0 = 0; c0 < l_max; c0 += kUnChunk) {
        for (int i = tid; i < D * kUnChunkWords; i += kUnThreads) bits[i] = 0u;
        __syncthreads();  // also orders the staging above before the first chunk's reads
        for (int i = tid; i < D * u.budget; i += kUnThreads) {
            const int32_t e = lists[i];
            if (e >= c0 && e < c0 + kUnChunk) {
                const int j = i / u.budget;
                atomicOr(&bits[j * kUnChunkWords + ((e - c0) >> 5)], 1u << (e & 31));
            }
        }
        __syncthreads();
        uint32_t word[kUnWordsPerThread];
        uint32_t cnt = 0;
#pragma unroll
        for (int q = 0; q < kUnWordsPerThread; ++q) {
            const int w = kUnWordsPerThread * tid + q;
            uint32_t x = 0;
            for (int j = 0; j < D; ++j) x |= bits[j * kUnChunkWords + w];
            word[q] = x;
            cnt += __popc(x);
        }
        // exclusive prefix of the counts over the CTA (threads in word order)
        uint32_t incl = cnt;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        if (lane == 31) s_warp[warp] = incl;
        __syncthreads();
        uint32_t before = 0, total = 0;
        for (int w = 0; w < kUnWarps; ++w) {
            const uint32_t c = s_warp[w];
            before += w < warp ? c : 0u;
            total += c;
        }
        uint32_t k = base + before + incl - cnt;
#pragma unroll
        for (int q = 0; q < kUnWordsPerThread; ++q) {
            const int w = kUnWordsPerThread * tid + q;
            uint32_t x = word[q];
            while (x != 0u) {
                const int b = __ffs(x) - 1;
                x &= x - 1u;
                uint32_t m = 0;
                for (int j = 0; j < D; ++j) m |= ((bits[j * kUnChunkWords + w] >> b) & 1u) << j;
                if (k < (uint32_t)u.union_cap) {  // at most D x budget distinct entries: always true
                    out_pos[k] = c0 + 32 * w + b;
                    out_msk[k] = (uint8_t)m;
                }
                ++k;
            }
        }
        base += total;
        __syncthreads();  // the bitmaps and s_warp are rewritten by the next chunk
    }
    // The attention splits the union into n_splits stretches of equal work
    // (members summed over the rows, not entries: the window run is held by
    // every row, the selected tokens by few). The members before each entry
    // go to shared memory (over the staged lists, no longer needed), then
    // thread s finds the first entry of stretch s by binary search.
    const int U = (int)min(base, (uint32_t)u.union_cap);
    int32_t* cum = lists;  // U <= D x budget entries
    __syncthreads();       // the masks written above are visible to the whole CTA
    uint32_t run = 0;
    for (int c0 = 0; c0 < U; c0 += kUnThreads) {
        const int k = c0 + tid;
        const uint32_t w = k < U ? (uint32_t)__popc(out_msk[k]) : 0u;
        uint32_t incl = w;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        if (lane == 31) s_warp[warp] = incl;
        __syncthreads();
        uint32_t before = 0, total = 0;
        for (int w2 = 0; w2 < kUnWarps; ++w2) {
            const uint32_t c = s_warp[w2];
            before += w2 < warp ? c : 0u;
            total += c;
        }
        if (k < U) cum[k] = (int32_t)(run + before + incl - w);
        run += total;
        __syncthreads();
    }
    pdl_trigger();
    int32_t* split = u.union_split + (int64_t)grp * (u.n_splits + 1);
    for (int sp = tid; sp <= u.n_splits; sp += kUnThreads) {
        const int64_t target = (int64_t)run * sp / u.n_splits;
        int lo = 0, hi = U;  // first entry whose members-before reach the target (U if none)
        while (lo < hi) {
            const int mid = (lo + hi) >> 1;
            if ((int64_t)cum[mid] >= target) hi = mid;
            else lo = mid + 1;
        }
        split[sp] = sp == u.n_splits ? U : lo;
    }
    if (tid == 0) u.union_len[grp] = U;
}

}  // namespace

size_t union_smem_bytes(int group_rows, int budget) {
    return (size_t)group_rows * kUnChunkWords * 4 + (size_t)group_rows * budget * 4;
}

cudaError_t launch_union_sets(const UnionArgs& u, cudaStream_t stream) {
    const size_t smem = union_smem_bytes(u.group_rows, u.budget);
    cudaError_t e = cudaFuncSetAttribute(union_sets_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    return launch_pdl(union_sets_kernel, dim3((unsigned)u.n_groups), dim3(kUnThreads), smem, stream, 0, u);
}

}  // namespace lsa
