// append.cuh — the block-sum reduction and the decode append's per-CTA work,
// shared by the block-sum kernels and by the block selection, which can run
// a decode step's append in CTAs of its own grid.
//
// Hierarchical Indexing scores whole blocks on the exact sum of their indexer
// keys ("LongCat-Flash-Lite-Sparse (aitrends.kr)", section "기술적 특징", HI
// bullet); the append keeps those sums exact as a decode loop adds tokens.
#pragma once

#include "common.cuh"
#include "internal.h"

namespace lsa {

__device__ __forceinline__ int sbyte(uint32_t w, int i) { return static_cast<int>(static_cast<int8_t>(w >> (8 * i))); }

// The sequence's cache span and block rows, checked; false when they are out
// of range (with LSA_DEV_BAD_LENGTH set by the CTA that has `report`). The
// check is uniform over the CTA.
__device__ __forceinline__ bool seq_ok(const BlockSumArgs& a, int seq, int64_t& off, int& len, bool report) {
    off = a.kv_offset[seq];
    len = a.seq_lens[seq];
    bool ok = len >= 1 && len <= a.max_len && off >= 0 && off + len <= a.total_tokens;
    if (ok && a.hi_block > 0) {
        const int64_t boff = a.blk_offset[seq];
        const int nblk = (len + a.hi_block - 1) / a.hi_block;
        ok = boff >= 0 && boff + nblk <= a.block_rows;
    }
    if (!ok && report && threadIdx.x == 0) flag(a.dev_status, LSA_DEV_BAD_LENGTH);
    return ok;
}

// Sum of rows [0, n) of one block, by a CTA of THREADS threads: thread t owns
// 16-byte chunk (t % CPR) of rows t / CPR, t / CPR + RPP, ..., so the block
// is read in B / RPP rounds of coalesced 16-byte loads (ROWS rows in flight
// per thread). row_ptr(i) is the address of the block's row i; the sum goes
// to out_row as the two byte planes (S >> 8 as int8, S & 0xFF as uint8).
// s_part: THREADS / 32 * D_I ints of shared memory. Every thread of the CTA
// calls it (one CTA barrier).
template <int D_I, int ROWS, int THREADS, typename RowPtr>
__device__ __forceinline__ void sum_block(RowPtr row_ptr, int n, int8_t* out_row, int* s_part) {
    constexpr int kCPR = D_I / 16;        // 16-byte chunks per row
    constexpr int kRPP = THREADS / kCPR;  // rows per pass
    constexpr int kWarps = THREADS / kWarp;
    const int tid = threadIdx.x, lane = lane_id(), warp = warp_id();
    const int c = tid % kCPR;
    int acc[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) acc[i] = 0;
    for (int row0 = tid / kCPR; row0 < n; row0 += kRPP * ROWS) {
        uint4 v[ROWS];
#pragma unroll
        for (int u = 0; u < ROWS; ++u) {
            const int row = row0 + u * kRPP;
            v[u] = row < n ? ldg16(row_ptr(row) + c * 16) : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int u = 0; u < ROWS; ++u) {
            const uint32_t w[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
            for (int q = 0; q < 4; ++q)
#pragma unroll
                for (int b = 0; b < 4; ++b) acc[4 * q + b] += sbyte(w[q], b);
        }
    }
    // lanes with the same chunk differ in the bits above log2(kCPR)
#pragma unroll
    for (int m = kCPR; m < kWarp; m <<= 1)
#pragma unroll
        for (int i = 0; i < 16; ++i) acc[i] += __shfl_xor_sync(0xffffffffu, acc[i], m);
    if (lane < kCPR) {
#pragma unroll
        for (int i = 0; i < 16; ++i) s_part[warp * D_I + lane * 16 + i] = acc[i];
    }
    __syncthreads();
    if (tid < D_I) {
        int S = 0;
#pragma unroll
        for (int w2 = 0; w2 < kWarps; ++w2) S += s_part[w2 * D_I + tid];
        // S = 256 * hi + lo with hi = S >> 8 (arithmetic), lo = S & 0xFF.
        out_row[tid] = static_cast<int8_t>(S >> 8);
        reinterpret_cast<uint8_t*>(out_row)[D_I + tid] = static_cast<uint8_t>(S & 0xFF);
    }
}

template <int THREADS>
__device__ __forceinline__ void copy16(uint8_t* dst, const uint8_t* src, int64_t bytes) {
    for (int64_t i = threadIdx.x; i < bytes / 16; i += THREADS)
        reinterpret_cast<uint4*>(dst)[i] = ldg16(src + 16 * i);
}

// One CTA's share of the decode append. Task (x, seq, role): role 0 copies the
// new tokens of sequence seq that fall in block first + x (HI on) or in the
// x-th run of kAppendRowsPerCta new tokens (HI off) — their indexer keys and
// every layer's K and V rows; role 1 (HI on) recomputes that block's sum,
// reading the new rows from the inputs and the older rows from the cache, so
// no task reads what any task writes. Uniform over the CTA.
template <int D_I, int THREADS>
__device__ void append_task(const AppendArgs& p, int x, int seq, int role, int* s_part) {
    const BlockSumArgs& a = p.bs;
    int64_t off;
    int len;
    if (!seq_ok(a, seq, off, len, x == 0 && role == 0)) return;
    const int n_new = a.n_new;
    if (n_new > len) {
        if (threadIdx.x == 0 && x == 0 && role == 0) flag(a.dev_status, LSA_DEV_BAD_LENGTH);
        return;
    }
    const int from = len - n_new;  // first new position
    int lo, hi, t0 = 0, n = 0, j = 0;
    if (p.sums) {
        const int B = a.hi_block;
        j = from / B + x;
        if (j >= (len + B - 1) / B) return;
        t0 = j * B;
        n = min(t0 + B, len) - t0;
        lo = max(t0, from);
        hi = t0 + n;
    } else {
        lo = from + x * kAppendRowsPerCta;
        hi = min(len, lo + kAppendRowsPerCta);
        if (lo >= hi) return;
    }
    if (role == 0) {
        const int64_t src0 = (int64_t)seq * n_new + (lo - from);  // first input row
        const int nr = hi - lo;
        copy16<THREADS>(reinterpret_cast<uint8_t*>(p.k_idx_cache) + (off + lo) * D_I,
                        reinterpret_cast<const uint8_t*>(p.k_idx_new) + src0 * D_I, (int64_t)nr * D_I);
        const int64_t kvb = p.kv_row_bytes;
        for (int g = 0; g < p.layers; ++g) {
            copy16<THREADS>(reinterpret_cast<uint8_t*>(p.k_cache[g]) + (off + lo) * kvb,
                            reinterpret_cast<const uint8_t*>(p.k_new[g]) + src0 * kvb, nr * kvb);
            copy16<THREADS>(reinterpret_cast<uint8_t*>(p.v_cache[g]) + (off + lo) * kvb,
                            reinterpret_cast<const uint8_t*>(p.v_new[g]) + src0 * kvb, nr * kvb);
        }
    } else if (p.sums) {
        const int8_t* cache = a.k_idx + (off + t0) * D_I;
        const int8_t* fresh = p.k_idx_new + (int64_t)seq * n_new * D_I;
        sum_block<D_I, 4, THREADS>(
            [&](int row) {
                const int pos = t0 + row;
                return pos >= from ? fresh + (int64_t)(pos - from) * D_I : cache + (int64_t)row * D_I;
            },
            n, a.block_sums + (a.blk_offset[seq] + j) * (2 * D_I), s_part);
    }
}

}  // namespace lsa
