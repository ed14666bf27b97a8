// block_sums.cu — HI block-sum pre-pass, and the decode append that writes
// the newest tokens' keys and K/V rows and refreshes their blocks' sums.
//
// Hierarchical Indexing first scores whole blocks ("LongCat-Flash-Lite-Sparse
// (aitrends.kr)", section "기술적 특징", HI bullet). The block score uses the
// exact sum of the block's indexer keys, S_b[d] = sum_t k_t[d], over the
// present tokens of the block (blocks aligned at position 0).
//
// One CTA reduces one block with 16-byte loads spread over all its threads
// (a single dependent round trip for the decode append update); partial sums
// are folded with shuffles and shared memory. The sum is stored as two byte
// planes (S >> 8 as int8, S & 0xFF as uint8) so that the coarse pass can feed
// it straight to the 8-bit tensor-core MMA.
#include "common.cuh"
#include "internal.h"

namespace lsa {
namespace {

constexpr int kBsThreads = 256;
constexpr int kBsWarps = kBsThreads / kWarp;

__device__ __forceinline__ int sbyte(uint32_t w, int i) { return static_cast<int>(static_cast<int8_t>(w >> (8 * i))); }

// Thread t owns 16-byte chunk (t % CPR) of rows t / CPR, t / CPR + RPP, ...
// of the block, so the block is read in B / RPP rounds of coalesced 16-byte
// loads (one round for hi_block <= 32 at d_I = 128). Keeping four rows in
// flight per thread was measured and dropped: 63 registers instead of 48
// cost resident CTAs, and the full build got slower. row_ptr(i) is
// the address of the block's row i; the sum of rows [0, n) goes to out_row as
// the two byte planes. Every thread of the CTA calls it (one CTA barrier).
// ROWS: rows each thread loads at once (the decode append, one block per
// CTA and latency-bound, issues a whole block's loads in one round).
template <int D_I, int ROWS = 1, typename RowPtr>
__device__ __forceinline__ void sum_block(RowPtr row_ptr, int n, int8_t* out_row, int (&s_part)[kBsWarps][D_I]) {
    constexpr int kCPR = D_I / 16;           // 16-byte chunks per row
    constexpr int kRPP = kBsThreads / kCPR;  // rows per pass
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
        for (int i = 0; i < 16; ++i) s_part[warp][lane * 16 + i] = acc[i];
    }
    __syncthreads();
    if (tid < D_I) {
        int S = 0;
#pragma unroll
        for (int w2 = 0; w2 < kBsWarps; ++w2) S += s_part[w2][tid];
        // S = 256 * hi + lo with hi = S >> 8 (arithmetic), lo = S & 0xFF.
        out_row[tid] = static_cast<int8_t>(S >> 8);
        reinterpret_cast<uint8_t*>(out_row)[D_I + tid] = static_cast<uint8_t>(S & 0xFF);
    }
}

// The sequence's cache span and block rows, checked; false (and a status
// bit) when they are out of range. The check is uniform over the CTA.
__device__ __forceinline__ bool seq_ok(const BlockSumArgs& a, int seq, int64_t& off, int& len) {
    off = a.kv_offset[seq];
    len = a.seq_lens[seq];
    bool ok = len >= 1 && len <= a.max_len && off >= 0 && off + len <= a.total_tokens;
    if (ok && a.hi_block > 0) {
        const int64_t boff = a.blk_offset[seq];
        const int nblk = (len + a.hi_block - 1) / a.hi_block;
        ok = boff >= 0 && boff + nblk <= a.block_rows;
    }
    if (!ok && threadIdx.x == 0 && blockIdx.x == 0) flag(a.dev_status, LSA_DEV_BAD_LENGTH);
    return ok;
}

// One CTA per block (full build) or per block holding the n_new newest tokens
// (append update).
template <int D_I>
__global__ void __launch_bounds__(kBsThreads) block_sums_kernel(const BlockSumArgs a) {
    pdl_enter();
    __shared__ int s_part[kBsWarps][D_I];
    const int seq = blockIdx.y;
    int64_t off;
    int len;
    if (!seq_ok(a, seq, off, len)) return;
    const int B = a.hi_block;
    const int nblk = (len + B - 1) / B;
    int first = 0;
    if (a.n_new > 0) {
        const int from = len - a.n_new;
        first = from > 0 ? from / B : 0;
    }
    const int j = first + blockIdx.x;
    if (j >= nblk) return;  // uniform over the CTA
    const int t0 = j * B;
    const int n = min(t0 + B, len) - t0;
    const int8_t* base = a.k_idx + (off + t0) * D_I;
    sum_block<D_I>([&](int row) { return base + (int64_t)row * D_I; }, n,
                   a.block_sums + (a.blk_offset[seq] + j) * (2 * D_I), s_part);
}

__device__ __forceinline__ void copy16(uint8_t* dst, const uint8_t* src, int64_t bytes) {
    for (int64_t i = threadIdx.x; i < bytes / 16; i += kBsThreads)
        reinterpret_cast<uint4*>(dst)[i] = ldg16(src + 16 * i);
}

constexpr int kAppendRowsPerCta = 64;  // HI off: new tokens per CTA

// Decode append. CTA (x, b, 0) owns the new tokens of sequence b that fall in
// block first + x (HI on) or the x-th run of kAppendRowsPerCta new tokens
// (HI off) and copies their indexer keys and every layer's K and V rows into
// the caches; with HI on, CTA (x, b, 1) recomputes that block's sum in the
// same launch (one round of loads each). The block sum reads the new rows
// from the inputs and the older rows from the cache, so no CTA reads what it
// (or another CTA) writes in this launch.
template <int D_I>
__global__ void __launch_bounds__(kBsThreads) append_kernel(const AppendArgs p) {
    pdl_enter();
    // a small grid: the next call's first kernel may be resident beside it
    // (it still waits for this grid's completion before reading the caches)
    pdl_trigger();
    __shared__ int s_part[kBsWarps][D_I];
    const BlockSumArgs& a = p.bs;
    const int seq = blockIdx.y;
    int64_t off;
    int len;
    if (!seq_ok(a, seq, off, len)) return;
    const int n_new = a.n_new;
    if (n_new > len) {
        if (threadIdx.x == 0 && blockIdx.x == 0) flag(a.dev_status, LSA_DEV_BAD_LENGTH);
        return;
    }
    const int from = len - n_new;  // first new position
    int lo, hi, t0 = 0, n = 0, j = 0;
    if (p.sums) {
        const int B = a.hi_block;
        j = from / B + blockIdx.x;
        if (j >= (len + B - 1) / B) return;  // uniform over the CTA
        t0 = j * B;
        n = min(t0 + B, len) - t0;
        lo = max(t0, from);
        hi = t0 + n;
    } else {
        lo = from + blockIdx.x * kAppendRowsPerCta;
        hi = min(len, lo + kAppendRowsPerCta);
        if (lo >= hi) return;
    }
    if (blockIdx.z == 0) {
        const int64_t src0 = (int64_t)seq * n_new + (lo - from);  // first input row
        const int nr = hi - lo;
        copy16(reinterpret_cast<uint8_t*>(p.k_idx_cache) + (off + lo) * D_I,
               reinterpret_cast<const uint8_t*>(p.k_idx_new) + src0 * D_I, (int64_t)nr * D_I);
        const int64_t kvb = p.kv_row_bytes;
        for (int g = 0; g < p.layers; ++g) {
            copy16(reinterpret_cast<uint8_t*>(p.k_cache[g]) + (off + lo) * kvb,
                   reinterpret_cast<const uint8_t*>(p.k_new[g]) + src0 * kvb, nr * kvb);
            copy16(reinterpret_cast<uint8_t*>(p.v_cache[g]) + (off + lo) * kvb,
                   reinterpret_cast<const uint8_t*>(p.v_new[g]) + src0 * kvb, nr * kvb);
        }
    } else if (p.sums) {
        const int8_t* cache = a.k_idx + (off + t0) * D_I;
        const int8_t* fresh = p.k_idx_new + (int64_t)seq * n_new * D_I;
        sum_block<D_I, 4>(
            [&](int row) {
                const int pos = t0 + row;
                return pos >= from ? fresh + (int64_t)(pos - from) * D_I : cache + (int64_t)row * D_I;
            },
            n, a.block_sums + (a.blk_offset[seq] + j) * (2 * D_I), s_part);
    }
}

}  // namespace

cudaError_t launch_block_sums(const BlockSumArgs& a, int d_I, cudaStream_t stream) {
    dim3 grid((unsigned)a.blocks_per_seq, (unsigned)a.n_seq);
    switch (d_I) {
        case 32: return launch_pdl(block_sums_kernel<32>, grid, dim3(kBsThreads), 0, stream, 0, a);
        case 64: return launch_pdl(block_sums_kernel<64>, grid, dim3(kBsThreads), 0, stream, 0, a);
        case 128: return launch_pdl(block_sums_kernel<128>, grid, dim3(kBsThreads), 0, stream, 0, a);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_append(const AppendArgs& a, int d_I, cudaStream_t stream) {
    const int n_new = a.bs.n_new;
    unsigned gx;
    if (a.sums) {
        int64_t full = ((int64_t)a.bs.max_len + a.bs.hi_block - 1) / a.bs.hi_block;
        int64_t cover = ((int64_t)n_new + a.bs.hi_block - 1) / a.bs.hi_block + 1;
        gx = (unsigned)(cover < full ? cover : full);
    } else {
        gx = (unsigned)((n_new + kAppendRowsPerCta - 1) / kAppendRowsPerCta);
    }
    dim3 grid(gx, (unsigned)a.bs.n_seq, a.sums ? 2u : 1u);
    switch (d_I) {
        case 32: return launch_pdl(append_kernel<32>, grid, dim3(kBsThreads), 0, stream, 0, a);
        case 64: return launch_pdl(append_kernel<64>, grid, dim3(kBsThreads), 0, stream, 0, a);
        case 128: return launch_pdl(append_kernel<128>, grid, dim3(kBsThreads), 0, stream, 0, a);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace lsa
