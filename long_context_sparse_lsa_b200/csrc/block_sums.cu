// block_sums.cu — HI block-sum pre-pass.
//
// Hierarchical Indexing first scores whole blocks ("LongCat-Flash-Lite-Sparse
// (aitrends.kr)", section "기술적 특징", HI bullet). The block score uses the
// exact sum of the block's indexer keys, S_b[d] = sum_t k_t[d], over the
// present tokens of the block (blocks aligned at position 0).
//
// One warp reduces one block: D_I/4 lanes cover one key row with 4-byte
// loads, so a warp reads 32*4 = 128 contiguous bytes per step; partial sums of
// the row groups are folded with shuffles. The sum is stored as two byte
// planes (S >> 8 as int8, S & 0xFF as uint8) so that the coarse pass can feed
// it straight to the 8-bit tensor-core MMA.
#include "common.cuh"
#include "internal.h"

namespace lsa {
namespace {

constexpr int kBsThreads = 256;
constexpr int kBsWarps = kBsThreads / kWarp;

__device__ __forceinline__ int sbyte(uint32_t w, int i) { return static_cast<int>(static_cast<int8_t>(w >> (8 * i))); }

template <int D_I>
__global__ void __launch_bounds__(kBsThreads) block_sums_kernel(const BlockSumArgs a) {
    constexpr int kLanesPerRow = D_I / 4;       // 8, 16 or 32
    constexpr int kRowsPerStep = kWarp / kLanesPerRow;
    const int seq = blockIdx.y;
    const int lane = lane_id();
    const int64_t off = a.kv_offset[seq];
    const int32_t len = a.seq_lens[seq];
    if (len < 1 || len > a.max_len || off < 0 || off + len > a.total_tokens) {
        if (threadIdx.x == 0 && blockIdx.x == 0) flag(a.dev_status, LSA_DEV_BAD_LENGTH);
        return;
    }
    const int B = a.hi_block;
    const int nblk = (len + B - 1) / B;
    const int64_t boff = a.blk_offset[seq];
    if (boff < 0 || boff + nblk > a.block_rows) {
        if (threadIdx.x == 0 && blockIdx.x == 0) flag(a.dev_status, LSA_DEV_BAD_LENGTH);
        return;
    }
    int first = 0;
    if (a.n_new > 0) {
        int from = len - a.n_new;
        first = from > 0 ? from / B : 0;
    }
    const int j = first + blockIdx.x * kBsWarps + warp_id();
    if (j >= nblk) return;
    const int t0 = j * B;
    const int t1 = min(t0 + B, len);
    const int sub = lane / kLanesPerRow;        // row within a step
    const int col = (lane % kLanesPerRow) * 4;  // first dim of this lane
    int acc0 = 0, acc1 = 0, acc2 = 0, acc3 = 0;
    const int8_t* base = a.k_idx + (off + t0) * D_I + col;
    int t = sub;
    const int n = t1 - t0;
    // four rows in flight per lane
    for (; t + 3 * kRowsPerStep < n; t += 4 * kRowsPerStep) {
        uint32_t w0 = __ldg(reinterpret_cast<const uint32_t*>(base + (int64_t)t * D_I));
        uint32_t w1 = __ldg(reinterpret_cast<const uint32_t*>(base + (int64_t)(t + kRowsPerStep) * D_I));
        uint32_t w2 = __ldg(reinterpret_cast<const uint32_t*>(base + (int64_t)(t + 2 * kRowsPerStep) * D_I));
        uint32_t w3 = __ldg(reinterpret_cast<const uint32_t*>(base + (int64_t)(t + 3 * kRowsPerStep) * D_I));
        acc0 += sbyte(w0, 0) + sbyte(w1, 0) + sbyte(w2, 0) + sbyte(w3, 0);
        acc1 += sbyte(w0, 1) + sbyte(w1, 1) + sbyte(w2, 1) + sbyte(w3, 1);
        acc2 += sbyte(w0, 2) + sbyte(w1, 2) + sbyte(w2, 2) + sbyte(w3, 2);
        acc3 += sbyte(w0, 3) + sbyte(w1, 3) + sbyte(w2, 3) + sbyte(w3, 3);
    }
    for (; t < n; t += kRowsPerStep) {
        uint32_t w0 = __ldg(reinterpret_cast<const uint32_t*>(base + (int64_t)t * D_I));
        acc0 += sbyte(w0, 0);
        acc1 += sbyte(w0, 1);
        acc2 += sbyte(w0, 2);
        acc3 += sbyte(w0, 3);
    }
#pragma unroll
    for (int m = kLanesPerRow; m < kWarp; m <<= 1) {
        acc0 += __shfl_xor_sync(0xffffffffu, acc0, m);
        acc1 += __shfl_xor_sync(0xffffffffu, acc1, m);
        acc2 += __shfl_xor_sync(0xffffffffu, acc2, m);
        acc3 += __shfl_xor_sync(0xffffffffu, acc3, m);
    }
    if (sub == 0) {
        // S = 256 * hi + lo with hi = S >> 8 (arithmetic), lo = S & 0xFF.
        uint32_t hi = (uint32_t)((acc0 >> 8) & 0xFF) | ((uint32_t)((acc1 >> 8) & 0xFF) << 8) |
                      ((uint32_t)((acc2 >> 8) & 0xFF) << 16) | ((uint32_t)((acc3 >> 8) & 0xFF) << 24);
        uint32_t lo = (uint32_t)(acc0 & 0xFF) | ((uint32_t)(acc1 & 0xFF) << 8) | ((uint32_t)(acc2 & 0xFF) << 16) |
                      ((uint32_t)(acc3 & 0xFF) << 24);
        int8_t* row = a.block_sums + (boff + j) * (2 * D_I);
        *reinterpret_cast<uint32_t*>(row + col) = hi;
        *reinterpret_cast<uint32_t*>(row + D_I + col) = lo;
    }
}

}  // namespace

cudaError_t launch_block_sums(const BlockSumArgs& a, int d_I, cudaStream_t stream) {
    dim3 grid((a.blocks_per_seq + kBsWarps - 1) / kBsWarps, a.n_seq);
    switch (d_I) {
        case 32: block_sums_kernel<32><<<grid, kBsThreads, 0, stream>>>(a); break;
        case 64: block_sums_kernel<64><<<grid, kBsThreads, 0, stream>>>(a); break;
        case 128: block_sums_kernel<128><<<grid, kBsThreads, 0, stream>>>(a); break;
        default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

}  // namespace lsa
