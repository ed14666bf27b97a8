// block_sums.cu — HI block-sum pre-pass.
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

// One CTA per block: thread t owns 16-byte chunk (t % CPR) of rows t / CPR,
// t / CPR + RPP, ... so the whole block is read in B / RPP dependent rounds
// of coalesced 16-byte loads (one round for hi_block <= 32 at d_I = 128).
template <int D_I>
__global__ void __launch_bounds__(kBsThreads) block_sums_kernel(const BlockSumArgs a) {
    pdl_enter();
    constexpr int kCPR = D_I / 16;           // 16-byte chunks per row
    constexpr int kRPP = kBsThreads / kCPR;  // rows per pass
    __shared__ int s_part[kBsWarps][D_I];
    const int seq = blockIdx.y;
    const int tid = threadIdx.x, lane = lane_id(), warp = warp_id();
    const int64_t off = a.kv_offset[seq];
    const int32_t len = a.seq_lens[seq];
    if (len < 1 || len > a.max_len || off < 0 || off + len > a.total_tokens) {
        if (tid == 0 && blockIdx.x == 0) flag(a.dev_status, LSA_DEV_BAD_LENGTH);
        return;
    }
    const int B = a.hi_block;
    const int nblk = (len + B - 1) / B;
    const int64_t boff = a.blk_offset[seq];
    if (boff < 0 || boff + nblk > a.block_rows) {
        if (tid == 0 && blockIdx.x == 0) flag(a.dev_status, LSA_DEV_BAD_LENGTH);
        return;
    }
    int first = 0;
    if (a.n_new > 0) {
        const int from = len - a.n_new;
        first = from > 0 ? from / B : 0;
    }
    const int j = first + blockIdx.x;
    if (j >= nblk) return;  // uniform over the CTA
    const int t0 = j * B;
    const int n = min(t0 + B, len) - t0;
    const int c = tid % kCPR;
    int acc[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) acc[i] = 0;
    const int8_t* base = a.k_idx + (off + t0) * D_I + c * 16;
    for (int row = tid / kCPR; row < n; row += kRPP) {
        const uint4 v = ldg16(base + (int64_t)row * D_I);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int q = 0; q < 4; ++q)
#pragma unroll
            for (int b = 0; b < 4; ++b) acc[4 * q + b] += sbyte(w[q], b);
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
        int8_t* row = a.block_sums + (boff + j) * (2 * D_I);
        row[tid] = static_cast<int8_t>(S >> 8);
        reinterpret_cast<uint8_t*>(row)[D_I + tid] = static_cast<uint8_t>(S & 0xFF);
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

}  // namespace lsa
