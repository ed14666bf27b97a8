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
#include "append.cuh"
#include "common.cuh"
#include "internal.h"

namespace lsa {
namespace {

constexpr int kBsThreads = 256;
constexpr int kBsWarps = kBsThreads / kWarp;

// Keeping four rows in flight per thread in the full build was measured and
// dropped: 63 registers instead of 48 cost resident CTAs, and the build got
// slower; the decode append, one block per CTA and latency-bound, issues a
// whole block's loads in one round (sum_block<.., 4, ..>).

// One CTA per block (full build) or per block holding the n_new newest tokens
// (append update).
template <int D_I>
__global__ void __launch_bounds__(kBsThreads) block_sums_kernel(const BlockSumArgs a) {
    pdl_enter();
    __shared__ int s_part[kBsWarps * D_I];
    const int seq = blockIdx.y;
    int64_t off;
    int len;
    if (!seq_ok(a, seq, off, len, blockIdx.x == 0)) return;
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
    sum_block<D_I, 1, kBsThreads>([&](int row) { return base + (int64_t)row * D_I; }, n,
                                  a.block_sums + (a.blk_offset[seq] + j) * (2 * D_I), s_part);
}

// Decode append, one task per CTA (append_task): CTA (x, b, role).
template <int D_I>
__global__ void __launch_bounds__(kBsThreads) append_kernel(const AppendArgs p) {
    pdl_enter();
    // a small grid: the next call's first kernel may be resident beside it
    // (it still waits for this grid's completion before reading the caches)
    pdl_trigger();
    __shared__ int s_part[kBsWarps * D_I];
    append_task<D_I, kBsThreads>(p, blockIdx.x, blockIdx.y, blockIdx.z, s_part);
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
    const unsigned gx = (unsigned)append_ctas_per_seq(a.bs.n_new, a.sums ? a.bs.hi_block : 0, a.bs.max_len);
    dim3 grid(gx, (unsigned)a.bs.n_seq, a.sums ? 2u : 1u);
    switch (d_I) {
        case 32: return launch_pdl(append_kernel<32>, grid, dim3(kBsThreads), 0, stream, 0, a);
        case 64: return launch_pdl(append_kernel<64>, grid, dim3(kBsThreads), 0, stream, 0, a);
        case 128: return launch_pdl(append_kernel<128>, grid, dim3(kBsThreads), 0, stream, 0, a);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace lsa
