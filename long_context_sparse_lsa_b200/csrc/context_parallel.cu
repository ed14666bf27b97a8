// context_parallel.cu — the two per-GPU steps of context-parallel attention
// around lsa_attend_lse: each GPU's part of a row's index set, and the exact
// combination of the GPUs' partial attentions.
//
// With one sequence's cache split by token range over GPUs, the softmax
// attention over a row's selected rows ("LongCat-2.0 (molayo1419.me)",
// section "1M 토큰에서의 Sparse Attention 문제") is a sum over the GPUs'
// ranges: GPU p attends over the entries it holds and returns its normalised
// output o_p and lse_p = ln sum_{j in p} exp(s_j); then
//   o = sum_p exp(lse_p - M) o_p / sum_p exp(lse_p - M),  M = max_p lse_p,
// which is the attention over all the entries up to rounding.
//
// Design: shard_sets_kernel compacts one row per CTA in set order (warp
// ballots and one CTA prefix per 256-entry chunk); combine_kernel takes one
// warp per output row, lanes striding over float4 chunks of d.
#include "common.cuh"
#include "internal.h"

namespace lsa {
namespace {

constexpr int kShThreads = 256;
constexpr int kShWarps = kShThreads / kWarp;

__global__ void __launch_bounds__(kShThreads) shard_sets_kernel(const int32_t* __restrict__ sets, int32_t budget,
                                                                 int32_t lo, int32_t hi, int32_t* __restrict__ local,
                                                                 int32_t* dev_status) {
    __shared__ uint32_t s_warp[kShWarps];
    pdl_enter();
    const int r = blockIdx.x, tid = threadIdx.x, lane = lane_id(), warp = warp_id();
    const int32_t* in = sets + (int64_t)r * budget;
    int32_t* out = local + (int64_t)r * budget;
    uint32_t base = 0;  // entries kept so far (identical in every thread)
    for (int c0 = 0; c0 < budget; c0 += kShThreads) {
        const int i = c0 + tid;
        const int32_t e = i < budget ? in[i] : -1;
        if (e < -1) flag(dev_status, LSA_DEV_BAD_INDEX);
        const bool keep = e >= lo && e < hi;
        const uint32_t bal = __ballot_sync(0xffffffffu, keep);
        if (lane == 0) s_warp[warp] = __popc(bal);
        __syncthreads();
        uint32_t before = 0, total = 0;
#pragma unroll
        for (int w = 0; w < kShWarps; ++w) {
            const uint32_t c = s_warp[w];
            before += w < warp ? c : 0u;
            total += c;
        }
        if (keep) out[base + before + __popc(bal & ((1u << lane) - 1u))] = e - lo;
        base += total;
        __syncthreads();  // s_warp is rewritten by the next chunk
    }
    pdl_trigger();
    for (int i = (int)base + tid; i < budget; i += kShThreads) out[i] = -1;
}

constexpr int kCbThreads = 256;
constexpr int kCbRowsPerCta = kCbThreads / kWarp;

__global__ void __launch_bounds__(kCbThreads) combine_kernel(const float* __restrict__ o_parts,
                                                              const float* __restrict__ lse_parts, int32_t n_parts,
                                                              int64_t rows, int32_t d, float* __restrict__ out,
                                                              float* __restrict__ lse_out) {
    pdl_enter();
    const int64_t row = (int64_t)blockIdx.x * kCbRowsPerCta + warp_id();
    if (row >= rows) return;
    const int lane = lane_id();
    // the parts' maximum lse, lanes striding over the parts
    float M = -INFINITY;
    for (int p = lane; p < n_parts; p += kWarp) M = fmaxf(M, lse_parts[(int64_t)p * rows + row]);
#pragma unroll
    for (int s = 16; s > 0; s >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, s));
    const int nc = d / 4;
    float* orow = out + row * d;
    if (M == -INFINITY) {  // every part is empty
        for (int c = lane; c < nc; c += kWarp) reinterpret_cast<float4*>(orow)[c] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (lane == 0 && lse_out != nullptr) lse_out[row] = -INFINITY;
        return;
    }
    float den = 0.f;
    for (int p = 0; p < n_parts; ++p) {
        const float lp = lse_parts[(int64_t)p * rows + row];
        den += lp == -INFINITY ? 0.f : expf(lp - M);
    }
    const float inv = 1.f / den;  // den >= 1: the part holding M contributes exp(0)
    for (int c = lane; c < nc; c += kWarp) {
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int p = 0; p < n_parts; ++p) {
            const float lp = lse_parts[(int64_t)p * rows + row];
            if (lp == -INFINITY) continue;
            const float wgt = expf(lp - M);
            const float4 v = reinterpret_cast<const float4*>(o_parts + ((int64_t)p * rows + row) * d)[c];
            acc.x += wgt * v.x;
            acc.y += wgt * v.y;
            acc.z += wgt * v.z;
            acc.w += wgt * v.w;
        }
        reinterpret_cast<float4*>(orow)[c] = make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
    }
    if (lane == 0 && lse_out != nullptr) lse_out[row] = M + logf(den);
}

}  // namespace

cudaError_t launch_shard_sets(const int32_t* sets, int n_q, int budget, int lo, int hi, int32_t* local,
                              int32_t* dev_status, cudaStream_t stream) {
    return launch_pdl(shard_sets_kernel, dim3((unsigned)n_q), dim3(kShThreads), 0, stream, 0, sets, (int32_t)budget,
                      (int32_t)lo, (int32_t)hi, local, dev_status);
}

cudaError_t launch_combine(const float* o_parts, const float* lse_parts, int n_parts, int64_t rows, int d, float* out,
                           float* lse_out, cudaStream_t stream) {
    const int64_t ctas = (rows + kCbRowsPerCta - 1) / kCbRowsPerCta;
    return launch_pdl(combine_kernel, dim3((unsigned)ctas), dim3(kCbThreads), 0, stream, 0, o_parts, lse_parts,
                      (int32_t)n_parts, rows, (int32_t)d, out, lse_out);
}

}  // namespace lsa
