// index_points.cu — indexer scores of given token positions and of given HI
// blocks, for callers that choose the candidates themselves (the ranks of a
// context-parallel index, each holding one token range of a sequence).
//
// The scores are the indexer's: score_t = sum_h w_h * max(0, q_h . k_t) over
// the int8 keys, and the HI coarse score, the same formula on a block's key
// sum ("LongCat-2.0 (molayo1419.me)", section "1M 토큰에서의 Sparse Attention
// 문제"; "LongCat-Flash-Lite-Sparse (aitrends.kr)", section "기술적 특징", HI
// bullet). Keys are written as score + 1 (0 for an empty slot), the layout
// lsa_merge_pairs takes after packing.
//
// Design: one warp scores 16 slots with the exact int8 tensor-core tiles of
// the indexer (fine_tile / coarse_tile); 8 warps per CTA, grid (slot chunks,
// query rows).
#include "index_common.cuh"

namespace lsa {
namespace {

constexpr int kPtThreads = 256;
constexpr int kPtWarps = kPtThreads / kWarp;
constexpr int kPtChunk = kPtWarps * 16;

template <int D_I, int NT>
__global__ void __launch_bounds__(kPtThreads) point_scores_kernel(const __grid_constant__ PointArgs p) {
    pdl_enter();
    const int r = blockIdx.y;
    const int lane = lane_id(), warp = warp_id(), g = lane >> 2, t4 = lane & 3;
    const int j0 = blockIdx.x * kPtChunk + warp * 16;
    if (j0 >= p.n) return;  // warp-uniform
    const int ja = j0 + g, jb = ja + 8;
    const int32_t* ids = p.ids + (int64_t)r * p.n;
    const int ia = ja < p.n ? ids[ja] : -1, ib = jb < p.n ? ids[jb] : -1;
    // ids are token positions (blocks == 0) or block indices, relative to the
    // row's first cache row / block row; out of range reads as empty
    const int64_t base = p.row_base[r];
    const int64_t lim = p.rows;
    const bool va = ia >= 0 && base + ia < lim, vb = ib >= 0 && base + ib < lim;
    if ((ia >= 0 && !va) || (ib >= 0 && !vb)) flag(p.a.dev_status, LSA_DEV_BAD_INDEX);
    QueryFrag<D_I, NT> qf;
    load_query<D_I, NT>(qf, p.a, r);
    if (p.blocks) {
        const int8_t* rows = p.a.block_sums;
        RowFrag<D_I> hg, lg, hg8, lg8;
        const int64_t ra = va ? base + ia : 0, rb = vb ? base + ib : 0;
        hg.load(rows + ra * (2 * D_I), t4, va);
        lg.load(rows + ra * (2 * D_I) + D_I, t4, va);
        hg8.load(rows + rb * (2 * D_I), t4, vb);
        lg8.load(rows + rb * (2 * D_I) + D_I, t4, vb);
        long long x, y;
        coarse_tile<D_I, NT>(qf, hg, lg, hg8, lg8, x, y);
        uint64_t* out = p.out_blocks + (int64_t)r * p.n;
        if (t4 == 0 && ja < p.n) out[ja] = va ? (unsigned long long)x + 1ull : 0ull;
        if (t4 == 1 && jb < p.n) out[jb] = vb ? (unsigned long long)y + 1ull : 0ull;
    } else {
        RowFrag<D_I> fa, fb;
        fa.load(p.a.k_idx + (va ? base + ia : 0) * D_I, t4, va);
        fb.load(p.a.k_idx + (vb ? base + ib : 0) * D_I, t4, vb);
        const int2 sc = fine_tile<D_I, NT>(qf, fa, fb);
        uint32_t* out = p.out_tokens + (int64_t)r * p.n;
        if (t4 == 0 && ja < p.n) out[ja] = va ? (uint32_t)sc.x + 1u : 0u;
        if (t4 == 1 && jb < p.n) out[jb] = vb ? (uint32_t)sc.y + 1u : 0u;
    }
}

template <int D_I>
cudaError_t launch_points_d(const PointArgs& p, cudaStream_t st) {
    const dim3 grid((unsigned)((p.n + kPtChunk - 1) / kPtChunk), (unsigned)p.a.n_q);
    const int nt = (p.a.H_I + 7) / 8;
    if (nt <= 1) return launch_pdl(point_scores_kernel<D_I, 1>, grid, dim3(kPtThreads), 0, st, 0, p);
    if (nt <= 2) return launch_pdl(point_scores_kernel<D_I, 2>, grid, dim3(kPtThreads), 0, st, 0, p);
    if (nt <= 4) return launch_pdl(point_scores_kernel<D_I, 4>, grid, dim3(kPtThreads), 0, st, 0, p);
    return launch_pdl(point_scores_kernel<D_I, 8>, grid, dim3(kPtThreads), 0, st, 0, p);
}

}  // namespace

cudaError_t launch_point_scores(const PointArgs& p, int d_I, cudaStream_t stream) {
    switch (d_I) {
        case 32: return launch_points_d<32>(p, stream);
        case 64: return launch_points_d<64>(p, stream);
        case 128: return launch_points_d<128>(p, stream);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace lsa
