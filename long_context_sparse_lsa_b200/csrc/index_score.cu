// index_score.cu — the streaming half of the LSA indexer: HI coarse scores of
// candidate blocks and fine scores of candidate tokens.
//
// The method ("LongCat-2.0 (molayo1419.me)", section "1M 토큰에서의 Sparse
// Attention 문제"; "LongCat-Flash-Lite-Sparse (aitrends.kr)", section
// "기술적 특징"): a DSA-style indexer scores cached tokens; HI first scores
// whole blocks on their key sums and scores fine tokens only inside the kept
// blocks.
//
// Design (B200): both kernels are bandwidth kernels. Each CTA scores one
// chunk of one query's candidates (128 blocks, or 256 token slots) with plain
// 16-byte vector loads straight into MMA fragments; small CTAs and modest
// register use keep several CTAs — and thus many loads in flight — on every
// SM. Scores are written as keys (score + 1; 0 = not a candidate) to an
// L2-resident workspace for the selection kernels.
#include "index_common.cuh"

namespace lsa {
namespace {

constexpr int kScThreads = 256;
constexpr int kScWarps = kScThreads / kWarp;
constexpr int kCoarseChunk = kScWarps * 16;     // 128 blocks per CTA

// Validates query row r; on success sets the row's cache offset and visible
// length. Uniform over a CTA; flags nothing (the selection kernel reports).
__device__ __forceinline__ bool row_ok(const IndexArgs& a, int r, int64_t& off, int& L) {
    const int seq = a.q_seq[r];
    L = a.q_len[r];
    if (seq < 0 || seq >= a.n_seq) return false;
    off = a.kv_offset[seq];
    const int slen = a.seq_lens[seq];
    if (L < 1 || L > a.max_len || L > slen || off < 0 || off + slen > a.total_tokens) return false;
    if (a.hi_block > 0) {
        const int64_t bo = a.blk_offset[seq];
        if (bo < 0 || bo + (L + a.hi_block - 1) / a.hi_block > a.block_rows) return false;
    }
    return true;
}

template <int D_I, int NT>
__global__ void __launch_bounds__(kScThreads) coarse_score_kernel(const __grid_constant__ IndexArgs a) {
    pdl_enter();
    const int r = blockIdx.y;
    int64_t off;
    int L;
    if (!row_ok(a, r, off, L)) return;
    const int s = min(a.sink, L);
    const int ws = max(s, L - a.window);
    if (ws <= s) return;
    const int B = a.hi_block;
    const int b_lo = s / B, b_hi = (ws + B - 1) / B;
    const int c0 = b_lo + blockIdx.x * kCoarseChunk;
    if (c0 >= b_hi) return;
    const int lane = lane_id(), warp = warp_id(), g = lane >> 2, t4 = lane & 3;
    const int j0 = c0 + warp * 16 + g, j1 = j0 + 8;  // block indices of rows g and g+8
    if (c0 + warp * 16 >= b_hi) return;                // warp-uniform
    const bool v0 = j0 < b_hi, v1 = j1 < b_hi;
    const int8_t* rows = a.block_sums + a.blk_offset[a.q_seq[r]] * (2 * D_I);
    RowFrag<D_I> hg, lg, hg8, lg8;
    hg.load(rows + (int64_t)j0 * (2 * D_I), t4, v0);
    lg.load(rows + (int64_t)j0 * (2 * D_I) + D_I, t4, v0);
    hg8.load(rows + (int64_t)j1 * (2 * D_I), t4, v1);
    lg8.load(rows + (int64_t)j1 * (2 * D_I) + D_I, t4, v1);
    QueryFrag<D_I, NT> qf;
    load_query<D_I, NT>(qf, a, r);
    long long x, y;
    coarse_tile<D_I, NT>(qf, hg, lg, hg8, lg8, x, y);
    uint64_t* keys = a.coarse_keys + (int64_t)r * a.coarse_cap;
    if (t4 == 0 && v0) keys[j0 - b_lo] = (unsigned long long)x + 1ull;
    if (t4 == 1 && v1) keys[j1 - b_lo] = (unsigned long long)y + 1ull;
}

// Fine scores: a persistent grid of kFineCtasPerSm CTAs per SM. With n_q <=
// warps, each row gets warps / n_q warps and each warp streams a contiguous
// range of the row's 16-slot tiles; with more rows, warps take whole rows in
// turn. Per warp the tile loop is software-pipelined: the key rows of tile
// j+1 (and the kept-block ids of tile j+2) are in flight while tile j is
// scored, so the dependent chain (row metadata, kept ids, key rows) is paid
// once per warp range rather than once per CTA.
constexpr int kFineCtasPerSm = 2;

template <int D_I>
struct FineTile {
    RowFrag<D_I> ra, rb;  // key rows of slots 16j + g and 16j + g + 8
    bool va, vb;          // slot holds a candidate token
};

template <int D_I, int NT>
__global__ void __launch_bounds__(kScThreads, kFineCtasPerSm) fine_score_kernel(const __grid_constant__ IndexArgs a) {
    pdl_enter();
    const int lane = lane_id(), g = lane >> 2, t4 = lane & 3;
    const int W = gridDim.x * kScWarps;
    const int gw = blockIdx.x * kScWarps + warp_id();
    const bool few_rows = a.n_q <= W;
    const int wpr = few_rows ? W / a.n_q : 1;  // warps per row
    const int seg = few_rows ? gw % wpr : 0;
    const int r0 = few_rows ? gw / wpr : gw;
    const int rstep = few_rows ? a.n_q : W;
    const bool hi = a.hi_block > 0;
    const int B = a.hi_block;
    const int lgB = (hi && (B & (B - 1)) == 0) ? __ffs(B) - 1 : -1;  // power-of-two block: shift, not divide
    for (int r = r0; r < a.n_q; r += rstep) {  // warp-uniform
        int64_t off;
        int L;
        if (!row_ok(a, r, off, L)) continue;
        const int s = min(a.sink, L);
        const int ws = max(s, L - a.window);
        const int n_slots = hi ? a.n_kept[r] * B : ws - s;
        const int nt = (n_slots + 15) / 16;
        const int j_lo = (int)((int64_t)nt * seg / wpr), j_hi = (int)((int64_t)nt * (seg + 1) / wpr);
        if (j_lo >= j_hi) continue;
        const int8_t* kseq = a.k_idx + off * D_I;
        const int32_t* kept = a.kept + (int64_t)r * a.hi_topblocks;
        uint32_t* keys = a.fine_keys + (int64_t)r * a.fine_cap;
        // kept-block ids of this lane's two slots of tile j (HI), or unused
        auto kept_ids = [&](int j, int& ka, int& kb) {
            ka = kb = 0;
            if (!hi) return;
            const int sa = 16 * j + g, sb = sa + 8;
            if (sa < n_slots) ka = __ldg(kept + (lgB >= 0 ? sa >> lgB : sa / B));
            if (sb < n_slots) kb = __ldg(kept + (lgB >= 0 ? sb >> lgB : sb / B));
        };
        auto token_of = [&](int slot, int kid, bool& valid) -> int {
            if (slot >= n_slots) {
                valid = false;
                return 0;
            }
            if (!hi) {
                valid = true;
                return s + slot;
            }
            const int kb = lgB >= 0 ? slot >> lgB : slot / B;
            const int tok = kid * B + (slot - kb * B);
            valid = tok >= s && tok < ws;
            return tok;
        };
        auto issue = [&](FineTile<D_I>& t, int j, int ka, int kb) {
            const int sa = 16 * j + g;
            const int ta = token_of(sa, ka, t.va);
            const int tb = token_of(sa + 8, kb, t.vb);
            t.ra.load(kseq + (int64_t)ta * D_I, t4, t.va);
            t.rb.load(kseq + (int64_t)tb * D_I, t4, t.vb);
        };
        QueryFrag<D_I, NT> qf;
        load_query<D_I, NT>(qf, a, r);
        auto score = [&](const FineTile<D_I>& t, int j) {
            const int2 sc = fine_tile<D_I, NT>(qf, t.ra, t.rb);
            const int sa = 16 * j + g, sb = sa + 8;
            if (t4 == 0 && sa < n_slots) keys[sa] = t.va ? (uint32_t)sc.x + 1u : 0u;
            if (t4 == 1 && sb < n_slots) keys[sb] = t.vb ? (uint32_t)sc.y + 1u : 0u;
        };
        FineTile<D_I> t0, t1;
        int ka0, kb0, ka1 = 0, kb1 = 0;
        kept_ids(j_lo, ka0, kb0);
        issue(t0, j_lo, ka0, kb0);
        if (j_lo + 1 < j_hi) kept_ids(j_lo + 1, ka1, kb1);
        for (int j = j_lo; j < j_hi; j += 2) {
            // tile j is in t0; the kept ids of tile j+1 are in (ka1, kb1)
            if (j + 1 < j_hi) issue(t1, j + 1, ka1, kb1);
            if (j + 2 < j_hi) kept_ids(j + 2, ka0, kb0);
            score(t0, j);
            if (j + 1 >= j_hi) break;
            if (j + 2 < j_hi) issue(t0, j + 2, ka0, kb0);
            if (j + 3 < j_hi) kept_ids(j + 3, ka1, kb1);
            score(t1, j + 1);
        }
    }
}

template <int D_I, int NT>
cudaError_t launch_scores_t(const IndexArgs& a, bool coarse, cudaStream_t st) {
    if (coarse) {
        dim3 grid((unsigned)((a.coarse_cap + kCoarseChunk - 1) / kCoarseChunk), (unsigned)a.n_q);
        return launch_pdl(coarse_score_kernel<D_I, NT>, grid, dim3(kScThreads), 0, st, 0, a);
    } else {
        dim3 grid((unsigned)(kFineCtasPerSm * device_sm_count()));
        return launch_pdl(fine_score_kernel<D_I, NT>, grid, dim3(kScThreads), 0, st, 0, a);
    }
}

template <int D_I>
cudaError_t launch_scores_d(const IndexArgs& a, bool coarse, cudaStream_t st) {
    const int nt = (a.H_I + 7) / 8;
    if (nt <= 1) return launch_scores_t<D_I, 1>(a, coarse, st);
    if (nt <= 2) return launch_scores_t<D_I, 2>(a, coarse, st);
    if (nt <= 4) return launch_scores_t<D_I, 4>(a, coarse, st);
    return launch_scores_t<D_I, 8>(a, coarse, st);
}

}  // namespace

cudaError_t launch_index_scores(const IndexArgs& a, int d_I, bool coarse, cudaStream_t stream) {
    switch (d_I) {
        case 32: return launch_scores_d<32>(a, coarse, stream);
        case 64: return launch_scores_d<64>(a, coarse, stream);
        case 128: return launch_scores_d<128>(a, coarse, stream);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace lsa
