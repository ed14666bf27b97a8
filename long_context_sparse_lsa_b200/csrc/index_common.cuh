// index_common.cuh — register fragments and scoring tiles shared by the
// indexer kernels (coarse and fine scoring).
//
// Scores are exact int8 dot products on the tensor cores (mma.m16n8k32.s8):
// 16 key rows form the A tile, the query's indexer heads (padded to multiples
// of 8) the B tile. Because a dot product is a sum, each lane may own any
// consistent subset of the dims: lane t owns 16-byte chunks t and 4+t of a
// 128-byte row and the query fragment uses the same permutation, so one warp
// load reads 8 rows x 64 contiguous bytes.
#pragma once

#include "common.cuh"
#include "internal.h"

namespace lsa {

// ----------------------------------------------------------------------------
// Row fragments: the bytes of a D_I-byte row that lane t (= lane % 4) owns.
// ----------------------------------------------------------------------------
template <int D_I>
struct RowFrag {
    static constexpr int kWords = D_I / 16;  // 32-bit words per lane
    uint32_t w[kWords];

    __device__ __forceinline__ void load(const int8_t* row, int t, bool valid) {
        if constexpr (D_I == 128) {
            uint4 x = make_uint4(0, 0, 0, 0), y = make_uint4(0, 0, 0, 0);
            if (valid) {
                x = ldg16(row + 16 * t);
                y = ldg16(row + 64 + 16 * t);
            }
            w[0] = x.x; w[1] = x.y; w[2] = x.z; w[3] = x.w;
            w[4] = y.x; w[5] = y.y; w[6] = y.z; w[7] = y.w;
        } else if constexpr (D_I == 64) {
            uint4 x = make_uint4(0, 0, 0, 0);
            if (valid) x = ldg16(row + 16 * t);
            w[0] = x.x; w[1] = x.y; w[2] = x.z; w[3] = x.w;
        } else {
            uint2 x = make_uint2(0, 0);
            if (valid) x = ldg8(row + 8 * t);
            w[0] = x.x; w[1] = x.y;
        }
    }
};

// The query's indexer heads as MMA B fragments, plus the per-lane weights.
template <int D_I, int NT>
struct QueryFrag {
    uint32_t b[NT][D_I / 32][2];
    int32_t wlo[NT], whi[NT];  // weights of heads 8n + 2t and 8n + 2t + 1
};

template <int D_I, int NT>
__device__ __forceinline__ void load_query(QueryFrag<D_I, NT>& qf, const IndexArgs& a, int r) {
    const int lane = lane_id(), g = lane >> 2, t = lane & 3;
    bool bad_w = false;
#pragma unroll
    for (int n = 0; n < NT; ++n) {
        const int head = 8 * n + g;
        RowFrag<D_I> f;
        f.load(a.q_idx + ((int64_t)r * a.H_I + head) * D_I, t, head < a.H_I);
#pragma unroll
        for (int s = 0; s < D_I / 32; ++s) {
            qf.b[n][s][0] = f.w[2 * s];
            qf.b[n][s][1] = f.w[2 * s + 1];
        }
        const int h0 = 8 * n + 2 * t, h1 = h0 + 1;
        int32_t w0 = h0 < a.H_I ? a.w[(int64_t)r * a.H_I + h0] : 0;
        int32_t w1 = h1 < a.H_I ? a.w[(int64_t)r * a.H_I + h1] : 0;
        if (w0 < 0 || w0 > a.w_max) { bad_w = true; w0 = 0; }
        if (w1 < 0 || w1 > a.w_max) { bad_w = true; w1 = 0; }
        qf.wlo[n] = w0;
        qf.whi[n] = w1;
    }
    if (bad_w) flag(a.dev_status, LSA_DEV_BAD_WEIGHT);
}

// Fine scores of 16 key rows (rows g and g+8 of this lane). Returns the
// weighted-ReLU sums for rows g (x) and g + 8 (y), reduced over the 4 lanes of
// the row group.
template <int D_I, int NT>
__device__ __forceinline__ int2 fine_tile(const QueryFrag<D_I, NT>& qf, const RowFrag<D_I>& rg,
                                          const RowFrag<D_I>& rg8) {
    int32_t acc[NT][4];
#pragma unroll
    for (int n = 0; n < NT; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0;
#pragma unroll
    for (int s = 0; s < D_I / 32; ++s) {
        const uint32_t a[4] = {rg.w[2 * s], rg8.w[2 * s], rg.w[2 * s + 1], rg8.w[2 * s + 1]};
#pragma unroll
        for (int n = 0; n < NT; ++n) mma_s8s8(acc[n], a, qf.b[n][s][0], qf.b[n][s][1]);
    }
    int32_t x = 0, y = 0;
#pragma unroll
    for (int n = 0; n < NT; ++n) {
        x += qf.wlo[n] * max(acc[n][0], 0) + qf.whi[n] * max(acc[n][1], 0);
        y += qf.wlo[n] * max(acc[n][2], 0) + qf.whi[n] * max(acc[n][3], 0);
    }
    x += __shfl_xor_sync(0xffffffffu, x, 1);
    y += __shfl_xor_sync(0xffffffffu, y, 1);
    x += __shfl_xor_sync(0xffffffffu, x, 2);
    y += __shfl_xor_sync(0xffffffffu, y, 2);
    return make_int2(x, y);
}

// Coarse scores of 16 block-sum rows (two byte planes each).
template <int D_I, int NT>
__device__ __forceinline__ void coarse_tile(const QueryFrag<D_I, NT>& qf, const RowFrag<D_I>& hg,
                                            const RowFrag<D_I>& lg, const RowFrag<D_I>& hg8,
                                            const RowFrag<D_I>& lg8, long long& x, long long& y) {
    int32_t ah[NT][4], al[NT][4];
#pragma unroll
    for (int n = 0; n < NT; ++n) {
        ah[n][0] = ah[n][1] = ah[n][2] = ah[n][3] = 0;
        al[n][0] = al[n][1] = al[n][2] = al[n][3] = 0;
    }
#pragma unroll
    for (int s = 0; s < D_I / 32; ++s) {
        const uint32_t a_hi[4] = {hg.w[2 * s], hg8.w[2 * s], hg.w[2 * s + 1], hg8.w[2 * s + 1]};
        const uint32_t a_lo[4] = {lg.w[2 * s], lg8.w[2 * s], lg.w[2 * s + 1], lg8.w[2 * s + 1]};
#pragma unroll
        for (int n = 0; n < NT; ++n) {
            mma_s8s8(ah[n], a_hi, qf.b[n][s][0], qf.b[n][s][1]);
            mma_u8s8(al[n], a_lo, qf.b[n][s][0], qf.b[n][s][1]);
        }
    }
    x = 0;
    y = 0;
#pragma unroll
    for (int n = 0; n < NT; ++n) {
        const int32_t d0 = ah[n][0] * 256 + al[n][0], d1 = ah[n][1] * 256 + al[n][1];
        const int32_t d2 = ah[n][2] * 256 + al[n][2], d3 = ah[n][3] * 256 + al[n][3];
        x += (long long)qf.wlo[n] * max(d0, 0) + (long long)qf.whi[n] * max(d1, 0);
        y += (long long)qf.wlo[n] * max(d2, 0) + (long long)qf.whi[n] * max(d3, 0);
    }
    x += __shfl_xor_sync(0xffffffffu, x, 1);
    y += __shfl_xor_sync(0xffffffffu, y, 1);
    x += __shfl_xor_sync(0xffffffffu, x, 2);
    y += __shfl_xor_sync(0xffffffffu, y, 2);
}

// HI blocks are summed over the tokens a row can see ([b*B, min((b+1)*B, L))).
// The block-sum cache holds one sum per block over every cached token, so for
// a row that sees fewer tokens than its sequence holds (L < seq_lens: a
// prefill chunk, draft rows) the block holding its last visible token L-1 may
// also count tokens the row cannot see. partial_block_fix() tells whether
// that block is a candidate of the row and needs its sum recomputed;
// partial_block_score() recomputes its coarse score from the keys.
__device__ __forceinline__ bool partial_block_fix(int L, int slen, int B, int ws, int& b_p) {
    b_p = (L - 1) / B;
    return L < slen && L % B != 0 && b_p * B < ws;
}

// The coarse score of the block [t0, t0 + n) of `rows` (the sequence's keys)
// for query row r, computed by every thread of the CTA (THREADS threads).
// s_sum: D_I ints of shared scratch. Returns the score in every thread; holds
// CTA barriers, so every thread must call it.
template <int D_I, int THREADS>
__device__ __noinline__ long long partial_block_score(const IndexArgs& a, int r, const int8_t* rows, int t0, int n,
                                         int32_t* s_sum, long long* s_out) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    constexpr int kWarps = THREADS / 32;
    constexpr int kLanes = D_I / 4;  // lanes owning 4 dims each
    for (int i = tid; i < D_I; i += THREADS) s_sum[i] = 0;
    __syncthreads();
    if (lane < kLanes) {
        int s0 = 0, s1 = 0, s2 = 0, s3 = 0;
        for (int i = warp; i < n; i += kWarps) {
            const uint32_t w = __ldg(reinterpret_cast<const uint32_t*>(rows + (int64_t)(t0 + i) * D_I) + lane);
            s0 += (int)(int8_t)(w & 0xffu);
            s1 += (int)(int8_t)((w >> 8) & 0xffu);
            s2 += (int)(int8_t)((w >> 16) & 0xffu);
            s3 += (int)(int8_t)(w >> 24);
        }
        atomicAdd(&s_sum[4 * lane + 0], s0);
        atomicAdd(&s_sum[4 * lane + 1], s1);
        atomicAdd(&s_sum[4 * lane + 2], s2);
        atomicAdd(&s_sum[4 * lane + 3], s3);
    }
    __syncthreads();
    if (warp == 0) {
        long long score = 0;
        for (int h = 0; h < a.H_I; ++h) {
            int dot = 0;
            if (lane < kLanes) {
                const uint32_t qw =
                    __ldg(reinterpret_cast<const uint32_t*>(a.q_idx + ((int64_t)r * a.H_I + h) * D_I) + lane);
                dot = (int)(int8_t)(qw & 0xffu) * s_sum[4 * lane] + (int)(int8_t)((qw >> 8) & 0xffu) * s_sum[4 * lane + 1] +
                      (int)(int8_t)((qw >> 16) & 0xffu) * s_sum[4 * lane + 2] + (int)(int8_t)(qw >> 24) * s_sum[4 * lane + 3];
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
            int32_t wh = __ldg(a.w + (int64_t)r * a.H_I + h);
            if (wh < 0 || wh > a.w_max) wh = 0;  // flagged by the query loads of the scoring passes
            score += (long long)wh * (long long)max(dot, 0);
        }
        if (lane == 0) *s_out = score;
    }
    __syncthreads();
    return *s_out;
}

}  // namespace lsa
