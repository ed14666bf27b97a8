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


}  // namespace lsa
