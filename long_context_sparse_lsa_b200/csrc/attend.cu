// attend.cu — sparse GQA softmax attention over LSA index sets, split over
// the set entries, and the merge of the split partials.
//
// The method: attention runs only over the tokens the indexer selected; SI
// makes the sink and window parts contiguous KV runs ("LongCat-Flash-Lite-
// Sparse (aitrends.kr)", section "기술적 특징", SI bullet); CLI lets G
// consecutive layers reuse one index set (same section, CLI bullet).
//
// Design (B200):
//  * grid = (splits x kv-head groups, query rows, layers); one CTA per SM.
//    A CTA covers up to 4 kv heads, whose rows of one token are contiguous
//    (4 x 256 B), over one contiguous range of index-set entries whose
//    indices are staged in shared memory first.
//  * The gather uses two independent load paths so that neither caps the
//    bandwidth: K rows come through the TMA engine (one cp.async.bulk of
//    hpc*256 bytes per selected token into a ring of 16-token stages, padded
//    by 16 bytes per row so ldmatrix reads of 8 tokens hit 8 bank groups,
//    completing on an mbarrier); V rows are loaded by the consumer warps
//    themselves with 16-byte vector loads straight into registers, two tiles
//    ahead of their use. (16-byte cp.async copies issued by one producer warp
//    instead of the bulk copies measured 2.2x slower.)
//  * Eight consumer warps: each owns one kv head and every (8/hpc)-th stage.
//    S^T = K Q^T on bf16 tensor cores (mma.m16n8k16): the 16 tokens are M and
//    the GQA group's query heads (8 per tile) are N. Online softmax in fp32
//    (exp2f, log2(e)/sqrt(d) scale). O^T = V^T P^T: P^T is moved into the B
//    operand with movmatrix.trans and split into a bf16 high part plus a bf16
//    remainder (two MMAs, ~16 significant bits). For V^T the output dims are
//    permuted so that lane (g, t) needs 16-byte chunks g and 8+g of tokens
//    2t, 2t+1, 2t+8, 2t+9; byte permutes assemble the A fragments.
//  * The consumers of one kv head merge in registers (log-sum-exp rule; the
//    partner warps park their fragments in shared memory); each CTA writes
//    its output directly when there is one split, else one partial per query
//    head, which a small merge kernel (one warp per query head, every partial
//    loaded at once) combines.
//  * Every mbarrier wait is bounded by a time limit; on expiry the kernel
//    flags LSA_DEV_TIMEOUT, waits (bounded) for the copies it issued and
//    returns.
#include <type_traits>

#include "common.cuh"
#include "internal.h"

namespace lsa {
namespace {

constexpr int kConsumers = 8;
constexpr int kAtThreads = (kConsumers + 1) * kWarp;  // + one producer warp
constexpr int kTile = 16;                              // tokens per stage
constexpr int kD = 128;
constexpr int kHeadBytes = kD * 2;                     // one (token, kv head) row
constexpr int kMaxEntriesPerSplit = 4096;
constexpr int kMaxStages = 8;
constexpr size_t kAtSmemBudget = 200 * 1024;
constexpr size_t kSmemPerSm = 228 * 1024;  // the shared-memory carveout's 100%

// V rows of one 16-token tile for one kv head, in the registers of lane
// (g, t): tokens 2t, 2t+1, 2t+8, 2t+9 (index j = 0..3), 16-byte chunks g and
// 8+g (index c = 0..1).
struct VTile {
    uint4 r[4][2];
};

__device__ __forceinline__ void load_vtile(VTile& v, const uint16_t* vbase, int64_t tok_stride, const int32_t* ent,
                                           int g, int t4) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const int row = 2 * t4 + (j & 1) + 8 * (j >> 1);
        const int e = ent[row];
        if (e >= 0) {
            const uint16_t* p = vbase + (int64_t)e * tok_stride;
            v.r[j][0] = ldg16(p + 8 * g);
            v.r[j][1] = ldg16(p + 64 + 8 * g);
        } else {
            v.r[j][0] = make_uint4(0, 0, 0, 0);
            v.r[j][1] = make_uint4(0, 0, 0, 0);
        }
    }
}

__device__ __forceinline__ uint32_t word(const uint4& x, int j) {
    return j == 0 ? x.x : (j == 1 ? x.y : (j == 2 ? x.z : x.w));
}

// Online softmax of one 16-token tile's scores (sacc: S^T fragments, tokens g
// and g+8 of this lane, masked where ok_g / ok_g8 is false) and O^T += V^T P^T
// from the tile's V registers.
template <int NT, bool F16 = false>
__device__ __forceinline__ void softmax_pv(const float (&sacc)[NT][4], bool ok_g, bool ok_g8, float scale_log2,
                                           float (&m_run)[NT][2], float (&l_run)[NT][2], float (&o)[NT][kD / 16][4],
                                           const VTile& v) {
    uint32_t phi[NT][2], plo[NT][2];
#pragma unroll
    for (int n = 0; n < NT; ++n) {
        const float z0 = ok_g ? sacc[n][0] * scale_log2 : -INFINITY;   // (tok g,   head 2t)
        const float z1 = ok_g ? sacc[n][1] * scale_log2 : -INFINITY;   // (tok g,   head 2t+1)
        const float z2 = ok_g8 ? sacc[n][2] * scale_log2 : -INFINITY;  // (tok g+8, head 2t)
        const float z3 = ok_g8 ? sacc[n][3] * scale_log2 : -INFINITY;  // (tok g+8, head 2t+1)
        float mx0 = fmaxf(z0, z2), mx1 = fmaxf(z1, z3);
#pragma unroll
        for (int msk = 4; msk < 32; msk <<= 1) {
            mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, msk));
            mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, msk));
        }
        const float mn0 = fmaxf(m_run[n][0], mx0), mn1 = fmaxf(m_run[n][1], mx1);
        const float base0 = mn0 == -INFINITY ? 0.f : mn0;
        const float base1 = mn1 == -INFINITY ? 0.f : mn1;
        const float al0 = exp2f(m_run[n][0] - base0), al1 = exp2f(m_run[n][1] - base1);
        const float p0 = exp2f(z0 - base0), p1 = exp2f(z1 - base1);
        const float p2 = exp2f(z2 - base0), p3 = exp2f(z3 - base1);
        // the running max rarely moves after the first tiles: rescale o
        // only when it did for some head of this warp
        const bool moved = __any_sync(0xffffffffu, mn0 != m_run[n][0] || mn1 != m_run[n][1]);
        m_run[n][0] = mn0;
        m_run[n][1] = mn1;
        l_run[n][0] = l_run[n][0] * al0 + p0 + p2;
        l_run[n][1] = l_run[n][1] * al1 + p1 + p3;
        if (moved) {
#pragma unroll
            for (int mt = 0; mt < kD / 16; ++mt) {
                o[n][mt][0] *= al0;
                o[n][mt][1] *= al1;
                o[n][mt][2] *= al0;
                o[n][mt][3] *= al1;
            }
        }
        if constexpr (F16) {
            const __half2 h01 = __floats2half2_rn(p0, p1);
            const __half2 h23 = __floats2half2_rn(p2, p3);
            const float2 fh01 = __half22float2(h01), fh23 = __half22float2(h23);
            phi[n][0] = movmatrix_trans(*reinterpret_cast<const uint32_t*>(&h01));
            phi[n][1] = movmatrix_trans(*reinterpret_cast<const uint32_t*>(&h23));
            plo[n][0] = movmatrix_trans(pack_f16(p0 - fh01.x, p1 - fh01.y));
            plo[n][1] = movmatrix_trans(pack_f16(p2 - fh23.x, p3 - fh23.y));
        } else {
            const __nv_bfloat162 h01 = __floats2bfloat162_rn(p0, p1);
            const __nv_bfloat162 h23 = __floats2bfloat162_rn(p2, p3);
            const float2 fh01 = __bfloat1622float2(h01), fh23 = __bfloat1622float2(h23);
            phi[n][0] = movmatrix_trans(*reinterpret_cast<const uint32_t*>(&h01));
            phi[n][1] = movmatrix_trans(*reinterpret_cast<const uint32_t*>(&h23));
            plo[n][0] = movmatrix_trans(pack_bf16(p0 - fh01.x, p1 - fh01.y));
            plo[n][1] = movmatrix_trans(pack_bf16(p2 - fh23.x, p3 - fh23.y));
        }
    }
    // O^T += V^T P^T from the registers of this tile's V
#pragma unroll
    for (int mt = 0; mt < kD / 16; ++mt) {
        const int c = mt >> 2, j = mt & 3;
        const uint32_t w0 = word(v.r[0][c], j), w1 = word(v.r[1][c], j);
        const uint32_t w8 = word(v.r[2][c], j), w9 = word(v.r[3][c], j);
        const uint32_t vfr[4] = {__byte_perm(w0, w1, 0x5410), __byte_perm(w0, w1, 0x7632),
                                 __byte_perm(w8, w9, 0x5410), __byte_perm(w8, w9, 0x7632)};
#pragma unroll
        for (int n = 0; n < NT; ++n) {
            mma_16<F16>(o[n][mt], vfr, phi[n][0], phi[n][1]);
            mma_16<F16>(o[n][mt], vfr, plo[n][0], plo[n][1]);
        }
    }
}

// ln(sum_j exp(s_j)) from the running max m (log2 units of the scaled
// scores) and the denominator l = sum_j exp2(m_j - m): (m + log2 l) ln 2.
__device__ __forceinline__ float lse_of(float m, float l) {
    return l > 0.f ? (m + log2f(l)) * 0.6931471805599453f : -INFINITY;
}

// Zeroes the output of an invalid row's query heads [h0, h0 + nh) and marks
// their lse empty (split 0 of the row does it).
__device__ __forceinline__ void clear_row(const AttendArgs& a, int layer, int r, int h0, int nh, int tid,
                                          int nthreads) {
    float* orow = a.out[layer] + ((int64_t)r * a.H_q + h0) * kD;
    for (int i = tid; i < nh * kD; i += nthreads) orow[i] = 0.f;
    if (a.lse[layer] != nullptr)
        for (int i = tid; i < nh; i += nthreads) a.lse[layer][(int64_t)r * a.H_q + h0 + i] = -INFINITY;
}

// Merges the consumer warps of each kv head (in registers: warps with
// wsel > 0 park their fragments in `merge_area`, lane-major, and the wsel == 0
// warp folds them in with the log-sum-exp rule), then writes the head's query
// heads: the final output when there is one split, else one partial. Every
// thread of the CTA calls it (it holds a CTA barrier); warps >= kConsumers
// only take part in the barrier.
// GROUPED (draft-row groups): hpc is the CTA's (kv head, row) pairs; the
// warps w % hpc == key work for kv head hgrp * kvpc + key % kvpc of row
// r + key / kvpc.
template <int NT, bool GROUPED = false>
__device__ __forceinline__ void merge_and_store(const AttendArgs& a, uint8_t* merge_area, float (&o)[NT][kD / 16][4],
                                                float (&m_run)[NT][2], float (&l_run)[NT][2], int warp, int lane,
                                                int hpc, int hgrp, int r, int layer, int split, int ratio,
                                                float vs = 1.f, int kvpc = 1) {
    const int g = lane >> 2, t4 = lane & 3;
    // ---- merge the consumers of each kv head, in registers ----
    // All warps hold O^T in the same fragment layout, so warps with wsel > 0
    // park theirs in shared memory (lane-major: conflict free) and the wsel ==
    // 0 warp of the head folds them in with the log-sum-exp rule.
    constexpr int kRegs = NT * (kD / 16) * 4;
    float* xo = reinterpret_cast<float*>(merge_area);  // [kConsumers][kRegs][32]
    float* xml = xo + kConsumers * kRegs * kWarp;              // [kConsumers][NT*4][32]
    const int wsel_me = warp / hpc;
    if (warp < kConsumers && wsel_me > 0) {
#pragma unroll
        for (int n = 0; n < NT; ++n) {
#pragma unroll
            for (int mt = 0; mt < kD / 16; ++mt)
#pragma unroll
                for (int c = 0; c < 4; ++c) xo[(warp * kRegs + (n * (kD / 16) + mt) * 4 + c) * kWarp + lane] = o[n][mt][c];
            xml[(warp * NT * 4 + n * 4 + 0) * kWarp + lane] = m_run[n][0];
            xml[(warp * NT * 4 + n * 4 + 1) * kWarp + lane] = m_run[n][1];
            xml[(warp * NT * 4 + n * 4 + 2) * kWarp + lane] = l_run[n][0];
            xml[(warp * NT * 4 + n * 4 + 3) * kWarp + lane] = l_run[n][1];
        }
    }
    __syncthreads();
    const bool direct = a.n_splits == 1;
    if (warp < kConsumers && wsel_me == 0) {
        const int h_local = warp % hpc;
        if (GROUPED) r += h_local / kvpc;
        const int64_t row_q = (int64_t)layer * a.n_q + r;
        const int n_sel = kConsumers / hpc;
        for (int j = 1; j < n_sel; ++j) {
            const int w = h_local + hpc * j;
#pragma unroll
            for (int n = 0; n < NT; ++n) {
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    const float mb = xml[(w * NT * 4 + n * 4 + c) * kWarp + lane];
                    const float lb = xml[(w * NT * 4 + n * 4 + 2 + c) * kWarp + lane];
                    const float M = fmaxf(m_run[n][c], mb);
                    const float sa = M == -INFINITY ? 0.f : exp2f(m_run[n][c] - M);
                    const float sb = M == -INFINITY ? 0.f : exp2f(mb - M);
                    m_run[n][c] = M;
                    l_run[n][c] = l_run[n][c] * sa + lb * sb;
#pragma unroll
                    for (int mt = 0; mt < kD / 16; ++mt) {
                        o[n][mt][c] = o[n][mt][c] * sa + xo[(w * kRegs + (n * (kD / 16) + mt) * 4 + c) * kWarp + lane] * sb;
                        o[n][mt][c + 2] =
                            o[n][mt][c + 2] * sa + xo[(w * kRegs + (n * (kD / 16) + mt) * 4 + c + 2) * kWarp + lane] * sb;
                    }
                }
            }
        }
        // write this kv head's query heads: the final output, or one split partial
        const int kvh = GROUPED ? hgrp * kvpc + h_local % kvpc : hgrp * hpc + h_local;
#pragma unroll
        for (int n = 0; n < NT; ++n) {
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                const int hh = 8 * n + 2 * t4 + c;
                if (hh >= ratio) continue;
                const int64_t qh = (int64_t)kvh * ratio + hh;
                const float inv = l_run[n][c] > 0.f ? 1.f / l_run[n][c] : 0.f;
                float* dst = direct ? a.out[layer] + ((int64_t)r * a.H_q + qh) * kD
                                    : a.part_o + ((row_q * a.n_splits + split) * a.H_q + qh) * kD;
                const float sc = direct ? inv * vs : vs;  // vs: the FP8 V scale (1 for bf16)
#pragma unroll
                for (int mt = 0; mt < kD / 16; ++mt) {
                    const int d0 = 8 * ((mt >> 2) ? 8 + g : g) + 2 * (mt & 3);
                    *reinterpret_cast<float2*>(dst + d0) = make_float2(o[n][mt][c] * sc, o[n][mt][c + 2] * sc);
                }
                if (!direct && g == 0)
                    *reinterpret_cast<float2*>(a.part_ml + ((row_q * a.n_splits + split) * a.H_q + qh) * 2) =
                        make_float2(m_run[n][c], l_run[n][c]);
                if (direct && g == 0 && a.lse[layer] != nullptr)
                    a.lse[layer][(int64_t)r * a.H_q + qh] = lse_of(m_run[n][c], l_run[n][c]);
            }
        }
    }
}

template <int NT>
__global__ void __launch_bounds__(kAtThreads, 1) attend_kernel(const __grid_constant__ AttendArgs a) {
    pdl_enter();
    extern __shared__ __align__(128) uint8_t smem[];
    __shared__ uint32_t s_fail;

    const int tid = threadIdx.x, lane = lane_id(), warp = warp_id();
    const int g = lane >> 2, t4 = lane & 3;
    const int split = blockIdx.x / a.head_groups;
    const int hgrp = blockIdx.x % a.head_groups;
    const int r = blockIdx.y;
    const int layer = blockIdx.z;
    const int ratio = a.H_q / a.H_kv;
    const int hpc = a.hpc;
    const int NS = a.n_stages;
    const int row_stride = a.row_stride;
    const int stage_bytes = kTile * row_stride;
    const int q_heads_cta = hpc * ratio;

    // ---- query row validation (uniform over the CTA) ----
    const int seq = a.q_seq[r];
    const int L = a.q_len[r];
    bool bad = seq < 0 || seq >= a.n_seq;
    int64_t off = 0;
    if (!bad) {
        off = a.kv_offset[seq];
        const int slen = a.seq_lens[seq];
        bad = L < 1 || L > a.max_len || L > slen || off < 0 || off + slen > a.total_tokens;
    }
    if (bad) {
        if (tid == 0 && blockIdx.x == 0 && layer == 0)
            flag(a.dev_status, seq < 0 || seq >= a.n_seq ? LSA_DEV_BAD_SEQ : LSA_DEV_BAD_LENGTH);
        if (split == 0) clear_row(a, layer, r, hgrp * q_heads_cta, q_heads_cta, tid, kAtThreads);
        return;
    }

    const int n_entries = min(L, a.budget);
    const int e0 = split * a.entries_per_split;
    const int n_local = max(0, min(n_entries - e0, a.entries_per_split));
    const int n_tiles = (n_local + kTile - 1) / kTile;
    const int32_t* set = a.sets + (int64_t)r * a.budget + e0;

    int32_t* s_ent = reinterpret_cast<int32_t*>(smem);
    const uint32_t bar_base = smem_u32(smem + a.bar_off);
    const uint32_t st_base = smem_u32(smem + a.stage_off);
    auto full_bar = [&](int s) { return bar_base + 8u * (uint32_t)s; };
    auto empty_bar = [&](int s) { return bar_base + 8u * (uint32_t)(NS + s); };

    if (tid == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(full_bar(s), 1);
            mbar_init(empty_bar(s), (uint32_t)hpc);
        }
        mbar_fence_init();
        s_fail = 0;
    }
    __syncthreads();
    // Entry i of this split, validated (invalid entries read as -1).
    auto entry = [&](int i) -> int {
        if (i >= n_local) return -1;
        const int v = set[i];
        if (v < -1 || v >= L) {
            flag(a.dev_status, LSA_DEV_BAD_INDEX);
            return -1;
        }
        return v;
    };
    if (warp < kConsumers) {
        // the consumers stage the split's entries; the producer reads its own
        // straight from global memory so its first copies start at once
        for (int i = tid; i < n_tiles * kTile; i += kConsumers * kWarp) s_ent[i] = entry(i);
        asm volatile("bar.sync 1, %0;" ::"r"(kConsumers * kWarp) : "memory");
    }

    // per-consumer state
    float o[NT][kD / 16][4];
    float m_run[NT][2], l_run[NT][2];
#pragma unroll
    for (int n = 0; n < NT; ++n) {
#pragma unroll
        for (int mt = 0; mt < kD / 16; ++mt) o[n][mt][0] = o[n][mt][1] = o[n][mt][2] = o[n][mt][3] = 0.f;
        m_run[n][0] = m_run[n][1] = -INFINITY;
        l_run[n][0] = l_run[n][1] = 0.f;
    }
    int issued = 0;  // producer: tiles whose copies were issued
    const int64_t tok_stride = (int64_t)a.H_kv * kD;  // elements between tokens

    if (warp == kConsumers) {
        // ------------------------------ producer (K) --------------------------
        const uint16_t* kb = a.k[layer] + (off * a.H_kv + (int64_t)hgrp * hpc) * kD;
        const uint32_t bytes = (uint32_t)(hpc * kHeadBytes);
        for (int i = 0; i < n_tiles; ++i) {
            const int s = i % NS;
            const int u = i / NS;
            if (u > 0 && !mbar_wait_bounded(empty_bar(s), (uint32_t)((u - 1) & 1), kWaitLimitNs)) {
                if (lane == 0) s_fail = 1;
                break;
            }
            const int ent = lane < kTile ? entry(i * kTile + lane) : -1;
            const bool valid = ent >= 0;
            const uint32_t nv = __popc(__ballot_sync(0xffffffffu, valid));
            if (lane == 0) mbar_arrive_expect_tx(full_bar(s), nv * bytes);
            __syncwarp();
            if (valid)
                bulk_g2s(st_base + (uint32_t)(s * stage_bytes + lane * row_stride), kb + (int64_t)ent * tok_stride,
                         bytes, full_bar(s));
            issued = i + 1;
        }
    } else {
        // ------------------------------ consumers -----------------------------
        const int h_local = warp % hpc;
        const int wsel = warp / hpc;
        const int n_sel = kConsumers / hpc;
        const int kvh = hgrp * hpc + h_local;
        const uint16_t* vbase = a.v[layer] + (off * a.H_kv + (int64_t)kvh) * kD;
        uint32_t qb[NT][kD / 16][2];
        {
            const uint16_t* qrow = a.q[layer] + ((int64_t)r * a.H_q + (int64_t)kvh * ratio) * kD;
#pragma unroll
            for (int n = 0; n < NT; ++n) {
                const int hh = 8 * n + g;
                const bool ok = hh < ratio;
#pragma unroll
                for (int ks = 0; ks < kD / 16; ++ks) {
                    qb[n][ks][0] = ok ? __ldg(reinterpret_cast<const uint32_t*>(qrow + hh * kD + 16 * ks + 2 * t4)) : 0u;
                    qb[n][ks][1] =
                        ok ? __ldg(reinterpret_cast<const uint32_t*>(qrow + hh * kD + 16 * ks + 8 + 2 * t4)) : 0u;
                }
            }
        }
        const uint32_t head_off = (uint32_t)(h_local * kHeadBytes);
        // V of this warp's next two tiles stays in flight (double buffer;
        // the loop is unrolled by two so each buffer is a fixed register set)
        VTile va, vbuf;
        if (wsel < n_tiles) load_vtile(va, vbase, tok_stride, s_ent + wsel * kTile, g, t4);
        if (wsel + n_sel < n_tiles) load_vtile(vbuf, vbase, tok_stride, s_ent + (wsel + n_sel) * kTile, g, t4);
        auto tile = [&](int i, VTile& v) -> bool {
            const int s = i % NS;
            const int u = i / NS;
            if (!mbar_wait_bounded(full_bar(s), (uint32_t)(u & 1), kWaitLimitNs)) {
                if (lane == 0) s_fail = 1;
                return false;
            }
            const uint32_t kst = st_base + (uint32_t)(s * stage_bytes) + head_off;
            const int ent_lane = lane < kTile ? s_ent[i * kTile + lane] : 0;
            const uint32_t masked = __ballot_sync(0xffffffffu, lane < kTile && ent_lane < 0);
            const bool ok_g = !((masked >> g) & 1u);
            const bool ok_g8 = !((masked >> (g + 8)) & 1u);
            // S^T tile: 16 tokens x (8 * NT) heads
            float sacc[NT][4];
#pragma unroll
            for (int n = 0; n < NT; ++n) sacc[n][0] = sacc[n][1] = sacc[n][2] = sacc[n][3] = 0.f;
            {
                const int mi = lane >> 3, rr = lane & 7;
                const uint32_t kaddr = kst + (uint32_t)((rr + 8 * (mi & 1)) * row_stride + (mi >> 1) * 16);
#pragma unroll
                for (int ks = 0; ks < kD / 16; ++ks) {
                    uint32_t afr[4];
                    ldmatrix_x4(afr, kaddr + ks * 32);
#pragma unroll
                    for (int n = 0; n < NT; ++n) mma_bf16(sacc[n], afr, qb[n][ks][0], qb[n][ks][1]);
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(empty_bar(s));  // K of this stage is no longer read
            softmax_pv<NT>(sacc, ok_g, ok_g8, a.scale_log2, m_run, l_run, o, v);
            // V two tiles ahead, in flight during the next tile's K wait and math
            if (i + 2 * n_sel < n_tiles) load_vtile(v, vbase, tok_stride, s_ent + (i + 2 * n_sel) * kTile, g, t4);
                    return true;
        };
        for (int i = wsel; i < n_tiles; i += 2 * n_sel) {
            if (!tile(i, va)) break;
            if (i + n_sel < n_tiles && !tile(i + n_sel, vbuf)) break;
        }
#pragma unroll
        for (int n = 0; n < NT; ++n)
#pragma unroll
            for (int j = 0; j < 2; ++j)
#pragma unroll
                for (int msk = 4; msk < 32; msk <<= 1)
                    l_run[n][j] += __shfl_xor_sync(0xffffffffu, l_run[n][j], msk);
    }
    __syncthreads();

    if (s_fail) {
        // wait (bounded) for every copy this CTA issued, then give up
        if (warp == kConsumers) {
            for (int i = max(0, issued - NS); i < issued; ++i)
                mbar_wait_bounded(full_bar(i % NS), (uint32_t)((i / NS) & 1), kWaitLimitNs);
        }
        if (tid == 0) flag(a.dev_status, LSA_DEV_TIMEOUT);
        return;
    }

    merge_and_store<NT>(a, smem + a.stage_off, o, m_run, l_run, warp, lane, hpc, hgrp, r, layer, split, ratio);
}

// K rows of one 16-token tile for one kv head, in the registers of lane
// (g, t): tokens g and g+8 (index rr), 16-byte chunks t, t+4, t+8, t+12 of
// the 256-byte row (index j). The QK^T contraction runs over the head dims in
// the matching permuted order: MMA k-step ks takes chunk ks/2, words
// 2*(ks&1) (k = 2t, 2t+1) and 2*(ks&1)+1 (k = 2t+8, 2t+9); the query
// fragments are read in the same order, so the dot products are unchanged.
struct KTile {
    uint4 r[2][4];
};

__device__ __forceinline__ void load_ktile(KTile& k, const uint16_t* kbase, int64_t tok_stride, const int32_t* ent,
                                           int g, int t4) {
#pragma unroll
    for (int rr = 0; rr < 2; ++rr) {
        const int e = ent[g + 8 * rr];
        if (e >= 0) {
            const uint16_t* p = kbase + (int64_t)e * tok_stride + 8 * t4;
#pragma unroll
            for (int j = 0; j < 4; ++j) k.r[rr][j] = ldg16(p + 32 * j);
        } else {
#pragma unroll
            for (int j = 0; j < 4; ++j) k.r[rr][j] = make_uint4(0, 0, 0, 0);
        }
    }
}

// ---- FP8 (E4M3) K/V ---------------------------------------------------------
// With an FP8 cache each element is one byte: a lane loads the same dims as in
// the bf16 tiles (8-byte chunks instead of 16-byte ones) and converts them to
// fp16 at use. Every E4M3 value is an fp16 exactly, and so is every bf16 query
// element in [2^-14, 65504] (the rest are fp16 subnormals or zero), so the
// MMAs run in fp16; the per-layer scales multiply the scores (K) and the
// output (V) in fp32.
struct KTile8 {
    uint2 r[2][4];
};
struct VTile8 {
    uint2 r[4][2];
};

__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t two) {  // bits 0..15: two codes, low first
    const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(two & 0xffffu), __NV_E4M3);
    return (uint32_t)h.x | ((uint32_t)h.y << 16);
}

__device__ __forceinline__ uint4 e4m3x8_to_f16(uint2 c) {
    return make_uint4(e4m3x2_to_f16x2(c.x), e4m3x2_to_f16x2(c.x >> 16), e4m3x2_to_f16x2(c.y),
                      e4m3x2_to_f16x2(c.y >> 16));
}

// True when either bf16 of the pair has magnitude >= 65536 (0x4780: above
// fp16's largest finite value 65504) or is not finite.
__device__ __forceinline__ bool bf16x2_beyond_f16(uint32_t x) {
    return (x & 0x7fffu) >= 0x4780u || ((x >> 16) & 0x7fffu) >= 0x4780u;
}

__device__ __forceinline__ uint32_t bf16x2_to_f16x2(uint32_t x) {
    const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&x));
    return pack_f16(f.x, f.y);
}

__device__ __forceinline__ void load_ktile8(KTile8& k, const uint8_t* kbase, int64_t tok_stride, const int32_t* ent,
                                            int g, int t4) {
#pragma unroll
    for (int rr = 0; rr < 2; ++rr) {
        const int e = ent[g + 8 * rr];
        if (e >= 0) {
            const uint8_t* p = kbase + (int64_t)e * tok_stride + 8 * t4;
#pragma unroll
            for (int j = 0; j < 4; ++j) k.r[rr][j] = ldg8(p + 32 * j);
        } else {
#pragma unroll
            for (int j = 0; j < 4; ++j) k.r[rr][j] = make_uint2(0, 0);
        }
    }
}

__device__ __forceinline__ void load_vtile8(VTile8& v, const uint8_t* vbase, int64_t tok_stride, const int32_t* ent,
                                            int g, int t4) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const int row = 2 * t4 + (j & 1) + 8 * (j >> 1);
        const int e = ent[row];
        if (e >= 0) {
            const uint8_t* p = vbase + (int64_t)e * tok_stride;
            v.r[j][0] = ldg8(p + 8 * g);
            v.r[j][1] = ldg8(p + 64 + 8 * g);
        } else {
            v.r[j][0] = make_uint2(0, 0);
            v.r[j][1] = make_uint2(0, 0);
        }
    }
}

// The 16-bit fragments of a tile: bf16 tiles as they are, FP8 tiles converted.
__device__ __forceinline__ const KTile& frag16(const KTile& k) { return k; }
__device__ __forceinline__ const VTile& frag16(const VTile& v) { return v; }
__device__ __forceinline__ KTile frag16(const KTile8& k) {
    KTile x;
#pragma unroll
    for (int rr = 0; rr < 2; ++rr)
#pragma unroll
        for (int j = 0; j < 4; ++j) x.r[rr][j] = e4m3x8_to_f16(k.r[rr][j]);
    return x;
}
__device__ __forceinline__ VTile frag16(const VTile8& v) {
    VTile x;
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
        for (int c = 0; c < 2; ++c) x.r[j][c] = e4m3x8_to_f16(v.r[j][c]);
    return x;
}

// The register-streaming variant (GQA groups of at most 8 query heads): every
// warp gathers its own K and V rows with 16-byte loads straight into MMA
// fragments, two tiles ahead of use, so no copy engine, shared-memory ring or
// producer warp sits between HBM and the tensor cores. Eight warps per CTA;
// warp w owns kv head w % hpc of the CTA and every (8/hpc)-th tile.
// FP8: the K/V caches hold E4M3 codes (see the FP8 tiles above).
template <bool FP8>
__global__ void __launch_bounds__(kConsumers * kWarp, 1) attend_rk_kernel(const __grid_constant__ AttendArgs a) {
    constexpr int NT = 1;
    extern __shared__ __align__(128) uint8_t smem[];
    const int tid = threadIdx.x, lane = lane_id(), warp = warp_id();
    const int g = lane >> 2, t4 = lane & 3;
    const int split = blockIdx.x / a.head_groups;
    const int hgrp = blockIdx.x % a.head_groups;
    const int r = blockIdx.y;
    const int layer = blockIdx.z;
    const int ratio = a.H_q / a.H_kv;
    const int hpc = a.hpc;
    const int q_heads_cta = hpc * ratio;

    // The set entries and the row's sequence metadata are fetched together
    // (the entries are checked against q_len once it is known); nothing is
    // written before the row check.
    // (the row's metadata is the caller's, never written by a kernel of this
    // library: it is read before the wait for the preceding kernel)
    const int seq = a.q_seq[r];
    const int L = a.q_len[r];
    const int seq_c = min(max(seq, 0), a.n_seq - 1);
    const int64_t off = a.kv_offset[seq_c];
    const int slen = a.seq_lens[seq_c];
    // the row's entries: the whole set, or (lsa_attend_si) its selected
    // entries [s, s + m) only, m = min(topk, ws - s)
    int e_begin = 0, e_end = a.budget;
    if (a.si_split) {
        const int Lc = min(max(L, 0), a.max_len);
        const int s = min(a.si_sink, Lc);
        const int ws = max(s, Lc - a.si_window);
        e_begin = min(s, a.budget);
        e_end = min(e_begin + min(a.si_topk, ws - s), a.budget);
    }
    pdl_enter();
    const int e0 = split * a.entries_per_split;
    const int32_t* set = a.sets + (int64_t)r * a.budget + e_begin + e0;
    const int n_cap = max(0, min(e_end - e_begin - e0, a.entries_per_split));  // entries this split may own
    int32_t* s_ent = reinterpret_cast<int32_t*>(smem);
    for (int i = tid; i < n_cap; i += kConsumers * kWarp) s_ent[i] = set[i];
    const bool bad = seq < 0 || seq >= a.n_seq || L < 1 || L > a.max_len || L > slen || off < 0 ||
                     off + slen > a.total_tokens;
    if (bad) {
        if (tid == 0 && blockIdx.x == 0 && layer == 0)
            flag(a.dev_status, seq < 0 || seq >= a.n_seq ? LSA_DEV_BAD_SEQ : LSA_DEV_BAD_LENGTH);
        if (split == 0) clear_row(a, layer, r, hgrp * q_heads_cta, q_heads_cta, tid, kConsumers * kWarp);
        return;
    }
    const int n_entries = a.si_split ? e_end - e_begin : min(L, a.budget);
    const int n_local = max(0, min(n_entries - e0, a.entries_per_split));
    const int n_tiles = (n_local + kTile - 1) / kTile;
    for (int i = tid; i < n_tiles * kTile; i += kConsumers * kWarp) {
        int v = -1;
        if (i < n_local) {
            v = s_ent[i];  // written by this thread above (same index and stride)
            if (v < -1 || v >= L) {
                flag(a.dev_status, LSA_DEV_BAD_INDEX);
                v = -1;
            }
        }
        s_ent[i] = v;
    }
    __syncthreads();

    float o[NT][kD / 16][4];
    float m_run[NT][2], l_run[NT][2];
#pragma unroll
    for (int mt = 0; mt < kD / 16; ++mt) o[0][mt][0] = o[0][mt][1] = o[0][mt][2] = o[0][mt][3] = 0.f;
    m_run[0][0] = m_run[0][1] = -INFINITY;
    l_run[0][0] = l_run[0][1] = 0.f;

    const int h_local = warp % hpc;
    const int wsel = warp / hpc;
    const int n_sel = kConsumers / hpc;
    const int kvh = hgrp * hpc + h_local;
    const int64_t tok_stride = (int64_t)a.H_kv * kD;  // elements (= bytes for FP8)
    constexpr int kEB = FP8 ? 1 : 2;                    // bytes per element
    const uint8_t* kbase = reinterpret_cast<const uint8_t*>(a.k[layer]) + (off * a.H_kv + (int64_t)kvh) * kD * kEB;
    const uint8_t* vbase = reinterpret_cast<const uint8_t*>(a.v[layer]) + (off * a.H_kv + (int64_t)kvh) * kD * kEB;
    using KT = std::conditional_t<FP8, KTile8, KTile>;
    using VT = std::conditional_t<FP8, VTile8, VTile>;
    auto load_k = [&](KT& k, const int32_t* ent) {
        if constexpr (FP8) load_ktile8(k, kbase, tok_stride, ent, g, t4);
        else load_ktile(k, reinterpret_cast<const uint16_t*>(kbase), tok_stride, ent, g, t4);
    };
    auto load_v = [&](VT& v, const int32_t* ent) {
        if constexpr (FP8) load_vtile8(v, vbase, tok_stride, ent, g, t4);
        else load_vtile(v, reinterpret_cast<const uint16_t*>(vbase), tok_stride, ent, g, t4);
    };
    // query fragments in the permuted dim order of KTile (fp16 for FP8 caches)
    uint32_t qb[kD / 16][2];
    {
        const uint16_t* qrow = a.q[layer] + ((int64_t)r * a.H_q + (int64_t)kvh * ratio) * kD;
        const bool ok = g < ratio;
        bool qbad = false;  // FP8: a query element fp16 cannot hold
#pragma unroll
        for (int ks = 0; ks < kD / 16; ++ks) {
            const uint16_t* p = qrow + g * kD + 8 * (t4 + 4 * (ks >> 1)) + 4 * (ks & 1);
            qb[ks][0] = ok ? __ldg(reinterpret_cast<const uint32_t*>(p)) : 0u;
            qb[ks][1] = ok ? __ldg(reinterpret_cast<const uint32_t*>(p + 2)) : 0u;
            if constexpr (FP8) {
                qbad |= bf16x2_beyond_f16(qb[ks][0]) | bf16x2_beyond_f16(qb[ks][1]);
                qb[ks][0] = bf16x2_to_f16x2(qb[ks][0]);
                qb[ks][1] = bf16x2_to_f16x2(qb[ks][1]);
            }
        }
        if (FP8 && __any_sync(0xffffffffu, qbad) && lane == 0) flag(a.dev_status, LSA_DEV_BAD_QUERY);
    }
    const float sl2 = FP8 ? a.scale_log2 * a.kscale[layer] : a.scale_log2;
    KT ka, kb2;
    VT va, vb2;
    if (wsel < n_tiles) {
        load_k(ka, s_ent + wsel * kTile);
        load_v(va, s_ent + wsel * kTile);
    }
    if (wsel + n_sel < n_tiles) {
        load_k(kb2, s_ent + (wsel + n_sel) * kTile);
        load_v(vb2, s_ent + (wsel + n_sel) * kTile);
    }
    auto tile = [&](int i, KT& k, VT& v) {
        const int ent_lane = lane < kTile ? s_ent[i * kTile + lane] : 0;
        const uint32_t masked = __ballot_sync(0xffffffffu, lane < kTile && ent_lane < 0);
        const bool ok_g = !((masked >> g) & 1u);
        const bool ok_g8 = !((masked >> (g + 8)) & 1u);
        float sacc[NT][4] = {{0.f, 0.f, 0.f, 0.f}};
        {
            const auto& kf = frag16(k);
#pragma unroll
            for (int ks = 0; ks < kD / 16; ++ks) {
                const int j = ks >> 1, w = 2 * (ks & 1);
                const uint32_t afr[4] = {word(kf.r[0][j], w), word(kf.r[1][j], w), word(kf.r[0][j], w + 1),
                                         word(kf.r[1][j], w + 1)};
                mma_16<FP8>(sacc[0], afr, qb[ks][0], qb[ks][1]);
            }
        }
        softmax_pv<NT, FP8>(sacc, ok_g, ok_g8, sl2, m_run, l_run, o, frag16(v));
        // K and V two tiles ahead, in flight during the next tile's math
        if (i + 2 * n_sel < n_tiles) {
            load_k(k, s_ent + (i + 2 * n_sel) * kTile);
            load_v(v, s_ent + (i + 2 * n_sel) * kTile);
        }
    };
    for (int i = wsel; i < n_tiles; i += 2 * n_sel) {
        tile(i, ka, va);
        if (i + n_sel < n_tiles) tile(i + n_sel, kb2, vb2);
    }
    pdl_trigger();  // only the head merge and the stores are left
#pragma unroll
    for (int j = 0; j < 2; ++j)
#pragma unroll
        for (int msk = 4; msk < 32; msk <<= 1) l_run[0][j] += __shfl_xor_sync(0xffffffffu, l_run[0][j], msk);
    __syncthreads();  // the merge area reuses the entry list
    merge_and_store<NT>(a, smem + a.stage_off, o, m_run, l_run, warp, lane, hpc, hgrp, r, layer, split, ratio,
                        FP8 ? a.vscale[layer] : 1.f);
}

// Draft-row groups: rows come in groups of D consecutive rows of one
// sequence (the draft tokens of a decode step), whose index sets share the
// sink run, nearly all of the window run and, where the drafts' indexer
// queries agree, much of the selection. A CTA covers hpc kv heads (whole
// tokens, as attend_rk_kernel) for rpc rows of a group, one warp per (kv
// head, row), all over the same stretch of their sets: entries [B s / n,
// B (s + 1) / n) of every row for split s. Sets as lsa_index writes them
// are ascending with the sink run first and the window run last, so the
// rows' stretches cover the same positions (exactly, for the sink and window
// runs), and a K/V row that several rows hold is fetched from L2 once and
// served from L1 to the others; the work per warp is the same as in
// attend_rk_kernel. The tile loop, the fragments and the softmax are
// attend_rk_kernel's (bf16 caches, GQA groups of at most 8 query heads); the
// partials merge as lsa_attend's.
__global__ void __launch_bounds__(kConsumers * kWarp, 1) attend_group_kernel(const __grid_constant__ AttendArgs a) {
    constexpr int NT = 1;
    extern __shared__ __align__(128) uint8_t smem[];
    const int tid = threadIdx.x, lane = lane_id(), warp = warp_id();
    const int g = lane >> 2, t4 = lane & 3;
    const int D = a.group_rows;
    // CTA (split, kv-head group, row block): hpc kv heads x rpc rows of the
    // group, n_ph warps on each (kv head, row); warp w: key w % (hpc rpc)
    const int hpc = a.hpc, rpc = a.rows_per_cta;
    const int keys = hpc * rpc;
    const int row_blocks = D / rpc;
    const int rb = blockIdx.x % row_blocks;
    const int hgrp = (blockIdx.x / row_blocks) % a.head_groups;
    const int split = blockIdx.x / (row_blocks * a.head_groups);
    const int grp = blockIdx.y;
    const int layer = blockIdx.z;
    const int ratio = a.H_q / a.H_kv;
    const int key = warp % keys;
    const int kvh = hgrp * hpc + key % hpc;
    const int jl = key / hpc;            // this warp's row of the CTA
    const int jr = rb * rpc + jl;        // ... of the group
    const int ph = warp / keys, n_ph = kConsumers / keys;
    const int r = grp * D + jr;
    // the row's metadata (the caller's) before the wait
    const int seq = a.q_seq[r];
    const int L = a.q_len[r];
    const int seq_c = min(max(seq, 0), a.n_seq - 1);
    const int64_t off = a.kv_offset[seq_c];
    const int slen = a.seq_lens[seq_c];
    pdl_enter();
    const bool bad = seq < 0 || seq >= a.n_seq || L < 1 || L > a.max_len || L > slen || off < 0 ||
                     off + slen > a.total_tokens;
    if (bad && split == 0 && hgrp == 0 && key % hpc == 0 && layer == 0 && lane == 0 && ph == 0)
        flag(a.dev_status, seq < 0 || seq >= a.n_seq ? LSA_DEV_BAD_SEQ : LSA_DEV_BAD_LENGTH);
    if (bad && split == 0 && ph == 0) {  // an invalid row's output is zero
        float* orow = a.out[layer] + ((int64_t)r * a.H_q + (int64_t)kvh * ratio) * kD;
        for (int i = lane; i < ratio * kD; i += kWarp) orow[i] = 0.f;
    }
    // split s of each of the CTA's rows: entries [B s / n, B (s + 1) / n) of
    // its set, checked as lsa_attend checks them (entries below -1 or at or
    // past q_len flagged and skipped; an invalid row's entries all skipped)
    // and padded with -1 to whole tiles
    const int B = a.budget;
    const int stride = a.entries_per_split;  // per-row list capacity
    int32_t* s_work = reinterpret_cast<int32_t*>(smem);  // [rpc][stride]
    __shared__ int32_t s_len[kMaxGroupRows];
    if (tid < rpc) {
        const int rr = grp * D + rb * rpc + tid;
        const int sq = a.q_seq[rr], Lr = a.q_len[rr];
        const int sc = min(max(sq, 0), a.n_seq - 1);
        const int64_t o2 = a.kv_offset[sc];
        const int sl = a.seq_lens[sc];
        const bool ok = sq >= 0 && sq < a.n_seq && Lr >= 1 && Lr <= a.max_len && Lr <= sl && o2 >= 0 &&
                        o2 + sl <= a.total_tokens;
        s_len[tid] = ok ? Lr : 0;
    }
    __syncthreads();
    const int e_lo = (int)((int64_t)B * split / a.n_splits);
    const int n_mine = (int)((int64_t)B * (split + 1) / a.n_splits) - e_lo;  // the same for every row
    const int n_tiles = (n_mine + kTile - 1) / kTile;
    bool bad_entry = false;
    for (int q = tid; q < rpc * n_tiles * kTile; q += kConsumers * kWarp) {
        const int j = q / (n_tiles * kTile), i = q - j * (n_tiles * kTile);
        int32_t e = -1;
        if (i < n_mine) {
            e = a.sets[(int64_t)(grp * D + rb * rpc + j) * B + e_lo + i];
            const int Lj = s_len[j];
            if (e < -1 || e >= Lj) {
                bad_entry |= Lj > 0;
                e = -1;
            }
        }
        s_work[j * stride + i] = e;
    }
    if (bad_entry) flag(a.dev_status, LSA_DEV_BAD_INDEX);
    __syncthreads();
    int32_t* s_ent = s_work + jl * stride;

    float o[NT][kD / 16][4];
    float m_run[NT][2], l_run[NT][2];
#pragma unroll
    for (int mt = 0; mt < kD / 16; ++mt) o[0][mt][0] = o[0][mt][1] = o[0][mt][2] = o[0][mt][3] = 0.f;
    m_run[0][0] = m_run[0][1] = -INFINITY;
    l_run[0][0] = l_run[0][1] = 0.f;
    const int64_t tok_stride = (int64_t)a.H_kv * kD;
    const uint16_t* kbase = a.k[layer] + (off * a.H_kv + (int64_t)kvh) * kD;
    const uint16_t* vbase = a.v[layer] + (off * a.H_kv + (int64_t)kvh) * kD;
    uint32_t qb[kD / 16][2];
    {
        const uint16_t* qrow = a.q[layer] + ((int64_t)r * a.H_q + (int64_t)kvh * ratio) * kD;
        const bool ok = g < ratio;
#pragma unroll
        for (int ks = 0; ks < kD / 16; ++ks) {
            const uint16_t* p = qrow + g * kD + 8 * (t4 + 4 * (ks >> 1)) + 4 * (ks & 1);
            qb[ks][0] = ok ? __ldg(reinterpret_cast<const uint32_t*>(p)) : 0u;
            qb[ks][1] = ok ? __ldg(reinterpret_cast<const uint32_t*>(p + 2)) : 0u;
        }
    }
    KTile ka, kb2;
    VTile va, vb2;
    if (ph < n_tiles) {
        load_ktile(ka, kbase, tok_stride, s_ent + ph * kTile, g, t4);
        load_vtile(va, vbase, tok_stride, s_ent + ph * kTile, g, t4);
    }
    if (ph + n_ph < n_tiles) {
        load_ktile(kb2, kbase, tok_stride, s_ent + (ph + n_ph) * kTile, g, t4);
        load_vtile(vb2, vbase, tok_stride, s_ent + (ph + n_ph) * kTile, g, t4);
    }
    auto tile = [&](int i, KTile& k, VTile& v) {
        const int ent_lane = lane < kTile ? s_ent[i * kTile + lane] : 0;
        const uint32_t masked = __ballot_sync(0xffffffffu, lane < kTile && ent_lane < 0);
        const bool ok_g = !((masked >> g) & 1u);
        const bool ok_g8 = !((masked >> (g + 8)) & 1u);
        float sacc[NT][4] = {{0.f, 0.f, 0.f, 0.f}};
#pragma unroll
        for (int ks = 0; ks < kD / 16; ++ks) {
            const int j = ks >> 1, w = 2 * (ks & 1);
            const uint32_t afr[4] = {word(k.r[0][j], w), word(k.r[1][j], w), word(k.r[0][j], w + 1),
                                     word(k.r[1][j], w + 1)};
            mma_16<false>(sacc[0], afr, qb[ks][0], qb[ks][1]);
        }
        softmax_pv<NT, false>(sacc, ok_g, ok_g8, a.scale_log2, m_run, l_run, o, v);
        if (i + 2 * n_ph < n_tiles) {
            load_ktile(k, kbase, tok_stride, s_ent + (i + 2 * n_ph) * kTile, g, t4);
            load_vtile(v, vbase, tok_stride, s_ent + (i + 2 * n_ph) * kTile, g, t4);
        }
    };
    for (int i = ph; i < n_tiles; i += 2 * n_ph) {
        tile(i, ka, va);
        if (i + n_ph < n_tiles) tile(i + n_ph, kb2, vb2);
    }
    pdl_trigger();
#pragma unroll
    for (int j = 0; j < 2; ++j)
#pragma unroll
        for (int msk = 4; msk < 32; msk <<= 1) l_run[0][j] += __shfl_xor_sync(0xffffffffu, l_run[0][j], msk);
    __syncthreads();  // the merge area reuses the entry lists
    if (bad) {        // keep the zeros written above (a partial of nothing merges to zero too)
#pragma unroll
        for (int mt = 0; mt < kD / 16; ++mt) o[0][mt][0] = o[0][mt][1] = o[0][mt][2] = o[0][mt][3] = 0.f;
    }
    merge_and_store<NT, true>(a, smem + a.stage_off, o, m_run, l_run, warp, lane, keys, hgrp,
                              grp * D + rb * rpc, layer, split, ratio, 1.f, hpc);
}

// Split merge: one CTA per (query head, row, layer) with one warp per
// kMergeSplitsPerWarp splits, so every partial is loaded in one round of
// loads; lane l owns dims 4l..4l+3. Each warp folds its splits with the
// log-sum-exp rule, and warp 0 folds the warps' results from shared memory.
constexpr int kMergeSplitsPerWarp = 8;
constexpr int kMergeMaxWarps = 16;

__global__ void __launch_bounds__(kMergeMaxWarps * kWarp) attend_merge_kernel(const __grid_constant__ AttendArgs a) {
    pdl_enter();
    __shared__ float s_m[kMergeMaxWarps], s_den[kMergeMaxWarps];
    __shared__ float4 s_acc[kMergeMaxWarps][kWarp];
    const int h = blockIdx.x, r = blockIdx.y, layer = blockIdx.z, lane = lane_id(), w = warp_id();
    const int nw = (int)(blockDim.x / kWarp);
    // the row check's loads overlap the partials' loads; the output is only
    // written for a valid row (an invalid row's output was zeroed already)
    const int seq = a.q_seq[r];
    const int L = a.q_len[r];
    const int seq_c = min(max(seq, 0), a.n_seq - 1);
    const int64_t off = a.kv_offset[seq_c];
    const int slen = a.seq_lens[seq_c];
    const int64_t row_q = (int64_t)layer * a.n_q + r;
    const float* P = a.part_o + (row_q * a.n_splits * a.H_q + h) * kD;
    const float* PML = a.part_ml + (row_q * a.n_splits * a.H_q + h) * 2;
    const int64_t pstride = (int64_t)a.H_q;  // between consecutive splits, in rows
    const int per = (a.n_splits + nw - 1) / nw;
    const int p_lo = w * per, p_hi = min(a.n_splits, p_lo + per);
    float M = -INFINITY, den = 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int p0 = p_lo; p0 < p_hi; p0 += kMergeSplitsPerWarp) {
        float2 ml[kMergeSplitsPerWarp];
        float4 v[kMergeSplitsPerWarp];
#pragma unroll
        for (int u = 0; u < kMergeSplitsPerWarp; ++u) {
            const int p = p0 + u;
            const bool ok = p < p_hi;
            ml[u] = ok ? __ldcg(reinterpret_cast<const float2*>(PML + p * pstride * 2)) : make_float2(-INFINITY, 0.f);
            v[u] = ok ? __ldcg(reinterpret_cast<const float4*>(P + p * pstride * kD) + lane)
                      : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int u = 0; u < kMergeSplitsPerWarp; ++u) {
            if (ml[u].x == -INFINITY) continue;
            const float nm = fmaxf(M, ml[u].x);
            const float so = exp2f(M - nm), sn = exp2f(ml[u].x - nm);
            den = den * so + ml[u].y * sn;
            acc.x = acc.x * so + v[u].x * sn;
            acc.y = acc.y * so + v[u].y * sn;
            acc.z = acc.z * so + v[u].z * sn;
            acc.w = acc.w * so + v[u].w * sn;
            M = nm;
        }
    }
    if (nw > 1) {
        s_acc[w][lane] = acc;
        if (lane == 0) {
            s_m[w] = M;
            s_den[w] = den;
        }
        __syncthreads();
        if (w != 0) return;
        M = -INFINITY;
        den = 0.f;
        acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int j = 0; j < nw; ++j) {
            const float mj = s_m[j];
            if (mj == -INFINITY) continue;
            const float nm = fmaxf(M, mj);
            const float so = exp2f(M - nm), sn = exp2f(mj - nm);
            const float4 aj = s_acc[j][lane];
            den = den * so + s_den[j] * sn;
            acc.x = acc.x * so + aj.x * sn;
            acc.y = acc.y * so + aj.y * sn;
            acc.z = acc.z * so + aj.z * sn;
            acc.w = acc.w * so + aj.w * sn;
            M = nm;
        }
    }
    if (seq < 0 || seq >= a.n_seq || L < 1 || L > a.max_len || L > slen || off < 0 || off + slen > a.total_tokens)
        return;
    const float inv = den > 0.f ? 1.f / den : 0.f;
    reinterpret_cast<float4*>(a.out[layer] + ((int64_t)r * a.H_q + h) * kD)[lane] =
        make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
    if (lane == 0 && a.lse[layer] != nullptr) a.lse[layer][(int64_t)r * a.H_q + h] = lse_of(M, den);
}

}  // namespace

AttendPlan plan_attend(int n_q, int max_len, int H_q, int H_kv, int d, int budget, int G, int num_sms, bool fp8) {
    AttendPlan p;
    (void)d;
    p.hpc = H_kv < 4 ? H_kv : 4;
    p.head_groups = H_kv / p.hpc;
    p.row_stride = p.hpc * kHeadBytes + 16;
    const int entries = budget < max_len ? budget : max_len;
    const long rows = (long)n_q * G * p.head_groups;
    int splits = rows > 0 ? (int)((num_sms + rows / 2) / rows) : 1;
    if (splits < 1) splits = 1;
    const int min_splits = (entries + kMaxEntriesPerSplit - 1) / kMaxEntriesPerSplit;
    const int max_splits = (entries + 63) / 64;  // at least 4 tiles per split
    if (splits > max_splits) splits = max_splits;
    if (splits < min_splits) splits = min_splits;
    if (splits < 1) splits = 1;
    int eps = (entries + splits - 1) / splits;
    eps = (eps + kTile - 1) / kTile * kTile;
    if (eps < kTile) eps = kTile;
    splits = (entries + eps - 1) / eps;
    if (splits < 1) splits = 1;
    p.n_splits = splits;
    p.entries_per_split = eps;
    // shared memory: entries | barriers | stages (the stages are reused for the merge)
    const size_t ent = ((size_t)eps * 4 + 127) / 128 * 128;
    (void)fp8;
    const size_t stage = (size_t)kTile * p.row_stride;
    const size_t bars = ((2 * (size_t)kMaxStages * 8 + 127) / 128) * 128;
    int ns = (int)((kAtSmemBudget - ent - bars - 128) / stage);
    if (ns > kMaxStages) ns = kMaxStages;
    // tile i uses stage i mod ns and the warps of wsel i mod (8 / hpc): with ns
    // a multiple of that, every use of a stage has the same warps, which saw
    // its previous phase complete before they wait on the next one
    const int n_sel = kConsumers / p.hpc;
    if (ns >= n_sel) ns = ns / n_sel * n_sel;
    p.n_stages = ns;
    p.bar_off = (int)ent;
    p.stage_off = (int)(ent + bars);
    const int NT = (H_q / H_kv + 7) / 8;
    size_t merge = (size_t)kConsumers * (NT * (kD / 16) * 4 + NT * 4) * kWarp * 4;
    size_t stages_bytes = (size_t)ns * stage;
    // groups of at most 8 query heads run the register-streaming kernel: no K stages
    if (H_q / H_kv <= 8) stages_bytes = 0;
    p.smem_bytes = p.stage_off + (stages_bytes > merge ? stages_bytes : merge);
    const size_t rows_q = (size_t)G * n_q;
    size_t ws = 256;
    if (splits > 1) {
        ws = rows_q * splits * H_q * kD * 4;
        ws = (ws + 255) / 256 * 256;
        ws += rows_q * splits * H_q * 2 * 4;
        ws = (ws + 255) / 256 * 256;
    }
    p.ws_bytes = ws;
    return p;
}

AttendPlan plan_attend_grouped(int n_q, int group_rows, int H_q, int H_kv, int budget, int G, int num_sms) {
    AttendPlan p;
    // a CTA reads whole tokens (all its kv heads, as attend_rk_kernel) for as
    // many rows of the group as its 8 warps hold
    p.hpc = H_kv < 4 ? H_kv : 4;
    p.head_groups = H_kv / p.hpc;
    p.rows_per_cta = group_rows < kConsumers / p.hpc ? group_rows : kConsumers / p.hpc;
    const int row_blocks = group_rows / p.rows_per_cta;
    const long units = (long)(n_q / group_rows) * p.head_groups * row_blocks * G;
    // one CTA per SM: the grid must not pass one wave (a few CTAs of a second
    // wave would double the call)
    int splits = units > 0 ? (int)(num_sms / units) : 1;
    const int min_splits = (budget + kMaxEntriesPerSplit - 1) / kMaxEntriesPerSplit;
    const int max_splits = (budget + 63) / 64;  // at least 4 tiles per split
    if (splits > max_splits) splits = max_splits;
    if (splits < min_splits) splits = min_splits;
    if (splits < 1) splits = 1;
    p.n_splits = splits;
    int eps = (budget + splits - 1) / splits;  // each row's entries in a split
    eps = (eps + kTile - 1) / kTile * kTile;
    p.entries_per_split = eps < kTile ? kTile : eps;
    const size_t lists = (size_t)p.rows_per_cta * p.entries_per_split * 4;
    const size_t merge = (size_t)kConsumers * ((kD / 16) * 4 + 4) * kWarp * 4;
    p.stage_off = 0;  // the merge area reuses the lists once the tiles are done
    p.smem_bytes = (lists + 127) / 128 * 128 > merge ? (lists + 127) / 128 * 128 : merge;
    const size_t rows_q = (size_t)G * n_q;
    size_t ws = 256;
    if (splits > 1) {
        ws = rows_q * splits * H_q * kD * 4;
        ws = (ws + 255) / 256 * 256;
        ws += rows_q * splits * H_q * 2 * 4;
        ws = (ws + 255) / 256 * 256;
    }
    p.ws_bytes = ws;
    return p;
}

cudaError_t launch_attend_grouped(const AttendArgs& a, size_t smem_bytes, cudaStream_t stream) {
    cudaError_t e = cudaFuncSetAttribute(attend_group_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem_bytes);
    if (e != cudaSuccess) return e;
    const int pct = (int)(((smem_bytes + 2048) * 100 + kSmemPerSm - 1) / kSmemPerSm);
    e = cudaFuncSetAttribute(attend_group_kernel, cudaFuncAttributePreferredSharedMemoryCarveout, pct < 100 ? pct : 100);
    if (e != cudaSuccess) return e;
    const dim3 grid((unsigned)(a.n_splits * a.head_groups * (a.group_rows / a.rows_per_cta)),
                    (unsigned)(a.n_q / a.group_rows), (unsigned)a.G);
    e = launch_pdl(attend_group_kernel, grid, dim3(kConsumers * kWarp), smem_bytes, stream, 0, a);
    if (e != cudaSuccess || a.n_splits == 1) return e;
    int nw = (a.n_splits + kMergeSplitsPerWarp - 1) / kMergeSplitsPerWarp;
    if (nw > kMergeMaxWarps) nw = kMergeMaxWarps;
    return launch_pdl(attend_merge_kernel, dim3((unsigned)a.H_q, (unsigned)a.n_q, (unsigned)a.G),
                      dim3((unsigned)(nw * kWarp)), 0, stream, 0, a);
}

cudaError_t launch_attend(const AttendArgs& a, size_t smem_bytes, cudaStream_t stream) {
    const int ratio = a.H_q / a.H_kv;
    dim3 grid((unsigned)(a.n_splits * a.head_groups), (unsigned)a.n_q, (unsigned)a.G);
    if (ratio <= 8) {
        auto kern = a.kv_fp8 ? attend_rk_kernel<true> : attend_rk_kernel<false>;
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_bytes);
        if (e != cudaSuccess) return e;
        // the register-streaming gather keeps its loads in flight in L1: ask
        // for the smallest shared-memory carveout that holds the CTA, so the
        // rest of the SM's 256 KB stays L1 whatever the previous kernel used
        const int pct = (int)(((smem_bytes + 2048) * 100 + kSmemPerSm - 1) / kSmemPerSm);
        e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, pct < 100 ? pct : 100);
        if (e != cudaSuccess) return e;
        e = launch_pdl(kern, grid, dim3(kConsumers * kWarp), smem_bytes, stream, 0, a);
        if (e != cudaSuccess) return e;
    } else {
        if (a.kv_fp8) return cudaErrorInvalidValue;  // FP8 caches: groups of at most 8 query heads
        cudaError_t e = cudaFuncSetAttribute(attend_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)smem_bytes);
        if (e != cudaSuccess) return e;
        e = launch_pdl(attend_kernel<2>, grid, dim3(kAtThreads), smem_bytes, stream, 0, a);
        if (e != cudaSuccess) return e;
    }
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess || a.n_splits == 1) return e;
    int nw = (a.n_splits + kMergeSplitsPerWarp - 1) / kMergeSplitsPerWarp;
    if (nw > kMergeMaxWarps) nw = kMergeMaxWarps;
    return launch_pdl(attend_merge_kernel, dim3((unsigned)a.H_q, (unsigned)a.n_q, (unsigned)a.G),
                      dim3((unsigned)(nw * kWarp)), 0, stream, 0, a);
}

}  // namespace lsa
