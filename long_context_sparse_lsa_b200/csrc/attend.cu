// attend.cu — sparse GQA softmax attention over LSA index sets, split over
// the set entries, with the split partials merged in the same launch.
//
// The method: attention runs only over the tokens the indexer selected; SI
// makes the sink and window parts contiguous KV runs ("LongCat-Flash-Lite-
// Sparse (aitrends.kr)", section "기술적 특징", SI bullet); CLI lets G
// consecutive layers reuse one index set (same section, CLI bullet).
//
// Design (B200):
//  * grid = (splits x head groups, query rows, layers). A CTA has 4 warps;
//    each warp owns one (kv head, sub-range of entries) and gathers its
//    selected 256-byte K and V rows with 16-byte cp.async into a 4-stage
//    shared-memory ring (XOR-swizzled so ldmatrix is conflict-free). Masked
//    entries are zero-filled without touching memory.
//  * S^T = K Q^T on bf16 tensor cores (mma.m16n8k16): the 16 gathered tokens
//    are the M dimension and the GQA group's query heads (8 per tile) the N
//    dimension, so no MMA row is wasted on padding.
//  * Online softmax in fp32 with exp2f and a log2(e)/sqrt(d) scale.
//  * O^T = V^T P^T: P^T is moved from the accumulator layout into the B
//    operand with movmatrix.trans; P is split into a bf16 high part and a
//    bf16 remainder (two MMAs) so it keeps ~16 significant bits, and V^T comes
//    from ldmatrix.trans.
//  * Each warp writes an unnormalised partial (m, l, o). The last CTA to
//    finish a (layer, query) — found with an atomic ticket, never a wait —
//    merges the partials with the log-sum-exp rule and resets the ticket.
#include "common.cuh"
#include "internal.h"

namespace lsa {
namespace {

constexpr int kAtThreads = 128;
constexpr int kAtWarps = 4;
constexpr int kTile = 16;       // tokens per pipeline stage
constexpr int kStages = 4;
constexpr int kRowBytes = 256;  // one (token, kv head) row at d = 128
constexpr int kD = 128;
constexpr int kStageBytes = 2 * kTile * kRowBytes;  // K and V
constexpr int kWarpSmem = kStages * kStageBytes;
constexpr int kAtSmem = kAtWarps * kWarpSmem;

// Byte offset of 16-byte chunk c of row r inside a [16 rows][256 B] tile.
__device__ __forceinline__ uint32_t swz(int r, int c) { return (uint32_t)(r * kRowBytes + ((c ^ (r & 7)) << 4)); }

template <int NT>
__global__ void __launch_bounds__(kAtThreads) attend_kernel(const __grid_constant__ AttendArgs a) {
    extern __shared__ __align__(128) uint8_t smem[];
    __shared__ uint32_t s_last;

    const int lane = lane_id(), wid = warp_id();
    const int g = lane >> 2, t4 = lane & 3;
    const int split = blockIdx.x / a.head_groups;
    const int hgrp = blockIdx.x % a.head_groups;
    const int r = blockIdx.y;
    const int layer = blockIdx.z;
    const int ratio = a.H_q / a.H_kv;
    const int heads_per_cta = kAtWarps / a.wph;
    const int kvh = hgrp * heads_per_cta + wid / a.wph;
    const int sub = wid % a.wph;
    const int n_parts = a.n_splits * a.wph;
    const int part = split * a.wph + sub;

    // ---- query row validation ----
    const int seq = a.q_seq[r];
    const int L = a.q_len[r];
    bool bad = seq < 0 || seq >= a.n_seq;
    int64_t off = 0;
    if (!bad) {
        off = a.kv_offset[seq];
        const int slen = a.seq_lens[seq];
        bad = L < 1 || L > a.max_len || L > slen || off < 0 || off + slen > a.total_tokens;
    }
    if (bad && threadIdx.x == 0 && blockIdx.x == 0 && layer == 0)
        flag(a.dev_status, seq < 0 || seq >= a.n_seq ? LSA_DEV_BAD_SEQ : LSA_DEV_BAD_LENGTH);
    const bool warp_live = !bad && kvh < a.H_kv;

    // entries of this warp
    const int n_entries = bad ? 0 : min(L, a.budget);
    const int per_sub = a.entries_per_split / a.wph;
    const int e_begin = split * a.entries_per_split + sub * per_sub;
    const int e_end = warp_live ? min(n_entries, e_begin + per_sub) : e_begin;
    const int32_t* set = a.sets + (int64_t)r * a.budget;

    const uint16_t* kbase = a.k[layer] + (off * a.H_kv + kvh) * kD;
    const uint16_t* vbase = a.v[layer] + (off * a.H_kv + kvh) * kD;
    const int64_t tok_stride = (int64_t)a.H_kv * kD;  // elements between consecutive tokens

    uint8_t* wsm = smem + wid * kWarpSmem;
    const uint32_t wsm_u32 = smem_u32(wsm);

    // ---- query fragments (B operand of S^T = K Q^T) ----
    uint32_t qb[NT][kD / 16][2];
    {
        const uint16_t* qrow = a.q[layer] + ((int64_t)r * a.H_q + (int64_t)kvh * ratio) * kD;
#pragma unroll
        for (int n = 0; n < NT; ++n) {
            const int hh = 8 * n + g;
            const bool ok = warp_live && hh < ratio;
#pragma unroll
            for (int ks = 0; ks < kD / 16; ++ks) {
                uint32_t b0 = 0, b1 = 0;
                if (ok) {
                    b0 = __ldg(reinterpret_cast<const uint32_t*>(qrow + hh * kD + 16 * ks + 2 * t4));
                    b1 = __ldg(reinterpret_cast<const uint32_t*>(qrow + hh * kD + 16 * ks + 8 + 2 * t4));
                }
                qb[n][ks][0] = b0;
                qb[n][ks][1] = b1;
            }
        }
    }

    // ---- gather pipeline ----
    // Entry of tile i, row j (j = lane for lanes < 16): token position or -1.
    auto fetch_entry = [&](int e) -> int {
        if (e >= e_end) return -1;
        const int idx = set[e];
        if (idx < -1 || idx >= L) {
            flag(a.dev_status, LSA_DEV_BAD_INDEX);
            return -1;
        }
        return idx;
    };
    const int n_tiles = e_end > e_begin ? (e_end - e_begin + kTile - 1) / kTile : 0;
    auto issue = [&](int tile, int stage) {
        // lane < 16 holds the token of row `lane`
        const int my_tok = lane < kTile ? fetch_entry(e_begin + tile * kTile + lane) : -1;
        const uint32_t kst = wsm_u32 + stage * kStageBytes;
        const uint32_t vst = kst + kTile * kRowBytes;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int c = lane + 32 * j;  // chunk id in [0, 256): row = c / 16, chunk-in-row = c % 16
            const int row = c >> 4, cir = c & 15;
            const int tok = __shfl_sync(0xffffffffu, my_tok, row);
            const bool ok = tok >= 0;
            const int64_t eo = ok ? (int64_t)tok * tok_stride + cir * 8 : 0;
            cp_async16(kst + swz(row, cir), kbase + eo, ok ? 16u : 0u);
            cp_async16(vst + swz(row, cir), vbase + eo, ok ? 16u : 0u);
        }
        return (uint64_t)__ballot_sync(0xffffffffu, lane < kTile && my_tok >= 0);  // valid rows
    };

    float o[NT][kD / 16][4];
#pragma unroll
    for (int n = 0; n < NT; ++n)
#pragma unroll
        for (int mt = 0; mt < kD / 16; ++mt) o[n][mt][0] = o[n][mt][1] = o[n][mt][2] = o[n][mt][3] = 0.f;
    float m_run[NT][2], l_run[NT][2];
#pragma unroll
    for (int n = 0; n < NT; ++n) {
        m_run[n][0] = m_run[n][1] = -INFINITY;
        l_run[n][0] = l_run[n][1] = 0.f;
    }

    // bits [16 s, 16 s + 16) of vmask: valid rows of pipeline stage s
    uint64_t vmask = 0;
#pragma unroll
    for (int st = 0; st < kStages - 1; ++st) {
        if (st < n_tiles) vmask |= issue(st, st) << (16 * st);
        cp_async_commit();
    }

    for (int tile = 0; tile < n_tiles; ++tile) {
        const int stage = tile % kStages;
        {
            const int nt = tile + kStages - 1;
            if (nt < n_tiles) {
                const int ns = nt % kStages;
                const uint64_t m = issue(nt, ns);
                vmask = (vmask & ~(0xFFFFull << (16 * ns))) | (m << (16 * ns));
            }
            cp_async_commit();
        }
        cp_async_wait<kStages - 1>();
        __syncwarp();
        const uint32_t kst = wsm_u32 + stage * kStageBytes;
        const uint32_t vst = kst + kTile * kRowBytes;
        const uint32_t rows_ok = (uint32_t)(vmask >> (16 * stage)) & 0xFFFFu;
        const bool ok_g = (rows_ok >> g) & 1u;
        const bool ok_g8 = (rows_ok >> (g + 8)) & 1u;

        // S^T tile: 16 tokens x (8 * NT) heads
        float sacc[NT][4];
#pragma unroll
        for (int n = 0; n < NT; ++n) sacc[n][0] = sacc[n][1] = sacc[n][2] = sacc[n][3] = 0.f;
#pragma unroll
        for (int ks = 0; ks < kD / 16; ++ks) {
            const int mi = lane >> 3, rr = lane & 7;
            const int row = rr + 8 * (mi & 1);
            const int chunk = 2 * ks + (mi >> 1);
            uint32_t afr[4];
            ldmatrix_x4(afr, kst + swz(row, chunk));
#pragma unroll
            for (int n = 0; n < NT; ++n) mma_bf16(sacc[n], afr, qb[n][ks][0], qb[n][ks][1]);
        }
        // online softmax (log2 domain)
        uint32_t phi[NT][2], plo[NT][2];
#pragma unroll
        for (int n = 0; n < NT; ++n) {
            float z0 = ok_g ? sacc[n][0] * a.scale_log2 : -INFINITY;   // (tok g,   head 2t)
            float z1 = ok_g ? sacc[n][1] * a.scale_log2 : -INFINITY;   // (tok g,   head 2t+1)
            float z2 = ok_g8 ? sacc[n][2] * a.scale_log2 : -INFINITY;  // (tok g+8, head 2t)
            float z3 = ok_g8 ? sacc[n][3] * a.scale_log2 : -INFINITY;  // (tok g+8, head 2t+1)
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
            m_run[n][0] = mn0;
            m_run[n][1] = mn1;
            l_run[n][0] = l_run[n][0] * al0 + p0 + p2;
            l_run[n][1] = l_run[n][1] * al1 + p1 + p3;
#pragma unroll
            for (int mt = 0; mt < kD / 16; ++mt) {
                o[n][mt][0] *= al0;
                o[n][mt][1] *= al1;
                o[n][mt][2] *= al0;
                o[n][mt][3] *= al1;
            }
            // P split into bf16 high part + bf16 remainder; transpose into B fragments.
            const __nv_bfloat162 h01 = __floats2bfloat162_rn(p0, p1);
            const __nv_bfloat162 h23 = __floats2bfloat162_rn(p2, p3);
            const float2 fh01 = __bfloat1622float2(h01), fh23 = __bfloat1622float2(h23);
            const uint32_t l01 = pack_bf16(p0 - fh01.x, p1 - fh01.y);
            const uint32_t l23 = pack_bf16(p2 - fh23.x, p3 - fh23.y);
            phi[n][0] = movmatrix_trans(*reinterpret_cast<const uint32_t*>(&h01));
            phi[n][1] = movmatrix_trans(*reinterpret_cast<const uint32_t*>(&h23));
            plo[n][0] = movmatrix_trans(l01);
            plo[n][1] = movmatrix_trans(l23);
        }
        // O^T += V^T P^T
#pragma unroll
        for (int mt = 0; mt < kD / 16; ++mt) {
            const int mi = lane >> 3, rr = lane & 7;
            const int row = rr + 8 * (mi >> 1);
            const int chunk = 2 * mt + (mi & 1);
            uint32_t vfr[4];
            ldmatrix_x4_trans(vfr, vst + swz(row, chunk));
#pragma unroll
            for (int n = 0; n < NT; ++n) {
                mma_bf16(o[n][mt], vfr, phi[n][0], phi[n][1]);
                mma_bf16(o[n][mt], vfr, plo[n][0], plo[n][1]);
            }
        }
        __syncwarp();  // the stage is refilled on the next iteration
    }
    cp_async_wait<0>();

    // ---- finish this warp's partial ----
#pragma unroll
    for (int n = 0; n < NT; ++n)
#pragma unroll
        for (int j = 0; j < 2; ++j)
#pragma unroll
            for (int msk = 4; msk < 32; msk <<= 1) l_run[n][j] += __shfl_xor_sync(0xffffffffu, l_run[n][j], msk);

    const int64_t row_q = (int64_t)layer * a.n_q + r;
    if (warp_live) {
        if (n_parts == 1) {
            float* orow = a.out[layer] + ((int64_t)r * a.H_q + (int64_t)kvh * ratio) * kD;
#pragma unroll
            for (int n = 0; n < NT; ++n) {
                const int h0 = 8 * n + 2 * t4, h1 = h0 + 1;
                const float i0 = l_run[n][0] > 0.f ? 1.f / l_run[n][0] : 0.f;
                const float i1 = l_run[n][1] > 0.f ? 1.f / l_run[n][1] : 0.f;
#pragma unroll
                for (int mt = 0; mt < kD / 16; ++mt) {
                    const int d0 = 16 * mt + g, d1 = d0 + 8;
                    if (h0 < ratio) {
                        orow[h0 * kD + d0] = o[n][mt][0] * i0;
                        orow[h0 * kD + d1] = o[n][mt][2] * i0;
                    }
                    if (h1 < ratio) {
                        orow[h1 * kD + d0] = o[n][mt][1] * i1;
                        orow[h1 * kD + d1] = o[n][mt][3] * i1;
                    }
                }
            }
        } else {
            const int64_t pbase = (row_q * n_parts + part) * a.H_q + (int64_t)kvh * ratio;
            float* po = a.part_o + pbase * kD;
            float* pml = a.part_ml + pbase * 2;
#pragma unroll
            for (int n = 0; n < NT; ++n) {
                const int h0 = 8 * n + 2 * t4, h1 = h0 + 1;
#pragma unroll
                for (int mt = 0; mt < kD / 16; ++mt) {
                    const int d0 = 16 * mt + g, d1 = d0 + 8;
                    if (h0 < ratio) {
                        po[h0 * kD + d0] = o[n][mt][0];
                        po[h0 * kD + d1] = o[n][mt][2];
                    }
                    if (h1 < ratio) {
                        po[h1 * kD + d0] = o[n][mt][1];
                        po[h1 * kD + d1] = o[n][mt][3];
                    }
                }
                if (g == 0) {
                    if (h0 < ratio) {
                        pml[h0 * 2] = m_run[n][0];
                        pml[h0 * 2 + 1] = l_run[n][0];
                    }
                    if (h1 < ratio) {
                        pml[h1 * 2] = m_run[n][1];
                        pml[h1 * 2 + 1] = l_run[n][1];
                    }
                }
            }
        }
    }
    if (n_parts == 1 || bad) {
        if (bad) {
            // zero this CTA's heads so the output is defined
            for (int i = threadIdx.x; i < heads_per_cta * ratio * kD; i += kAtThreads) {
                const int hh = hgrp * heads_per_cta * ratio + i / kD;
                if (hh < a.H_q && split == 0) a.out[layer][((int64_t)r * a.H_q + hh) * kD + i % kD] = 0.f;
            }
        }
        return;
    }

    // ---- last-arriving CTA of this (layer, row) merges ----
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) {
        const uint32_t total = (uint32_t)(a.n_splits * a.head_groups);
        const uint32_t prev = atomicAdd(&a.counters[row_q], 1u);
        s_last = (prev == total - 1) ? 1u : 0u;
    }
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    float* orow = a.out[layer] + (int64_t)r * a.H_q * kD;
    const float* po = a.part_o + row_q * n_parts * a.H_q * kD;
    const float* pml = a.part_ml + row_q * n_parts * a.H_q * 2;
    for (int hd = threadIdx.x; hd < a.H_q * kD; hd += kAtThreads) {
        const int h = hd / kD;
        float M = -INFINITY;
        for (int p = 0; p < n_parts; ++p) M = fmaxf(M, __ldcg(pml + ((int64_t)p * a.H_q + h) * 2));
        float acc = 0.f, den = 0.f;
        if (M != -INFINITY) {
            for (int p = 0; p < n_parts; ++p) {
                const float mp = __ldcg(pml + ((int64_t)p * a.H_q + h) * 2);
                const float wgt = exp2f(mp - M);
                den += wgt * __ldcg(pml + ((int64_t)p * a.H_q + h) * 2 + 1);
                acc += wgt * __ldcg(po + ((int64_t)p * a.H_q) * kD + hd);
            }
        }
        orow[hd] = den > 0.f ? acc / den : 0.f;
    }
    if (threadIdx.x == 0) a.counters[row_q] = 0u;
}

}  // namespace

AttendPlan plan_attend(int n_q, int max_len, int H_q, int H_kv, int d, int budget, int G, int num_sms) {
    AttendPlan p;
    (void)d;
    p.wph = H_kv >= kAtWarps ? 1 : kAtWarps / H_kv;
    p.head_groups = H_kv >= kAtWarps ? H_kv / kAtWarps : 1;
    const int entries = budget < max_len ? budget : max_len;
    const long rows = (long)n_q * G * p.head_groups;
    int splits = rows > 0 ? (int)((num_sms + rows / 2) / rows) : 1;
    if (splits < 1) splits = 1;
    const int gran = kTile * p.wph;
    const int max_splits = (entries + 4 * gran - 1) / (4 * gran);  // >= 64 entries per warp
    if (splits > max_splits) splits = max_splits < 1 ? 1 : max_splits;
    int eps = (entries + splits - 1) / splits;
    eps = (eps + gran - 1) / gran * gran;
    if (eps < gran) eps = gran;
    splits = (entries + eps - 1) / eps;
    if (splits < 1) splits = 1;
    p.n_splits = splits;
    p.entries_per_split = eps;
    const size_t n_parts = (size_t)splits * p.wph;
    const size_t rows_q = (size_t)G * n_q;
    size_t ws = (rows_q * 4 + 255) / 256 * 256;  // counters first
    if (n_parts > 1) {
        ws += rows_q * n_parts * H_q * 128 * 4;
        ws = (ws + 255) / 256 * 256;
        ws += rows_q * n_parts * H_q * 2 * 4;
    }
    p.ws_bytes = ws;
    return p;
}

cudaError_t launch_attend(const AttendArgs& a, cudaStream_t stream) {
    const int ratio = a.H_q / a.H_kv;
    dim3 grid((unsigned)(a.n_splits * a.head_groups), (unsigned)a.n_q, (unsigned)a.G);
    if (ratio <= 8) {
        cudaError_t e = cudaFuncSetAttribute(attend_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, kAtSmem);
        if (e != cudaSuccess) return e;
        attend_kernel<1><<<grid, kAtThreads, kAtSmem, stream>>>(a);
    } else {
        cudaError_t e = cudaFuncSetAttribute(attend_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, kAtSmem);
        if (e != cudaSuccess) return e;
        attend_kernel<2><<<grid, kAtThreads, kAtSmem, stream>>>(a);
    }
    return cudaGetLastError();
}

}  // namespace lsa
