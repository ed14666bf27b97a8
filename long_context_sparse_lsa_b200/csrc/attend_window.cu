// attend_window.cu — the sink and window part of lsa_attend_si for the rows
// of a prefill chunk, as a dense tile contraction shared by neighbouring rows.
//
// The method: every row's index set keeps the sink run [0, s) and the local
// window [ws, L) besides its selected tokens ("LongCat-Flash-Lite-Sparse
// (aitrends.kr)", section "기술적 특징", SI bullet), and the attention is the
// softmax over all of them ("LongCat-2.0 (molayo1419.me)", section "1M 토큰에서의
// Sparse Attention 문제"). Rows i and i + 1 of a causal chunk see windows that
// differ by one position, so 16 consecutive rows read the same sink run and
// windows spanning window + 15 positions: one K/V tile in shared memory serves
// all of them. attend_rk_kernel attends each row over its selected entries
// only and leaves its normalised output and log-sum-exp; this kernel attends
// the rows over their sink and window runs and combines the two partials.
//
// Design: one CTA of 8 warps per (16 consecutive rows, kv head, layer), two
// CTAs per SM (128 registers). K and V tiles of 16 positions (the kv head's
// 256-byte rows, padded to 272 bytes so fragment loads are conflict free)
// stream through a 4-stage shared-memory ring filled by 16-byte cp.async
// copies from all threads (positions outside the runs are zero-filled). Warp
// w takes rows 2w and 2w + 1 of the CTA with the group's query heads as the
// 16 rows of an m16n8k16 MMA (its Q rows staged in shared memory, read as
// ldmatrix fragments): S = Q K^T from the tile's K rows (ldmatrix; even and
// odd k-steps in separate accumulators), a mask per (row, position), online
// softmax in fp32, and O += P V in fp16: each V tile is converted from bf16
// to fp16 once in shared memory (exact for magnitudes below 65520, else
// LSA_DEV_BAD_VALUE), and P in fp16 keeps 11 significant bits, so one MMA
// does what the gather kernel's bf16 high part and remainder do in two.
#include "common.cuh"
#include "internal.h"

namespace lsa {
namespace {

constexpr int kWinRows = 16;                 // query rows per CTA (2 per warp)
constexpr int kWinWarps = kWinRows / 2;
constexpr int kWinThreads = kWinWarps * kWarp;
constexpr int kWinTile = 16;                 // positions per K/V tile
constexpr int kWinStages = 4;
constexpr int kWinRow = 128 * 2 + 16;        // bytes of one staged (position, kv head) row
constexpr int kWinStageBytes = 2 * kWinTile * kWinRow;  // K rows then V rows
constexpr int kD = 128;

// Tile t's V rows from bf16 to fp16 in place, one 16-byte chunk per thread:
// every bf16 of magnitude below 65520 is an fp16 (subnormal below 2^-14), so
// P V can run with P in fp16 (11 significant bits: one MMA instead of a bf16
// pair); returns false if an element does not fit.
__device__ __forceinline__ bool v_to_f16(uint8_t* vtile, int tid) {
    bool fits = true;
    for (int c = tid; c < kWinTile * 16; c += kWinThreads) {
        uint4* p = reinterpret_cast<uint4*>(vtile + (c / 16) * kWinRow + 16 * (c % 16));
        uint4 x = *p;
        uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[i]));
            const uint32_t h = pack_f16(f.x, f.y);
            fits &= (h & 0x7c00u) != 0x7c00u && ((h >> 16) & 0x7c00u) != 0x7c00u;
            w[i] = h;
        }
        *p = make_uint4(w[0], w[1], w[2], w[3]);
    }
    return fits;
}

__global__ void __launch_bounds__(kWinThreads, 2) attend_window_kernel(const __grid_constant__ AttendArgs a) {
    extern __shared__ __align__(128) uint8_t win_dyn[];
    uint8_t* ring = win_dyn;                                        // kWinStages x (K tile, V tile)
    uint8_t* s_qall = win_dyn + kWinStages * kWinStageBytes;        // each warp's 16 MMA rows of Q
    __shared__ int32_t s_L[kWinRows], s_s[kWinRows], s_ws[kWinRows];
    __shared__ int32_t s_span[3];  // sink run end, window runs start, end (over the CTA's rows)
    const int tid = threadIdx.x, lane = lane_id(), warp = warp_id();
    const int g = lane >> 2, t4 = lane & 3;
    const int r0 = blockIdx.x * kWinRows;
    const int kvh = blockIdx.y, layer = blockIdx.z;
    const int ratio = a.H_q / a.H_kv;
    const int64_t off = a.kv_offset[0];
    const int slen = a.seq_lens[0];
    // the rows' metadata (the caller's) before the wait for the selected part
    if (tid < kWinRows) {
        const int r = r0 + tid;
        int L = 0;
        if (r < a.n_q) {
            const int Lr = a.q_len[r];
            const bool ok = a.q_seq[r] == 0 && Lr >= 1 && Lr <= a.max_len && Lr <= slen && off >= 0 &&
                            off + slen <= a.total_tokens;
            L = ok ? Lr : 0;  // an invalid row attends nothing here (the gather kernel zeroed and flagged it)
        }
        const int s = min(a.si_sink, L);
        s_L[tid] = L;
        s_s[tid] = s;
        s_ws[tid] = max(s, L - a.si_window);
    }
    __syncthreads();
    if (tid == 0) {
        int s_max = 0, ws_min = 0x7fffffff, l_max = 0;
        for (int i = 0; i < kWinRows; ++i) {
            if (s_L[i] <= 0) continue;
            s_max = max(s_max, s_s[i]);
            if (s_L[i] > s_ws[i]) {
                ws_min = min(ws_min, s_ws[i]);
                l_max = max(l_max, s_L[i]);
            }
        }
        const int b0 = max(ws_min, s_max);
        s_span[0] = s_max;
        s_span[1] = l_max > b0 ? b0 : s_max;
        s_span[2] = l_max > b0 ? l_max : s_max;
    }
    pdl_enter();
    __syncthreads();
    const int a_end = s_span[0], b_lo = s_span[1], b_hi = s_span[2];
    const int n_a = (a_end + kWinTile - 1) / kWinTile;
    const int n_t = n_a + (b_hi - b_lo + kWinTile - 1) / kWinTile;
    auto tile_base = [&](int t) { return t < n_a ? t * kWinTile : b_lo + (t - n_a) * kWinTile; };
    auto tile_end = [&](int t) { return t < n_a ? a_end : b_hi; };

    // stage tile t: 16 positions x (K row, V row) of this kv head, 16 bytes a copy
    const uint16_t* kg = a.k[layer] + (off * a.H_kv + kvh) * kD;
    const uint16_t* vg = a.v[layer] + (off * a.H_kv + kvh) * kD;
    const int64_t tok = (int64_t)a.H_kv * kD;
    auto stage = [&](int t) {
        if (t < n_t) {
            const int pb = tile_base(t), pe = tile_end(t);
            const uint32_t sb = smem_u32(ring + (t % kWinStages) * kWinStageBytes);
            for (int c = tid; c < 2 * kWinTile * 16; c += kWinThreads) {
                const int kv = c / (kWinTile * 16), rem = c % (kWinTile * 16);
                const int j = rem / 16, ch = rem % 16;  // position j of the tile, 16-byte chunk ch
                const int p = pb + j;
                const bool in = p < pe;
                const uint16_t* src = (kv ? vg : kg) + (int64_t)(in ? p : pb) * tok + 8 * ch;
                cp_async16(sb + (uint32_t)(kv * kWinTile * kWinRow + j * kWinRow + 16 * ch), src, in ? 16u : 0u);
            }
        }
        cp_async_commit();
    };
    for (int t = 0; t < kWinStages - 1; ++t) stage(t);

    // the warp's 16 MMA rows: rows 2w (m < 8) and 2w + 1 (m >= 8) of the CTA,
    // query head m % 8 of the kv head's group (heads >= ratio are zero)
    const int ra = 2 * warp, rb = ra + 1;
    const int La = s_L[ra], sa = s_s[ra], wsa = s_ws[ra];
    const int Lb = s_L[rb], sb_ = s_s[rb], wsb = s_ws[rb];
    // the warp's Q rows into shared memory (MMA row m: row 2w + m / 8, head m % 8),
    // read back per k-step as ldmatrix A fragments
    {
        uint8_t* qs = s_qall + warp * 16 * kWinRow;
        for (int c = lane; c < 16 * 16; c += kWarp) {  // 16 rows x 16 chunks of 16 bytes
            const int m = c / 16, ch = c % 16;
            const int rl = ra + (m >> 3), h = m & 7;
            const bool ok = h < ratio && s_L[rl] > 0;
            uint4 v = make_uint4(0u, 0u, 0u, 0u);
            if (ok)
                v = __ldg(reinterpret_cast<const uint4*>(
                    a.q[layer] + ((int64_t)(r0 + rl) * a.H_q + (int64_t)kvh * ratio + h) * kD) + ch);
            *reinterpret_cast<uint4*>(qs + m * kWinRow + 16 * ch) = v;
        }
        __syncwarp();
    }
    // lane l addresses row (l & 7) + 8 ((l >> 3) & 1), 16-byte column (l >> 4)
    // of each k-step's 16 x 16 block: the four 8 x 8 matrices of the A fragment
    const uint32_t qrow = smem_u32(s_qall + warp * 16 * kWinRow) + (uint32_t)(((lane & 7) + 8 * ((lane >> 3) & 1)) * kWinRow + 16 * (lane >> 4));
    // and for K: matrices (positions 0-7 | 8-15) x (dims lo | hi) of a k-step
    const uint32_t krow_off = (uint32_t)(((lane & 7) + 8 * (lane >> 4)) * kWinRow + 16 * ((lane >> 3) & 1));
    float o[kD / 8][4];
#pragma unroll
    for (int j = 0; j < kD / 8; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
    float mA = -INFINITY, mB = -INFINITY, lA = 0.f, lB = 0.f;
    const float sl2 = a.scale_log2;

    bool v_fits = true;
    if (n_t > 0) {
        cp_async_wait<kWinStages - 2>();
        __syncthreads();
        v_fits &= v_to_f16(ring + kWinTile * kWinRow, tid);  // tile 0's V rows
    }
    for (int t = 0; t < n_t; ++t) {
        // tiles t and t + 1 have landed for every thread, tile t's V rows are
        // fp16 (converted an iteration ago), tile t - 1 is no longer read
        cp_async_wait<kWinStages - 3>();
        __syncthreads();
        if (t + 1 < n_t) v_fits &= v_to_f16(ring + ((t + 1) % kWinStages) * kWinStageBytes + kWinTile * kWinRow, tid);
        stage(t + kWinStages - 1);       // into the stage tile t - 1 used
        const uint8_t* st = ring + (t % kWinStages) * kWinStageBytes;
        const uint32_t kbase = smem_u32(st), vbase = smem_u32(st + kWinTile * kWinRow);
        const int pb = tile_base(t), pe = tile_end(t);
        // S = Q K^T: two n-tiles of 8 positions, even and odd k-steps in
        // separate accumulators (four independent MMA chains)
        float sacc[2][4], sodd[2][4];
#pragma unroll
        for (int n = 0; n < 2; ++n)
#pragma unroll
            for (int c = 0; c < 4; ++c) sacc[n][c] = sodd[n][c] = 0.f;
#pragma unroll
        for (int ks = 0; ks < kD / 16; ++ks) {
            uint32_t qa[4], kb[4];
            ldmatrix_x4(qa, qrow + (uint32_t)(32 * ks));
            ldmatrix_x4(kb, kbase + krow_off + (uint32_t)(32 * ks));
            mma_16<false>((ks & 1) ? sodd[0] : sacc[0], qa, kb[0], kb[1]);
            mma_16<false>((ks & 1) ? sodd[1] : sacc[1], qa, kb[2], kb[3]);
        }
#pragma unroll
        for (int n = 0; n < 2; ++n)
#pragma unroll
            for (int c = 0; c < 4; ++c) sacc[n][c] += sodd[n][c];
        // mask: row A holds positions [0, sa) and [wsa, La), row B likewise
        float z[2][4];
#pragma unroll
        for (int n = 0; n < 2; ++n) {
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                const int p = pb + 8 * n + 2 * t4 + c;
                const bool inb = p < pe;
                const bool okA = inb && (p < sa || (p >= wsa && p < La));
                const bool okB = inb && (p < sb_ || (p >= wsb && p < Lb));
                z[n][c] = okA ? sacc[n][c] * sl2 : -INFINITY;
                z[n][2 + c] = okB ? sacc[n][2 + c] * sl2 : -INFINITY;
            }
        }
        float xA = fmaxf(fmaxf(z[0][0], z[0][1]), fmaxf(z[1][0], z[1][1]));
        float xB = fmaxf(fmaxf(z[0][2], z[0][3]), fmaxf(z[1][2], z[1][3]));
#pragma unroll
        for (int msk = 1; msk < 4; msk <<= 1) {
            xA = fmaxf(xA, __shfl_xor_sync(0xffffffffu, xA, msk));
            xB = fmaxf(xB, __shfl_xor_sync(0xffffffffu, xB, msk));
        }
        const float nA = fmaxf(mA, xA), nB = fmaxf(mB, xB);
        const float bA = nA == -INFINITY ? 0.f : nA, bB = nB == -INFINITY ? 0.f : nB;
        const float alA = exp2f(mA - bA), alB = exp2f(mB - bB);
        float p[2][4];
#pragma unroll
        for (int n = 0; n < 2; ++n) {
            p[n][0] = exp2f(z[n][0] - bA);
            p[n][1] = exp2f(z[n][1] - bA);
            p[n][2] = exp2f(z[n][2] - bB);
            p[n][3] = exp2f(z[n][3] - bB);
        }
        lA = lA * alA + p[0][0] + p[0][1] + p[1][0] + p[1][1];
        lB = lB * alB + p[0][2] + p[0][3] + p[1][2] + p[1][3];
        if (__any_sync(0xffffffffu, nA != mA || nB != mB)) {
#pragma unroll
            for (int j = 0; j < kD / 8; ++j) {
                o[j][0] *= alA;
                o[j][1] *= alA;
                o[j][2] *= alB;
                o[j][3] *= alB;
            }
        }
        mA = nA;
        mB = nB;
        // P as the A operand (the two n-tiles' accumulators are the k16
        // fragment), in fp16: p in [0, 1] keeps 11 significant bits
        const uint32_t ph[4] = {pack_f16(p[0][0], p[0][1]), pack_f16(p[0][2], p[0][3]), pack_f16(p[1][0], p[1][1]),
                                pack_f16(p[1][2], p[1][3])};
        // O += P V: the tile's fp16 V rows (positions) x dims through
        // ldmatrix.trans, two n-tiles of 8 dims per load
        const uint32_t vrow = vbase + (uint32_t)(((lane & 7) + 8 * ((lane >> 3) & 1)) * kWinRow + 16 * (lane >> 4));
#pragma unroll
        for (int j = 0; j < kD / 8; j += 2) {
            uint32_t vb[4];
            ldmatrix_x4_trans(vb, vrow + (uint32_t)(16 * j));
            mma_16<true>(o[j], ph, vb[0], vb[1]);
            mma_16<true>(o[j + 1], ph, vb[2], vb[3]);
        }
    }
    cp_async_wait<0>();
    if (!v_fits) flag(a.dev_status, LSA_DEV_BAD_VALUE);

    // the rows' denominators over their quad, then the window part's lse and
    // its combination with the selected part (attend_rk_kernel's output and
    // lse for the same row and head)
#pragma unroll
    for (int msk = 1; msk < 4; msk <<= 1) {
        lA += __shfl_xor_sync(0xffffffffu, lA, msk);
        lB += __shfl_xor_sync(0xffffffffu, lB, msk);
    }
    if (g >= ratio) return;
#pragma unroll
    for (int half = 0; half < 2; ++half) {
        const int rl = half ? rb : ra;
        const int r = r0 + rl;
        if (s_L[rl] <= 0) continue;  // invalid or past the batch: left as the gather kernel wrote it
        const float m = half ? mB : mA, l = half ? lB : lA;
        const int64_t qh = (int64_t)kvh * ratio + g;
        float* out = a.out[layer] + ((int64_t)r * a.H_q + qh) * kD;
        float* lse_sel = a.lse[layer] + (int64_t)r * a.H_q + qh;
        const float ls = *lse_sel;  // ln of the selected part's denominator (-inf: none)
        const float lw = l > 0.f ? (m + log2f(l)) * 0.6931471805599453f : -INFINITY;
        const float M = fmaxf(ls, lw);
        const float ws = ls == -INFINITY ? 0.f : expf(ls - M);
        const float ww = lw == -INFINITY ? 0.f : expf(lw - M);
        const float den = ws + ww;
        const float inv = den > 0.f ? 1.f / den : 0.f;
        const float cw = l > 0.f ? ww / l * inv : 0.f;  // the window part's O is unnormalised
        const float cs = ws * inv;
#pragma unroll
        for (int j = 0; j < kD / 8; ++j) {
            float2* dst = reinterpret_cast<float2*>(out + 8 * j + 2 * t4);
            const float2 osel = *dst;
            const float ox = o[j][half ? 2 : 0], oy = o[j][half ? 3 : 1];
            *dst = make_float2(cs * osel.x + cw * ox, cs * osel.y + cw * oy);
        }
    }
}

}  // namespace

cudaError_t launch_attend_window(const AttendArgs& a, cudaStream_t stream) {
    constexpr size_t smem = (size_t)kWinStages * kWinStageBytes + (size_t)kWinWarps * 16 * kWinRow;
    cudaError_t e = cudaFuncSetAttribute(attend_window_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const dim3 grid((unsigned)((a.n_q + kWinRows - 1) / kWinRows), (unsigned)a.H_kv, (unsigned)a.G);
    return launch_pdl(attend_window_kernel, grid, dim3(kWinThreads), smem, stream, 0, a);
}

}  // namespace lsa
