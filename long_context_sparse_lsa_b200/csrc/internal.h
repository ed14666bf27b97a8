// internal.h — argument blocks and launchers shared between the C-ABI layer
// (abi.cu) and the kernel translation units. Host and device code only.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "../../include/lsa.h"

namespace lsa {

constexpr int kMaxLayers = LSA_MAX_LAYERS;

// ---- HI block sums --------------------------------------------------------
struct BlockSumArgs {
    const int8_t* k_idx;
    int8_t* block_sums;
    const int64_t* kv_offset;
    const int32_t* seq_lens;
    const int64_t* blk_offset;
    int32_t* dev_status;
    int64_t total_tokens;
    int64_t block_rows;
    int32_t n_seq;
    int32_t max_len;
    int32_t hi_block;
    int32_t n_new;           // <= 0: every block
    int32_t blocks_per_seq;  // grid coverage along x (blocks of one sequence)
};
cudaError_t launch_block_sums(const BlockSumArgs& a, int d_I, cudaStream_t stream);

// Decode append: the n_new newest tokens of every sequence receive their
// indexer key and per-layer K/V rows, and (HI on) the block sums of their
// blocks are recomputed, in one launch.
struct AppendArgs {
    BlockSumArgs bs;               // k_idx: the cache being written; n_new > 0
    const int8_t* k_idx_new;       // [n_seq][n_new][d_I]
    int8_t* k_idx_cache;           // == bs.k_idx
    const void* k_new[kMaxLayers];  // [n_seq][n_new] rows of kv_row_bytes, per layer
    const void* v_new[kMaxLayers];
    void* k_cache[kMaxLayers];      // [total_tokens] rows of kv_row_bytes, per layer
    void* v_cache[kMaxLayers];
    int32_t layers;
    int32_t kv_row_bytes;          // one token's K (or V) row of one layer
    int32_t sums;                  // 1: recompute the block sums (HI on)
};
cudaError_t launch_append(const AppendArgs& a, int d_I, cudaStream_t stream);
constexpr int kAppendRowsPerCta = 64;  // HI off: new tokens per append CTA
// CTAs per sequence and role of the decode append: with HI on, the blocks that
// the n_new newest tokens can fall in; otherwise runs of kAppendRowsPerCta.
__host__ __device__ __forceinline__ int append_ctas_per_seq(int n_new, int hi_block, int max_len) {
    if (hi_block > 0) {
        const int64_t full = ((int64_t)max_len + hi_block - 1) / hi_block;
        const int64_t cover = ((int64_t)n_new + hi_block - 1) / hi_block + 1;
        return (int)(cover < full ? cover : full);
    }
    return (n_new + kAppendRowsPerCta - 1) / kAppendRowsPerCta;
}

// ---- indexer: scoring kernels + selection kernels -------------------------
// Keys (score + 1) are histogrammed on a monotone logarithmic scale: the bit
// length of the key and the 6 bits after its leading one (keys below 64 map
// to themselves). 3776 bins cover every 64-bit key.
constexpr int kHistBins = 4096;
__host__ __device__ __forceinline__ uint32_t key_bin(unsigned long long key) {
#ifdef __CUDA_ARCH__
    const int nb = 64 - __clzll((long long)key);
#else
    const int nb = key ? 64 - __builtin_clzll(key) : 0;
#endif
    if (nb <= 6) return (uint32_t)key;
    return ((uint32_t)(nb - 6) << 6) | (uint32_t)((key >> (nb - 7)) & 63ull);
}
struct IndexArgs {
    const int8_t* q_idx;
    const int8_t* k_idx;
    const int32_t* w;
    const int8_t* block_sums;
    int32_t* index_sets;
    int32_t* dev_status;
    const int64_t* kv_offset;
    const int32_t* seq_lens;
    const int64_t* blk_offset;
    const int32_t* q_seq;
    const int32_t* q_len;
    int64_t total_tokens;
    int64_t block_rows;
    int32_t n_seq, n_q, max_len;
    int32_t H_I, w_max;
    int32_t sink, window, topk, hi_block, hi_topblocks, budget;
    // workspace (see plan_index)
    uint64_t* coarse_keys;  // [n_q][coarse_cap] HI block keys (score + 1)
    int32_t* kept;          // [n_q][hi_topblocks] kept block ids, ascending
    int32_t* n_kept;        // [n_q]
    uint32_t* fine_keys;    // [n_q][fine_cap] token keys (score + 1, 0 = none)
    uint64_t* cand;         // prefill chunks: [n_q][fine_cap] candidate pairs (key << 32 | position)
    int32_t* cand_seg;      // prefill chunks: [n_q][LSA_TC_MAX_SPLITS][4][2] (first slot, count) per token split
                            // and lane quarter of the scoring
    uint32_t* ghist;        // prefill chunks: [n_q][LSA_TC_BINS] candidate-filter counts over all splits
    int32_t tc_splits;      // prefill chunks: token splits of the tensor-core scoring
    int32_t coarse_cap, fine_cap;
    // selection: keys of one CTA's slice staged in shared memory (0 = read
    // from global memory) and kept-block slots per slice
    int32_t coarse_stage, fine_stage, kept_slots;
    // a decode append run by extra CTAs of the block selection's grid (rows
    // n_q onwards): app_tasks tasks of app_per_seq CTAs per sequence and role
    // (0 = no append in this call)
    AppendArgs app;
    int32_t app_tasks, app_per_seq, app_dI;
};

struct IndexPlan {
    int coarse_cap = 0, fine_cap = 0;
    int cluster = 8;                          // CTAs per query row in the selection kernels
    int coarse_stage = 0, fine_stage = 0, kept_slots = 0;
    size_t smem_blocks = 0, smem_tokens = 0;  // dynamic smem of the selection kernels
    size_t off_coarse = 0, off_kept = 0, off_nkept = 0, off_fine = 0, off_cand = 0, off_count = 0, off_ghist = 0;
    size_t ws_bytes = 0;
};
// dense: the batch is a prefill chunk scored by the tensor-core contraction
// (candidate pairs instead of one key per token)
IndexPlan plan_index(int n_q, int max_len, const lsa_budget_t& b, bool dense = false);
cudaError_t launch_index_scores(const IndexArgs& a, int d_I, bool coarse, cudaStream_t stream);
// Fine scores of a causal chunk of rows of one sequence (HI off) on the
// tcgen05 tensor cores; same keys as launch_index_scores(coarse = false).
bool prefill_tc_supported(int H_I, int d_I, int n_seq, int64_t total_tokens);
// TMA tensor maps over [rows, 128] byte matrices (128-byte swizzle, box of
// box_rows x 128 bytes, rows past the end read as zero).
bool tensor_maps_available();
bool tensor_map_rows128(CUtensorMap* m, const void* base, uint64_t rows, uint32_t box_rows);
cudaError_t launch_fine_scores_tc(const IndexArgs& a, cudaStream_t stream);
// Token splits of each 16-row tile in the tensor-core scoring (<= LSA_TC_MAX_SPLITS).
#define LSA_TC_MAX_SPLITS 16
#define LSA_TC_SEGS 4     // candidate segments per token split (one per TMEM lane quarter)
#define LSA_TC_BINS 512   // candidate-filter histogram bins per row
#define LSA_TC_TOKENS 128 // cached tokens per tensor-core tile
int prefill_tc_splits(int n_q);
// HI block selection computes the coarse scores itself when each cluster
// CTA's slice of blocks fits in shared memory, the query has at most 16
// indexer heads (more would not fit the selection kernel's 64 registers) and
// there are enough rows for the clusters to cover the GPU (with a few rows
// the coarse scoring kernel spreads the block sums over more SMs); otherwise
// the coarse scoring kernel writes the scores to the workspace first.
inline bool coarse_in_select(int hi_block, int coarse_stage, int H_I, int n_q) {
    return hi_block > 0 && coarse_stage > 0 && H_I <= 16 && n_q >= 8;
}
inline bool coarse_in_select(const IndexArgs& a) { return coarse_in_select(a.hi_block, a.coarse_stage, a.H_I, a.n_q); }
// Prefill chunks: exact top-k over each row's candidate pairs, SI assembly.
cudaError_t launch_topk_pairs(const IndexArgs& a, cudaStream_t stream);
// Context-parallel merge of (score, id) values (lsa_merge_pairs).
cudaError_t launch_merge_pairs(const uint64_t* pairs, const int32_t* counts, int n_rows, int cap, int k, int32_t* out,
                               uint64_t* out_values, int32_t* dev_status, cudaStream_t stream);
cudaError_t launch_index_select(const IndexArgs& a, bool blocks, int d_I, int cluster, size_t smem,
                                cudaStream_t stream);
// Grid rows the block selection adds for a fused append (a.app_tasks tasks).
int index_select_append_rows(const IndexArgs& a, int cluster);

// Indexer scores of given token positions or HI blocks (lsa_score_tokens,
// lsa_score_blocks): q_idx, k_idx, w, w_max, H_I, n_q, block_sums and
// dev_status of `a` are used.
struct PointArgs {
    IndexArgs a;
    const int32_t* ids;       // [n_q][n] positions or block indices (-1: empty slot)
    const int64_t* row_base;  // [n_q] first cache row / block-sum row of each query row's sequence
    int64_t rows;             // rows of the key cache / block-sum cache
    uint32_t* out_tokens;     // [n_q][n]
    uint64_t* out_blocks;     // [n_q][n]
    int32_t n;
    int32_t blocks;
};
cudaError_t launch_point_scores(const PointArgs& p, int d_I, cudaStream_t stream);

// Draft-row groups (attend_group_kernel): at most this many rows per group.
constexpr int kMaxGroupRows = 8;

// Context-parallel attention (context_parallel.cu).
cudaError_t launch_shard_sets(const int32_t* sets, int n_q, int budget, int lo, int hi, int32_t* local,
                              int32_t* dev_status, cudaStream_t stream);
cudaError_t launch_combine(const float* o_parts, const float* lse_parts, int n_parts, int64_t rows, int d, float* out,
                           float* lse_out, cudaStream_t stream);

// ---- sparse attention -----------------------------------------------------
struct AttendArgs {
    const uint16_t* q[kMaxLayers];
    const uint16_t* k[kMaxLayers];
    const uint16_t* v[kMaxLayers];
    float* out[kMaxLayers];
    float* lse[kMaxLayers];  // optional: ln of the softmax denominator per (row, query head)
    const int32_t* sets;
    const int64_t* kv_offset;
    const int32_t* seq_lens;
    const int32_t* q_seq;
    const int32_t* q_len;
    int32_t* dev_status;
    float* part_o;        // [G][n_q][n_splits][H_q][d]
    float* part_ml;       // [G][n_q][n_splits][H_q][2]
    int64_t total_tokens;
    int32_t n_seq, n_q, max_len;
    int32_t H_q, H_kv, budget, G;
    int32_t n_splits, entries_per_split, head_groups;
    int32_t hpc;          // kv heads per CTA
    int32_t n_stages, row_stride, bar_off, stage_off;  // shared-memory plan
    float scale_log2;     // log2(e) / sqrt(d)
    int32_t kv_fp8;       // K/V caches hold FP8 E4M3 codes (k, v point at bytes)
    float kscale[kMaxLayers], vscale[kMaxLayers];  // FP8: value = scale * E4M3(code)
    // draft-row groups (attend_group_kernel): rows per group and per CTA
    int32_t group_rows, rows_per_cta;
    // lsa_attend_si: the gather kernel attends only the selected entries
    // [s, s + m) of each set; the sink and window runs are attend_window_kernel's
    int32_t si_split, si_sink, si_window, si_topk;
};

struct AttendPlan {
    int n_splits = 1, entries_per_split = 16, head_groups = 1, hpc = 1, rows_per_cta = 1;
    int n_stages = 2, row_stride = 272, bar_off = 0, stage_off = 0;
    size_t smem_bytes = 0;
    size_t ws_bytes = 0;
};
AttendPlan plan_attend(int n_q, int max_len, int H_q, int H_kv, int d, int budget, int G, int num_sms,
                       bool fp8 = false);
cudaError_t launch_attend(const AttendArgs& a, size_t smem_bytes, cudaStream_t stream);
// Draft-row groups: splits, shared memory and workspace of attend_group_kernel.
AttendPlan plan_attend_grouped(int n_q, int group_rows, int H_q, int H_kv, int budget, int G, int num_sms);
cudaError_t launch_attend_grouped(const AttendArgs& a, size_t smem_bytes, cudaStream_t stream);
// lsa_attend_si's sink and window part (attend_window.cu), after the gather.
cudaError_t launch_attend_window(const AttendArgs& a, cudaStream_t stream);

int device_sm_count();

// Launches `kernel` with programmatic stream serialisation (the kernel calls
// pdl_enter() first) and, when cluster > 0, that cluster size along x.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                       int cluster, Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    unsigned n = 0;
    attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
    if (cluster > 0) {
        attr[n].id = cudaLaunchAttributeClusterDimension;
        attr[n].val.clusterDim.x = (unsigned)cluster;
        attr[n].val.clusterDim.y = 1;
        attr[n].val.clusterDim.z = 1;
        ++n;
    }
    cfg.attrs = attr;
    cfg.numAttrs = n;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<Args&&>(args)...);
}

}  // namespace lsa
