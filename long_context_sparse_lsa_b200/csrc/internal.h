// internal.h — argument blocks and launchers shared between the C-ABI layer
// (abi.cu) and the kernel translation units. Host and device code only.
#pragma once

#include <cstddef>
#include <cstdint>
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

// ---- fused decode indexer -------------------------------------------------
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
    // storage plan (see plan_index)
    int32_t coarse_cap;   // coarse key slots per CTA
    int32_t fine_cap;     // fine key slots per CTA
    int32_t kept_cap;     // kept-block list entries (leader CTA)
    int32_t smem_coarse;  // byte offset in dynamic smem, or -1 (global)
    int32_t smem_fine;    // byte offset in dynamic smem, or -1 (global)
    int32_t smem_kept;    // byte offset in dynamic smem
    int32_t smem_kept_local;
    uint64_t* g_coarse;   // [n_q * C * coarse_cap] when smem_coarse < 0
    uint32_t* g_fine;     // [n_q * C * fine_cap] when smem_fine < 0
};

struct IndexPlan {
    int cluster = 1;
    int coarse_cap = 0, fine_cap = 0, kept_cap = 0;
    int smem_coarse = -1, smem_fine = -1, smem_kept = 0, smem_kept_local = 0;
    size_t dyn_smem = 0;
    size_t ws_coarse = 0, ws_fine = 0;  // global bytes
};

// Storage plan for a given cluster size (pure host arithmetic).
IndexPlan plan_index(int cluster, int n_q, int max_len, const lsa_budget_t& b);
// Chooses the cluster size for this device and batch.
cudaError_t choose_index_cluster(int d_I, int H_I, int n_q, int max_len, const lsa_budget_t& b,
                                 IndexPlan* out);
cudaError_t launch_index(const IndexArgs& a, const IndexPlan& plan, int d_I, cudaStream_t stream);

// ---- sparse attention -----------------------------------------------------
struct AttendArgs {
    const uint16_t* q[kMaxLayers];
    const uint16_t* k[kMaxLayers];
    const uint16_t* v[kMaxLayers];
    float* out[kMaxLayers];
    const int32_t* sets;
    const int64_t* kv_offset;
    const int32_t* seq_lens;
    const int32_t* q_seq;
    const int32_t* q_len;
    int32_t* dev_status;
    float* part_o;        // [G][n_q][n_parts][H_q][d]
    float* part_ml;       // [G][n_q][n_parts][H_q][2]
    uint32_t* counters;   // [G][n_q]
    int64_t total_tokens;
    int32_t n_seq, n_q, max_len;
    int32_t H_q, H_kv, budget, G;
    int32_t n_splits, entries_per_split, wph, head_groups;
    float scale_log2;     // log2(e) / sqrt(d)
};

struct AttendPlan {
    int n_splits = 1, entries_per_split = 16, wph = 1, head_groups = 1;
    size_t ws_bytes = 0;
};
AttendPlan plan_attend(int n_q, int max_len, int H_q, int H_kv, int d, int budget, int G, int num_sms);
cudaError_t launch_attend(const AttendArgs& a, cudaStream_t stream);

int device_sm_count();

}  // namespace lsa
