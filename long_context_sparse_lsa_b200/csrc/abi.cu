// abi.cu — the extern "C" entry points of liblsa.so (declared in
// include/lsa.h): argument validation, launch planning, and the launches.
// Every check that can be made on the host is made here, before any launch;
// nothing in this file allocates device memory or synchronises.
#include <cmath>
#include <cstring>
#include <map>
#include <mutex>
#include <tuple>

#include "internal.h"

namespace {

thread_local int32_t g_last_cuda = 0;

lsa_status_t cuda_fail(cudaError_t e) {
    g_last_cuda = (int32_t)e;
    return LSA_ERR_CUDA;
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

bool batch_ok(const lsa_batch_t* b, bool need_queries) {
    if (b == nullptr) return false;
    if (b->n_seq < 1 || b->n_q < 0 || b->max_len < 1 || b->reserved != 0 || b->total_tokens < 0) return false;
    if (b->kv_offset == nullptr || b->seq_lens == nullptr) return false;
    if (need_queries && b->n_q > 0 && (b->q_seq == nullptr || b->q_len == nullptr)) return false;
    return true;
}

bool budget_ok(const lsa_budget_t& b) {
    return b.sink >= 0 && b.window >= 0 && b.topk >= 0 && b.hi_block >= 0 && b.hi_topblocks >= 0;
}

int64_t budget_len(const lsa_budget_t& b) { return (int64_t)b.sink + b.window + b.topk; }

std::mutex g_mu;
std::map<int, int> g_sms;

int current_device() {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return -1;
    }
    return dev;
}

}  // namespace

namespace lsa {
int device_sm_count() {
    const int dev = current_device();
    std::lock_guard<std::mutex> lk(g_mu);
    auto it = g_sms.find(dev);
    if (it != g_sms.end()) return it->second;
    int n = 0;
    if (dev < 0 || cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
        cudaGetLastError();
        n = 148;  // B200
    }
    g_sms[dev] = n;
    return n;
}
}  // namespace lsa

extern "C" {

int32_t lsa_version(void) { return 100; }

int32_t lsa_last_cuda_error(void) { return g_last_cuda; }

const char* lsa_status_string(int32_t status) {
    switch (status) {
        case LSA_OK: return "LSA_OK";
        case LSA_ERR_INVALID_ARG: return "LSA_ERR_INVALID_ARG";
        case LSA_ERR_UNSUPPORTED: return "LSA_ERR_UNSUPPORTED";
        case LSA_ERR_CUDA: return "LSA_ERR_CUDA";
        case LSA_ERR_WORKSPACE: return "LSA_ERR_WORKSPACE";
        default: return "LSA_ERR_UNKNOWN";
    }
}

// ---------------------------------------------------------------------------
lsa_status_t lsa_hi_block_sums(const int8_t* k_idx_cache, int32_t d_I, int32_t hi_block, const lsa_batch_t* batch,
                               int32_t n_new, int8_t* block_sums, int64_t block_rows, int32_t* dev_status,
                               void* stream) {
    if (!batch_ok(batch, false)) return LSA_ERR_INVALID_ARG;
    if (k_idx_cache == nullptr || block_sums == nullptr || batch->blk_offset == nullptr || block_rows < 0)
        return LSA_ERR_INVALID_ARG;
    if (hi_block < 1 || d_I < 1) return LSA_ERR_INVALID_ARG;
    if (d_I != 32 && d_I != 64 && d_I != 128) return LSA_ERR_UNSUPPORTED;
    if (hi_block > LSA_MAX_HI_BLOCK) return LSA_ERR_UNSUPPORTED;
    if (!aligned(k_idx_cache, 16) || !aligned(block_sums, 16)) return LSA_ERR_INVALID_ARG;
    lsa::BlockSumArgs a;
    a.k_idx = k_idx_cache;
    a.block_sums = block_sums;
    a.kv_offset = batch->kv_offset;
    a.seq_lens = batch->seq_lens;
    a.blk_offset = batch->blk_offset;
    a.dev_status = dev_status;
    a.total_tokens = batch->total_tokens;
    a.block_rows = block_rows;
    a.n_seq = batch->n_seq;
    a.max_len = batch->max_len;
    a.hi_block = hi_block;
    a.n_new = n_new;
    const int64_t full = ((int64_t)batch->max_len + hi_block - 1) / hi_block;
    int64_t cover = n_new > 0 ? ((int64_t)n_new + hi_block - 1) / hi_block + 1 : full;
    if (cover > full) cover = full;
    a.blocks_per_seq = (int32_t)cover;
    if (batch->n_seq > 65535) return LSA_ERR_UNSUPPORTED;
    cudaError_t e = lsa::launch_block_sums(a, d_I, reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? LSA_OK : cuda_fail(e);
}

}  // extern "C"

// Checks lsa_append's arguments and fills the kernel arguments.
static lsa_status_t append_args(const int8_t* k_idx_new, int8_t* k_idx_cache, int32_t d_I, const void* const* k_new,
                                const void* const* v_new, void* const* k_cache, void* const* v_cache,
                                int32_t kv_row_bytes, int32_t layers, int32_t hi_block, int8_t* block_sums,
                                int64_t block_rows, const lsa_batch_t* batch, int32_t n_new, int32_t* dev_status,
                                lsa::AppendArgs& a) {
    if (!batch_ok(batch, false)) return LSA_ERR_INVALID_ARG;
    if (n_new < 1 || d_I < 1 || layers < 0 || hi_block < 0 || block_rows < 0) return LSA_ERR_INVALID_ARG;
    if (d_I != 32 && d_I != 64 && d_I != 128) return LSA_ERR_UNSUPPORTED;
    if (hi_block > LSA_MAX_HI_BLOCK || layers > LSA_MAX_LAYERS) return LSA_ERR_UNSUPPORTED;
    if (k_idx_new == nullptr || k_idx_cache == nullptr || !aligned(k_idx_new, 16) || !aligned(k_idx_cache, 16))
        return LSA_ERR_INVALID_ARG;
    if (hi_block > 0 && (block_sums == nullptr || batch->blk_offset == nullptr || !aligned(block_sums, 16)))
        return LSA_ERR_INVALID_ARG;
    if (layers > 0) {
        if (kv_row_bytes < 16 || kv_row_bytes % 16 != 0) return LSA_ERR_INVALID_ARG;
        if (k_new == nullptr || v_new == nullptr || k_cache == nullptr || v_cache == nullptr)
            return LSA_ERR_INVALID_ARG;
        for (int g = 0; g < layers; ++g) {
            if (k_new[g] == nullptr || v_new[g] == nullptr || k_cache[g] == nullptr || v_cache[g] == nullptr)
                return LSA_ERR_INVALID_ARG;
            if (!aligned(k_new[g], 16) || !aligned(v_new[g], 16) || !aligned(k_cache[g], 16) ||
                !aligned(v_cache[g], 16))
                return LSA_ERR_INVALID_ARG;
        }
    }
    if (batch->n_seq > 65535) return LSA_ERR_UNSUPPORTED;
    std::memset(&a, 0, sizeof a);
    a.bs.k_idx = k_idx_cache;
    a.bs.block_sums = block_sums;
    a.bs.kv_offset = batch->kv_offset;
    a.bs.seq_lens = batch->seq_lens;
    a.bs.blk_offset = batch->blk_offset;
    a.bs.dev_status = dev_status;
    a.bs.total_tokens = batch->total_tokens;
    a.bs.block_rows = block_rows;
    a.bs.n_seq = batch->n_seq;
    a.bs.max_len = batch->max_len;
    a.bs.hi_block = hi_block;
    a.bs.n_new = n_new;
    a.k_idx_new = k_idx_new;
    a.k_idx_cache = k_idx_cache;
    for (int g = 0; g < layers; ++g) {
        a.k_new[g] = k_new[g];
        a.v_new[g] = v_new[g];
        a.k_cache[g] = k_cache[g];
        a.v_cache[g] = v_cache[g];
    }
    a.layers = layers;
    a.kv_row_bytes = layers > 0 ? kv_row_bytes : 0;
    a.sums = hi_block > 0 ? 1 : 0;
    return LSA_OK;
}

extern "C" {

lsa_status_t lsa_append(const int8_t* k_idx_new, int8_t* k_idx_cache, int32_t d_I, const void* const* k_new,
                        const void* const* v_new, void* const* k_cache, void* const* v_cache,
                        int32_t kv_row_bytes, int32_t layers, int32_t hi_block, int8_t* block_sums,
                        int64_t block_rows, const lsa_batch_t* batch, int32_t n_new, int32_t* dev_status,
                        void* stream) {
    lsa::AppendArgs a;
    const lsa_status_t st = append_args(k_idx_new, k_idx_cache, d_I, k_new, v_new, k_cache, v_cache, kv_row_bytes,
                                        layers, hi_block, block_sums, block_rows, batch, n_new, dev_status, a);
    if (st != LSA_OK) return st;
    cudaError_t e = lsa::launch_append(a, d_I, reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? LSA_OK : cuda_fail(e);
}

// ---------------------------------------------------------------------------
}  // extern "C"

// Rows from which a chunk of one sequence is scored as a dense contraction.
constexpr int32_t kDenseMinRows = 64;

static bool index_dense(const lsa_batch_t* batch, int32_t H_I, int32_t d_I, const lsa_budget_t& budget) {
    return budget.hi_block == 0 && batch->n_q >= kDenseMinRows &&
           lsa::prefill_tc_supported(H_I, d_I, batch->n_seq, batch->total_tokens);
}

extern "C" {

size_t lsa_index_workspace_size(const lsa_batch_t* batch, int32_t H_I, int32_t d_I, lsa_budget_t budget) {
    if (batch == nullptr || batch->n_q <= 0 || batch->max_len < 1 || !budget_ok(budget)) return 0;
    if (budget.hi_block == 0) budget.hi_topblocks = 0;
    return lsa::plan_index(batch->n_q, batch->max_len, budget, index_dense(batch, H_I, d_I, budget)).ws_bytes;
}

int32_t lsa_index_uses_tensor_cores(const lsa_batch_t* batch, int32_t H_I, int32_t d_I,
                                               lsa_budget_t budget) {
    if (batch == nullptr || !budget_ok(budget)) return 0;
    return index_dense(batch, H_I, d_I, budget) ? 1 : 0;
}

int32_t lsa_index_launches(const lsa_batch_t* batch, int32_t H_I, int32_t d_I, lsa_budget_t budget) {
    if (batch == nullptr || batch->n_q <= 0 || batch->max_len < 1 || !budget_ok(budget)) return 0;
    (void)d_I;
    if (budget.hi_block == 0) return 2;  // fine scores, token selection
    const lsa::IndexPlan plan = lsa::plan_index(batch->n_q, batch->max_len, budget);
    const bool fused = lsa::coarse_in_select(budget.hi_block, plan.coarse_stage, H_I, batch->n_q);
    return (fused ? 1 : 2) + 2;  // [coarse scores,] block selection, fine scores, token selection
}

static lsa_status_t index_validate(const int8_t* q_idx, const int8_t* k_idx_cache, const int32_t* w, int32_t w_max,
                                   int32_t H_I, int32_t d_I, const lsa_batch_t* batch, lsa_budget_t budget,
                                   const int8_t* block_sums, int64_t block_rows, const int32_t* index_sets) {
    if (!batch_ok(batch, true) || !budget_ok(budget)) return LSA_ERR_INVALID_ARG;
    if (H_I < 1 || d_I < 1 || w_max < 0) return LSA_ERR_INVALID_ARG;
    if (batch->n_q > 0 && (q_idx == nullptr || k_idx_cache == nullptr || w == nullptr || index_sets == nullptr))
        return LSA_ERR_INVALID_ARG;
    if (!aligned(q_idx, 16) || !aligned(k_idx_cache, 16) || !aligned(w, 4) || !aligned(index_sets, 4))
        return LSA_ERR_INVALID_ARG;
    if (d_I != 32 && d_I != 64 && d_I != 128) return LSA_ERR_UNSUPPORTED;
    if (H_I > LSA_MAX_HEADS_I) return LSA_ERR_UNSUPPORTED;
    if (budget_len(budget) > LSA_MAX_BUDGET) return LSA_ERR_UNSUPPORTED;
    // fine scores are exact in int32 when H_I * w_max * d_I * 128 * 128 < 2^31
    if ((double)H_I * (double)w_max * (double)d_I * 16384.0 >= 2147483648.0) return LSA_ERR_UNSUPPORTED;
    if (budget.hi_block > 0) {
        if (budget.hi_block > LSA_MAX_HI_BLOCK || budget.hi_topblocks > LSA_MAX_TOPBLOCKS) return LSA_ERR_UNSUPPORTED;
        if (block_sums == nullptr || batch->blk_offset == nullptr || block_rows < 0) return LSA_ERR_INVALID_ARG;
        if (!aligned(block_sums, 16)) return LSA_ERR_INVALID_ARG;
    }
    return LSA_OK;
}

}  // extern "C"

// The append may run inside the block selection when the two touch disjoint
// memory: HI on, and the n_new newest tokens' blocks inside every row's
// window (window >= hi_block + n_new - 1), so that no candidate block sum
// and no candidate key is written by the append; the fine scores and the
// token selection wait for the whole block-selection grid.
static bool append_fusable(const lsa_budget_t& b, int32_t n_new) {
    return b.hi_block > 0 && n_new >= 1 && (int64_t)b.window >= (int64_t)b.hi_block + n_new - 1;
}

// lsa_index after validation; app (nullable) is a decode append to run in
// extra CTAs of the block selection (append_fusable holds).
static lsa_status_t index_impl(const int8_t* q_idx, const int8_t* k_idx_cache, const int32_t* w, int32_t w_max,
                               int32_t H_I, int32_t d_I, const lsa_batch_t* batch, lsa_budget_t budget,
                               const int8_t* block_sums, int64_t block_rows, int32_t* index_sets, void* workspace,
                               size_t workspace_bytes, int32_t* dev_status, void* stream,
                               const lsa::AppendArgs* app) {
    if (budget.hi_block == 0) budget.hi_topblocks = 0;

    const bool dense = index_dense(batch, H_I, d_I, budget);
    const lsa::IndexPlan plan = lsa::plan_index(batch->n_q, batch->max_len, budget, dense);
    if (plan.ws_bytes > 0 && (workspace == nullptr || workspace_bytes < plan.ws_bytes || !aligned(workspace, 256)))
        return LSA_ERR_WORKSPACE;
    if (batch->n_q > 65535) return LSA_ERR_UNSUPPORTED;

    lsa::IndexArgs a;
    std::memset(&a, 0, sizeof a);
    a.q_idx = q_idx;
    a.k_idx = k_idx_cache;
    a.w = w;
    a.block_sums = block_sums;
    a.index_sets = index_sets;
    a.dev_status = dev_status;
    a.kv_offset = batch->kv_offset;
    a.seq_lens = batch->seq_lens;
    a.blk_offset = batch->blk_offset;
    a.q_seq = batch->q_seq;
    a.q_len = batch->q_len;
    a.total_tokens = batch->total_tokens;
    a.block_rows = block_rows;
    a.n_seq = batch->n_seq;
    a.n_q = batch->n_q;
    a.max_len = batch->max_len;
    a.H_I = H_I;
    a.w_max = w_max;
    a.sink = budget.sink;
    a.window = budget.window;
    a.topk = budget.topk;
    a.hi_block = budget.hi_block;
    a.hi_topblocks = budget.hi_topblocks;
    a.budget = (int32_t)budget_len(budget);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    a.coarse_keys = reinterpret_cast<uint64_t*>(ws + plan.off_coarse);
    a.kept = reinterpret_cast<int32_t*>(ws + plan.off_kept);
    a.n_kept = reinterpret_cast<int32_t*>(ws + plan.off_nkept);
    a.fine_keys = reinterpret_cast<uint32_t*>(ws + plan.off_fine);
    a.cand = dense ? reinterpret_cast<uint64_t*>(ws + plan.off_cand) : nullptr;
    a.cand_seg = dense ? reinterpret_cast<int32_t*>(ws + plan.off_count) : nullptr;
    a.ghist = dense ? reinterpret_cast<uint32_t*>(ws + plan.off_ghist) : nullptr;
    a.tc_splits = dense ? lsa::prefill_tc_splits(batch->n_q) : 0;
    a.coarse_cap = plan.coarse_cap;
    a.fine_cap = plan.fine_cap;
    a.coarse_stage = plan.coarse_stage;
    a.fine_stage = plan.fine_stage;
    a.kept_slots = plan.kept_slots;
    if (app != nullptr) {
        a.app = *app;
        a.app_per_seq = lsa::append_ctas_per_seq(app->bs.n_new, app->bs.hi_block, app->bs.max_len);
        a.app_tasks = a.app_per_seq * app->bs.n_seq * 2;  // copy and block-sum roles
        a.app_dI = d_I;
        if ((int64_t)batch->n_q + lsa::index_select_append_rows(a, plan.cluster) > 65535) return LSA_ERR_UNSUPPORTED;
    }
    cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = cudaSuccess;
    if (budget.hi_block > 0) {
        if (!lsa::coarse_in_select(a)) e = lsa::launch_index_scores(a, d_I, true, cs);
        if (e == cudaSuccess) e = lsa::launch_index_select(a, true, d_I, plan.cluster, plan.smem_blocks, cs);
        a.app_tasks = 0;  // the later kernels carry no append
    }
    if (e == cudaSuccess) {
        // a prefill chunk (many rows of one sequence, HI off) is one dense
        // contraction: tensor-core path; otherwise per-row streaming scores
        e = dense ? lsa::launch_fine_scores_tc(a, cs) : lsa::launch_index_scores(a, d_I, false, cs);
    }
    if (e == cudaSuccess) {
        e = dense ? lsa::launch_topk_pairs(a, cs)
                  : lsa::launch_index_select(a, false, d_I, plan.cluster, plan.smem_tokens, cs);
    }
    return e == cudaSuccess ? LSA_OK : cuda_fail(e);
}

extern "C" {

lsa_status_t lsa_index(const int8_t* q_idx, const int8_t* k_idx_cache, const int32_t* w, int32_t w_max, int32_t H_I,
                       int32_t d_I, const lsa_batch_t* batch, lsa_budget_t budget, const int8_t* block_sums,
                       int64_t block_rows, int32_t* index_sets, void* workspace, size_t workspace_bytes,
                       int32_t* dev_status, void* stream) {
    const lsa_status_t st = index_validate(q_idx, k_idx_cache, w, w_max, H_I, d_I, batch, budget, block_sums,
                                           block_rows, index_sets);
    if (st != LSA_OK) return st;
    if (batch->n_q == 0) return LSA_OK;
    return index_impl(q_idx, k_idx_cache, w, w_max, H_I, d_I, batch, budget, block_sums, block_rows, index_sets,
                      workspace, workspace_bytes, dev_status, stream, nullptr);
}

int32_t lsa_append_index_launches(const lsa_batch_t* batch, int32_t H_I, int32_t d_I, lsa_budget_t budget,
                                  int32_t n_new) {
    if (batch == nullptr || n_new < 1) return 0;
    const int32_t n_idx = batch->n_q > 0 ? lsa_index_launches(batch, H_I, d_I, budget) : 0;
    if (n_idx == 0 && batch->n_q > 0) return 0;
    return n_idx + (batch->n_q > 0 && append_fusable(budget, n_new) ? 0 : 1);
}

lsa_status_t lsa_append_index(const int8_t* k_idx_new, const void* const* k_new, const void* const* v_new,
                              void* const* k_cache, void* const* v_cache, int32_t kv_row_bytes, int32_t layers,
                              int32_t n_new, const int8_t* q_idx, int8_t* k_idx_cache, const int32_t* w,
                              int32_t w_max, int32_t H_I, int32_t d_I, const lsa_batch_t* batch, lsa_budget_t budget,
                              int8_t* block_sums, int64_t block_rows, int32_t* index_sets, void* workspace,
                              size_t workspace_bytes, int32_t* dev_status, void* stream) {
    if (!budget_ok(budget)) return LSA_ERR_INVALID_ARG;
    lsa::AppendArgs app;
    lsa_status_t st = append_args(k_idx_new, k_idx_cache, d_I, k_new, v_new, k_cache, v_cache, kv_row_bytes, layers,
                                  budget.hi_block, block_sums, block_rows, batch, n_new, dev_status, app);
    if (st != LSA_OK) return st;
    st = index_validate(q_idx, k_idx_cache, w, w_max, H_I, d_I, batch, budget, block_sums, block_rows, index_sets);
    if (st != LSA_OK) return st;
    if (batch->n_q > 0 && append_fusable(budget, n_new))  // (index_impl checks everything before its first launch)
        return index_impl(q_idx, k_idx_cache, w, w_max, H_I, d_I, batch, budget, block_sums, block_rows, index_sets,
                          workspace, workspace_bytes, dev_status, stream, &app);
    if (batch->n_q > 0) {
        // the checks index_impl makes before its first launch, ahead of the
        // append's launch, so that a refused call launches nothing
        lsa_budget_t b = budget;
        if (b.hi_block == 0) b.hi_topblocks = 0;
        const lsa::IndexPlan plan = lsa::plan_index(batch->n_q, batch->max_len, b, index_dense(batch, H_I, d_I, b));
        if (plan.ws_bytes > 0 && (workspace == nullptr || workspace_bytes < plan.ws_bytes || !aligned(workspace, 256)))
            return LSA_ERR_WORKSPACE;
        if (batch->n_q > 65535) return LSA_ERR_UNSUPPORTED;
    }
    cudaError_t e = lsa::launch_append(app, d_I, reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e);
    if (batch->n_q == 0) return LSA_OK;
    return index_impl(q_idx, k_idx_cache, w, w_max, H_I, d_I, batch, budget, block_sums, block_rows, index_sets,
                      workspace, workspace_bytes, dev_status, stream, nullptr);
}

// ---------------------------------------------------------------------------
static bool attend_shape_ok(int32_t H_q, int32_t H_kv, int32_t d, int32_t budget, int32_t G) {
    if (d != 128) return false;
    if (H_kv < 1 || H_q < 1 || H_q % H_kv != 0) return false;
    const int ratio = H_q / H_kv;
    if (ratio != 1 && ratio != 2 && ratio != 4 && ratio != 8 && ratio != 16) return false;
    if (!(H_kv == 1 || H_kv == 2 || H_kv == 4 || H_kv % 4 == 0)) return false;
    if (G < 1 || G > LSA_MAX_LAYERS) return false;
    if (budget < 0 || budget > LSA_MAX_BUDGET) return false;
    return true;
}

size_t lsa_attend_workspace_size(const lsa_batch_t* batch, int32_t H_q, int32_t H_kv, int32_t d, int32_t budget,
                                 int32_t layers_per_index) {
    if (batch == nullptr || batch->n_q <= 0 || batch->max_len < 1) return 0;
    if (!attend_shape_ok(H_q, H_kv, d, budget, layers_per_index)) return 0;
    lsa::AttendPlan p = lsa::plan_attend(batch->n_q, batch->max_len, H_q, H_kv, d, budget, layers_per_index,
                                         lsa::device_sm_count());
    return p.ws_bytes;
}

int32_t lsa_attend_launches(const lsa_batch_t* batch, int32_t H_q, int32_t H_kv, int32_t d, int32_t budget,
                            int32_t layers_per_index) {
    if (batch == nullptr || batch->n_q <= 0 || !attend_shape_ok(H_q, H_kv, d, budget, layers_per_index)) return 0;
    const lsa::AttendPlan p = lsa::plan_attend(batch->n_q, batch->max_len, H_q, H_kv, d, budget, layers_per_index,
                                               lsa::device_sm_count());
    return p.n_splits > 1 ? 2 : 1;  // attention[, split merge]
}

}  // extern "C"

// lsa_attend and lsa_attend_fp8: k_cache / v_cache point at bf16 elements, or
// at E4M3 codes when kscale / vscale are given (FP8).
static lsa_status_t attend_impl(const uint16_t* const* q, const void* const* k_cache, const void* const* v_cache,
                                const float* kscale, const float* vscale, int32_t H_q, int32_t H_kv, int32_t d,
                                const int32_t* index_sets, int32_t budget, const lsa_batch_t* batch,
                                int32_t layers_per_index, float* const* out, float* const* lse, void* workspace,
                                size_t workspace_bytes, int32_t* dev_status, void* stream) {
    const bool fp8 = kscale != nullptr;
    if (!batch_ok(batch, true)) return LSA_ERR_INVALID_ARG;
    if (H_q < 1 || H_kv < 1 || d < 1 || budget < 0 || layers_per_index < 1) return LSA_ERR_INVALID_ARG;
    if (H_q % H_kv != 0) return LSA_ERR_INVALID_ARG;
    if (!attend_shape_ok(H_q, H_kv, d, budget, layers_per_index)) return LSA_ERR_UNSUPPORTED;
    if (fp8 && H_q / H_kv > 8) return LSA_ERR_UNSUPPORTED;
    if (q == nullptr || k_cache == nullptr || v_cache == nullptr || out == nullptr) return LSA_ERR_INVALID_ARG;
    if (fp8) {
        if (vscale == nullptr) return LSA_ERR_INVALID_ARG;
        for (int g = 0; g < layers_per_index; ++g)
            if (!std::isfinite(kscale[g]) || !std::isfinite(vscale[g])) return LSA_ERR_INVALID_ARG;
    }
    if (batch->n_q == 0) return LSA_OK;
    if (budget > 0 && (index_sets == nullptr || !aligned(index_sets, 4))) return LSA_ERR_INVALID_ARG;
    for (int g = 0; g < layers_per_index; ++g) {
        if (q[g] == nullptr || k_cache[g] == nullptr || v_cache[g] == nullptr || out[g] == nullptr)
            return LSA_ERR_INVALID_ARG;
        if (!aligned(q[g], 16) || !aligned(k_cache[g], 16) || !aligned(v_cache[g], 16) || !aligned(out[g], 16))
            return LSA_ERR_INVALID_ARG;
        if (lse != nullptr && (lse[g] == nullptr || !aligned(lse[g], 4))) return LSA_ERR_INVALID_ARG;
    }
    if ((int64_t)batch->n_q > 65535) return LSA_ERR_UNSUPPORTED;
    lsa::AttendPlan p = lsa::plan_attend(batch->n_q, batch->max_len, H_q, H_kv, d, budget, layers_per_index,
                                         lsa::device_sm_count(), fp8);
    if (workspace == nullptr || workspace_bytes < p.ws_bytes || !aligned(workspace, 256)) return LSA_ERR_WORKSPACE;
    lsa::AttendArgs a;
    std::memset(&a, 0, sizeof a);
    for (int g = 0; g < layers_per_index; ++g) {
        a.q[g] = q[g];
        a.k[g] = static_cast<const uint16_t*>(k_cache[g]);
        a.v[g] = static_cast<const uint16_t*>(v_cache[g]);
        a.out[g] = out[g];
        a.lse[g] = lse != nullptr ? lse[g] : nullptr;
        a.kscale[g] = fp8 ? kscale[g] : 1.f;
        a.vscale[g] = fp8 ? vscale[g] : 1.f;
    }
    a.kv_fp8 = fp8 ? 1 : 0;
    a.sets = index_sets;
    a.kv_offset = batch->kv_offset;
    a.seq_lens = batch->seq_lens;
    a.q_seq = batch->q_seq;
    a.q_len = batch->q_len;
    a.dev_status = dev_status;
    const size_t rows_q = (size_t)layers_per_index * batch->n_q;
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    if (p.n_splits > 1) {
        a.part_o = reinterpret_cast<float*>(ws);
        const size_t off = (rows_q * p.n_splits * H_q * 128 * 4 + 255) / 256 * 256;
        a.part_ml = reinterpret_cast<float*>(ws + off);
    }
    a.total_tokens = batch->total_tokens;
    a.n_seq = batch->n_seq;
    a.n_q = batch->n_q;
    a.max_len = batch->max_len;
    a.H_q = H_q;
    a.H_kv = H_kv;
    a.budget = budget;
    a.G = layers_per_index;
    a.n_splits = p.n_splits;
    a.entries_per_split = p.entries_per_split;
    a.head_groups = p.head_groups;
    a.hpc = p.hpc;
    a.n_stages = p.n_stages;
    a.row_stride = p.row_stride;
    a.bar_off = p.bar_off;
    a.stage_off = p.stage_off;
    a.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)d));
    cudaError_t e = lsa::launch_attend(a, p.smem_bytes, reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? LSA_OK : cuda_fail(e);
}

extern "C" {

lsa_status_t lsa_attend(const uint16_t* const* q, const uint16_t* const* k_cache, const uint16_t* const* v_cache,
                        int32_t H_q, int32_t H_kv, int32_t d, const int32_t* index_sets, int32_t budget,
                        const lsa_batch_t* batch, int32_t layers_per_index, float* const* out, void* workspace,
                        size_t workspace_bytes, int32_t* dev_status, void* stream) {
    return attend_impl(q, reinterpret_cast<const void* const*>(k_cache), reinterpret_cast<const void* const*>(v_cache),
                       nullptr, nullptr, H_q, H_kv, d, index_sets, budget, batch, layers_per_index, out, nullptr,
                       workspace, workspace_bytes, dev_status, stream);
}

lsa_status_t lsa_attend_lse(const uint16_t* const* q, const uint16_t* const* k_cache, const uint16_t* const* v_cache,
                            int32_t H_q, int32_t H_kv, int32_t d, const int32_t* index_sets, int32_t budget,
                            const lsa_batch_t* batch, int32_t layers_per_index, float* const* out,
                            float* const* lse, void* workspace, size_t workspace_bytes, int32_t* dev_status,
                            void* stream) {
    if (lse == nullptr) return LSA_ERR_INVALID_ARG;
    return attend_impl(q, reinterpret_cast<const void* const*>(k_cache), reinterpret_cast<const void* const*>(v_cache),
                       nullptr, nullptr, H_q, H_kv, d, index_sets, budget, batch, layers_per_index, out, lse,
                       workspace, workspace_bytes, dev_status, stream);
}

// ---- SI split attention (prefill chunks) ---------------------------------------
static bool si_shape_ok(const lsa_batch_t* batch, int32_t H_q, int32_t H_kv, int32_t d, const lsa_budget_t& b,
                        int32_t G) {
    const int32_t budget = b.sink + b.window + b.topk;
    if (b.sink < 0 || b.window < 0 || b.topk < 0) return false;
    if (!attend_shape_ok(H_q, H_kv, d, budget, G) || H_q / H_kv > 8) return false;
    return batch->n_seq == 1 && (batch->n_q + 15) / 16 <= 0x7fffffff;
}

static lsa::AttendPlan si_plan(const lsa_batch_t* batch, int32_t H_q, int32_t H_kv, int32_t d,
                               const lsa_budget_t& b, int32_t G, size_t* lse_off) {
    // the gather kernel's splits cover the selected entries only
    lsa::AttendPlan p = lsa::plan_attend(batch->n_q, batch->max_len, H_q, H_kv, d, b.topk > 0 ? b.topk : 1, G,
                                         lsa::device_sm_count());
    *lse_off = (p.ws_bytes + 255) / 256 * 256;
    p.ws_bytes = *lse_off + ((size_t)G * batch->n_q * H_q * 4 + 255) / 256 * 256;
    return p;
}

size_t lsa_attend_si_workspace_size(const lsa_batch_t* batch, int32_t H_q, int32_t H_kv, int32_t d,
                                    lsa_budget_t budget, int32_t layers_per_index) {
    if (batch == nullptr || batch->n_q <= 0 || batch->max_len < 1) return 0;
    if (!si_shape_ok(batch, H_q, H_kv, d, budget, layers_per_index)) return 0;
    size_t lo;
    return si_plan(batch, H_q, H_kv, d, budget, layers_per_index, &lo).ws_bytes;
}

int32_t lsa_attend_si_launches(const lsa_batch_t* batch, int32_t H_q, int32_t H_kv, int32_t d, lsa_budget_t budget,
                               int32_t layers_per_index) {
    if (batch == nullptr || batch->n_q <= 0) return 0;
    if (!si_shape_ok(batch, H_q, H_kv, d, budget, layers_per_index)) return 0;
    size_t lo;
    const lsa::AttendPlan p = si_plan(batch, H_q, H_kv, d, budget, layers_per_index, &lo);
    return p.n_splits > 1 ? 3 : 2;  // gather[, split merge], sink and window tiles
}

lsa_status_t lsa_attend_si(const uint16_t* const* q, const uint16_t* const* k_cache, const uint16_t* const* v_cache,
                           int32_t H_q, int32_t H_kv, int32_t d, const int32_t* index_sets, lsa_budget_t budget,
                           const lsa_batch_t* batch, int32_t layers_per_index, float* const* out, void* workspace,
                           size_t workspace_bytes, int32_t* dev_status, void* stream) {
    if (!batch_ok(batch, true)) return LSA_ERR_INVALID_ARG;
    if (H_q < 1 || H_kv < 1 || d < 1 || layers_per_index < 1) return LSA_ERR_INVALID_ARG;
    if (budget.sink < 0 || budget.window < 0 || budget.topk < 0 || H_q % H_kv != 0) return LSA_ERR_INVALID_ARG;
    if (!si_shape_ok(batch, H_q, H_kv, d, budget, layers_per_index)) return LSA_ERR_UNSUPPORTED;
    if (q == nullptr || k_cache == nullptr || v_cache == nullptr || out == nullptr) return LSA_ERR_INVALID_ARG;
    if (batch->n_q == 0) return LSA_OK;
    const int32_t nb = budget.sink + budget.window + budget.topk;
    if (nb > 0 && (index_sets == nullptr || !aligned(index_sets, 4))) return LSA_ERR_INVALID_ARG;
    for (int g = 0; g < layers_per_index; ++g) {
        if (q[g] == nullptr || k_cache[g] == nullptr || v_cache[g] == nullptr || out[g] == nullptr)
            return LSA_ERR_INVALID_ARG;
        if (!aligned(q[g], 16) || !aligned(k_cache[g], 16) || !aligned(v_cache[g], 16) || !aligned(out[g], 16))
            return LSA_ERR_INVALID_ARG;
    }
    size_t lse_off = 0;
    const lsa::AttendPlan p = si_plan(batch, H_q, H_kv, d, budget, layers_per_index, &lse_off);
    if (workspace == nullptr || workspace_bytes < p.ws_bytes || !aligned(workspace, 256)) return LSA_ERR_WORKSPACE;
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    lsa::AttendArgs a;
    std::memset(&a, 0, sizeof a);
    for (int g = 0; g < layers_per_index; ++g) {
        a.q[g] = q[g];
        a.k[g] = k_cache[g];
        a.v[g] = v_cache[g];
        a.out[g] = out[g];
        a.lse[g] = reinterpret_cast<float*>(ws + lse_off) + (size_t)g * batch->n_q * H_q;
        a.kscale[g] = 1.f;
        a.vscale[g] = 1.f;
    }
    a.sets = index_sets;
    a.kv_offset = batch->kv_offset;
    a.seq_lens = batch->seq_lens;
    a.q_seq = batch->q_seq;
    a.q_len = batch->q_len;
    a.dev_status = dev_status;
    const size_t rows_q = (size_t)layers_per_index * batch->n_q;
    if (p.n_splits > 1) {
        a.part_o = reinterpret_cast<float*>(ws);
        const size_t off = (rows_q * p.n_splits * H_q * 128 * 4 + 255) / 256 * 256;
        a.part_ml = reinterpret_cast<float*>(ws + off);
    }
    a.total_tokens = batch->total_tokens;
    a.n_seq = batch->n_seq;
    a.n_q = batch->n_q;
    a.max_len = batch->max_len;
    a.H_q = H_q;
    a.H_kv = H_kv;
    a.budget = nb;
    a.G = layers_per_index;
    a.n_splits = p.n_splits;
    a.entries_per_split = p.entries_per_split;
    a.head_groups = p.head_groups;
    a.hpc = p.hpc;
    a.n_stages = p.n_stages;
    a.row_stride = p.row_stride;
    a.bar_off = p.bar_off;
    a.stage_off = p.stage_off;
    a.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)d));
    a.si_split = 1;
    a.si_sink = budget.sink;
    a.si_window = budget.window;
    a.si_topk = budget.topk;
    const cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = lsa::launch_attend(a, p.smem_bytes, cs);
    if (e == cudaSuccess) e = lsa::launch_attend_window(a, cs);
    return e == cudaSuccess ? LSA_OK : cuda_fail(e);
}

// ---- draft-row groups --------------------------------------------------------
static bool grouped_shape_ok(const lsa_batch_t* batch, int32_t H_q, int32_t H_kv, int32_t d, int32_t budget,
                             int32_t G, int32_t group_rows) {
    if (!attend_shape_ok(H_q, H_kv, d, budget, G) || H_q / H_kv > 8) return false;
    if (group_rows != 1 && group_rows != 2 && group_rows != 4 && group_rows != 8) return false;
    if (batch->n_q % group_rows != 0 || batch->n_q / group_rows > 65535) return false;
    const lsa::AttendPlan p =
        lsa::plan_attend_grouped(batch->n_q, group_rows, H_q, H_kv, budget, G, lsa::device_sm_count());
    return p.smem_bytes <= 220 * 1024;  // the rows' sets are staged in shared memory
}

size_t lsa_attend_grouped_workspace_size(const lsa_batch_t* batch, int32_t H_q, int32_t H_kv, int32_t d,
                                         int32_t budget, int32_t layers_per_index, int32_t group_rows) {
    if (batch == nullptr || batch->n_q <= 0 || batch->max_len < 1) return 0;
    if (!grouped_shape_ok(batch, H_q, H_kv, d, budget, layers_per_index, group_rows)) return 0;
    return lsa::plan_attend_grouped(batch->n_q, group_rows, H_q, H_kv, budget, layers_per_index,
                                    lsa::device_sm_count())
        .ws_bytes;
}

int32_t lsa_attend_grouped_launches(const lsa_batch_t* batch, int32_t H_q, int32_t H_kv, int32_t d, int32_t budget,
                                    int32_t layers_per_index, int32_t group_rows) {
    if (batch == nullptr || batch->n_q <= 0) return 0;
    if (!grouped_shape_ok(batch, H_q, H_kv, d, budget, layers_per_index, group_rows)) return 0;
    const lsa::AttendPlan p = lsa::plan_attend_grouped(batch->n_q, group_rows, H_q, H_kv, budget, layers_per_index,
                                                       lsa::device_sm_count());
    return p.n_splits > 1 ? 2 : 1;  // attention[, split merge]
}

lsa_status_t lsa_attend_grouped(const uint16_t* const* q, const uint16_t* const* k_cache,
                                const uint16_t* const* v_cache, int32_t H_q, int32_t H_kv, int32_t d,
                                const int32_t* index_sets, int32_t budget, const lsa_batch_t* batch,
                                int32_t layers_per_index, int32_t group_rows, float* const* out, void* workspace,
                                size_t workspace_bytes, int32_t* dev_status, void* stream) {
    if (!batch_ok(batch, true)) return LSA_ERR_INVALID_ARG;
    if (H_q < 1 || H_kv < 1 || d < 1 || budget < 0 || layers_per_index < 1 || group_rows < 1)
        return LSA_ERR_INVALID_ARG;
    if (H_q % H_kv != 0 || batch->n_q % group_rows != 0) return LSA_ERR_INVALID_ARG;
    if (!grouped_shape_ok(batch, H_q, H_kv, d, budget, layers_per_index, group_rows)) return LSA_ERR_UNSUPPORTED;
    if (q == nullptr || k_cache == nullptr || v_cache == nullptr || out == nullptr) return LSA_ERR_INVALID_ARG;
    if (batch->n_q == 0) return LSA_OK;
    if (budget > 0 && (index_sets == nullptr || !aligned(index_sets, 4))) return LSA_ERR_INVALID_ARG;
    for (int g = 0; g < layers_per_index; ++g) {
        if (q[g] == nullptr || k_cache[g] == nullptr || v_cache[g] == nullptr || out[g] == nullptr)
            return LSA_ERR_INVALID_ARG;
        if (!aligned(q[g], 16) || !aligned(k_cache[g], 16) || !aligned(v_cache[g], 16) || !aligned(out[g], 16))
            return LSA_ERR_INVALID_ARG;
    }
    const lsa::AttendPlan p = lsa::plan_attend_grouped(batch->n_q, group_rows, H_q, H_kv, budget, layers_per_index,
                                                       lsa::device_sm_count());
    if (workspace == nullptr || workspace_bytes < p.ws_bytes || !aligned(workspace, 256)) return LSA_ERR_WORKSPACE;
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    lsa::AttendArgs a;
    std::memset(&a, 0, sizeof a);
    for (int g = 0; g < layers_per_index; ++g) {
        a.q[g] = q[g];
        a.k[g] = k_cache[g];
        a.v[g] = v_cache[g];
        a.out[g] = out[g];
        a.kscale[g] = 1.f;
        a.vscale[g] = 1.f;
    }
    a.sets = index_sets;
    a.kv_offset = batch->kv_offset;
    a.seq_lens = batch->seq_lens;
    a.q_seq = batch->q_seq;
    a.q_len = batch->q_len;
    a.dev_status = dev_status;
    const size_t rows_q = (size_t)layers_per_index * batch->n_q;
    if (p.n_splits > 1) {
        a.part_o = reinterpret_cast<float*>(ws);
        const size_t off = (rows_q * p.n_splits * H_q * 128 * 4 + 255) / 256 * 256;
        a.part_ml = reinterpret_cast<float*>(ws + off);
    }
    a.total_tokens = batch->total_tokens;
    a.n_seq = batch->n_seq;
    a.n_q = batch->n_q;
    a.max_len = batch->max_len;
    a.H_q = H_q;
    a.H_kv = H_kv;
    a.budget = budget;
    a.G = layers_per_index;
    a.n_splits = p.n_splits;
    a.entries_per_split = p.entries_per_split;
    a.head_groups = p.head_groups;
    a.hpc = p.hpc;
    a.rows_per_cta = p.rows_per_cta;
    a.stage_off = p.stage_off;
    a.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)d));
    a.group_rows = group_rows;
    cudaError_t e = lsa::launch_attend_grouped(a, p.smem_bytes, reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? LSA_OK : cuda_fail(e);
}

lsa_status_t lsa_shard_sets(const int32_t* index_sets, int32_t n_q, int32_t budget, int32_t lo, int32_t hi,
                            int32_t* local_sets, int32_t* dev_status, void* stream) {
    if (n_q < 0 || budget < 0 || lo < 0 || hi < lo) return LSA_ERR_INVALID_ARG;
    if (budget > LSA_MAX_BUDGET || n_q > 65535) return LSA_ERR_UNSUPPORTED;
    if (n_q == 0 || budget == 0) return LSA_OK;
    if (index_sets == nullptr || local_sets == nullptr || index_sets == local_sets) return LSA_ERR_INVALID_ARG;
    if (!aligned(index_sets, 4) || !aligned(local_sets, 4)) return LSA_ERR_INVALID_ARG;
    cudaError_t e = lsa::launch_shard_sets(index_sets, n_q, budget, lo, hi, local_sets, dev_status,
                                           reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? LSA_OK : cuda_fail(e);
}

lsa_status_t lsa_combine(const float* o_parts, const float* lse_parts, int32_t n_parts, int64_t rows, int32_t d,
                         float* out, float* lse_out, void* stream) {
    if (n_parts < 1 || rows < 0 || d < 0 || d % 4 != 0) return LSA_ERR_INVALID_ARG;
    if (n_parts > 65535 || (rows + 7) / 8 > 0x7fffffff) return LSA_ERR_UNSUPPORTED;
    if (rows == 0 || d == 0) return LSA_OK;
    if (o_parts == nullptr || lse_parts == nullptr || out == nullptr) return LSA_ERR_INVALID_ARG;
    if (!aligned(o_parts, 16) || !aligned(lse_parts, 4) || !aligned(out, 16)) return LSA_ERR_INVALID_ARG;
    if (lse_out != nullptr && !aligned(lse_out, 4)) return LSA_ERR_INVALID_ARG;
    cudaError_t e = lsa::launch_combine(o_parts, lse_parts, n_parts, rows, d, out, lse_out,
                                        reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? LSA_OK : cuda_fail(e);
}

static lsa_status_t point_common(const int8_t* q_idx, const int32_t* w, int32_t w_max, int32_t H_I, int32_t d_I,
                                 int32_t n_q, const int64_t* row_base, const int32_t* ids, int32_t n,
                                 lsa::PointArgs& p) {
    if (n_q < 0 || n < 0 || H_I < 1 || d_I < 1 || w_max < 0) return LSA_ERR_INVALID_ARG;
    if (d_I != 32 && d_I != 64 && d_I != 128) return LSA_ERR_UNSUPPORTED;
    if (H_I > LSA_MAX_HEADS_I || n_q > 65535) return LSA_ERR_UNSUPPORTED;
    if ((double)H_I * (double)w_max * (double)d_I * 16384.0 >= 2147483648.0) return LSA_ERR_UNSUPPORTED;
    if (n_q == 0 || n == 0) return LSA_OK;
    if (q_idx == nullptr || w == nullptr || row_base == nullptr || ids == nullptr) return LSA_ERR_INVALID_ARG;
    if (!aligned(q_idx, 16) || !aligned(w, 4) || !aligned(row_base, 8) || !aligned(ids, 4))
        return LSA_ERR_INVALID_ARG;
    std::memset(&p, 0, sizeof p);
    p.a.q_idx = q_idx;
    p.a.w = w;
    p.a.w_max = w_max;
    p.a.H_I = H_I;
    p.a.n_q = n_q;
    p.ids = ids;
    p.row_base = row_base;
    p.n = n;
    return LSA_OK;
}

lsa_status_t lsa_score_tokens(const int8_t* q_idx, const int8_t* k_idx_cache, const int32_t* w, int32_t w_max,
                              int32_t H_I, int32_t d_I, int32_t n_q, const int64_t* row_offset, int64_t total_tokens,
                              const int32_t* positions, int32_t n, uint32_t* keys, int32_t* dev_status,
                              void* stream) {
    lsa::PointArgs p;
    lsa_status_t st = point_common(q_idx, w, w_max, H_I, d_I, n_q, row_offset, positions, n, p);
    if (st != LSA_OK || n_q == 0 || n == 0) return st;
    if (k_idx_cache == nullptr || keys == nullptr || total_tokens < 0) return LSA_ERR_INVALID_ARG;
    if (!aligned(k_idx_cache, 16) || !aligned(keys, 4)) return LSA_ERR_INVALID_ARG;
    p.a.k_idx = k_idx_cache;
    p.a.dev_status = dev_status;
    p.rows = total_tokens;
    p.out_tokens = keys;
    p.blocks = 0;
    cudaError_t e = lsa::launch_point_scores(p, d_I, reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? LSA_OK : cuda_fail(e);
}

lsa_status_t lsa_score_blocks(const int8_t* q_idx, const int32_t* w, int32_t w_max, int32_t H_I, int32_t d_I,
                              int32_t n_q, const int8_t* block_sums, int64_t block_rows, const int64_t* blk_row_offset,
                              const int32_t* blocks, int32_t n, uint64_t* keys, int32_t* dev_status, void* stream) {
    lsa::PointArgs p;
    lsa_status_t st = point_common(q_idx, w, w_max, H_I, d_I, n_q, blk_row_offset, blocks, n, p);
    if (st != LSA_OK || n_q == 0 || n == 0) return st;
    if (block_sums == nullptr || keys == nullptr || block_rows < 0) return LSA_ERR_INVALID_ARG;
    if (!aligned(block_sums, 16) || !aligned(keys, 8)) return LSA_ERR_INVALID_ARG;
    p.a.block_sums = block_sums;
    p.a.dev_status = dev_status;
    p.rows = block_rows;
    p.out_blocks = keys;
    p.blocks = 1;
    cudaError_t e = lsa::launch_point_scores(p, d_I, reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? LSA_OK : cuda_fail(e);
}

lsa_status_t lsa_merge_pairs(const uint64_t* pairs, const int32_t* counts, int32_t n_rows, int32_t cap, int32_t k,
                             int32_t* out, uint64_t* out_values, int32_t* dev_status, void* stream) {
    if (n_rows < 0 || cap < 0 || k < 0) return LSA_ERR_INVALID_ARG;
    if (k > LSA_MAX_BUDGET || n_rows > 65535) return LSA_ERR_UNSUPPORTED;
    if (n_rows == 0 || k == 0) return LSA_OK;
    if (pairs == nullptr || counts == nullptr || out == nullptr) return LSA_ERR_INVALID_ARG;
    if (!aligned(pairs, 16) || !aligned(counts, 4) || !aligned(out, 4)) return LSA_ERR_INVALID_ARG;
    if (out_values != nullptr && !aligned(out_values, 8)) return LSA_ERR_INVALID_ARG;
    cudaError_t e = lsa::launch_merge_pairs(pairs, counts, n_rows, cap, k, out, out_values, dev_status,
                                            reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? LSA_OK : cuda_fail(e);
}

lsa_status_t lsa_attend_fp8(const uint16_t* const* q, const uint8_t* const* k_cache, const uint8_t* const* v_cache,
                            const float* k_scale, const float* v_scale, int32_t H_q, int32_t H_kv, int32_t d,
                            const int32_t* index_sets, int32_t budget, const lsa_batch_t* batch,
                            int32_t layers_per_index, float* const* out, void* workspace, size_t workspace_bytes,
                            int32_t* dev_status, void* stream) {
    if (k_scale == nullptr || v_scale == nullptr) return LSA_ERR_INVALID_ARG;
    return attend_impl(q, reinterpret_cast<const void* const*>(k_cache), reinterpret_cast<const void* const*>(v_cache),
                       k_scale, v_scale, H_q, H_kv, d, index_sets, budget, batch, layers_per_index, out, nullptr,
                       workspace, workspace_bytes, dev_status, stream);
}

}  // extern "C"
