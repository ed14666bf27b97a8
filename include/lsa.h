/*
 * lsa.h — C ABI of liblsa.so, the B200 (sm_100a) implementation of the
 * LongCat Sparse Attention (LSA) decode/prefill hot path.
 *
 * What the method is (the pages give mechanisms, not formulas):
 *  - "LongCat-2.0: Meituan이 Nvidia GPU 없이 ... (molayo1419.me)", section
 *    "1M 토큰에서의 Sparse Attention 문제": LSA extends DeepSeek Sparse
 *    Attention (an indexer scores every cached token and a top-k is kept)
 *    with Streaming-aware Indexing (SI), Cross-Layer Indexing (CLI) and
 *    Hierarchical Indexing (HI).
 *  - "LongCat-Flash-Lite-Sparse (aitrends.kr)", section "기술적 특징": SI
 *    gives part of the budget to fixed sinks and a local sliding window so KV
 *    reads become contiguous; CLI reuses one index result over adjacent
 *    layers; HI keeps coarse candidate blocks first and selects fine tokens
 *    only inside them.
 *  The arithmetic this library fixes:
 *    fine score   score_t = sum_h w_h * max(0, q_h . k_t), int8 q and k,
 *                 exact integer accumulation;
 *    coarse score c_b     = the same formula on S_b, the exact sum of the
 *                 indexer keys of block b;
 *    selection    the topk highest scores of the "middle" tokens, ties to
 *                 the lower position (blocks: the lower block index);
 *    index set    [0, s) U selected U [ws, L), ascending, padded with -1,
 *                 where s = min(sink, L) and ws = max(s, L - window);
 *    attention    o = softmax(q . k_j / sqrt(d)) v_j over the set, GQA with
 *                 query head h reading kv head floor(h * H_kv / H_q), bf16
 *                 inputs, fp32 accumulation and fp32 output.
 *
 * Conventions for every entry point:
 *  - Pointers marked "device" are CUDA device pointers (e.g. a torch tensor's
 *    data_ptr()); pointers marked "host" are ordinary host memory read during
 *    the call. The caller owns every buffer; the library allocates nothing
 *    and never frees caller memory. Between calls it keeps only read-only
 *    facts (each device's SM count, the driver's tensor-map entry point) and
 *    the static scratch of lsa_attend_noalloc.
 *  - `stream` is a cudaStream_t passed as void*. Every call is asynchronous
 *    on that stream and returns without synchronising.
 *  - Argument and shape errors are returned synchronously, before any launch,
 *    as an lsa_status_t. LSA_ERR_CUDA reports a failed launch (call
 *    lsa_last_cuda_error() for the CUDA error code).
 *  - Errors only the device can see (bad lengths or indices in device arrays)
 *    are OR-ed as LSA_DEV_* bits into *dev_status (device int32, may be
 *    NULL); the caller reads it after synchronising. The offending query's
 *    output is then unspecified but every access stays in bounds.
 *  - No kernel spins on another CTA, kernel or device. The only cross-CTA
 *    waits are hardware barriers: thread-block-cluster barriers (a cluster's
 *    CTAs are scheduled together) and the programmatic-launch wait for the
 *    preceding kernel on the stream. Waits on a CTA's own asynchronous copies
 *    are bounded by a time limit after which the kernel sets LSA_DEV_TIMEOUT
 *    and returns, so no call can hang; no kernel traps.
 *  - Calls are thread-safe when they use distinct workspaces.
 *  - Kernels are launched with programmatic stream serialisation: a kernel
 *    may start before the preceding kernel on the stream has finished when
 *    that kernel allows it (griddepcontrol.launch_dependents), and it reads
 *    the batch's row metadata (q_seq, q_len, kv_offset, seq_lens, blk_offset)
 *    before waiting for it; everything else is read after the wait. A caller
 *    whose own kernels trigger dependent launches must write those arrays
 *    before triggering.
 */
#ifndef LSA_H_
#define LSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    LSA_OK = 0,
    LSA_ERR_INVALID_ARG = 1, /* null pointer, negative size, bad shape */
    LSA_ERR_UNSUPPORTED = 2, /* valid but outside the compiled range */
    LSA_ERR_CUDA = 3,        /* a CUDA runtime call or launch failed */
    LSA_ERR_WORKSPACE = 4    /* workspace pointer null or smaller than required */
} lsa_status_t;

/* Bits OR-ed into *dev_status by device-side checks. */
#define LSA_DEV_BAD_LENGTH 0x1 /* q_len/seq_lens outside [1, max_len] or past the cache */
#define LSA_DEV_BAD_SEQ 0x2    /* q_seq outside [0, n_seq) */
#define LSA_DEV_BAD_INDEX 0x4  /* an index-set entry < -1 or >= q_len (entry skipped) */
#define LSA_DEV_BAD_WEIGHT 0x8 /* an indexer head weight outside [0, w_max] (treated as 0) */
#define LSA_DEV_TIMEOUT 0x10   /* a bounded wait inside a kernel gave up (output unspecified) */
#define LSA_DEV_BAD_QUERY 0x20 /* lsa_attend_fp8: a query element outside the fp16 range
                                  (|q| >= 65536 as bf16, or not finite); the row's output is
                                  unspecified */
#define LSA_DEV_BAD_VALUE 0x40 /* lsa_attend_si: a V element of magnitude >= 65520 (or not
                                  finite) in a sink or window run, which that call multiplies
                                  in fp16; the outputs of the rows that read it are unspecified */

/* Selection budget. sink + window + topk is the index-set length ("budget").
 * hi_block == 0 switches HI off; otherwise blocks of hi_block tokens aligned
 * at position 0 are scored coarsely and the hi_topblocks best are kept. */
typedef struct {
    int32_t sink;
    int32_t window;
    int32_t topk;
    int32_t hi_block;
    int32_t hi_topblocks;
} lsa_budget_t;

/* A batch of query rows over packed sequences.
 *  Decode: one row per sequence, q_len[r] = seq_lens[q_seq[r]] (the current
 *  token's K/V and indexer key are already in the cache).
 *  Prefill: the rows of a chunk of n new tokens appended to a cache of C
 *  tokens see q_len = C + i + 1 for i = 0..n-1. */
typedef struct {
    int32_t n_seq;            /* number of sequences, >= 1 */
    int32_t n_q;              /* number of query rows, >= 0 */
    int32_t max_len;          /* host-side upper bound on every q_len and seq_lens */
    int32_t reserved;         /* must be 0 */
    int64_t total_tokens;     /* rows in the packed caches (bounds every access) */
    const int64_t *kv_offset; /* device [n_seq]: first cache row of each sequence */
    const int32_t *seq_lens;  /* device [n_seq]: tokens present in each sequence */
    const int64_t *blk_offset;/* device [n_seq]: first block-sum row of each sequence
                                 (HI only; NULL when HI is off) */
    const int32_t *q_seq;     /* device [n_q]: sequence of each query row */
    const int32_t *q_len;     /* device [n_q]: visible length of each query row */
} lsa_batch_t;

/* Largest sizes the kernels are compiled for. */
#define LSA_MAX_HEADS_I 64    /* H_I */
#define LSA_MAX_BUDGET 16384  /* sink + window + topk */
#define LSA_MAX_HI_BLOCK 256  /* hi_block (block sums stay exact in 16 bits) */
#define LSA_MAX_TOPBLOCKS 4096
#define LSA_MAX_LAYERS 8      /* layers sharing one index set (CLI group) */

/* Library version, as MAJOR*10000 + MINOR*100 + PATCH. */
int32_t lsa_version(void);

/* CUDA error code (cudaError_t) of the last LSA_ERR_CUDA on this thread. */
int32_t lsa_last_cuda_error(void);

/* Human-readable name of a status code (static string). */
const char *lsa_status_string(int32_t status);

/* ----------------------------------------------------------------------- */
/* HI block-sum pre-pass                                                     */
/* ----------------------------------------------------------------------- */
/* Computes the per-block key sums S_b[d] = sum of k_t[d] over the present
 * tokens t of block b (blocks of hi_block tokens aligned at position 0; the
 * last may be partial). HI's "fast approximate block-level pass" scores
 * these instead of every token (Flash-Lite-Sparse page, "기술적 특징",
 * Hierarchical Indexing bullet).
 *
 * k_idx_cache  device int8 [total_tokens][d_I], sequences packed by kv_offset.
 * block_sums   device int8 [rows][2*d_I]. Sequence b's blocks are the rows
 *              blk_offset[b] .. blk_offset[b] + ceil(seq_lens[b]/hi_block) - 1.
 *              Each row stores S_b exactly in two byte planes: bytes
 *              [0, d_I) hold S >> 8 as int8 and bytes [d_I, 2*d_I) hold
 *              S & 0xFF as uint8, so S = 256*hi + lo (|S| <= 128*hi_block).
 * block_rows   rows of block_sums (a sequence whose rows would fall outside
 *              sets LSA_DEV_BAD_LENGTH and is skipped).
 * n_new        <= 0: rebuild every block of every sequence. > 0: rebuild only
 *              the blocks that hold the last n_new tokens of each sequence
 *              (the decode append update; n_new = 1 for one new token).
 * Supported: d_I in {32, 64, 128}; 1 <= hi_block <= LSA_MAX_HI_BLOCK.
 */
lsa_status_t lsa_hi_block_sums(const int8_t *k_idx_cache, int32_t d_I,
                               int32_t hi_block, const lsa_batch_t *batch,
                               int32_t n_new, int8_t *block_sums,
                               int64_t block_rows, int32_t *dev_status,
                               void *stream);

/* ----------------------------------------------------------------------- */
/* Decode append                                                             */
/* ----------------------------------------------------------------------- */
/* Writes the n_new newest tokens of every sequence into the caches and, with
 * HI on, refreshes the block sums of the blocks that hold them, in one
 * launch: the step just before indexing in a decode loop, so that the block
 * sums stay resident and exact as the cache grows (the HI block pass of the
 * Flash-Lite-Sparse page, "기술적 특징", Hierarchical Indexing bullet, over
 * a cache that gains a token per step).
 *
 * For sequence b the new tokens are positions seq_lens[b] - n_new ..
 * seq_lens[b] - 1 (seq_lens already counts them; 1 <= n_new <= seq_lens[b],
 * else LSA_DEV_BAD_LENGTH and the sequence is skipped).
 * k_idx_new    device int8 [n_seq][n_new][d_I]: the new indexer keys.
 * k_idx_cache  device int8 [total_tokens][d_I], written at the new positions.
 * k_new, v_new host [layers] arrays of device [n_seq][n_new] rows of
 *              kv_row_bytes bytes each (one token's K or V of one layer:
 *              H_kv*d*2 for bf16 caches, H_kv*d for FP8 E4M3 caches).
 * k_cache, v_cache host [layers] arrays of device [total_tokens] rows of
 *              kv_row_bytes bytes, written at the new positions. The rows
 *              are copied as bytes. layers may be 0 (indexer keys only);
 *              the arrays may then be NULL.
 * block_sums   as for lsa_hi_block_sums, or NULL when hi_block == 0. The
 *              refreshed blocks are summed from the new keys (read from
 *              k_idx_new) and the older keys of the block (from the cache).
 * All device pointers 16-byte aligned; the inputs must not overlap the
 * cache rows being written. Supported: d_I in {32, 64, 128}; kv_row_bytes
 * a positive multiple of 16 (when layers > 0); 0 <= layers <=
 * LSA_MAX_LAYERS; 0 <= hi_block <= LSA_MAX_HI_BLOCK.
 */
lsa_status_t lsa_append(const int8_t *k_idx_new, int8_t *k_idx_cache, int32_t d_I,
                        const void *const *k_new, const void *const *v_new,
                        void *const *k_cache, void *const *v_cache,
                        int32_t kv_row_bytes, int32_t layers, int32_t hi_block,
                        int8_t *block_sums, int64_t block_rows,
                        const lsa_batch_t *batch, int32_t n_new,
                        int32_t *dev_status, void *stream);

/* ----------------------------------------------------------------------- */
/* Indexer: scores, HI, top-k, SI assembly                                   */
/* ----------------------------------------------------------------------- */
/* Workspace bytes lsa_index needs for this batch shape (reads only the host
 * fields of *batch). 0 means no workspace is needed. */
size_t lsa_index_workspace_size(const lsa_batch_t *batch, int32_t H_I,
                                int32_t d_I, lsa_budget_t budget);

/* 1 when lsa_index would score this batch's fine candidates as one dense
 * int8 contraction on the tcgen05 tensor cores, else 0 (reads only host
 * fields). That path serves a prefill chunk: HI off, every row in one
 * sequence (n_seq == 1), at least 64 rows, H_I == 16, d_I == 128; other
 * batches are scored per row. Both paths give bit-identical index sets. The
 * pages define the score, not how to evaluate it; this call only reports the
 * evaluation strategy. */
int32_t lsa_index_uses_tensor_cores(const lsa_batch_t *batch, int32_t H_I,
                                    int32_t d_I, lsa_budget_t budget);

/* Number of kernel launches lsa_index issues for this shape (host fields
 * only), e.g. for accounting in benchmarks. 0 for an invalid shape. */
int32_t lsa_index_launches(const lsa_batch_t *batch, int32_t H_I, int32_t d_I,
                           lsa_budget_t budget);

/* One index set per query row (CLI: call once per group of layers and pass
 * the result to lsa_attend with layers_per_index = G).
 *
 * What the set is: LSA keeps DeepSeek Sparse Attention's indexer (every
 * candidate cached token is scored, a top-k is kept) and adds three
 * mechanisms ("LongCat-2.0 (molayo1419.me)", section "1M 토큰에서의 Sparse
 * Attention 문제"). This call evaluates them as follows:
 *  - SI ("LongCat-Flash-Lite-Sparse (aitrends.kr)", section "기술적 특징",
 *    first bullet): the budget has a fixed sink run [0, s) and a local
 *    window run [ws, L) that are always kept; the top-k competes only over
 *    the middle [s, ws).
 *  - HI (same section, third bullet): with hi_block > 0 the middle's blocks
 *    are scored coarsely on their key sums, the hi_topblocks best are kept,
 *    and the fine top-k runs only over the middle tokens inside them.
 *  - CLI (same section, second bullet): one set serves G adjacent layers;
 *    lsa_index runs once per group.
 * The fine score, the coarse score and the tie rule are the ones fixed at
 * the top of this file.
 *
 * q_idx        device int8 [n_q][H_I][d_I] indexer queries.
 * k_idx_cache  device int8 [total_tokens][d_I] indexer keys (one per token,
 *              shared by all indexer heads).
 * w            device int32 [n_q][H_I] head weights in [0, w_max].
 * w_max        host bound on w; H_I * w_max * d_I * 16384 must be < 2^31 so
 *              that fine scores are exact in int32 (else LSA_ERR_UNSUPPORTED).
 * block_sums   device, as written by lsa_hi_block_sums (HI on), or NULL when
 *              hi_block == 0; block_rows is its row count.
 * index_sets   device int32 [n_q][sink+window+topk] output: positions relative
 *              to the sequence start, ascending, -1 padded.
 * workspace    device scratch of lsa_index_workspace_size() bytes (may be NULL
 *              when that size is 0). Not needed after the call returns on the
 *              stream.
 * Supported: d_I in {32, 64, 128}; 1 <= H_I <= LSA_MAX_HEADS_I;
 * budget <= LSA_MAX_BUDGET; hi_topblocks <= LSA_MAX_TOPBLOCKS. With HI on, a
 * row's blocks are summed over the tokens the row sees: a row that sees
 * fewer tokens than its sequence holds (q_len < seq_lens: prefill chunks,
 * draft rows) has the block holding its last visible token, when that block
 * is a candidate, re-summed from the keys instead of read from block_sums
 * (whose row covers every cached token of the block).
 */
lsa_status_t lsa_index(const int8_t *q_idx, const int8_t *k_idx_cache,
                       const int32_t *w, int32_t w_max, int32_t H_I, int32_t d_I,
                       const lsa_batch_t *batch, lsa_budget_t budget,
                       const int8_t *block_sums, int64_t block_rows,
                       int32_t *index_sets,
                       void *workspace, size_t workspace_bytes,
                       int32_t *dev_status, void *stream);

/* ----------------------------------------------------------------------- */
/* Decode append and index in one call                                       */
/* ----------------------------------------------------------------------- */
/* lsa_append followed by lsa_index on the same batch, with the results of
 * those two calls in that order (a decode step's first two calls: the new
 * tokens enter the cache whose keys and block sums the HI block pass of the
 * Flash-Lite-Sparse page, "기술적 특징", Hierarchical Indexing bullet,
 * scores).
 *
 * When HI is on and budget.window >= hi_block + n_new - 1, the n_new newest
 * tokens of every sequence lie in every row's window: the index call reads
 * no key, block sum or K/V row that the append writes, and the append runs in
 * extra CTAs of the block selection's grid instead of a launch of its own
 * (one kernel boundary fewer in the step). Otherwise the two calls' kernels
 * are launched one after the other.
 *
 * Arguments: those of lsa_append (k_idx_new, k_new, v_new, k_cache, v_cache,
 * kv_row_bytes, layers, n_new; hi_block is budget.hi_block) and of lsa_index
 * (q_idx, k_idx_cache, w, w_max, H_I, d_I, batch, budget, block_sums,
 * block_rows, index_sets, workspace, workspace_bytes), with the same meaning,
 * layout, ownership and support limits; workspace is lsa_index's. Every check
 * of both calls runs before the first launch: a refused call launches
 * nothing. Device errors set the same dev_status bits as the two calls.
 */
lsa_status_t lsa_append_index(const int8_t *k_idx_new, const void *const *k_new,
                              const void *const *v_new, void *const *k_cache,
                              void *const *v_cache, int32_t kv_row_bytes,
                              int32_t layers, int32_t n_new,
                              const int8_t *q_idx, int8_t *k_idx_cache,
                              const int32_t *w, int32_t w_max, int32_t H_I,
                              int32_t d_I, const lsa_batch_t *batch,
                              lsa_budget_t budget, int8_t *block_sums,
                              int64_t block_rows, int32_t *index_sets,
                              void *workspace, size_t workspace_bytes,
                              int32_t *dev_status, void *stream);

/* Kernel launches lsa_append_index makes for this shape (reads only host
 * fields): lsa_index_launches, plus one when the append is not fused. 0 for
 * invalid arguments. */
int32_t lsa_append_index_launches(const lsa_batch_t *batch, int32_t H_I,
                                  int32_t d_I, lsa_budget_t budget,
                                  int32_t n_new);

/* ----------------------------------------------------------------------- */
/* Sparse attention over the index sets (all G layers of a CLI group)        */
/* ----------------------------------------------------------------------- */
/* Workspace bytes lsa_attend needs (split partials; contents need no
 * initialisation: every call writes what it later reads). */
size_t lsa_attend_workspace_size(const lsa_batch_t *batch, int32_t H_q,
                                 int32_t H_kv, int32_t d, int32_t budget,
                                 int32_t layers_per_index);

/* Number of kernel launches lsa_attend issues for this shape (host fields
 * only): the attention kernel, plus a merge kernel when the budget is split
 * over several CTAs per row. 0 for an invalid shape. */
int32_t lsa_attend_launches(const lsa_batch_t *batch, int32_t H_q,
                            int32_t H_kv, int32_t d, int32_t budget,
                            int32_t layers_per_index);

/* o[g][r][h] = softmax_j(q . k_j / sqrt(d)) v_j over the entries j of
 * index_sets[r] that are not -1, for every layer g < layers_per_index
 * (Cross-Layer Indexing: all G layers share one set).
 *
 * This is the attention that follows LSA's token selection: softmax
 * attention restricted to the selected KV rows ("LongCat-2.0 (molayo1419.me)",
 * section "1M 토큰에서의 Sparse Attention 문제"). Its reads are the ones SI
 * makes contiguous: the sink and window runs of every set are sequential KV
 * reads ("LongCat-Flash-Lite-Sparse (aitrends.kr)", section "기술적 특징",
 * first bullet), and CLI lets one set drive the G layers of a group (same
 * section, second bullet). Scale 1/sqrt(d), GQA groups as fixed at the top
 * of this file.
 *
 * q            host [G] array of device bf16 [n_q][H_q][d] (bit patterns).
 * k_cache      host [G] array of device bf16 [total_tokens][H_kv][d].
 * v_cache      host [G] array of device bf16 [total_tokens][H_kv][d].
 * index_sets   device int32 [n_q][budget] (e.g. from lsa_index). Entries
 *              < -1 or >= q_len set LSA_DEV_BAD_INDEX and are skipped.
 * out          host [G] array of device fp32 [n_q][H_q][d]. A row whose set
 *              is empty is written as zeros.
 * Supported: d == 128; H_q % H_kv == 0 and H_q / H_kv in {1, 2, 4, 8, 16};
 * H_kv in {1, 2, 4} or a multiple of 4; 1 <= G <= LSA_MAX_LAYERS;
 * budget <= LSA_MAX_BUDGET.
 */
lsa_status_t lsa_attend(const uint16_t *const *q, const uint16_t *const *k_cache,
                        const uint16_t *const *v_cache, int32_t H_q, int32_t H_kv,
                        int32_t d, const int32_t *index_sets, int32_t budget,
                        const lsa_batch_t *batch, int32_t layers_per_index,
                        float *const *out, void *workspace, size_t workspace_bytes,
                        int32_t *dev_status, void *stream);

/* lsa_attend over an FP8 KV cache. The pages name FP8 variants of the
 * models and a KV-cache data type but fix neither the format nor its
 * scaling; this call reads the cache as OCP FP8 E4M3 codes (1 sign, 4
 * exponent bits with bias 7, 3 mantissa bits, subnormals, no infinities)
 * with one scale per layer for K and one for V: k = k_scale[g] * E4M3(code),
 * v = v_scale[g] * E4M3(code). Everything else — the set, the softmax, the
 * GQA mapping, the output, the workspace (lsa_attend_workspace_size) and the
 * device-side errors — is lsa_attend's.
 *
 * q                 as for lsa_attend. The products run on fp16 tensor cores:
 *                   every E4M3 value is an fp16, and so is every bf16 query
 *                   element of magnitude below 65536 (elements below 2^-14 keep
 *                   fp16's subnormal precision). A query element of magnitude
 *                   65536 or more, or not finite, sets LSA_DEV_BAD_QUERY.
 * k_cache, v_cache  host [G] arrays of device uint8 [total_tokens][H_kv][d]
 *                   E4M3 codes (NaN codes give unspecified output).
 * k_scale, v_scale  host [G] arrays of finite floats.
 * Supported: as lsa_attend, with H_q / H_kv <= 8 (else LSA_ERR_UNSUPPORTED).
 */
lsa_status_t lsa_attend_fp8(const uint16_t *const *q, const uint8_t *const *k_cache,
                            const uint8_t *const *v_cache, const float *k_scale,
                            const float *v_scale, int32_t H_q, int32_t H_kv, int32_t d,
                            const int32_t *index_sets, int32_t budget,
                            const lsa_batch_t *batch, int32_t layers_per_index,
                            float *const *out, void *workspace, size_t workspace_bytes,
                            int32_t *dev_status, void *stream);

/* ----------------------------------------------------------------------- */
/* Prefill attention: sink and window runs as dense tiles                    */
/* ----------------------------------------------------------------------- */
/* lsa_attend_si is the attention of lsa_attend over sets with the SI
 * structure lsa_index writes: the sink run [0, s), the selected tokens, the
 * window run [ws, L) ("LongCat-Flash-Lite-Sparse (aitrends.kr)", section
 * "기술적 특징", SI bullet; s = min(sink, L), ws = max(s, L - window)). It
 * attends each row over
 *    [0, s)  +  entries [s, s + m) of its set  +  [ws, L),   m = min(topk, ws - s),
 * taking the two runs from the positions, not from the set: for a set
 * lsa_index wrote with this budget it equals lsa_attend. Meant for the rows of
 * a causal prefill chunk, whose neighbouring rows share their sink and (all
 * but one position of) their window runs: those runs are attended as dense
 * tiles of 16 rows over K/V tiles in shared memory, the selected entries by
 * the per-row gather, and the two partials combined by their log-sum-exp.
 *
 * Arguments and device-side errors as lsa_attend, with the budget (sink,
 * window, topk; hi_block and hi_topblocks unused) instead of the set length
 * (sets are [n_q][sink + window + topk]); workspace of
 * lsa_attend_si_workspace_size() bytes.
 * The dense tiles multiply P V in fp16 (every bf16 below 65520 in magnitude
 * is an fp16; P keeps 11 significant bits): a V element of the sink or window
 * runs of magnitude 65520 or more sets LSA_DEV_BAD_VALUE.
 * Supported: one sequence (n_seq == 1), d == 128, H_q / H_kv <= 8, bf16 caches.
 */
size_t lsa_attend_si_workspace_size(const lsa_batch_t *batch, int32_t H_q, int32_t H_kv, int32_t d,
                                    lsa_budget_t budget, int32_t layers_per_index);
int32_t lsa_attend_si_launches(const lsa_batch_t *batch, int32_t H_q, int32_t H_kv, int32_t d,
                               lsa_budget_t budget, int32_t layers_per_index);
lsa_status_t lsa_attend_si(const uint16_t *const *q, const uint16_t *const *k_cache,
                           const uint16_t *const *v_cache, int32_t H_q, int32_t H_kv, int32_t d,
                           const int32_t *index_sets, lsa_budget_t budget,
                           const lsa_batch_t *batch, int32_t layers_per_index,
                           float *const *out, void *workspace, size_t workspace_bytes,
                           int32_t *dev_status, void *stream);

/* ----------------------------------------------------------------------- */
/* Draft rows sharing one gather                                             */
/* ----------------------------------------------------------------------- */
/* A decode step that verifies several draft tokens of a sequence at once
 * (multi-token prediction for speculative decoding, "LongCat-2.0
 * (molayo1419.me)", section "1M 토큰에서의 Sparse Attention 문제") has one
 * decode row per draft token. Their index sets share the sink run, nearly all
 * of the window run and, where the drafts' indexer queries agree, much of
 * the selection.
 *
 * lsa_attend_grouped computes exactly what lsa_attend computes for the same
 * arguments (every row over its own set, invalid entries flagged and
 * skipped alike), for batches whose rows come in groups of group_rows
 * consecutive rows of one sequence (row g * group_rows + j is draft j of group
 * g, as the decode rows of lsa_batch_t with several rows per sequence are laid
 * out). The rows of a group are attended together: each stretch of their
 * sets (the same entry range of every row) runs in one CTA, so for sets as
 * lsa_index writes them (ascending, sink run first, window run last) the rows
 * walk the same positions at the same time and a K/V row several of them hold
 * is read from HBM once and served to the others on chip. Any other set is
 * still attended exactly.
 *
 * Arguments, output and device-side errors as lsa_attend, plus
 * group_rows  1, 2, 4 or 8; n_q must be a multiple of it.
 * workspace   lsa_attend_grouped_workspace_size() bytes (split partials; no
 *             initialisation needed).
 * Supported: the shapes lsa_attend supports with H_q / H_kv <= 8 and bf16
 * caches, n_q / group_rows <= 65535. One launch, plus a split merge with
 * several splits.
 */
size_t lsa_attend_grouped_workspace_size(const lsa_batch_t *batch, int32_t H_q, int32_t H_kv,
                                         int32_t d, int32_t budget, int32_t layers_per_index,
                                         int32_t group_rows);
int32_t lsa_attend_grouped_launches(const lsa_batch_t *batch, int32_t H_q, int32_t H_kv,
                                    int32_t d, int32_t budget, int32_t layers_per_index,
                                    int32_t group_rows);
lsa_status_t lsa_attend_grouped(const uint16_t *const *q, const uint16_t *const *k_cache,
                                const uint16_t *const *v_cache, int32_t H_q, int32_t H_kv,
                                int32_t d, const int32_t *index_sets, int32_t budget,
                                const lsa_batch_t *batch, int32_t layers_per_index,
                                int32_t group_rows, float *const *out, void *workspace,
                                size_t workspace_bytes, int32_t *dev_status, void *stream);

/* ----------------------------------------------------------------------- */
/* Context-parallel merge                                                    */
/* ----------------------------------------------------------------------- */
/* When one sequence's cache is split by token range over several GPUs, each
 * GPU keeps its own best candidates (HI blocks, then middle tokens) and the
 * exact global choice is the best of their union: a block or token among
 * the global top-k is among the top-k of its own shard under the same order.
 * This call is that merge step, after the candidates of every shard have
 * been gathered (e.g. with one all-gather). It keeps the order of the
 * selection rules fixed at the top of this file (score descending, ties to
 * the lower id), the HI bullet and the top-k of "LongCat-Flash-Lite-Sparse
 * (aitrends.kr)", section "기술적 특징", and "LongCat-2.0 (molayo1419.me)",
 * section "1M 토큰에서의 Sparse Attention 문제".
 *
 * pairs   device uint64 [n_rows][cap]. Entry = (key << LSA_MERGE_ID_BITS) |
 *         (2^LSA_MERGE_ID_BITS - 1 - id) with 0 <= id < 2^LSA_MERGE_ID_BITS and
 *         1 <= key < 2^(64 - LSA_MERGE_ID_BITS) (e.g. the score + 1); a value of 0
 *         is an empty slot and is skipped. The entries of a row must be
 *         distinct (distinct ids). Larger values rank first: key descending,
 *         ties to the lower id.
 * counts  device int32 [n_rows]: slots used in each row (outside [0, cap]: the
 *         row is clamped and LSA_DEV_BAD_LENGTH is set).
 * out     device int32 [n_rows][k]: the ids of the k best entries of each row,
 *         ascending, then -1 for rows with fewer than k entries.
 * out_values  device uint64 [n_rows][k] or NULL: the kept entries themselves,
 *         in the order of out (0 after), e.g. for a second round of merging.
 * Supported: 0 <= k <= LSA_MAX_BUDGET, cap >= 0, n_rows <= 65535.
 */
#define LSA_MERGE_ID_BITS 24

/* The keys (score + 1) of given candidates, for callers that choose them
 * (the ranks of a context-parallel index, each scoring its own token range):
 * lsa_score_tokens gives the fine score of token positions, lsa_score_blocks
 * the HI coarse score of blocks from their stored sums (the block sums must
 * cover the tokens the row sees; see lsa_index for rows that see fewer).
 *
 * q_idx, w, w_max, H_I, d_I   as for lsa_index, n_q query rows.
 * row_offset    device int64 [n_q]: cache row of position 0 of each query row's
 *               sequence (lsa_score_tokens); total_tokens bounds the cache.
 * blk_row_offset device int64 [n_q]: block-sum row of block 0 of each query
 *               row's sequence (lsa_score_blocks); block_rows bounds block_sums.
 * positions, blocks device int32 [n_q][n]: the candidates (-1: empty slot,
 *               key 0). A candidate outside the cache sets LSA_DEV_BAD_INDEX
 *               and reads as empty.
 * keys          device uint32 [n_q][n] (tokens) or uint64 [n_q][n] (blocks).
 */
lsa_status_t lsa_score_tokens(const int8_t *q_idx, const int8_t *k_idx_cache, const int32_t *w,
                              int32_t w_max, int32_t H_I, int32_t d_I, int32_t n_q,
                              const int64_t *row_offset, int64_t total_tokens,
                              const int32_t *positions, int32_t n, uint32_t *keys,
                              int32_t *dev_status, void *stream);
lsa_status_t lsa_score_blocks(const int8_t *q_idx, const int32_t *w, int32_t w_max, int32_t H_I,
                              int32_t d_I, int32_t n_q, const int8_t *block_sums,
                              int64_t block_rows, const int64_t *blk_row_offset,
                              const int32_t *blocks, int32_t n, uint64_t *keys,
                              int32_t *dev_status, void *stream);
lsa_status_t lsa_merge_pairs(const uint64_t *pairs, const int32_t *counts, int32_t n_rows,
                             int32_t cap, int32_t k, int32_t *out, uint64_t *out_values,
                             int32_t *dev_status, void *stream);

/* Context-parallel attention: each GPU attends over the entries of the set
 * that fall in its token range and returns its partial as the normalised
 * output plus the log of the softmax denominator; the exact attention over
 * the whole set is the log-sum-exp combination of the partials. This is the
 * softmax attention over the selected rows of "LongCat-2.0 (molayo1419.me)",
 * section "1M 토큰에서의 Sparse Attention 문제", split by rows of the cache
 * instead of by entries of the set; the arithmetic is lsa_attend's.
 *
 * lsa_attend_lse is lsa_attend that also writes, for every layer g, row r
 * and query head h,
 *   lse[g][r][h] = ln( sum_j exp(q . k_j / sqrt(d)) )
 * over the row's entries (-INFINITY for a row with no entry, or an invalid
 * row, whose output is zero as for lsa_attend).
 * lse   host [G] array of device fp32 [n_q][H_q].
 * Every other argument, the workspace and the device-side errors are
 * lsa_attend's.
 */
lsa_status_t lsa_attend_lse(const uint16_t *const *q, const uint16_t *const *k_cache,
                            const uint16_t *const *v_cache, int32_t H_q, int32_t H_kv, int32_t d,
                            const int32_t *index_sets, int32_t budget,
                            const lsa_batch_t *batch, int32_t layers_per_index,
                            float *const *out, float *const *lse, void *workspace,
                            size_t workspace_bytes, int32_t *dev_status, void *stream);

/* The part of each row's index set that one GPU holds: the entries e with
 * lo <= e < hi, as e - lo, in the set's order, then -1 up to the budget.
 *
 * index_sets  device int32 [n_q][budget] (positions relative to the sequence
 *             start, -1 padded, e.g. from lsa_index).
 * local_sets  device int32 [n_q][budget] output (may not alias index_sets).
 * lo, hi      host: the GPU's token range of the sequence, 0 <= lo <= hi.
 * An entry below -1 sets LSA_DEV_BAD_INDEX in dev_status and is dropped.
 * Supported: budget <= LSA_MAX_BUDGET, n_q <= 65535.
 */
lsa_status_t lsa_shard_sets(const int32_t *index_sets, int32_t n_q, int32_t budget, int32_t lo,
                            int32_t hi, int32_t *local_sets, int32_t *dev_status, void *stream);

/* The exact combination of n_parts attention partials of the same rows:
 *   M      = max_p lse[p][i]
 *   out[i] = sum_p exp(lse[p][i] - M) * o[p][i] / sum_p exp(lse[p][i] - M)
 *   lse_out[i] = M + ln(sum_p exp(lse[p][i] - M))
 * (zeros and -INFINITY when every part of row i is empty).
 *
 * o_parts    device fp32 [n_parts][rows][d]: each part's normalised output.
 * lse_parts  device fp32 [n_parts][rows]: each part's lse (-INFINITY: empty).
 * out        device fp32 [rows][d]; lse_out device fp32 [rows] or NULL.
 * Supported: d % 4 == 0, 1 <= n_parts <= 65535.
 */
lsa_status_t lsa_combine(const float *o_parts, const float *lse_parts, int32_t n_parts, int64_t rows,
                         int32_t d, float *out, float *lse_out, void *stream);

/* ----------------------------------------------------------------------- */
/* Allocation-free attention (no counterpart in the pages)                   */
/* ----------------------------------------------------------------------- */
/* Largest scratch lsa_attend_noalloc can use. Every GPU on which the library
 * is loaded holds one array of this size until the process exits. */
#define LSA_NOALLOC_SCRATCH_BYTES (8u << 20)

/* lsa_attend without a workspace argument, for callers that cannot call
 * cudaMalloc on this path: an engine whose device memory belongs entirely to
 * its own pool allocator, or a decode loop that must not run an allocation
 * (cudaMalloc and cudaFree can synchronise the device). The scratch that
 * lsa_attend takes as `workspace` lives instead in a static device array of
 * LSA_NOALLOC_SCRATCH_BYTES bytes inside the library; nothing is allocated.
 *
 * Arguments, output and device-side errors are those of lsa_attend. The
 * caller still owns and passes every input and output buffer.
 *  - A shape whose lsa_attend_workspace_size() exceeds
 *    LSA_NOALLOC_SCRATCH_BYTES returns LSA_ERR_UNSUPPORTED before any launch.
 *  - The first call on each device looks up the array's device address with
 *    that device current; make that first call before any stream capture.
 *    The address is kept per device ordinal for the life of the process: it
 *    belongs to the device's primary context (the one the CUDA runtime uses),
 *    so do not call this after cudaDeviceReset() or from a context of your
 *    own made current with the driver API.
 *  - All calls on a device share the one array, which keeps the previous
 *    call's contents; nothing in it needs to start at zero, because every
 *    call writes the scratch it later reads. Calls that overlap on the GPU
 *    (other streams, other host threads on the same device) race on the
 *    array: order them on one stream.
 */
lsa_status_t lsa_attend_noalloc(const uint16_t *const *q, const uint16_t *const *k_cache,
                                const uint16_t *const *v_cache, int32_t H_q, int32_t H_kv,
                                int32_t d, const int32_t *index_sets, int32_t budget,
                                const lsa_batch_t *batch, int32_t layers_per_index,
                                float *const *out, int32_t *dev_status, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* LSA_H_ */
