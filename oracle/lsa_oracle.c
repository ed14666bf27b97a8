/*
 * lsa_oracle.c — plain, slow, obviously-correct CPU oracle for the LongCat
 * Sparse Attention (LSA) decode/prefill hot path.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing in the product path may call, link or
 * load this file: only the tests, the smoke check and the benchmark's CPU
 * baseline leg use it. It shares no code, header, table or helper with the
 * CUDA library; it reads the same seeded input bytes and nothing else.
 *
 * What it computes (the pages give mechanisms, not formulas):
 *  - "LongCat-2.0 ... (molayo1419.me)", section "1M 토큰에서의 Sparse Attention
 *    문제": LSA extends DeepSeek Sparse Attention (an indexer that scores every
 *    cached token, then a top-k) with three orthogonal mechanisms: SI, CLI, HI.
 *  - "LongCat-Flash-Lite-Sparse (aitrends.kr)", section "기술적 특징": SI spends
 *    part of the selection budget on fixed sink tokens and a local sliding
 *    window; CLI reuses one index result across adjacent layers; HI first
 *    keeps coarse candidate blocks, then selects fine tokens inside them.
 *  The arithmetic this library fixes for those mechanisms:
 *    fine score   score_t = sum_h w_h * max(0, q_h . k_t)   (int8 q/k, exact)
 *    coarse score c_b     = sum_h w_h * max(0, q_h . S_b)   (S_b = sum of the
 *                           keys in block b, exact)
 *    ties go to the lower index; attention is softmax(q.k/sqrt(d)) v over the
 *    selected rows, GQA with contiguous head groups.
 *  Integer work is done in int64 (wider than any bound the library supports);
 *  attention in double from the exact bf16 values. Single-threaded per query;
 *  the batch drivers may spread independent queries over POSIX threads.
 *
 * Readings where the pages are silent (each is the plainest one the rest
 * supports):
 *  - one indexer key per token, shared by all indexer heads;
 *  - w is given per (query, head);
 *  - top-k competes only over the "middle" [s, ws), s = min(sink, L),
 *    ws = max(s, L - window); sink and window are always kept;
 *  - HI blocks are aligned at position 0, the last may be partial, a block's
 *    sum covers every present token of the block, a block is a candidate iff
 *    it meets the middle, and only its middle tokens become candidates;
 *  - the index set holds positions relative to the sequence start, ascending,
 *    padded with -1 to the budget sink + window + topk;
 *  - a query whose set is empty produces a zero output row.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ----------------------------------------------------------------------- */
/* Scores                                                                    */
/* ----------------------------------------------------------------------- */

/* Fine indexer score of one key for one query (DSA-style lightning indexer,
 * weighted ReLU over heads). q: [H_I][d_I], w: [H_I], k: [d_I]. */
int64_t oracle_fine_score(const int8_t *q, const int32_t *w, const int8_t *k,
                          int H_I, int d_I)
{
    int64_t total = 0;
    for (int h = 0; h < H_I; ++h) {
        int64_t dot = 0;
        for (int d = 0; d < d_I; ++d)
            dot += (int64_t)q[h * d_I + d] * (int64_t)k[d];
        if (dot > 0)
            total += (int64_t)w[h] * dot;
    }
    return total;
}

/* Per-block key sums for Hierarchical Indexing. k: [L][d_I] (one sequence),
 * S: [ceil(L/B)][d_I]. Block b covers tokens [b*B, min((b+1)*B, L)). */
void oracle_block_sums(const int8_t *k, int64_t L, int d_I, int B, int64_t *S)
{
    int64_t nblk = (L + B - 1) / B;
    memset(S, 0, (size_t)nblk * (size_t)d_I * sizeof(int64_t));
    for (int64_t t = 0; t < L; ++t) {
        int64_t b = t / B;
        for (int d = 0; d < d_I; ++d)
            S[b * d_I + d] += k[t * d_I + d];
    }
}

/* Coarse HI score of one block: the fine formula applied to the block sum. */
int64_t oracle_coarse_score(const int8_t *q, const int32_t *w, const int64_t *S_b,
                            int H_I, int d_I)
{
    int64_t total = 0;
    for (int h = 0; h < H_I; ++h) {
        int64_t dot = 0;
        for (int d = 0; d < d_I; ++d)
            dot += (int64_t)q[h * d_I + d] * S_b[d];
        if (dot > 0)
            total += (int64_t)w[h] * dot;
    }
    return total;
}

/* ----------------------------------------------------------------------- */
/* Selection                                                                 */
/* ----------------------------------------------------------------------- */

typedef struct {
    int64_t score;
    int64_t pos;
} scored_t;

/* Order: higher score first; among equal scores the lower position first. */
static int by_score_then_pos(const void *a, const void *b)
{
    const scored_t *x = (const scored_t *)a, *y = (const scored_t *)b;
    if (x->score != y->score)
        return x->score > y->score ? -1 : 1;
    return x->pos < y->pos ? -1 : (x->pos > y->pos ? 1 : 0);
}

static int by_value(const void *a, const void *b)
{
    int32_t x = *(const int32_t *)a, y = *(const int32_t *)b;
    return x < y ? -1 : (x > y ? 1 : 0);
}

/* Index set of one query. q: [H_I][d_I], w: [H_I], kseq: [L][d_I] are the
 * query's indexer inputs and its sequence's keys. out: [sink+window+topk].
 * hi_block == 0 switches HI off. Returns the number of valid entries, or -1
 * on a bad argument or an allocation failure. */
int oracle_index_query(const int8_t *q, const int32_t *w, const int8_t *kseq,
                       int64_t L, int H_I, int d_I, int sink, int window,
                       int topk, int hi_block, int hi_topblocks, int32_t *out)
{
    if (L < 1 || sink < 0 || window < 0 || topk < 0 || hi_block < 0 ||
        hi_topblocks < 0 || H_I < 1 || d_I < 1)
        return -1;
    int budget = sink + window + topk;
    int64_t s = sink < L ? sink : L;               /* sink run   [0, s)  */
    int64_t ws = L - window > s ? L - window : s;  /* window run [ws, L) */
    int64_t n_mid = ws - s;                        /* middle     [s, ws) */

    /* Candidate mask over the middle. */
    unsigned char *is_cand = (unsigned char *)calloc((size_t)(n_mid > 0 ? n_mid : 1), 1);
    if (!is_cand)
        return -1;
    if (hi_block == 0) {
        memset(is_cand, 1, (size_t)n_mid);
    } else if (n_mid > 0) {
        int64_t B = hi_block;
        int64_t nblk = (L + B - 1) / B;
        int64_t *S = (int64_t *)malloc((size_t)nblk * (size_t)d_I * sizeof(int64_t));
        scored_t *blocks = (scored_t *)malloc((size_t)nblk * sizeof(scored_t));
        if (!S || !blocks) {
            free(S);
            free(blocks);
            free(is_cand);
            return -1;
        }
        oracle_block_sums(kseq, L, d_I, hi_block, S);
        int64_t n_cb = 0;
        for (int64_t b = 0; b < nblk; ++b) {
            int64_t lo = b * B, hi = (b + 1) * B < L ? (b + 1) * B : L;
            if (lo < ws && hi > s) { /* block meets the middle */
                blocks[n_cb].score = oracle_coarse_score(q, w, S + b * d_I, H_I, d_I);
                blocks[n_cb].pos = b;
                ++n_cb;
            }
        }
        qsort(blocks, (size_t)n_cb, sizeof(scored_t), by_score_then_pos);
        int64_t keep = n_cb < hi_topblocks ? n_cb : hi_topblocks;
        for (int64_t i = 0; i < keep; ++i) {
            int64_t b = blocks[i].pos;
            int64_t lo = b * B, hi = (b + 1) * B < L ? (b + 1) * B : L;
            for (int64_t t = lo; t < hi; ++t)
                if (t >= s && t < ws)
                    is_cand[t - s] = 1;
        }
        free(S);
        free(blocks);
    }

    /* Fine scores of the candidates, then the top-k by (score desc, pos asc). */
    scored_t *cand = (scored_t *)malloc((size_t)(n_mid > 0 ? n_mid : 1) * sizeof(scored_t));
    if (!cand) {
        free(is_cand);
        return -1;
    }
    int64_t n_cand = 0;
    for (int64_t i = 0; i < n_mid; ++i) {
        if (!is_cand[i])
            continue;
        int64_t t = s + i;
        cand[n_cand].score = oracle_fine_score(q, w, kseq + t * d_I, H_I, d_I);
        cand[n_cand].pos = t;
        ++n_cand;
    }
    qsort(cand, (size_t)n_cand, sizeof(scored_t), by_score_then_pos);
    int64_t n_sel = n_cand < topk ? n_cand : topk;

    /* Streaming-aware assembly: sink run, selected middle, window run. */
    int n = 0;
    for (int64_t t = 0; t < s; ++t)
        out[n++] = (int32_t)t;
    for (int64_t i = 0; i < n_sel; ++i)
        out[n++] = (int32_t)cand[i].pos;
    for (int64_t t = ws; t < L; ++t)
        out[n++] = (int32_t)t;
    qsort(out, (size_t)n, sizeof(int32_t), by_value);
    for (int i = n; i < budget; ++i)
        out[i] = -1;
    free(cand);
    free(is_cand);
    return n;
}

/* ----------------------------------------------------------------------- */
/* Attention                                                                 */
/* ----------------------------------------------------------------------- */

/* bf16 bit pattern -> double (exact: a bf16 is the top half of an fp32). */
static double bf16_to_double(uint16_t bits)
{
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* Sparse softmax attention of one query over its index set.
 * q: [H_q][d] bf16 bits; kseq/vseq: [L][H_kv][d] bf16 bits (the sequence's
 * rows); set: [budget] positions or -1; out: [H_q][d]. Query head h reads kv
 * head floor(h*H_kv/H_q). Scale 1/sqrt(d). */
void oracle_attend_query(const uint16_t *q, const uint16_t *kseq,
                         const uint16_t *vseq, const int32_t *set, int budget,
                         int H_q, int H_kv, int d, double *out)
{
    double scale = 1.0 / sqrt((double)d);
    double *z = (double *)malloc((size_t)(budget > 0 ? budget : 1) * sizeof(double));
    for (int h = 0; h < H_q; ++h) {
        int kvh = (int)(((int64_t)h * H_kv) / H_q);
        double zmax = -INFINITY;
        int any = 0;
        for (int j = 0; j < budget; ++j) {
            if (set[j] < 0)
                continue;
            const uint16_t *krow = kseq + ((int64_t)set[j] * H_kv + kvh) * d;
            double dot = 0.0;
            for (int e = 0; e < d; ++e)
                dot += bf16_to_double(q[h * d + e]) * bf16_to_double(krow[e]);
            z[j] = dot * scale;
            if (z[j] > zmax)
                zmax = z[j];
            any = 1;
        }
        for (int e = 0; e < d; ++e)
            out[h * d + e] = 0.0;
        if (!any)
            continue;
        double denom = 0.0;
        for (int j = 0; j < budget; ++j) {
            if (set[j] < 0)
                continue;
            double p = exp(z[j] - zmax);
            denom += p;
            const uint16_t *vrow = vseq + ((int64_t)set[j] * H_kv + kvh) * d;
            for (int e = 0; e < d; ++e)
                out[h * d + e] += p * bf16_to_double(vrow[e]);
        }
        for (int e = 0; e < d; ++e)
            out[h * d + e] /= denom;
    }
    free(z);
}

/* ----------------------------------------------------------------------- */
/* Attention over an FP8 KV cache                                            */
/* ----------------------------------------------------------------------- */
/* The pages name FP8 variants of the models and a KV-cache data type, but
 * not the FP8 format or its scaling. Reading used here: OCP FP8 E4M3 codes
 * (1 sign bit, 4 exponent bits with bias 7, 3 mantissa bits; exponent field
 * 0 holds the subnormals m/8 * 2^-6; no infinities; S.1111.111 is NaN) with
 * one scale per layer for K and one for V: value = scale * E4M3(code). */

/* E4M3 code -> double, from the format's definition. */
double oracle_e4m3_value(uint8_t code)
{
    int sign = code >> 7, E = (code >> 3) & 0xF, m = code & 7;
    double v;
    if (E == 15 && m == 7)
        return NAN;
    if (E == 0)
        v = ldexp((double)m / 8.0, -6);
    else
        v = ldexp(1.0 + (double)m / 8.0, E - 7);
    return sign ? -v : v;
}

/* oracle_attend_query with K and V given as E4M3 codes: k = k_scale *
 * E4M3(k code), v = v_scale * E4M3(v code); everything else (GQA mapping,
 * scale 1/sqrt(d), skipped -1 entries, empty set -> zeros) as there. */
void oracle_attend_query_fp8(const uint16_t *q, const uint8_t *kseq,
                             const uint8_t *vseq, double k_scale, double v_scale,
                             const int32_t *set, int budget, int H_q, int H_kv,
                             int d, double *out)
{
    const double inv_sqrt_d = 1.0 / sqrt((double)d);
    double *z = (double *)malloc((size_t)(budget > 0 ? budget : 1) * sizeof(double));
    for (int h = 0; h < H_q; ++h) {
        const int kv_head = (int)(((int64_t)h * H_kv) / H_q);
        double zmax = -INFINITY;
        int any = 0;
        for (int j = 0; j < budget; ++j) {
            if (set[j] < 0)
                continue;
            const uint8_t *krow = kseq + ((int64_t)set[j] * H_kv + kv_head) * d;
            double dot = 0.0;
            for (int e = 0; e < d; ++e)
                dot += bf16_to_double(q[h * d + e]) * (k_scale * oracle_e4m3_value(krow[e]));
            z[j] = dot * inv_sqrt_d;
            if (z[j] > zmax)
                zmax = z[j];
            any = 1;
        }
        for (int e = 0; e < d; ++e)
            out[h * d + e] = 0.0;
        if (!any)
            continue;
        double denom = 0.0;
        for (int j = 0; j < budget; ++j) {
            if (set[j] < 0)
                continue;
            double p = exp(z[j] - zmax);
            denom += p;
            const uint8_t *vrow = vseq + ((int64_t)set[j] * H_kv + kv_head) * d;
            for (int e = 0; e < d; ++e)
                out[h * d + e] += p * (v_scale * oracle_e4m3_value(vrow[e]));
        }
        for (int e = 0; e < d; ++e)
            out[h * d + e] = out[h * d + e] / denom;
    }
    free(z);
}

/* ----------------------------------------------------------------------- */
/* Batch drivers (independent queries; optionally spread over threads)       */
/* ----------------------------------------------------------------------- */

typedef struct {
    /* index */
    const int8_t *q_idx;       /* [n_q][H_I][d_I] */
    const int8_t *k_idx;       /* [T][d_I] packed sequences */
    const int32_t *w;          /* [n_q][H_I] */
    const int64_t *kv_offset;  /* [n_seq] first token of each sequence */
    const int32_t *q_seq;      /* [n_q] sequence of each query */
    const int32_t *q_len;      /* [n_q] visible length of each query */
    int H_I, d_I, sink, window, topk, hi_block, hi_topblocks;
    int32_t *sets;             /* [n_q][budget] */
    /* attend */
    const uint16_t *const *q;  /* [G] -> [n_q][H_q][d] */
    const uint16_t *const *k;  /* [G] -> [T][H_kv][d] */
    const uint16_t *const *v;  /* [G] -> [T][H_kv][d] */
    int H_q, H_kv, d, G, budget;
    double *const *out;        /* [G] -> [n_q][H_q][d] */
    /* work split */
    int64_t n_q;
    int n_threads;
    int tid;
    int status;
} batch_job_t;

static void *index_worker(void *arg)
{
    batch_job_t *j = (batch_job_t *)arg;
    int budget = j->sink + j->window + j->topk;
    for (int64_t r = j->tid; r < j->n_q; r += j->n_threads) {
        const int8_t *kseq = j->k_idx + j->kv_offset[j->q_seq[r]] * j->d_I;
        int n = oracle_index_query(j->q_idx + r * j->H_I * j->d_I, j->w + r * j->H_I,
                                   kseq, j->q_len[r], j->H_I, j->d_I, j->sink,
                                   j->window, j->topk, j->hi_block, j->hi_topblocks,
                                   j->sets + r * budget);
        if (n < 0)
            j->status = -1;
    }
    return NULL;
}

static void *attend_worker(void *arg)
{
    batch_job_t *j = (batch_job_t *)arg;
    int64_t row = (int64_t)j->H_kv * j->d;
    for (int64_t r = j->tid; r < j->n_q; r += j->n_threads) {
        int64_t base = j->kv_offset[j->q_seq[r]];
        for (int g = 0; g < j->G; ++g)
            oracle_attend_query(j->q[g] + r * j->H_q * j->d, j->k[g] + base * row,
                                j->v[g] + base * row, j->sets + r * j->budget,
                                j->budget, j->H_q, j->H_kv, j->d,
                                j->out[g] + r * j->H_q * j->d);
    }
    return NULL;
}

static int run_threads(batch_job_t *proto, void *(*fn)(void *))
{
    int nt = proto->n_threads < 1 ? 1 : proto->n_threads;
    if (nt > 256)
        nt = 256;
    batch_job_t jobs[256];
    pthread_t th[256];
    int status = 0;
    for (int i = 0; i < nt; ++i) {
        jobs[i] = *proto;
        jobs[i].n_threads = nt;
        jobs[i].tid = i;
        jobs[i].status = 0;
    }
    if (nt == 1) {
        fn(&jobs[0]);
        return jobs[0].status;
    }
    for (int i = 0; i < nt; ++i)
        pthread_create(&th[i], NULL, fn, &jobs[i]);
    for (int i = 0; i < nt; ++i) {
        pthread_join(th[i], NULL);
        if (jobs[i].status)
            status = jobs[i].status;
    }
    return status;
}

/* Index sets of n_q queries (CLI: one set per group of layers). */
int oracle_lsa_index(const int8_t *q_idx, const int8_t *k_idx, const int32_t *w,
                     const int64_t *kv_offset, const int32_t *q_seq,
                     const int32_t *q_len, int64_t n_q, int H_I, int d_I,
                     int sink, int window, int topk, int hi_block,
                     int hi_topblocks, int32_t *sets, int n_threads)
{
    batch_job_t j;
    memset(&j, 0, sizeof j);
    j.q_idx = q_idx;
    j.k_idx = k_idx;
    j.w = w;
    j.kv_offset = kv_offset;
    j.q_seq = q_seq;
    j.q_len = q_len;
    j.n_q = n_q;
    j.H_I = H_I;
    j.d_I = d_I;
    j.sink = sink;
    j.window = window;
    j.topk = topk;
    j.hi_block = hi_block;
    j.hi_topblocks = hi_topblocks;
    j.sets = sets;
    j.n_threads = n_threads;
    return run_threads(&j, index_worker);
}

/* Attention of n_q queries for G layers that share one index set per query. */
int oracle_lsa_attend(const uint16_t *const *q, const uint16_t *const *k,
                      const uint16_t *const *v, const int32_t *sets, int budget,
                      const int64_t *kv_offset, const int32_t *q_seq, int64_t n_q,
                      int H_q, int H_kv, int d, int G, double *const *out,
                      int n_threads)
{
    batch_job_t j;
    memset(&j, 0, sizeof j);
    j.q = q;
    j.k = k;
    j.v = v;
    j.sets = (int32_t *)sets;
    j.budget = budget;
    j.kv_offset = kv_offset;
    j.q_seq = q_seq;
    j.n_q = n_q;
    j.H_q = H_q;
    j.H_kv = H_kv;
    j.d = d;
    j.G = G;
    j.out = out;
    j.n_threads = n_threads;
    return run_threads(&j, attend_worker);
}
