/*
 * dsa_oracle.c -- the ORACLE for query-driven dynamic block-sparse attention.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the plain, slow CPU statement of
 * what the library computes.  Only the test suite, the smoke check and the
 * CPU-baseline leg of the benchmark may load it.  It shares no code, header,
 * table or helper with the CUDA library, and the CUDA library never calls it.
 *
 * Everything is straight nested loops over the definition.  Integers are
 * accumulated in int64, floating point in double.  Nothing is blocked, fused
 * or reordered beyond what the definition itself states.
 *
 * Sources (web pages, cited by title and section):
 *  [P1] "Day-0 Adaptation for Massive LLMs: Overcoming Sparse Attention and
 *       MXFP4 Expert Weights", section 4 "Challenge 1: Full Implementation of
 *       Dynamic Sparse Attention", parts (1) Index Selection, (2) KV Cache
 *       Layout, (3) Prefill and Decode.
 *  [P3] "Day-0 Adaptation for Trillion-Parameter Models: Engineering Practices
 *       and Technical Breakdown", section 4 "Sparse Attention Adaptation"
 *       (4.1 Index Selection, 4.2 KV Cache Layout).
 *  [P5] "Day-0 Readiness for Trillion-Parameter Models: Engineering Sparse
 *       Attention and Expert Weight Compression", sections "Index Selection
 *       Path" and "KV Cache Layout".
 *
 * Readings adopted where the pages are silent (each one is also listed with
 * its reason in the design notes of the repository):
 *  - Block score: S[t,b] = sum_h w[t,h] * max(0, sum_d q_idx[t,h,d]*kc[page(b),d]),
 *    one coarse key per KV block shared by all indexer heads, one weight per
 *    query and indexer head.  The pages only say "score the compressed
 *    representation against the query" [P1 4(1)], [P5 "Index Selection Path"].
 *  - Visible blocks of a query at position p: b = 0 .. floor(p/B).
 *  - Selection: the query's own block floor(p/B) is always taken; the other
 *    K-1 slots go to the other visible blocks ordered by (score descending,
 *    block index ascending).  When at most K blocks are visible all are taken.
 *    The output lists logical block ids ascending, padded with -1; the gather
 *    maps them through the block table [P5 "Index Selection Path": index
 *    semantics aligned with the downstream gather].
 *  - Attention: exact softmax attention over the tokens of the selected
 *    blocks with position <= p [P3 4: exact attention on the selected part;
 *    P1 4(3): the valid mask], logit scale given by the caller (1/sqrt(D)),
 *    query head h reads KV head floor(h / (Hq/Hkv)).
 *  - KV layout: pool[page][token_in_block][kv_head][dim] [P5 "KV Cache Layout"].
 */
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <math.h>

/* status codes of the oracle (not shared with the library) */
#define ORC_OK 0
#define ORC_BAD_ARG 1
#define ORC_BAD_PAGE 2
#define ORC_BAD_POS 3

/* bf16 is the top half of an IEEE binary32; decoding it is exact. */
static double bf16_bits_to_double(uint16_t bits)
{
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/*
 * Where new token i of sequence s lands [P5 "KV Cache Layout": prefill writes
 * blocks in batch, decode appends one token and keeps the block table].
 * Sequence s owns new tokens i in [cu_new[s], cu_new[s+1]); seq_lens[s] is
 * the length AFTER the append, so token i sits at position
 * seq_lens[s] - n_s + (i - cu_new[s]).
 */
static int new_token_position(const int32_t *seq_lens, const int32_t *cu_new, int s, int i)
{
    int n = cu_new[s + 1] - cu_new[s];
    return seq_lens[s] - n + (i - cu_new[s]);
}

/*
 * Append the new tokens' K and V rows to the fine-grained KV pool
 * [P1 4(2): the KV blocks used by attention; P5 "KV Cache Layout"].
 */
int oracle_kv_append(int num_seqs, const int32_t *block_table, int max_blocks,
                     const int32_t *seq_lens, const int32_t *cu_new,
                     int block_size, int num_kv_heads, int head_dim, int num_pages,
                     const uint16_t *k_new, const uint16_t *v_new,
                     uint16_t *k_pool, uint16_t *v_pool)
{
    const long row = (long)num_kv_heads * head_dim; /* elements per token */
    for (int s = 0; s < num_seqs; ++s) {
        int n = cu_new[s + 1] - cu_new[s];
        if (n < 0 || n > seq_lens[s]) return ORC_BAD_ARG;
        for (int i = cu_new[s]; i < cu_new[s + 1]; ++i) {
            int pos = new_token_position(seq_lens, cu_new, s, i);
            int blk = pos / block_size, slot = pos % block_size;
            if (blk >= max_blocks) return ORC_BAD_POS;
            int page = block_table[(long)s * max_blocks + blk];
            if (page < 0 || page >= num_pages) return ORC_BAD_PAGE;
            long dst = ((long)page * block_size + slot) * row;
            for (long e = 0; e < row; ++e) {
                k_pool[dst + e] = k_new[(long)i * row + e];
                v_pool[dst + e] = v_new[(long)i * row + e];
            }
        }
    }
    return ORC_OK;
}

/*
 * Update the coarse keys of the blocks the new tokens land in
 * [P1 4(2): the compressed index blocks used for selection].  Row i of
 * kc_new is the coarse key of the block that token i lands in, as it stands
 * after token i; a block keeps the row of the last new token in it.
 */
int oracle_kc_append(int num_seqs, const int32_t *block_table, int max_blocks,
                     const int32_t *seq_lens, const int32_t *cu_new,
                     int block_size, int idx_dim, int num_pages,
                     const int8_t *kc_new, int8_t *kc_pool)
{
    for (int s = 0; s < num_seqs; ++s) {
        int n = cu_new[s + 1] - cu_new[s];
        if (n < 0 || n > seq_lens[s]) return ORC_BAD_ARG;
        for (int i = cu_new[s]; i < cu_new[s + 1]; ++i) {
            int pos = new_token_position(seq_lens, cu_new, s, i);
            int blk = pos / block_size, slot = pos % block_size;
            if (blk >= max_blocks) return ORC_BAD_POS;
            int page = block_table[(long)s * max_blocks + blk];
            if (page < 0 || page >= num_pages) return ORC_BAD_PAGE;
            int last_in_block = (i == cu_new[s + 1] - 1) || (slot == block_size - 1);
            if (last_in_block)
                for (int d = 0; d < idx_dim; ++d)
                    kc_pool[(long)page * idx_dim + d] = kc_new[(long)i * idx_dim + d];
        }
    }
    return ORC_OK;
}

/*
 * Block scores of every query against every visible block
 * [P1 4(1) "Index Selection"; P3 4.1; P5 "Index Selection Path"].
 * Query t belongs to sequence q_seq[t] and sits at position q_pos[t].
 * scores[t][b] (int64, row stride max_blocks) is written for the visible
 * blocks b <= q_pos[t] / block_size and set to INT64_MIN elsewhere.
 */
int oracle_index_score(int total_q, const int32_t *q_seq, const int32_t *q_pos,
                       const int32_t *block_table, int max_blocks, int block_size,
                       int num_pages, const int8_t *kc_pool, int idx_dim,
                       const int8_t *q_idx, const int32_t *w, int num_idx_heads,
                       int64_t *scores)
{
    for (int t = 0; t < total_q; ++t) {
        int s = q_seq[t], p = q_pos[t];
        if (p < 0) return ORC_BAD_POS;
        int n_vis = p / block_size + 1;
        if (n_vis > max_blocks) return ORC_BAD_POS;
        for (int b = 0; b < max_blocks; ++b) scores[(long)t * max_blocks + b] = INT64_MIN;
        for (int b = 0; b < n_vis; ++b) {
            int page = block_table[(long)s * max_blocks + b];
            if (page < 0 || page >= num_pages) return ORC_BAD_PAGE;
            const int8_t *kc = kc_pool + (long)page * idx_dim;
            int64_t total = 0;
            for (int h = 0; h < num_idx_heads; ++h) {
                const int8_t *q = q_idx + ((long)t * num_idx_heads + h) * idx_dim;
                int64_t dot = 0;
                for (int d = 0; d < idx_dim; ++d) dot += (int64_t)q[d] * (int64_t)kc[d];
                int64_t relu = dot > 0 ? dot : 0;
                total += (int64_t)w[(long)t * num_idx_heads + h] * relu;
            }
            scores[(long)t * max_blocks + b] = total;
        }
    }
    return ORC_OK;
}

/*
 * The value of an FP8 E4M3 code times 2^9 ("low-precision inputs" of the
 * indexer [P5 "Index Selection Path"]; the format is the OCP 8-bit floating
 * point E4M3: one sign bit, four exponent bits with bias 7, three mantissa
 * bits, exponent field 0 for subnormals, codes 0x7F and 0xFF for NaN, no
 * infinities).  A subnormal is (f/8) * 2^-6 = f * 2^-9 and a normal is
 * (1 + f/8) * 2^(e-7) = (8 + f) * 2^(e-10), so every finite value times 2^9 is
 * an integer of magnitude at most 448 * 2^9.  *is_nan is set for a NaN code.
 */
int64_t oracle_e4m3_times_512(uint8_t code, int *is_nan)
{
    int sign = code >> 7, e = (code >> 3) & 15, f = code & 7;
    *is_nan = (e == 15 && f == 7);
    if (*is_nan) return 0;
    int64_t mag = (e == 0) ? (int64_t)f : ((int64_t)(8 + f) << (e - 1));
    return sign ? -mag : mag;
}

/*
 * Block scores of the FP8 indexer: the same formula as oracle_index_score
 * with q_idx and the coarse keys as E4M3 codes, computed EXACTLY and returned
 * times 2^18: S[t,b] * 2^18 = sum_h w[t,h] * max(0, sum_d (2^9 q[d]) (2^9 kc[d])).
 * Each factor is an integer (oracle_e4m3_times_512), so the sum is exact in
 * 128-bit integers; ORC_BAD_ARG if a code is NaN or a score does not fit int64.
 */
int oracle_index_score_fp8(int total_q, const int32_t *q_seq, const int32_t *q_pos,
                           const int32_t *block_table, int max_blocks, int block_size,
                           int num_pages, const uint8_t *kc_pool, int idx_dim,
                           const uint8_t *q_idx, const int32_t *w, int num_idx_heads,
                           int64_t *scores)
{
    for (int t = 0; t < total_q; ++t) {
        int s = q_seq[t], p = q_pos[t];
        if (p < 0) return ORC_BAD_POS;
        int n_vis = p / block_size + 1;
        if (n_vis > max_blocks) return ORC_BAD_POS;
        for (int b = 0; b < max_blocks; ++b) scores[(long)t * max_blocks + b] = INT64_MIN;
        for (int b = 0; b < n_vis; ++b) {
            int page = block_table[(long)s * max_blocks + b];
            if (page < 0 || page >= num_pages) return ORC_BAD_PAGE;
            const uint8_t *kc = kc_pool + (long)page * idx_dim;
            __int128 total = 0;
            for (int h = 0; h < num_idx_heads; ++h) {
                const uint8_t *q = q_idx + ((long)t * num_idx_heads + h) * idx_dim;
                __int128 dot = 0;
                for (int d = 0; d < idx_dim; ++d) {
                    int nan_q, nan_k;
                    int64_t qv = oracle_e4m3_times_512(q[d], &nan_q);
                    int64_t kv = oracle_e4m3_times_512(kc[d], &nan_k);
                    if (nan_q || nan_k) return ORC_BAD_ARG;
                    dot += (__int128)qv * kv;
                }
                __int128 relu = dot > 0 ? dot : 0;
                total += (__int128)w[(long)t * num_idx_heads + h] * relu;
            }
            if (total > (__int128)INT64_MAX || total <= (__int128)INT64_MIN) return ORC_BAD_ARG;
            scores[(long)t * max_blocks + b] = (int64_t)total;
        }
    }
    return ORC_OK;
}

/* candidate of the Top-K step: higher score first, then lower block id */
typedef struct { int64_t score; int32_t block; } orc_cand;

static int cand_rank_order(const void *a, const void *b)
{
    const orc_cand *x = (const orc_cand *)a, *y = (const orc_cand *)b;
    if (x->score != y->score) return x->score > y->score ? -1 : 1;
    return (x->block > y->block) - (x->block < y->block);
}

static int int_ascending(const void *a, const void *b)
{
    int32_t x = *(const int32_t *)a, y = *(const int32_t *)b;
    return (x > y) - (x < y);
}

/*
 * Top-K block selection [P1 4(1) "Scalable Top-K"; P5 "Index Selection Path"].
 * k = k_per_seq[q_seq[t]] (1 <= k <= k_max).  Writes sel[t][0..k_max) =
 * chosen logical block ids ascending, then -1; cnt[t] = number chosen.
 * A full sort of the candidates is the definition; no partial selection.
 */
int oracle_topk(int total_q, const int32_t *q_seq, const int32_t *q_pos,
                int block_size, const int64_t *scores, int max_blocks,
                const int32_t *k_per_seq, int k_max, int32_t *sel, int32_t *cnt)
{
    orc_cand *cand = (orc_cand *)malloc(sizeof(orc_cand) * (size_t)(max_blocks > 0 ? max_blocks : 1));
    if (!cand) return ORC_BAD_ARG;
    for (int t = 0; t < total_q; ++t) {
        int k = k_per_seq[q_seq[t]];
        if (k < 1 || k > k_max) { free(cand); return ORC_BAD_ARG; }
        int n_vis = q_pos[t] / block_size + 1;
        int32_t *out = sel + (long)t * k_max;
        int n = 0;
        if (n_vis <= k) {
            for (int b = 0; b < n_vis; ++b) out[n++] = b;
        } else {
            int own = n_vis - 1;
            for (int b = 0; b < own; ++b) {
                cand[b].score = scores[(long)t * max_blocks + b];
                cand[b].block = b;
            }
            qsort(cand, (size_t)own, sizeof(orc_cand), cand_rank_order);
            for (int i = 0; i < k - 1; ++i) out[n++] = cand[i].block;
            out[n++] = own;
            qsort(out, (size_t)n, sizeof(int32_t), int_ascending);
        }
        cnt[t] = n;
        for (int i = n; i < k_max; ++i) out[i] = -1;
    }
    free(cand);
    return ORC_OK;
}

/*
 * Exact attention over the selected blocks only [P1 4(3) decode schematic:
 * select, gather by block, attend under a valid mask; P3 4: exact attention
 * on the selected portion; P5 "KV Cache Layout" for the pool layout].
 * out[t][h][:] and lse[t][h] (natural log of the softmax denominator, with
 * the logits already scaled) are produced in double.
 */
int oracle_sparse_attention(int total_q, const int32_t *q_seq, const int32_t *q_pos,
                            const int32_t *block_table, int max_blocks, int block_size,
                            int num_pages, int num_q_heads, int num_kv_heads, int head_dim,
                            const uint16_t *q, const uint16_t *k_pool, const uint16_t *v_pool,
                            const int32_t *sel, const int32_t *cnt, int k_max,
                            double sm_scale, double *out, double *lse)
{
    if (num_kv_heads <= 0 || num_q_heads % num_kv_heads != 0) return ORC_BAD_ARG;
    int group = num_q_heads / num_kv_heads;
    long n_tok_max = (long)k_max * block_size;
    double *logit = (double *)malloc(sizeof(double) * (size_t)(n_tok_max > 0 ? n_tok_max : 1));
    long *tok_row = (long *)malloc(sizeof(long) * (size_t)(n_tok_max > 0 ? n_tok_max : 1));
    if (!logit || !tok_row) { free(logit); free(tok_row); return ORC_BAD_ARG; }
    int rc = ORC_OK;
    for (int t = 0; t < total_q && rc == ORC_OK; ++t) {
        int s = q_seq[t], p = q_pos[t];
        /* the token rows (page*block_size + slot) that the query may see */
        long n_tok = 0;
        for (int i = 0; i < cnt[t]; ++i) {
            int b = sel[(long)t * k_max + i];
            if (b < 0 || b >= max_blocks) { rc = ORC_BAD_ARG; break; }
            int page = block_table[(long)s * max_blocks + b];
            if (page < 0 || page >= num_pages) { rc = ORC_BAD_PAGE; break; }
            for (int slot = 0; slot < block_size; ++slot) {
                int pos = b * block_size + slot;
                if (pos <= p) tok_row[n_tok++] = (long)page * block_size + slot;
            }
        }
        if (rc != ORC_OK) break;
        for (int h = 0; h < num_q_heads; ++h) {
            int kvh = h / group;
            const uint16_t *qh = q + ((long)t * num_q_heads + h) * head_dim;
            double *o = out + ((long)t * num_q_heads + h) * head_dim;
            double m = -INFINITY;
            for (long j = 0; j < n_tok; ++j) {
                const uint16_t *kj = k_pool + (tok_row[j] * num_kv_heads + kvh) * head_dim;
                double dot = 0.0;
                for (int d = 0; d < head_dim; ++d)
                    dot += bf16_bits_to_double(qh[d]) * bf16_bits_to_double(kj[d]);
                logit[j] = dot * sm_scale;
                if (logit[j] > m) m = logit[j];
            }
            double denom = 0.0;
            for (long j = 0; j < n_tok; ++j) denom += exp(logit[j] - m);
            for (int d = 0; d < head_dim; ++d) o[d] = 0.0;
            for (long j = 0; j < n_tok; ++j) {
                double pj = exp(logit[j] - m) / denom;
                const uint16_t *vj = v_pool + (tok_row[j] * num_kv_heads + kvh) * head_dim;
                for (int d = 0; d < head_dim; ++d) o[d] += pj * bf16_bits_to_double(vj[d]);
            }
            lse[(long)t * num_q_heads + h] = n_tok > 0 ? m + log(denom) : -INFINITY;
        }
    }
    free(logit);
    free(tok_row);
    return rc;
}
