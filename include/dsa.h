/*
 * dsa.h -- C ABI of the B200 (sm_100a) library for query-driven dynamic
 * block-sparse attention over a block-paged KV cache.
 *
 * The pipeline follows the pages' statement of the problem:
 *   append new tokens -> score every visible KV block with a low-precision
 *   indexer -> keep the Top-K blocks (own block forced) -> exact attention over
 *   the selected blocks only, with separate decode and prefill paths.
 * Pages (cited by title and section):
 *   [P1] "Day-0 Adaptation for Massive LLMs: Overcoming Sparse Attention and
 *        MXFP4 Expert Weights", section 4 (1) Index Selection, (2) KV Cache
 *        Layout, (3) Prefill and Decode (decode schematic: select, gather by
 *        block, attend under a valid mask).
 *   [P3] "Day-0 Adaptation for Trillion-Parameter Models: Engineering
 *        Practices and Technical Breakdown", section 4 (4.1 index selection,
 *        4.2 KV cache layout, 4.3 dual prefill / decode paths).
 *   [P5] "Day-0 Readiness for Trillion-Parameter Models: Engineering Sparse
 *        Attention and Expert Weight Compression", sections "Index Selection
 *        Path", "KV Cache Layout", "Differentiated Adaptation of Prefill and
 *        Decode".
 *
 * Conventions shared by every entry point
 *  - Every array pointer is DEVICE memory owned by the caller, 16-byte
 *    aligned.  The library never allocates or frees device memory.
 *  - Calls are asynchronous on `stream` (a cudaStream_t; NULL = the legacy
 *    default stream).  Host-side validation is synchronous: a non-zero
 *    status means nothing was launched.
 *  - Kernels never trap.  A fault they detect in device-resident metadata
 *    (a page id outside the pool, a position outside its sequence, a
 *    selection outside the visible range) ORs a DSA_DEV_ERR_* bit into
 *    *dev_err (an int32 in device memory, may be NULL to ignore) and the
 *    offending item is skipped; the caller reads the word back when it likes.
 *  - Sizes in v1: block_size 64, 128, 256 or 512 tokens (one KV block is one
 *    page of the pools; dsa_decode_fused keeps 64), head_dim 128, idx_dim 64;
 *    query heads per KV head 1..16; indexer heads 1..16.  Anything else is
 *    DSA_ERR_UNSUPPORTED.
 *  - Consecutive calls on one stream overlap: each kernel lets the next one
 *    start early (programmatic dependent launch) and waits for its
 *    predecessor before it reads anything a library call writes (the pools,
 *    scores, selections).  Before that wait a kernel may already read the
 *    batch description and its own inputs (block_table, seq_lens, cu_q, q_pos,
 *    k_per_seq, q_idx, w, q): these must not be outputs of the library call
 *    issued just before it on the same stream.  Work from other kernels is
 *    waited for in full, as usual.
 *  - Calls on different streams may run at the same time (independent
 *    batches in flight, one stream each) as long as no call writes what
 *    another reads or writes: each needs its own outputs and workspaces.  The
 *    library keeps no device state between calls apart from the fixed
 *    scratch of dsa_sparse_attn_decode_noalloc.
 *
 * KV cache layout [P5 "KV Cache Layout"; P1 4(2) two storage types]:
 *   k_pool, v_pool : bf16  [num_pages][block_size][num_kv_heads][head_dim]
 *   kc_pool        : int8  [num_pages][idx_dim]  one coarse key per block
 *   block_table    : int32 [num_seqs][max_blocks] logical block -> page
 *
 * Queries are ragged: sequence s owns queries cu_q[s] .. cu_q[s+1]-1, query t
 * sits at position q_pos[t] (< seq_lens[s]).  A query sees the logical
 * blocks 0 .. q_pos[t]/block_size ("visible blocks"); the last of them is its
 * own block.
 */
#ifndef DSA_H
#define DSA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* cudaStream_t without pulling in the CUDA headers */
typedef struct CUstream_st *dsa_stream_t;

/* host-side status codes */
enum {
    DSA_OK = 0,
    DSA_ERR_INVALID_ARG = 1, /* NULL / misaligned pointer, negative or inconsistent size */
    DSA_ERR_UNSUPPORTED = 2, /* a size this version does not implement (see above) */
    DSA_ERR_RANGE = 3,       /* int32 scores could overflow for the stated |w| bound */
    DSA_ERR_WORKSPACE = 4,   /* workspace NULL or smaller than the size query says */
    DSA_ERR_CUDA = 5         /* a CUDA runtime call failed (launch or attribute) */
};

/* device-side error bits ORed into *dev_err */
#define DSA_DEV_ERR_PAGE 1u  /* block_table entry outside [0, num_pages) */
#define DSA_DEV_ERR_POS 2u   /* position / new-token count outside the sequence or table */
#define DSA_DEV_ERR_SEL 4u   /* selected block id outside the query's visible blocks */
#define DSA_DEV_ERR_K 8u     /* k_per_seq[s] outside [1, k_max] */
#define DSA_DEV_ERR_WAIT 16u /* a bounded in-kernel wait gave up (work of that unit skipped) */
#define DSA_DEV_ERR_VALUE 32u /* an FP8 input code is NaN (read as 0) */

typedef struct {
    void *k_pool;          /* bf16 [num_pages][block_size][num_kv_heads][head_dim] */
    void *v_pool;          /* bf16, same shape */
    int8_t *kc_pool;       /* int8 [num_pages][idx_dim] */
    int32_t num_pages;
    int32_t block_size;    /* tokens per block (= page): 64, 128, 256 or 512 */
    int32_t num_kv_heads;
    int32_t head_dim;      /* 128 */
    int32_t idx_dim;       /* 64 */
} dsa_kv_cache;

typedef struct {
    const int32_t *block_table; /* [num_seqs][max_blocks]; entries past a sequence's end are never read */
    int32_t max_blocks;
    const int32_t *seq_lens;    /* [num_seqs] context length INCLUDING any tokens appended this step */
    int32_t num_seqs;
} dsa_seqs;

typedef struct {
    const int32_t *cu_q;   /* [num_seqs + 1] ragged offsets of each sequence's queries */
    const int32_t *q_pos;  /* [total_q] absolute position of each query token */
    int32_t total_q;
} dsa_queries;

/*
 * dsa_kv_append -- write new tokens into the paged cache [P5 "KV Cache
 * Layout": prefill writes blocks in batch, decode appends incrementally and
 * keeps the block table; both share one block-index semantics].
 *   cu_new  [num_seqs+1]: sequence s appends tokens cu_new[s] .. cu_new[s+1]-1,
 *           landing at positions seq_lens[s]-n_s .. seq_lens[s]-1.
 *   k_new, v_new: bf16 [total_new][num_kv_heads][head_dim].
 *   kc_new: int8 [total_new][idx_dim] or NULL.  Row i is the coarse key of the
 *           block token i lands in, as that block stands after token i; each
 *           touched block keeps the row of its last new token.  NULL leaves
 *           kc_pool untouched.
 * Device errors: DSA_DEV_ERR_POS (n_s > seq_lens[s] or block >= max_blocks),
 * DSA_DEV_ERR_PAGE; the token is skipped.
 */
int dsa_kv_append(const dsa_kv_cache *cache, const dsa_seqs *seqs, const int32_t *cu_new,
                  int32_t total_new, const void *k_new, const void *v_new,
                  const int8_t *kc_new, int32_t *dev_err, dsa_stream_t stream);

/*
 * dsa_index_score -- block scores of every query against each visible block
 * [P1 4(1): the inner product of the compressed representation with the
 * query, in one fused kernel without intermediate writes; P5 "Index
 * Selection Path": low-precision inputs; P3 4.1].  The pages leave the
 * formula open; this library computes
 *     S[t][b] = sum_h w[t][h] * max(0, sum_d q_idx[t][h][d] * kc[page(s,b)][d])
 * exactly in int32.
 *   q_idx  int8  [total_q][num_idx_heads][idx_dim]
 *   w      int32 [total_q][num_idx_heads]; |w| <= w_abs_max (caller's bound)
 *   scores int32 [total_q][max_blocks]: entries b <= q_pos[t]/block_size are
 *          written, the rest of the row is left untouched.
 * DSA_ERR_RANGE when num_idx_heads * w_abs_max * idx_dim * 128 * 128 >= 2^31
 * (an int32 result could overflow).  Batches with at least 16 queries per
 * sequence on average (prefill) run as int8 tensor-core tiles of 128 blocks x
 * 16 queries (tcgen05, one persistent CTA per SM) when q_pos is 16-byte
 * aligned; the others (decode) scan 256 blocks of one sequence per CTA with
 * dp4a on the CUDA cores.  Both write identical scores.
 * Device errors: DSA_DEV_ERR_PAGE, DSA_DEV_ERR_POS.
 */
int dsa_index_score(const dsa_kv_cache *cache, const dsa_seqs *seqs, const dsa_queries *queries,
                    const int8_t *q_idx, const int32_t *w, int32_t num_idx_heads,
                    int32_t w_abs_max, int32_t *scores, int32_t *dev_err, dsa_stream_t stream);

/*
 * dsa_topk_blocks -- per-query block selection [P1 4(1) "Scalable Top-K";
 * P5 "Index Selection Path": index semantics aligned with the gather].
 * With n = q_pos[t]/block_size + 1 visible blocks and K = k_per_seq[s]:
 * if n <= K every visible block is taken; otherwise the own block n-1 plus
 * the K-1 best of blocks 0..n-2 under (score descending, block id ascending).
 *   scores   int32 [total_q][max_blocks] as written by dsa_index_score
 *   k_per_seq int32 [num_seqs], each in [1, k_max]
 *   sel      int32 [total_q][k_max]: LOGICAL block ids ascending, then -1
 *   cnt      int32 [total_q]: number of ids written
 *   block_size: tokens per block, as in the cache the scores were taken from
 * k_max <= 64 in v1.
 * Device errors: DSA_DEV_ERR_K (that query gets cnt 0), DSA_DEV_ERR_POS.
 */
int dsa_topk_blocks(const dsa_seqs *seqs, const dsa_queries *queries, const int32_t *scores,
                    const int32_t *k_per_seq, int32_t k_max, int32_t block_size, int32_t *sel,
                    int32_t *cnt, int32_t *dev_err, dsa_stream_t stream);

/*
 * Wide scores [P5 "Index Selection Path": the scoring operator takes
 * low-precision inputs; P1 4(1)].  The same formula as dsa_index_score, with
 * int64 results, for the cases the int32 path refuses or does not take:
 *
 * dsa_index_score_i64 -- int8 q_idx and coarse keys, any int32 weights (no
 *   w_abs_max bound): the dot products are exact in int32 and the weighted sum
 *   is accumulated in int64.  scores int64 [total_q][max_blocks], visible
 *   entries written as in dsa_index_score.
 *
 * dsa_index_score_fp8 -- q_idx and the coarse keys (cache->kc_pool, read as
 *   bytes) hold FP8 E4M3 codes (OCP 8-bit float: bias 7, 3 mantissa bits,
 *   subnormals, 0x7F and 0xFF are NaN).  Every finite E4M3 value times 2^9 is
 *   an integer, so the score is computed exactly and returned times 2^18:
 *       scores[t][b] = sum_h w[t][h] * max(0, sum_d (2^9 q[t][h][d]) (2^9 kc[d]))
 *   (int64; the selection it gives is exact and does not depend on any
 *   summation order).  |w| <= w_abs_max; DSA_ERR_RANGE when
 *   num_idx_heads * w_abs_max * idx_dim * (448 * 2^9)^2 >= 2^63.  A NaN code is
 *   read as 0 and sets DSA_DEV_ERR_VALUE.
 *
 * dsa_topk_blocks_i64 -- dsa_topk_blocks over int64 scores (either call above).
 *
 * Both scoring calls run on the CUDA cores (256 blocks of one sequence per
 * CTA).  Device errors: those of the int32 calls, and DSA_DEV_ERR_VALUE.
 */
int dsa_index_score_i64(const dsa_kv_cache *cache, const dsa_seqs *seqs, const dsa_queries *queries,
                        const int8_t *q_idx, const int32_t *w, int32_t num_idx_heads, int64_t *scores,
                        int32_t *dev_err, dsa_stream_t stream);

int dsa_index_score_fp8(const dsa_kv_cache *cache, const dsa_seqs *seqs, const dsa_queries *queries,
                        const uint8_t *q_idx_e4m3, const int32_t *w, int32_t num_idx_heads, int32_t w_abs_max,
                        int64_t *scores, int32_t *dev_err, dsa_stream_t stream);

int dsa_topk_blocks_i64(const dsa_seqs *seqs, const dsa_queries *queries, const int64_t *scores,
                        const int32_t *k_per_seq, int32_t k_max, int32_t block_size, int32_t *sel,
                        int32_t *cnt, int32_t *dev_err, dsa_stream_t stream);

/*
 * dsa_select_blocks -- dsa_index_score and dsa_topk_blocks in one pass, with
 * no score matrix in memory [P1 4(1): one fused scoring kernel with no
 * intermediate written to memory, block-wise reduction + partial selection;
 * P5 "Differentiated Adaptation of Prefill and Decode": fuse selection in
 * decode].  Same arguments and the same sel / cnt results as the two calls;
 * k_max <= 64 and max_blocks <= 131072 (an 8M-token context) in v1.  Each
 * query's visible blocks are scored in chunks by separate CTAs that keep their
 * local Top-(K-1); the last CTA of the query merges them.  Needs a workspace
 * of dsa_select_blocks_workspace_size(total_q) bytes, zero-filled before its
 * first use (each call leaves its counters at zero again).
 * Device errors: DSA_DEV_ERR_PAGE, DSA_DEV_ERR_POS, DSA_DEV_ERR_K.
 */
size_t dsa_select_blocks_workspace_size(int32_t total_q);

int dsa_select_blocks(const dsa_kv_cache *cache, const dsa_seqs *seqs, const dsa_queries *queries,
                      const int8_t *q_idx, const int32_t *w, int32_t num_idx_heads, int32_t w_abs_max,
                      const int32_t *k_per_seq, int32_t k_max, int32_t *sel, int32_t *cnt,
                      void *workspace, size_t workspace_bytes, int32_t *dev_err, dsa_stream_t stream);

/*
 * dsa_select_blocks_append -- dsa_select_blocks and dsa_kv_append in one
 * launch, for a decode batch: the token copies run in extra CTAs of the
 * selection's grid, overlapping the selection (which never reads them), and
 * whatever is launched after this call on `stream` sees both finished.  Same
 * arguments and results as the two calls; the kernel waits for all earlier
 * work on the stream before it starts.  With no queries only the append is
 * launched.
 *  - Every appended block of a sequence must lie at or after the own block of
 *    each of that sequence's queries; a query that breaks this gets
 *    DSA_DEV_ERR_POS and cnt 0 (its selection would read keys being written).
 * Device errors: those of the two calls.
 */
int dsa_select_blocks_append(const dsa_kv_cache *cache, const dsa_seqs *seqs, const dsa_queries *queries,
                             const int32_t *cu_new, int32_t total_new, const void *k_new, const void *v_new,
                             const int8_t *kc_new, const int8_t *q_idx, const int32_t *w, int32_t num_idx_heads,
                             int32_t w_abs_max, const int32_t *k_per_seq, int32_t k_max, int32_t *sel,
                             int32_t *cnt, void *workspace, size_t workspace_bytes, int32_t *dev_err,
                             dsa_stream_t stream);

/*
 * Exact attention over the selected blocks [P1 4(3) decode schematic; P3 4:
 * exact attention on the selected part; P4 "Day-0 Adaptation for Large
 * Language Models: From Architecture Analysis to Inference Serving", table:
 * only the token pairs named by the indexes].  For query t and query head h
 * (KV head h / (num_q_heads/num_kv_heads)), over the tokens j of the blocks
 * sel[t][0..cnt[t]) with position <= q_pos[t]:
 *     out[t][h] = sum_j softmax_j(sm_scale * q[t][h].k_j) v_j
 *     lse[t][h] = ln sum_j exp(sm_scale * q[t][h].k_j)
 * bf16 inputs, fp32 accumulation, bf16 out.
 *   q   bf16 [total_q][num_q_heads][head_dim];  out bf16, same shape
 *   lse fp32 [total_q][num_q_heads] (may be NULL)
 * Both entries run one persistent CTA per SM over the list of (query, KV
 * head, selected block) units, split evenly.  The decode entry may split a
 * (query, KV head) pair across CTAs and merge the partial softmax states
 * (through the workspace, or, when the batch has between a quarter and a half
 * as many pairs as the GPU has SMs, inside a 2-CTA cluster through
 * distributed shared memory); it needs a workspace of dsa_sparse_attn_decode_workspace_size() bytes (a
 * 4-byte counter per (query, KV head) pair plus room for two partial states
 * per CTA), zero-filled before its first use (each call leaves it zeroed
 * again).  The prefill entry keeps every pair
 * inside one CTA and needs no workspace.
 * Device errors: DSA_DEV_ERR_SEL, DSA_DEV_ERR_PAGE (that block is skipped).
 */
size_t dsa_sparse_attn_decode_workspace_size(int32_t total_q, int32_t num_q_heads,
                                             int32_t num_kv_heads, int32_t k_max);

int dsa_sparse_attn_decode(const dsa_kv_cache *cache, const dsa_seqs *seqs,
                           const dsa_queries *queries, const void *q, int32_t num_q_heads,
                           const int32_t *sel, const int32_t *cnt, int32_t k_max, float sm_scale,
                           void *out, float *lse, void *workspace, size_t workspace_bytes,
                           int32_t *dev_err, dsa_stream_t stream);

int dsa_sparse_attn_prefill(const dsa_kv_cache *cache, const dsa_seqs *seqs,
                            const dsa_queries *queries, const void *q, int32_t num_q_heads,
                            const int32_t *sel, const int32_t *cnt, int32_t k_max, float sm_scale,
                            void *out, float *lse, int32_t *dev_err, dsa_stream_t stream);

/*
 * dsa_decode_fused -- one decode step in a single launch: dsa_kv_append, the
 * selection of dsa_select_blocks and dsa_sparse_attn_decode run as phases of
 * one persistent kernel [P5 "Differentiated Adaptation of Prefill and
 * Decode": in decode, fuse index selection, the gather and attention; P1
 * 4(1): block-wise scoring with partial selection].  Arguments are those of
 * the three calls; the results (the pools after the append, sel, cnt, out,
 * lse) are the same bits.
 *  - Every appended block of a sequence must lie at or after the own block of
 *    each of that sequence's queries (decode: one new token per sequence,
 *    whose query sits at its position).  A query that breaks this gets
 *    DSA_DEV_ERR_POS and cnt 0.  With total_new == 0 nothing is appended.
 *  - total_q <= 1024, k_max <= 64, num_idx_heads <= 16.
 *  - Needs a workspace of dsa_decode_fused_workspace_size() bytes, zero-filled
 *    before its first use; each call leaves it ready for the next (it keeps a
 *    call counter, so calls that share one workspace must not overlap).
 *  - Every CTA of the grid must be resident at once (a cooperative launch):
 *    the call fails with DSA_ERR_CUDA if the GPU cannot give it one CTA per
 *    SM.  Waits between phases are bounded (DSA_DEV_ERR_WAIT on timeout).
 * Device errors: those of the three calls.
 */
size_t dsa_decode_fused_workspace_size(int32_t total_q, int32_t num_q_heads, int32_t num_kv_heads,
                                       int32_t k_max);

int dsa_decode_fused(const dsa_kv_cache *cache, const dsa_seqs *seqs, const dsa_queries *queries,
                     const int32_t *cu_new, int32_t total_new, const void *k_new, const void *v_new,
                     const int8_t *kc_new, const int8_t *q_idx, const int32_t *w, int32_t num_idx_heads,
                     int32_t w_abs_max, const int32_t *k_per_seq, int32_t k_max, const void *q,
                     int32_t num_q_heads, float sm_scale, int32_t *sel, int32_t *cnt, void *out, float *lse,
                     void *workspace, size_t workspace_bytes, int32_t *dev_err, dsa_stream_t stream);

/*
 * dsa_sparse_attn_decode_noalloc -- the decode attention above for callers
 * that cannot allocate device memory.  The pages have no counterpart to this
 * call; it exists for callers such as an engine plugin whose enqueue path must
 * not allocate or synchronise, or a runtime that owns all device memory
 * itself, which therefore cannot hand over a workspace from cudaMalloc.
 * Arguments are those of dsa_sparse_attn_decode without the workspace: the
 * split-KV scratch lives in a fixed array of DSA_NOALLOC_SCRATCH_BYTES inside
 * the library, held on every GPU that loads the library until the process
 * exits.  The call allocates nothing.
 *  - Limit: dsa_sparse_attn_decode_workspace_size(total_q, num_q_heads,
 *    num_kv_heads, k_max) must be <= DSA_NOALLOC_SCRATCH_BYTES (with 8 query
 *    heads per KV head that is about 2.1 MiB plus 4 bytes per (query, KV head),
 *    so up to roughly 3.6 million (query, KV head) pairs); larger problems get
 *    DSA_ERR_WORKSPACE and nothing is launched.
 *  - The first call on each device (with that device current) looks up the
 *    scratch array's device address; make that first call before any stream
 *    capture.
 *  - Every call first zeroes the scratch's split counters on `stream`.  All
 *    calls share the one array, so calls that overlap on the GPU (other
 *    streams or threads) race; the caller must serialise them.
 */
#define DSA_NOALLOC_SCRATCH_BYTES (16u << 20)

int dsa_sparse_attn_decode_noalloc(const dsa_kv_cache *cache, const dsa_seqs *seqs,
                                   const dsa_queries *queries, const void *q, int32_t num_q_heads,
                                   const int32_t *sel, const int32_t *cnt, int32_t k_max,
                                   float sm_scale, void *out, float *lse, int32_t *dev_err,
                                   dsa_stream_t stream);

/*
 * Host staging of repeated steps.  The pages have no counterpart to this
 * part: it is runtime plumbing for a loop that issues one step per batch from
 * the host, each step's inputs in pinned host memory and its results wanted
 * back on the host.  A stager owns two copy streams (created at
 * dsa_stager_create, on the device current then) and one set of events per
 * slot; a slot is one batch whose device buffers are reused step after step.
 * The copies of one slot overlap the kernels of the other slots' steps while
 * each step still sees its own inputs and leaves its own results:
 *
 *   dsa_stager_begin(st, slot, ...)   inputs host -> device
 *   <the step's library calls on the stager's stream>
 *   dsa_stager_end(st, slot, ...)     results device -> host
 *
 *  - dsa_stager_create: num_slots in 1..4096; `stream` is the compute stream
 *    the steps are issued on (the stager does not own it).  *out receives the
 *    handle.  DSA_ERR_CUDA if a stream or event cannot be created.
 *  - dsa_stager_begin: n regions (0..64), region i copies bytes[i] bytes from
 *    host_src[i] to dev_dst[i] (cudaMemcpyAsync; asynchronous only if the
 *    host memory is pinned).  The copies wait until the slot's previous step
 *    (the calls between its previous begin and end) has run, since that step
 *    reads those device buffers; then the compute stream waits for them and
 *    for the slot's previous read-back.  Any other reader or writer of those
 *    buffers must be ordered by the caller.  The host must not rewrite
 *    host_src before the copies have landed (dsa_stager_wait on the slot
 *    covers it).
 *  - dsa_stager_end: after the step's calls; region i copies bytes[i] bytes
 *    from dev_src[i] to host_dst[i] once the step has run.
 *  - dsa_stager_wait: blocks the host until the slot's last read-back has
 *    landed.  dsa_stager_join: makes the compute stream wait for every copy
 *    issued so far (before an event or a synchronisation on that stream).
 *  - dsa_stager_destroy: waits for the copy streams, then frees everything
 *    (NULL is a no-op).
 *  - Errors: DSA_ERR_INVALID_ARG for a NULL handle, a slot outside
 *    [0, num_slots), n outside 0..64 or a NULL pointer of a non-empty
 *    region (nothing is issued); DSA_ERR_CUDA when a CUDA call fails.
 *  - Call with the device of create current; not under stream capture (a
 *    graph captures the plain calls and torch-side copies instead); one
 *    thread at a time per stager.
 */
typedef struct dsa_stager dsa_stager;

int dsa_stager_create(int32_t num_slots, dsa_stream_t stream, dsa_stager **out);
int dsa_stager_destroy(dsa_stager *st);
int dsa_stager_begin(dsa_stager *st, int32_t slot, int32_t n, void *const *dev_dst, const void *const *host_src,
                     const size_t *bytes);
int dsa_stager_end(dsa_stager *st, int32_t slot, int32_t n, void *const *host_dst, const void *const *dev_src,
                   const size_t *bytes);
int dsa_stager_wait(dsa_stager *st, int32_t slot);
int dsa_stager_join(dsa_stager *st);

/* human-readable name of a status code (static string) */
const char *dsa_status_string(int status);

/* library version, e.g. 100 for 0.1.0 */
int dsa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* DSA_H */
