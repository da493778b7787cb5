// dsa_kernels.h -- internal kernel argument blocks and launchers (not part of the C ABI).
#pragma once

#include "dsa_common.cuh"

namespace dsa {

// launch `kern` with programmatic stream serialization (see pdl_wait)
template <typename Kern, typename... Args>
cudaError_t launch_pdl(Kern kern, dim3 grid, dim3 block, size_t smem, cudaStream_t stream, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, args...);
}

struct KvAppendArgs {
    void *k_pool, *v_pool;
    int8_t *kc_pool;
    int num_pages, num_kv_heads;
    int block_shift;         // tokens per KV block = 1 << block_shift (6..9)
    const int32_t *block_table;
    int max_blocks;
    const int32_t *seq_lens;
    int num_seqs;
    const int32_t *cu_new;
    int total_new;
    const void *k_new, *v_new;
    const int8_t *kc_new;
    int32_t *dev_err;
    // 0: an ordinary launch (waits for everything before it).  1: launched
    // as a programmatic dependent of a selection kernel that reads none of
    // the rows written here -- the copies overlap it, and the kernel waits
    // for it only before exiting, so whatever waits for the append also
    // waits for the selection.
    int overlap_prev;
};

struct IndexScoreArgs {
    const int8_t *kc_pool;
    int num_pages;
    int block_shift;
    const int32_t *block_table;
    int max_blocks;
    const int32_t *seq_lens;
    int num_seqs;
    const int32_t *cu_q;
    const int32_t *q_pos;
    int total_q;
    const int8_t *q_idx;     // [T][H][64]
    const int32_t *w;        // [T][H]
    int num_idx_heads;
    int32_t *scores;         // [T][max_blocks]
    int32_t *dev_err;
};

struct TopkArgs {
    int block_shift;
    const int32_t *seq_lens;
    int num_seqs;
    int max_blocks;
    const int32_t *cu_q;
    const int32_t *q_pos;
    int total_q;
    const int32_t *scores;
    const int32_t *k_per_seq;
    int k_max;
    int32_t *sel;
    int32_t *cnt;
    int32_t *dev_err;
};

// fused score + Top-K (decode-oriented): candidate workspace layout
constexpr int kSelMaxChunks = 32;   // chunks per query
constexpr int kSelMaxK = 64;        // largest k_max of the fused path
struct SelectArgs {
    const int8_t *kc_pool;
    int num_pages;
    int block_shift;
    const int32_t *block_table;
    int max_blocks;
    const int32_t *seq_lens;
    int num_seqs;
    const int32_t *cu_q;
    const int32_t *q_pos;
    int total_q;
    const int8_t *q_idx;     // [T][H][64]
    const int32_t *w;        // [T][H]
    int num_idx_heads;
    const int32_t *k_per_seq;
    int k_max;
    int32_t *sel;            // [T][k_max]
    int32_t *cnt;            // [T]
    unsigned long long *cand;   // [T][kSelMaxChunks][kSelMaxK-1] 64-bit selection keys, sorted descending
    int32_t *counters;       // [T] chunk CTAs done per query
    int32_t *dev_err;
    // append ordered after this selection (dsa_select_blocks_append): a
    // query whose sequence appends a block before its own block is refused
    // (DSA_DEV_ERR_POS, cnt 0) -- the selection must not read those keys; and
    // the kernel is launched after everything before it has completed
    const int32_t *cu_new;   // null: no append follows
    // the append itself (app.total_new > 0): extra CTAs of the selection grid,
    // rows sel_rows.. of blockIdx.y, copy the new tokens while the selection runs
    KvAppendArgs app;
    int sel_rows;            // set by the launcher: grid rows that select
};

struct AttnArgs {
    const __nv_bfloat16 *k_pool, *v_pool;
    int num_pages, num_kv_heads;
    // tokens per KV block = 1 << block_shift; the kernel works in 64-token
    // tiles, tile_shift = block_shift - 6 of them per block
    int block_shift, tile_shift;
    const int32_t *block_table;
    int max_blocks;
    const int32_t *seq_lens;
    int num_seqs;
    const int32_t *cu_q;
    const int32_t *q_pos;
    int total_q;
    const __nv_bfloat16 *q;  // [T][Hq][128]
    int num_q_heads;
    int group;               // Hq / Hkv
    const int32_t *sel;      // [T][k_max]
    const int32_t *cnt;      // [T]
    int k_max;
    float scale_log2;        // sm_scale * log2(e)
    __nv_bfloat16 *out;      // [T][Hq][128]
    float *lse;              // [T][Hq] or null
    // persistent schedule: work unit u = (query t, KV head, selection slot j,
    // 64-token tile i of that block), u = ((t * Hkv + kvh) * k_max + j) * m + i
    // with m = 1 << tile_shift; CTA c owns [c*U/C, (c+1)*U/C), rounded to whole
    // (t, kvh) pairs when pair_aligned
    long long total_units;   // U
    int num_ctas;            // C (= gridDim.x)
    int pair_aligned;
    // with pair_aligned: CTA c runs instead the pairs r = c, c + C, c + 2C, ...
    // of the KV-head-major order r = kvh * T + t, so that all CTAs work on
    // the same KV head at a time and its blocks are re-read from L2
    int interleave;
    // 1: pair p is run by the 2-CTA cluster (2p, 2p+1), each CTA taking half
    // of its units; the halves merge through distributed shared memory and
    // no workspace is touched
    int cluster2;
    float *part;             // [2*C][group][kAttnPartStride] partial (o[128], m, l) of split pairs
    int32_t *counters;       // [T*Hkv] units merged so far per split pair
    int32_t *dev_err;
};

// single-launch decode step (append + select + attention in one persistent
// kernel): the arguments beyond AttnArgs
constexpr int kFusedMaxQ = 1024;                            // queries per call
constexpr int kHdrEpoch = 0, kHdrDone = 1, kHdrAppended = 2;  // workspace header words
struct FusedArgs {
    // append (total_new == 0: nothing to append)
    const int32_t *cu_new;
    int total_new;
    const void *k_new, *v_new;
    const int8_t *kc_new;
    void *k_pool, *v_pool;   // the pools, writable
    int8_t *kc_pool;
    // indexer + selection
    const int8_t *q_idx;     // [T][H][64]
    const int32_t *w;        // [T][H]
    int num_idx_heads;
    const int32_t *k_per_seq;
    int32_t *sel;            // [T][k_max] (AttnArgs::sel, writable)
    int32_t *cnt;            // [T]
    // workspace
    int32_t *hdr;            // epoch, CTAs done, tokens appended
    int32_t *sel_count;      // [T] candidate groups merged per query
    int32_t *flags;          // [T] selection ready: the call's epoch + 1
    unsigned long long *cand;   // [C][2][kSelMaxK-1] per-CTA Top-(K-1) of split queries
};

cudaError_t launch_kv_append(const KvAppendArgs &a, cudaStream_t stream);
cudaError_t launch_index_score(const IndexScoreArgs &a, cudaStream_t stream);
// tensor-core (tcgen05 int8) scoring for batches with many queries per sequence
cudaError_t launch_index_score_tc(const IndexScoreArgs &a, int num_sms, cudaStream_t stream);
int index_score_tc_min_queries_per_seq();
cudaError_t launch_topk(const TopkArgs &a, cudaStream_t stream);
// int64 scores: the int8 indexer without the int32 bound, or (fp8) the E4M3
// indexer times 2^18; and the Top-K over such scores
cudaError_t launch_index_score_wide(const IndexScoreArgs &a, bool fp8, int64_t *scores, cudaStream_t stream);
cudaError_t launch_topk_wide(const TopkArgs &a, const int64_t *scores, cudaStream_t stream);
cudaError_t launch_select_blocks(const SelectArgs &a, cudaStream_t stream);
int topk_max_blocks();   // longest block table the standalone Top-K kernel accepts
// the K/V pool and Q tensor maps are built by the launcher from AttnArgs
cudaError_t launch_sparse_attn(const AttnArgs &a, cudaStream_t stream);
cudaError_t launch_decode_fused(const AttnArgs &a, const FusedArgs &f, cudaStream_t stream);
// host-side checks of dsa_sparse_attn_decode's arguments, without any CUDA
// call: DSA_OK or the status the entry point would return
int check_decode_attn_args(const dsa_kv_cache *cache, const dsa_seqs *seqs, const dsa_queries *queries,
                           const void *q, int32_t num_q_heads, const int32_t *sel, const int32_t *cnt,
                           int32_t k_max, float sm_scale, void *out, float *lse);
// largest grid the attention kernel uses (sizes the partial-state workspace)
constexpr int kAttnMaxCtas = 256;
// floats per partial-state row: o[128], m, l, padded to a 16-byte multiple
constexpr int kAttnPartStride = 132;

}  // namespace dsa
