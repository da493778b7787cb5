// dsa_kernels.h -- internal kernel argument blocks and launchers (not part of the C ABI).
#pragma once

#include "dsa_common.cuh"

namespace dsa {

struct KvAppendArgs {
    void *k_pool, *v_pool;
    int8_t *kc_pool;
    int num_pages, num_kv_heads;
    const int32_t *block_table;
    int max_blocks;
    const int32_t *seq_lens;
    int num_seqs;
    const int32_t *cu_new;
    int total_new;
    const void *k_new, *v_new;
    const int8_t *kc_new;
    int32_t *dev_err;
};

struct IndexScoreArgs {
    const int8_t *kc_pool;
    int num_pages;
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

struct AttnArgs {
    const __nv_bfloat16 *k_pool, *v_pool;
    int num_pages, num_kv_heads;
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
    int n_splits;            // CTAs per (query, kv head)
    int blocks_per_split;
    float *part_o;           // [T][Hq][n_splits][128]
    float *part_ml;          // [T][Hq][n_splits][2]
    int32_t *counters;       // [T][Hkv]
    int32_t *dev_err;
};

cudaError_t launch_kv_append(const KvAppendArgs &a, cudaStream_t stream);
cudaError_t launch_index_score(const IndexScoreArgs &a, cudaStream_t stream);
cudaError_t launch_topk(const TopkArgs &a, cudaStream_t stream);
cudaError_t launch_sparse_attn(const AttnArgs &a, cudaStream_t stream);

}  // namespace dsa
