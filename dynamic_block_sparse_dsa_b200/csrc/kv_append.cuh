// kv_append.cuh -- the copy of one new token into the block-paged KV cache,
// shared by the append kernel and the selection kernel that overlaps it.
//
// "Day-0 Readiness for Trillion-Parameter Models: Engineering Sparse Attention
// and Expert Weight Compression", section "KV Cache Layout": decode appends
// one token into the page slot block_table[s][pos / B], token pos % B (B the
// block size), and prefill writes whole blocks the same way.  Token i of sequence s (cu_new[s]
// <= i < cu_new[s+1]) lands at position seq_lens[s] - n_s + (i - cu_new[s]);
// its K and V rows (num_kv_heads * 256 bytes each) are copied with 16-byte
// vectors, and the last new token of each touched block also writes that
// block's coarse key.  `nthreads` threads numbered `tid` share the copy.
#pragma once

#include "dsa_kernels.h"

namespace dsa {

__device__ __forceinline__ void append_token(const KvAppendArgs &a, int i, int tid, int nthreads) {
    const int s = find_seq(a.cu_new, a.num_seqs, i);
    const int first = __ldg(a.cu_new + s), last = __ldg(a.cu_new + s + 1);
    if (i < first || i >= last) {            // total_new larger than cu_new[num_seqs]
        if (tid == 0) set_err(a.dev_err, DSA_DEV_ERR_POS);
        return;
    }
    const int len = __ldg(a.seq_lens + s);
    const int n = last - first;
    const int pos = len - n + (i - first);
    const int blk = pos >> a.block_shift, slot = pos & ((1 << a.block_shift) - 1);
    if (n > len || pos < 0 || blk >= a.max_blocks) {
        if (tid == 0) set_err(a.dev_err, DSA_DEV_ERR_POS);
        return;
    }
    const int page = __ldg(a.block_table + (size_t)s * a.max_blocks + blk);
    if (page < 0 || page >= a.num_pages) {
        if (tid == 0) set_err(a.dev_err, DSA_DEV_ERR_PAGE);
        return;
    }
    // one token row = num_kv_heads * head_dim bf16 = row16 16-byte vectors
    const int row16 = a.num_kv_heads * (kHeadDim * 2 / 16);
    const size_t dst = (((size_t)page << a.block_shift) + slot) * row16;
    const uint4 *ks = reinterpret_cast<const uint4 *>(a.k_new) + (size_t)i * row16;
    const uint4 *vs = reinterpret_cast<const uint4 *>(a.v_new) + (size_t)i * row16;
    uint4 *kd = reinterpret_cast<uint4 *>(a.k_pool) + dst;
    uint4 *vd = reinterpret_cast<uint4 *>(a.v_pool) + dst;
    for (int e = tid; e < row16; e += nthreads) {
        kd[e] = __ldg(ks + e);
        vd[e] = __ldg(vs + e);
    }
    const bool last_in_block = (i == last - 1) || (slot == (1 << a.block_shift) - 1);
    if (a.kc_new && last_in_block && tid < kIdxDim / 16) {
        const uint4 *cs = reinterpret_cast<const uint4 *>(a.kc_new) + (size_t)i * (kIdxDim / 16);
        uint4 *cd = reinterpret_cast<uint4 *>(a.kc_pool) + (size_t)page * (kIdxDim / 16);
        cd[tid] = __ldg(cs + tid);
    }
}

}  // namespace dsa
