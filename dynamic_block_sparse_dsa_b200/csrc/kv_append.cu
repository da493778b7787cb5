// kv_append.cu -- scatter new tokens into the block-paged KV cache.
//
// "Day-0 Readiness for Trillion-Parameter Models: Engineering Sparse Attention
// and Expert Weight Compression", section "KV Cache Layout": prefill writes
// blocks in batch, decode appends one token and maintains the block table,
// and both share one block-index semantics.  One CTA per new token copies its
// K and V rows (num_kv_heads * 256 bytes each) with 16-byte vector stores into
// the page slot block_table[s][pos / 64], token pos % 64; the last new token
// of each touched block also writes that block's coarse key.
#include "dsa_kernels.h"

namespace dsa {

__device__ __forceinline__ void append_one(const KvAppendArgs &a);

__global__ void __launch_bounds__(128) kv_append_kernel(KvAppendArgs a) {
    pdl_trigger();   // the next kernel may start its prologue; it waits for us before reading
    append_one(a);
    // overlapping a selection: finish only once it has (see KvAppendArgs)
    if (a.overlap_prev) pdl_wait();
}

__device__ __forceinline__ void append_one(const KvAppendArgs &a) {
    const int i = blockIdx.x;
    const int s = find_seq(a.cu_new, a.num_seqs, i);
    const int first = __ldg(a.cu_new + s), last = __ldg(a.cu_new + s + 1);
    if (i < first || i >= last) {            // total_new larger than cu_new[num_seqs]
        if (threadIdx.x == 0) set_err(a.dev_err, DSA_DEV_ERR_POS);
        return;
    }
    const int len = __ldg(a.seq_lens + s);
    const int n = last - first;
    const int pos = len - n + (i - first);
    const int blk = pos / kBlockSize, slot = pos % kBlockSize;
    if (n > len || pos < 0 || blk >= a.max_blocks) {
        if (threadIdx.x == 0) set_err(a.dev_err, DSA_DEV_ERR_POS);
        return;
    }
    const int page = __ldg(a.block_table + (size_t)s * a.max_blocks + blk);
    if (page < 0 || page >= a.num_pages) {
        if (threadIdx.x == 0) set_err(a.dev_err, DSA_DEV_ERR_PAGE);
        return;
    }
    // one token row = num_kv_heads * head_dim bf16 = row16 16-byte vectors
    const int row16 = a.num_kv_heads * (kHeadDim * 2 / 16);
    const size_t dst = ((size_t)page * kBlockSize + slot) * row16;
    const uint4 *ks = reinterpret_cast<const uint4 *>(a.k_new) + (size_t)i * row16;
    const uint4 *vs = reinterpret_cast<const uint4 *>(a.v_new) + (size_t)i * row16;
    uint4 *kd = reinterpret_cast<uint4 *>(a.k_pool) + dst;
    uint4 *vd = reinterpret_cast<uint4 *>(a.v_pool) + dst;
    for (int e = threadIdx.x; e < row16; e += blockDim.x) {
        kd[e] = __ldg(ks + e);
        vd[e] = __ldg(vs + e);
    }
    const bool last_in_block = (i == last - 1) || (slot == kBlockSize - 1);
    if (a.kc_new && last_in_block && threadIdx.x < kIdxDim / 16) {
        const uint4 *cs = reinterpret_cast<const uint4 *>(a.kc_new) + (size_t)i * (kIdxDim / 16);
        uint4 *cd = reinterpret_cast<uint4 *>(a.kc_pool) + (size_t)page * (kIdxDim / 16);
        cd[threadIdx.x] = __ldg(cs + threadIdx.x);
    }
}

cudaError_t launch_kv_append(const KvAppendArgs &a, cudaStream_t stream) {
    if (a.total_new == 0) return cudaSuccess;
    if (a.overlap_prev) return launch_pdl(kv_append_kernel, dim3(a.total_new), dim3(128), 0, stream, a);
    kv_append_kernel<<<a.total_new, 128, 0, stream>>>(a);
    return cudaGetLastError();
}

}  // namespace dsa
