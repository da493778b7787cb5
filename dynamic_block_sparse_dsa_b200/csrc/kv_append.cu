// kv_append.cu -- scatter new tokens into the block-paged KV cache.
//
// "Day-0 Readiness for Trillion-Parameter Models: Engineering Sparse Attention
// and Expert Weight Compression", section "KV Cache Layout": prefill writes
// blocks in batch, decode appends one token and maintains the block table,
// and both share one block-index semantics.  One CTA per new token copies its
// K and V rows (num_kv_heads * 256 bytes each) with 16-byte vector stores into
// the page slot block_table[s][pos / B], token pos % B (B the block size);
// the last new token of each touched block also writes that block's coarse key.
#include "dsa_kernels.h"
#include "kv_append.cuh"

namespace dsa {

__global__ void __launch_bounds__(128) kv_append_kernel(KvAppendArgs a) {
    pdl_trigger();   // the next kernel may start its prologue; it waits for us before reading
    append_token(a, blockIdx.x, threadIdx.x, blockDim.x);
    // overlapping a selection: finish only once it has (see KvAppendArgs)
    if (a.overlap_prev) pdl_wait();
}

cudaError_t launch_kv_append(const KvAppendArgs &a, cudaStream_t stream) {
    if (a.total_new == 0) return cudaSuccess;
    if (a.overlap_prev) return launch_pdl(kv_append_kernel, dim3(a.total_new), dim3(128), 0, stream, a);
    kv_append_kernel<<<a.total_new, 128, 0, stream>>>(a);
    return cudaGetLastError();
}

}  // namespace dsa
