// topk.cu -- per-query Top-K block selection from a score matrix.
//
// "Day-0 Adaptation for Massive LLMs: Overcoming Sparse Attention and MXFP4
// Expert Weights", section 4(1) "Scalable Top-K": the candidate count grows
// with the context, so no full sort -- an exact partial selection instead.
// "Day-0 Readiness for Trillion-Parameter Models ...", section "Index
// Selection Path": the indices follow the gather's semantics; here they are
// logical block ids, ascending, -1 padded.
//
// One CTA of 1024 threads per query.  The candidates (blocks 0..n-2; the own
// block n-1 is always kept) are loaded once into registers, E consecutive
// blocks per thread, and the K-1 winners under (score descending, block id
// ascending) are found by the radix selection of select_core.cuh; a prefix
// count over the threads writes them in ascending id order without a sort.
#include "dsa_kernels.h"
#include "select_core.cuh"

namespace dsa {

namespace {
constexpr int kTopkThreads = 1024;
}  // namespace

template <int E>
__global__ void __launch_bounds__(kTopkThreads) topk_kernel(TopkArgs a) {
    __shared__ SelectSmem sh;
    const int t = blockIdx.x, tid = threadIdx.x;
    int32_t *out = a.sel + (size_t)t * a.k_max;
    const int s = find_seq(a.cu_q, a.num_seqs, t);
    const int p = __ldg(a.q_pos + t);
    const int len = __ldg(a.seq_lens + s);
    const int K = __ldg(a.k_per_seq + s);
    const int n_vis = p / kBlockSize + 1;
    const bool bad_pos = p < 0 || p >= len || n_vis > a.max_blocks;
    const bool bad_k = K < 1 || K > a.k_max;
    if (bad_pos || bad_k) {
        if (tid == 0) {
            set_err(a.dev_err, bad_k ? DSA_DEV_ERR_K : DSA_DEV_ERR_POS);
            a.cnt[t] = 0;
        }
        for (int i = tid; i < a.k_max; i += kTopkThreads) out[i] = -1;
        return;
    }
    if (n_vis <= K) {   // every visible block is taken
        for (int i = tid; i < a.k_max; i += kTopkThreads) out[i] = i < n_vis ? i : -1;
        if (tid == 0) a.cnt[t] = n_vis;
        return;
    }
    const int n = n_vis - 1;   // candidates 0..n-1 (n >= K)
    const int kk = K - 1;
    const int32_t *row = a.scores + (size_t)t * a.max_blocks;
    uint32_t key[E];
    bool valid[E];
#pragma unroll
    for (int e = 0; e < E; ++e) {
        const int b = tid * E + e;
        valid[e] = b < n;
        key[e] = valid[e] ? order_key(__ldg(row + b)) : 0u;
    }
    bool take[E];
    cta_select<kTopkThreads, E>(key, valid, kk, take, sh);
    int nt = 0;
#pragma unroll
    for (int e = 0; e < E; ++e) nt += take[e];
    int tot;
    int pos = cta_exclusive_scan<kTopkThreads>(nt, sh, &tot);
#pragma unroll
    for (int e = 0; e < E; ++e)
        if (take[e]) out[pos++] = tid * E + e;
    if (tid == 0) {
        out[kk] = n;   // the own block, the largest visible id
        a.cnt[t] = K;
    }
    for (int i = K + tid; i < a.k_max; i += kTopkThreads) out[i] = -1;
}

int topk_max_blocks() { return kTopkThreads * 32; }

cudaError_t launch_topk(const TopkArgs &a, cudaStream_t stream) {
    if (a.total_q == 0) return cudaSuccess;
    const int e = (a.max_blocks + kTopkThreads - 1) / kTopkThreads;
    if (e <= 1) topk_kernel<1><<<a.total_q, kTopkThreads, 0, stream>>>(a);
    else if (e <= 2) topk_kernel<2><<<a.total_q, kTopkThreads, 0, stream>>>(a);
    else if (e <= 4) topk_kernel<4><<<a.total_q, kTopkThreads, 0, stream>>>(a);
    else if (e <= 8) topk_kernel<8><<<a.total_q, kTopkThreads, 0, stream>>>(a);
    else if (e <= 16) topk_kernel<16><<<a.total_q, kTopkThreads, 0, stream>>>(a);
    else if (e <= 32) topk_kernel<32><<<a.total_q, kTopkThreads, 0, stream>>>(a);
    else return cudaErrorInvalidValue;   // the host rejects longer tables first
    return cudaGetLastError();
}

}  // namespace dsa
