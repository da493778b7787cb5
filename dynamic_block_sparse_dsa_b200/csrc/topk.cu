// topk.cu -- per-query Top-K block selection from a score matrix.
//
// "Day-0 Adaptation for Massive LLMs: Overcoming Sparse Attention and MXFP4
// Expert Weights", section 4(1) "Scalable Top-K": the candidate count grows
// with the context, so no full sort -- an exact partial selection instead.
// "Day-0 Readiness for Trillion-Parameter Models ...", section "Index
// Selection Path": the indices follow the gather's semantics; here they are
// logical block ids, ascending, -1 padded.
//
// One CTA of 256 threads per query (several resident per SM).  Each warp
// streams groups of 64 candidates (coalesced loads): it sorts its first group
// with a warp bitonic network and folds later ones into its running Top-64,
// skipping, after one vote, every group with no key above the current
// (K-1)-th (warp_topk.cuh); a merge tree over the 8 warps leaves the query's
// Top-64 in warp 0, which appends the own block and writes the winners in
// ascending block order.
#include "dsa_kernels.h"
#include "warp_topk.cuh"

namespace dsa {

namespace {
constexpr int kTopkThreads = 256;
constexpr int kTopkWarps = kTopkThreads / 32;
}  // namespace

__global__ void __launch_bounds__(kTopkThreads) topk_kernel(TopkArgs a) {
    __shared__ key64 s_lists[kTopkWarps * 64];
    pdl_trigger();
    pdl_wait();   // the scores come from the preceding kernel
    const int t = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    int32_t *out = a.sel + (size_t)t * a.k_max;
    const int s = find_seq(a.cu_q, a.num_seqs, t);
    const int p = __ldg(a.q_pos + t);
    const int len = __ldg(a.seq_lens + s);
    const int K = __ldg(a.k_per_seq + s);
    const int n_vis = (p >> a.block_shift) + 1;
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
    key64 acc[2] = {0ull, 0ull};
    bool first = true;
    for (int g0 = warp * 64; g0 < n; g0 += kTopkWarps * 64) {
        const int i0 = g0 + lane, i1 = g0 + 32 + lane;
        key64 v[2] = {i0 < n ? make_key64(__ldg(row + i0), (uint32_t)i0) : 0ull,
                      i1 < n ? make_key64(__ldg(row + i1), (uint32_t)i1) : 0ull};
        if (first) {
            warp_sort64_desc(v);
            acc[0] = v[0];
            acc[1] = v[1];
            first = false;
        } else {
            warp_fold_topk(acc, v, kk);   // groups with nothing above the kk-th key cost one vote
        }
    }
    cta_merge_top64<kTopkWarps>(acc, s_lists);
    if (warp == 0) {
        const bool v0 = lane < kk, v1 = 32 + lane < kk;
        uint32_t ids[2] = {v0 ? key64_id(acc[0]) : 0xffffffffu, v1 ? key64_id(acc[1]) : 0xffffffffu};
        warp_sort64_asc_u32(ids);
        if (v0) out[lane] = (int32_t)ids[0];
        if (v1) out[32 + lane] = (int32_t)ids[1];
        if (lane == 0) {
            out[kk] = n;   // the own block, the largest visible id
            a.cnt[t] = K;
        }
        for (int i = K + lane; i < a.k_max; i += 32) out[i] = -1;
    }
}

int topk_max_blocks() { return 1 << 20; }

cudaError_t launch_topk(const TopkArgs &a, cudaStream_t stream) {
    if (a.total_q == 0) return cudaSuccess;
    if (a.k_max > 64) return cudaErrorInvalidValue;   // the host rejects these first
    return launch_pdl(topk_kernel, dim3(a.total_q), dim3(kTopkThreads), 0, stream, a);
}

}  // namespace dsa
