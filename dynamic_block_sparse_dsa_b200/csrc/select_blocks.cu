// select_blocks.cu -- fused block scoring + Top-K selection (no score matrix).
//
// "Day-0 Adaptation for Massive LLMs: Overcoming Sparse Attention and MXFP4
// Expert Weights", section 4(1): score the compressed block representation in
// one fused kernel without writing intermediates to memory, and make the
// Top-K scalable with a block-wise reduction plus partial selection instead of
// a full sort.  "Day-0 Readiness ...", section "Differentiated Adaptation of
// Prefill and Decode": fuse index selection for decode to cut launches and
// write-backs.
//
// Grid: (query, chunk of 256*E candidate blocks).  Each CTA scores its chunk
// with the CUDA-core int8 indexer (one thread per E consecutive blocks: page
// id, 64-byte coarse key, dp4a), keeps the chunk's local Top-(K-1) in id order
// (warp-level bitonic Top-64 on unique 64-bit keys, then a merge tree over
// the warps) and writes it to the workspace.  The last CTA of the query --
// elected with an atomic counter, nothing waits -- merges the chunks' sorted
// lists the same way, appends the query's own block and writes the ascending
// selection.  Result is identical to dsa_index_score followed by
// dsa_topk_blocks.
#include "dsa_kernels.h"
#include "indexer_core.cuh"
#include "warp_topk.cuh"

namespace dsa {

namespace {
constexpr int kSelThreads = 256;
constexpr int kSelWarps = kSelThreads / 32;
constexpr int kCuqCache = 1024;   // cu_q entries staged in shared memory
}  // namespace

template <int E>
__global__ void __launch_bounds__(kSelThreads) select_blocks_kernel(SelectArgs a) {
    __shared__ int4 s_q[kMaxIdxHeads][kIdxDim / 16];
    __shared__ int s_w[kMaxIdxHeads];
    __shared__ int s_cuq[kCuqCache + 1];
    __shared__ key64 s_lists[kSelWarps * 64];
    __shared__ int s_last;
    constexpr int CH = kSelThreads * E;
    const int t = blockIdx.x, c = blockIdx.y, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int H = a.num_idx_heads;

    // ---- query facts: the sequence from a shared-memory copy of cu_q
    const bool cached = a.num_seqs + 1 <= kCuqCache;
    if (cached)
        for (int i = tid; i <= a.num_seqs; i += kSelThreads) s_cuq[i] = __ldg(a.cu_q + i);
    for (int e = tid; e < H * 4; e += kSelThreads)
        s_q[e >> 2][e & 3] = __ldg(reinterpret_cast<const int4 *>(a.q_idx + (size_t)t * H * kIdxDim) + e);
    if (tid < H) s_w[tid] = __ldg(a.w + (size_t)t * H + tid);
    __syncthreads();
    int s;
    if (cached) {
        int lo = 0, hi = a.num_seqs - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (s_cuq[mid] <= t) lo = mid; else hi = mid - 1;
        }
        s = lo;
    } else {
        s = find_seq(a.cu_q, a.num_seqs, t);
    }
    const int p = __ldg(a.q_pos + t);
    const int len = __ldg(a.seq_lens + s);
    const int K = __ldg(a.k_per_seq + s);
    const int n_vis = p / kBlockSize + 1;
    int32_t *out = a.sel + (size_t)t * a.k_max;
    const bool bad_pos = p < 0 || p >= len || n_vis > a.max_blocks;
    const bool bad_k = K < 1 || K > a.k_max;
    if (bad_pos || bad_k) {
        if (c == 0) {
            if (tid == 0) {
                set_err(a.dev_err, bad_k ? DSA_DEV_ERR_K : DSA_DEV_ERR_POS);
                a.cnt[t] = 0;
            }
            for (int i = tid; i < a.k_max; i += kSelThreads) out[i] = -1;
        }
        return;
    }
    const int own = n_vis - 1;
    const int kk = K - 1;
    if (n_vis <= K || kk == 0) {   // every visible block, or only the own block
        if (c == 0) {
            const int n = n_vis <= K ? n_vis : 1;
            for (int i = tid; i < a.k_max; i += kSelThreads) out[i] = i < n ? (n == 1 ? own : i) : -1;
            if (tid == 0) a.cnt[t] = n;
        }
        return;
    }
    const int n_chunks = (own + CH - 1) / CH;   // candidates: blocks 0 .. own-1
    if (c >= n_chunks) return;

    // ---- score this chunk: E consecutive blocks per thread
    key64 key[E];
    uint32_t err_bits = 0;
    const int b0 = c * CH + tid * E;
#pragma unroll
    for (int e = 0; e < E; ++e) {
        const int b = b0 + e;
        key[e] = 0;
        if (b < own) {
            const int page = __ldg(a.block_table + (size_t)s * a.max_blocks + b);
            if (page >= 0 && page < a.num_pages) {
                int kc[16];
                load_coarse_key(a.kc_pool, page, kc);
                key[e] = make_key64(block_score(kc, s_q, s_w, H), (uint32_t)b);
            } else {
                err_bits |= DSA_DEV_ERR_PAGE;
            }
        }
    }
    if (err_bits) set_err(a.dev_err, err_bits);

    // ---- chunk Top-64: per warp, then a merge tree over the warps
    key64 acc[2];
#pragma unroll
    for (int g = 0; g < (E + 1) / 2; ++g) {
        key64 v[2] = {key[2 * g], 2 * g + 1 < E ? key[2 * g + 1] : 0ull};
        warp_sort64_desc(v);
        if (g == 0) { acc[0] = v[0]; acc[1] = v[1]; }
        else warp_merge64_desc(acc, v);
    }
    cta_merge_top64<kSelWarps>(acc, s_lists);
    key64 *cand = a.cand + ((size_t)t * kSelMaxChunks + c) * (kSelMaxK - 1);
    if (warp == 0) {
        if (lane < kk) cand[lane] = acc[0];
        if (32 + lane < kk) cand[32 + lane] = acc[1];
    }

    // ---- the last chunk CTA of this query merges the chunks' lists
    __threadfence();
    __syncthreads();
    if (tid == 0) {
        const int old = atomicAdd(a.counters + t, 1);
        s_last = (old == n_chunks - 1);
    }
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    acc[0] = acc[1] = 0ull;
    for (int ci = warp; ci < n_chunks; ci += kSelWarps) {
        const key64 *src = a.cand + ((size_t)t * kSelMaxChunks + ci) * (kSelMaxK - 1);
        const key64 b[2] = {lane < kk ? __ldcg(src + lane) : 0ull, 32 + lane < kk ? __ldcg(src + 32 + lane) : 0ull};
        if (ci == warp) { acc[0] = b[0]; acc[1] = b[1]; }
        else warp_merge64_desc(acc, b);
    }
    cta_merge_top64<kSelWarps>(acc, s_lists);
    if (warp == 0) {
        // the winners (non-zero keys among the first kk) in ascending block order
        const bool v0 = lane < kk && acc[0] != 0ull, v1 = 32 + lane < kk && acc[1] != 0ull;
        const int km = __popc(__ballot_sync(0xffffffffu, v0)) + __popc(__ballot_sync(0xffffffffu, v1));
        uint32_t ids[2] = {v0 ? key64_id(acc[0]) : 0xffffffffu, v1 ? key64_id(acc[1]) : 0xffffffffu};
        warp_sort64_asc_u32(ids);
        if (lane < km) out[lane] = (int32_t)ids[0];
        if (32 + lane < km) out[32 + lane] = (int32_t)ids[1];
        if (lane == 0) {
            out[km] = own;              // the own block: the largest visible id, last in order
            a.cnt[t] = km + 1;
            a.counters[t] = 0;          // ready for the next call
        }
        for (int i = km + 1 + lane; i < a.k_max; i += 32) out[i] = -1;
    }
}

cudaError_t launch_select_blocks(const SelectArgs &a, cudaStream_t stream) {
    if (a.total_q == 0) return cudaSuccess;
    // the chunk size keeps every query at <= kSelMaxChunks chunks
    const int need = (a.max_blocks + kSelMaxChunks - 1) / kSelMaxChunks;   // blocks per chunk
    const int e = (need + kSelThreads - 1) / kSelThreads;
    auto go = [&](auto kern, int E) {
        const int chunks = (a.max_blocks + kSelThreads * E - 1) / (kSelThreads * E);
        kern<<<dim3(a.total_q, chunks), kSelThreads, 0, stream>>>(a);
    };
    if (e <= 1) go(select_blocks_kernel<1>, 1);
    else if (e <= 2) go(select_blocks_kernel<2>, 2);
    else if (e <= 4) go(select_blocks_kernel<4>, 4);
    else if (e <= 8) go(select_blocks_kernel<8>, 8);
    else if (e <= 16) go(select_blocks_kernel<16>, 16);
    else return cudaErrorInvalidValue;   // the host rejects contexts this long first
    return cudaGetLastError();
}

}  // namespace dsa
