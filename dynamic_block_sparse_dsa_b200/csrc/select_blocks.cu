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
// (exact radix select on register-resident keys) and writes it to the
// workspace.  The last CTA of the query -- elected with an atomic counter,
// nothing waits -- merges the chunks' candidates with the same selection,
// appends the query's own block and writes the ascending selection.  Result
// is identical to dsa_index_score followed by dsa_topk_blocks.
#include "dsa_kernels.h"
#include "indexer_core.cuh"
#include "select_core.cuh"

namespace dsa {

namespace {
constexpr int kSelThreads = 256;
constexpr int kMergeE = kSelMaxChunks * (kSelMaxK - 1) / kSelThreads + 1;   // candidates per thread
}  // namespace

template <int E>
__global__ void __launch_bounds__(kSelThreads) select_blocks_kernel(SelectArgs a) {
    __shared__ SelectSmem sh;
    __shared__ int4 s_q[kMaxIdxHeads][kIdxDim / 16];
    __shared__ int s_w[kMaxIdxHeads];
    __shared__ int s_last;
    constexpr int CH = kSelThreads * E;
    const int t = blockIdx.x, c = blockIdx.y, tid = threadIdx.x;
    const int H = a.num_idx_heads;

    const int s = find_seq(a.cu_q, a.num_seqs, t);
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

    // ---- score this chunk (E consecutive blocks per thread)
    for (int e = tid; e < H * 4; e += kSelThreads)
        s_q[e >> 2][e & 3] = __ldg(reinterpret_cast<const int4 *>(a.q_idx + (size_t)t * H * kIdxDim) + e);
    if (tid < H) s_w[tid] = __ldg(a.w + (size_t)t * H + tid);
    __syncthreads();
    uint32_t key[E];
    bool valid[E];
    uint32_t err_bits = 0;
    const int b0 = c * CH + tid * E;
#pragma unroll
    for (int e = 0; e < E; ++e) {
        const int b = b0 + e;
        valid[e] = false;
        key[e] = 0;
        if (b < own) {
            const int page = __ldg(a.block_table + (size_t)s * a.max_blocks + b);
            if (page >= 0 && page < a.num_pages) {
                int kc[16];
                load_coarse_key(a.kc_pool, page, kc);
                key[e] = order_key(block_score(kc, s_q, s_w, H));
                valid[e] = true;
            } else {
                err_bits |= DSA_DEV_ERR_PAGE;
            }
        }
    }
    if (err_bits) set_err(a.dev_err, err_bits);

    // ---- local Top-kk of the chunk, written in id order
    int nv = 0;
#pragma unroll
    for (int e = 0; e < E; ++e) nv += valid[e];
    int n_valid;
    cta_exclusive_scan<kSelThreads>(nv, sh, &n_valid);
    const int kl = min(kk, n_valid);
    bool take[E];
    if (kl == n_valid) {
#pragma unroll
        for (int e = 0; e < E; ++e) take[e] = valid[e];
    } else {
        cta_select<kSelThreads, E>(key, valid, kl, take, sh);
    }
    int nt = 0;
#pragma unroll
    for (int e = 0; e < E; ++e) nt += take[e];
    int tot;
    int pos = cta_exclusive_scan<kSelThreads>(nt, sh, &tot);
    uint2 *cand = a.cand + ((size_t)t * kSelMaxChunks + c) * (kSelMaxK - 1);
#pragma unroll
    for (int e = 0; e < E; ++e)
        if (take[e]) cand[pos++] = make_uint2(key[e], (uint32_t)(b0 + e));
    for (int i = kl + tid; i < kk; i += kSelThreads) cand[i] = make_uint2(0u, 0xffffffffu);   // padding

    // ---- the last chunk CTA of this query merges
    __threadfence();
    __syncthreads();
    if (tid == 0) {
        const int old = atomicAdd(a.counters + t, 1);
        s_last = (old == n_chunks - 1);
    }
    __syncthreads();
    if (!s_last) return;
    __threadfence();

    const int n_cand = n_chunks * kk;
    uint32_t mk[kMergeE];
    uint32_t mid[kMergeE];
    bool mv[kMergeE];
#pragma unroll
    for (int e = 0; e < kMergeE; ++e) {
        const int i = tid * kMergeE + e;
        mv[e] = false;
        mk[e] = 0;
        mid[e] = 0;
        if (i < n_cand) {
            const int ci = i / kk, j = i - ci * kk;
            const uint2 v = __ldcg(a.cand + ((size_t)t * kSelMaxChunks + ci) * (kSelMaxK - 1) + j);
            mk[e] = v.x;
            mid[e] = v.y;
            mv[e] = v.y != 0xffffffffu;
        }
    }
    nv = 0;
#pragma unroll
    for (int e = 0; e < kMergeE; ++e) nv += mv[e];
    cta_exclusive_scan<kSelThreads>(nv, sh, &n_valid);
    const int km = min(kk, n_valid);
    bool mt[kMergeE];
    if (km == n_valid) {
#pragma unroll
        for (int e = 0; e < kMergeE; ++e) mt[e] = mv[e];
    } else {
        cta_select<kSelThreads, kMergeE>(mk, mv, km, mt, sh);
    }
    nt = 0;
#pragma unroll
    for (int e = 0; e < kMergeE; ++e) nt += mt[e];
    pos = cta_exclusive_scan<kSelThreads>(nt, sh, &tot);
#pragma unroll
    for (int e = 0; e < kMergeE; ++e)
        if (mt[e]) out[pos++] = (int32_t)mid[e];
    if (tid == 0) {
        out[km] = own;              // the own block: the largest visible id, last in order
        a.cnt[t] = km + 1;
        a.counters[t] = 0;          // ready for the next call
    }
    for (int i = km + 1 + tid; i < a.k_max; i += kSelThreads) out[i] = -1;
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
