// index_score.cu -- block scores of the lightweight int8 indexer.
//
// "Day-0 Adaptation for Massive LLMs: Overcoming Sparse Attention and MXFP4
// Expert Weights", section 4(1): score the compressed per-block representation
// against each query in one fused kernel, writing no intermediate to memory;
// "Day-0 Readiness for Trillion-Parameter Models ...", section "Index
// Selection Path": low-precision scoring inputs.  The score is
//     S[t][b] = sum_h w[t][h] * max(0, q_idx[t][h] . kc[page(s,b)])
// in exact int32 (the host checks the range bound).
//
// CUDA-core path (decode; any sequence with few queries): the scan over a
// sequence's coarse keys is HBM-bound, 64 bytes per block.  One thread owns one
// block: it reads the page id and the 64-byte key with four 16-byte loads,
// keeps the key in 16 registers and runs 16 dp4a per indexer head against the
// query rows, which every thread of the CTA reads from shared memory as
// broadcasts.  Queries of the sequence are taken in batches of kQBatch.
#include "dsa_kernels.h"
#include "indexer_core.cuh"

namespace dsa {

namespace {
constexpr int kScoreThreads = 256;   // blocks scored per CTA
constexpr int kQBatch = 8;           // queries staged in shared memory at once
}  // namespace

__global__ void __launch_bounds__(kScoreThreads) index_score_dp4a_kernel(IndexScoreArgs a) {
    __shared__ int4 s_q[kQBatch][kMaxIdxHeads][kIdxDim / 16];
    __shared__ int s_w[kQBatch][kMaxIdxHeads];
    __shared__ int s_own[kQBatch];

    pdl_trigger();
    pdl_wait();   // coarse keys may come from the preceding append
    const int s = blockIdx.y;
    const int q0 = __ldg(a.cu_q + s), q1 = __ldg(a.cu_q + s + 1);
    if (q1 <= q0) return;
    if (q0 < 0 || q1 > a.total_q) {          // offsets outside the query arrays
        if (blockIdx.x == 0 && threadIdx.x == 0) set_err(a.dev_err, DSA_DEV_ERR_POS);
        return;
    }
    const int len = __ldg(a.seq_lens + s);
    const int b = blockIdx.x * kScoreThreads + threadIdx.x;
    const int H = a.num_idx_heads;

    // the coarse key of this thread's block (if it can be visible to anyone)
    const int n_blocks = (len + (1 << a.block_shift) - 1) >> a.block_shift;
    bool have = false;
    int kc[16];
    if (blockIdx.x * kScoreThreads >= n_blocks) return;   // the whole chunk is past the end
    if (b < n_blocks && b < a.max_blocks) {
        const int page = __ldg(a.block_table + (size_t)s * a.max_blocks + b);
        if (page >= 0 && page < a.num_pages) {
            load_coarse_key(a.kc_pool, page, kc);
            have = true;
        } else {
            set_err(a.dev_err, DSA_DEV_ERR_PAGE);
        }
    }

    for (int qb = q0; qb < q1; qb += kQBatch) {
        const int nq = min(kQBatch, q1 - qb);
        __syncthreads();
        // stage the batch's query rows, weights and own-block indices
        for (int e = threadIdx.x; e < nq * H * (kIdxDim / 16); e += kScoreThreads) {
            const int qi = e / (H * 4), rest = e % (H * 4);
            s_q[qi][rest / 4][rest % 4] =
                __ldg(reinterpret_cast<const int4 *>(a.q_idx + ((size_t)(qb + qi) * H) * kIdxDim) + rest);
        }
        for (int e = threadIdx.x; e < nq * H; e += kScoreThreads)
            s_w[e / H][e % H] = __ldg(a.w + (size_t)(qb + e / H) * H + e % H);
        if (threadIdx.x < nq) {
            const int p = __ldg(a.q_pos + qb + threadIdx.x);
            int own = p >> a.block_shift;
            if (p < 0 || p >= len || own >= a.max_blocks) {
                if (blockIdx.x == 0) set_err(a.dev_err, DSA_DEV_ERR_POS);
                own = -1;
            }
            s_own[threadIdx.x] = own;
        }
        __syncthreads();
        if (!have) continue;
        for (int qi = 0; qi < nq; ++qi) {
            if (b > s_own[qi]) continue;
            const int total = block_score(kc, s_q[qi], s_w[qi], H);
            a.scores[(size_t)(qb + qi) * a.max_blocks + b] = total;
        }
    }
}

cudaError_t launch_index_score(const IndexScoreArgs &a, cudaStream_t stream) {
    if (a.total_q == 0 || a.num_seqs == 0) return cudaSuccess;
    dim3 grid((a.max_blocks + kScoreThreads - 1) / kScoreThreads, a.num_seqs);
    return launch_pdl(index_score_dp4a_kernel, grid, dim3(kScoreThreads), 0, stream, a);
}

}  // namespace dsa
