// topk_wide.cu -- per-query Top-K block selection from int64 scores (the
// wide and FP8 indexers of index_score_wide.cu).
//
// "Day-0 Adaptation for Massive LLMs: Overcoming Sparse Attention and MXFP4
// Expert Weights", section 4(1) "Scalable Top-K": an exact partial selection,
// no full sort.  The order is the one of dsa_topk_blocks -- the own block
// forced, then score descending, block id ascending -- over int64 scores.
//
// A candidate is a wide key (the score mapped to an unsigned order, ~block
// id): larger wins, so the total order is a lexicographic unsigned compare
// and no two keys tie.  One CTA of 512 threads per query: each warp sorts its
// first group of 64 candidates with a bitonic network and folds later groups
// into its running Top-64 (groups with no key above the current (K-1)-th are
// skipped after one vote); a merge tree over the 16 warps leaves the query's
// Top-64 in warp 0, which appends the own block and writes the winners in
// ascending block order.
#include "dsa_kernels.h"
#include "warp_topk.cuh"

namespace dsa {

namespace {
constexpr int kWtThreads = 512;
constexpr int kWtWarps = kWtThreads / 32;

struct WKey {
    unsigned long long ord;   // score ^ 2^63: larger scores give larger values, never 0 for a real score
    uint32_t inv;             // ~block id: the lower block wins a tie
};
__device__ __forceinline__ bool wk_gt(const WKey &x, const WKey &y) {
    return x.ord > y.ord || (x.ord == y.ord && x.inv > y.inv);
}
__device__ __forceinline__ WKey wk_xor(const WKey &v, int j) {
    return WKey{__shfl_xor_sync(0xffffffffu, v.ord, j), __shfl_xor_sync(0xffffffffu, v.inv, j)};
}
__device__ __forceinline__ WKey wk_from(const WKey &v, int src) {
    return WKey{__shfl_sync(0xffffffffu, v.ord, src), __shfl_sync(0xffffffffu, v.inv, src)};
}
__device__ __forceinline__ WKey wk_make(long long score, uint32_t id) {
    return WKey{(unsigned long long)score ^ 0x8000000000000000ull, ~id};
}
constexpr WKey kNone{0ull, 0u};

__device__ __forceinline__ void wk_cx(WKey &v, int j, bool keep_max) {
    const WKey w = wk_xor(v, j);
    const bool g = wk_gt(v, w);
    v = (keep_max == g) ? v : w;
}

// 64 keys held two per lane (element i in lane i % 32, register i / 32), sorted descending
__device__ __forceinline__ void wk_sort64_desc(WKey (&v)[2]) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int k = 2; k <= 64; k <<= 1) {
#pragma unroll
        for (int j = k >> 1; j > 0; j >>= 1) {
            if (j == 32) {
                if (wk_gt(v[1], v[0])) { const WKey t = v[0]; v[0] = v[1]; v[1] = t; }
            } else {
#pragma unroll
                for (int r = 0; r < 2; ++r) {
                    const int i = r * 32 + lane;
                    wk_cx(v[r], j, ((lane & j) == 0) == ((i & k) == 0));
                }
            }
        }
    }
}

// a bitonic sequence of 64 keys, sorted descending
__device__ __forceinline__ void wk_bitonic_merge64_desc(WKey (&v)[2]) {
    const int lane = threadIdx.x & 31;
    if (wk_gt(v[1], v[0])) { const WKey t = v[0]; v[0] = v[1]; v[1] = t; }
#pragma unroll
    for (int j = 16; j > 0; j >>= 1) {
        const bool lower = (lane & j) == 0;
        wk_cx(v[0], j, lower);
        wk_cx(v[1], j, lower);
    }
}

// a <- Top-64 of (a, b), both sorted descending
__device__ __forceinline__ void wk_merge64_desc(WKey (&a)[2], const WKey (&b)[2]) {
    const int lane = threadIdx.x & 31;
    const WKey r0 = wk_from(b[1], 31 - lane), r1 = wk_from(b[0], 31 - lane);
    a[0] = wk_gt(a[0], r0) ? a[0] : r0;
    a[1] = wk_gt(a[1], r1) ? a[1] : r1;
    wk_bitonic_merge64_desc(a);
}
}  // namespace

__global__ void __launch_bounds__(kWtThreads) topk_wide_kernel(TopkArgs a, const int64_t *scores) {
    __shared__ WKey s_lists[kWtWarps * 64];
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
        for (int i = tid; i < a.k_max; i += kWtThreads) out[i] = -1;
        return;
    }
    if (n_vis <= K) {
        for (int i = tid; i < a.k_max; i += kWtThreads) out[i] = i < n_vis ? i : -1;
        if (tid == 0) a.cnt[t] = n_vis;
        return;
    }
    const int n = n_vis - 1;   // candidates 0..n-1 (n >= K)
    const int kk = K - 1;
    const int64_t *row = scores + (size_t)t * a.max_blocks;
    WKey acc[2] = {kNone, kNone};
    bool first = true;
    for (int g0 = warp * 64; g0 < n; g0 += kWtWarps * 64) {
        const int i0 = g0 + lane, i1 = g0 + 32 + lane;
        WKey v[2] = {i0 < n ? wk_make(__ldg(reinterpret_cast<const long long *>(row) + i0), (uint32_t)i0) : kNone,
                     i1 < n ? wk_make(__ldg(reinterpret_cast<const long long *>(row) + i1), (uint32_t)i1) : kNone};
        if (!first) {
            // keys not above the current kk-th largest cannot reach the first kk
            const WKey thr = wk_from(kk <= 32 ? acc[0] : acc[1], (kk - 1) & 31);
            const bool p0 = wk_gt(v[0], thr), p1 = wk_gt(v[1], thr);
            if (!__any_sync(0xffffffffu, p0 || p1)) continue;
            if (!p0) v[0] = kNone;
            if (!p1) v[1] = kNone;
        }
        wk_sort64_desc(v);
        if (first) {
            acc[0] = v[0];
            acc[1] = v[1];
            first = false;
        } else {
            wk_merge64_desc(acc, v);
        }
    }
    // merge tree over the warps
#pragma unroll
    for (int step = 1; step < kWtWarps; step <<= 1) {
        if ((warp & (2 * step - 1)) == step) {
            s_lists[warp * 64 + lane] = acc[0];
            s_lists[warp * 64 + 32 + lane] = acc[1];
        }
        __syncthreads();
        if ((warp & (2 * step - 1)) == 0 && warp + step < kWtWarps) {
            const WKey b[2] = {s_lists[(warp + step) * 64 + lane], s_lists[(warp + step) * 64 + 32 + lane]};
            wk_merge64_desc(acc, b);
        }
        __syncthreads();
    }
    if (warp == 0) {
        const bool v0 = lane < kk, v1 = 32 + lane < kk;
        uint32_t ids[2] = {v0 ? ~acc[0].inv : 0xffffffffu, v1 ? ~acc[1].inv : 0xffffffffu};
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

cudaError_t launch_topk_wide(const TopkArgs &a, const int64_t *scores, cudaStream_t stream) {
    if (a.total_q == 0) return cudaSuccess;
    if (a.k_max > 64) return cudaErrorInvalidValue;   // the host rejects these first
    return launch_pdl(topk_wide_kernel, dim3(a.total_q), dim3(kWtThreads), 0, stream, a, scores);
}

}  // namespace dsa
