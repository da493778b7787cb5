// topk.cu -- per-query Top-K block selection.
//
// "Day-0 Adaptation for Massive LLMs: Overcoming Sparse Attention and MXFP4
// Expert Weights", section 4(1) "Scalable Top-K": the candidate count grows
// with the context, so no full sort -- a block-wise reduction and partial
// selection instead.  "Day-0 Readiness for Trillion-Parameter Models ...",
// section "Index Selection Path": the indices must follow the gather's
// semantics; here they are logical block ids, ascending, -1 padded.
//
// One CTA per query.  The K-1 winners among blocks 0..n-2 (the own block n-1
// is always kept) are found by an MSB-first radix select on the order-
// preserving unsigned image of the int32 score: four 8-bit passes, each a
// shared-memory histogram (warp-aggregated with match.any) followed by a
// one-warp search for the digit that holds the (K-1)-th largest key.  That
// yields the exact threshold key T and how many keys equal to T still fit.
// Ties at T go to the lowest block ids: a block-wide scan over contiguous
// per-thread ranges counts the T-keys before each thread, and a second scan
// places the winners, so the output comes out in ascending block order
// without any sort.
#include "dsa_kernels.h"

namespace dsa {

namespace {
constexpr int kTopkThreads = 1024;
constexpr int kWarps = kTopkThreads / 32;

__device__ __forceinline__ uint32_t order_key(int32_t v) { return static_cast<uint32_t>(v) ^ 0x80000000u; }

// exclusive prefix sum of v over the CTA; *total receives the sum of all v
__device__ __forceinline__ int block_exclusive_scan(int v, int *s_warp, int *total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) s_warp[warp] = x;
    __syncthreads();
    if (warp == 0) {
        int w = lane < kWarps ? s_warp[lane] : 0;
        int incl = w;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        if (lane < kWarps) s_warp[lane] = incl - w;   // exclusive warp offsets
        if (lane == 31) s_warp[kWarps] = incl;        // grand total
    }
    __syncthreads();
    const int res = s_warp[warp] + x - v;
    *total = s_warp[kWarps];
    __syncthreads();   // s_warp may be reused by the caller
    return res;
}
}  // namespace

__global__ void __launch_bounds__(kTopkThreads) topk_kernel(TopkArgs a) {
    __shared__ uint32_t s_hist[256];
    __shared__ uint32_t s_digit, s_rem;
    __shared__ int s_warp[kWarps + 1];

    const int t = blockIdx.x;
    const int tid = threadIdx.x, lane = tid & 31;
    int32_t *out = a.sel + (size_t)t * a.k_max;
    const int s = find_seq(a.cu_q, a.num_seqs, t);
    const int p = __ldg(a.q_pos + t);
    const int len = __ldg(a.seq_lens + s);
    const int K = __ldg(a.k_per_seq + s);
    const int n_vis = p / kBlockSize + 1;

    if (p < 0 || p >= len || n_vis > a.max_blocks || K < 1 || K > a.k_max) {
        if (tid == 0) {
            set_err(a.dev_err, (K < 1 || K > a.k_max) ? DSA_DEV_ERR_K : DSA_DEV_ERR_POS);
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

    const int n = n_vis - 1;          // candidates: blocks 0..n-1 (n >= K)
    const int kk = K - 1;             // winners among them
    const int32_t *row = a.scores + (size_t)t * a.max_blocks;

    uint32_t prefix = 0, mask = 0, remaining = kk;
    if (kk > 0) {
        for (int pass = 0; pass < 4; ++pass) {
            const int shift = 24 - 8 * pass;
            for (int i = tid; i < 256; i += kTopkThreads) s_hist[i] = 0;
            __syncthreads();
            for (int base = tid & ~31; base < n; base += kTopkThreads) {
                const int i = base + lane;
                bool valid = false;
                uint32_t d = 256u + lane;       // distinct per lane when not counted
                if (i < n) {
                    const uint32_t u = order_key(row[i]);
                    if ((u & mask) == prefix) {
                        valid = true;
                        d = (u >> shift) & 255u;
                    }
                }
                const uint32_t peers = __match_any_sync(0xffffffffu, d);
                if (valid && lane == __ffs(peers) - 1) atomicAdd(&s_hist[d], __popc(peers));
            }
            __syncthreads();
            if (tid < 32) {
                // lane l owns digits 8l..8l+7; count of keys in higher lanes' digits
                uint32_t c[8], sum = 0;
#pragma unroll
                for (int j = 0; j < 8; ++j) { c[j] = s_hist[8 * lane + j]; sum += c[j]; }
                uint32_t above = 0, x = sum;   // inclusive suffix sum over lanes >= l
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    uint32_t y = __shfl_down_sync(0xffffffffu, x, o);
                    if (lane + o < 32) x += y;
                }
                above = x - sum;               // keys with digit in lanes > l
                if (above < remaining && remaining <= above + sum) {
                    uint32_t acc = above;
                    for (int j = 7; j >= 0; --j) {
                        if (acc + c[j] >= remaining) {
                            s_digit = 8 * lane + j;
                            s_rem = remaining - acc;
                            break;
                        }
                        acc += c[j];
                    }
                }
            }
            __syncthreads();
            prefix |= s_digit << shift;
            mask |= 255u << shift;
            remaining = s_rem;
            __syncthreads();
        }
    }

    // kk winners: every key > T, plus the first `remaining` keys == T by block id
    const uint32_t T = prefix;
    const int per = (n + kTopkThreads - 1) / kTopkThreads;
    const int lo = min(n, tid * per), hi = min(n, lo + per);
    int n_eq = 0, n_gt = 0;
    if (kk > 0)
        for (int i = lo; i < hi; ++i) {
            const uint32_t u = order_key(row[i]);
            n_eq += (u == T);
            n_gt += (u > T);
        }
    int tot;
    const int eq_before = block_exclusive_scan(n_eq, s_warp, &tot);
    const int take_eq = kk > 0 ? max(0, min(n_eq, (int)remaining - eq_before)) : 0;
    const int out_before = block_exclusive_scan(n_gt + take_eq, s_warp, &tot);
    if (kk > 0) {
        int o = out_before, eq_seen = 0;
        for (int i = lo; i < hi; ++i) {
            const uint32_t u = order_key(row[i]);
            if (u > T) {
                out[o++] = i;
            } else if (u == T) {
                if (eq_seen < take_eq) out[o++] = i;
                ++eq_seen;
            }
        }
    }
    if (tid == 0) {
        out[kk] = n;                    // the own block, the largest visible id
        a.cnt[t] = K;
    }
    for (int i = K + tid; i < a.k_max; i += kTopkThreads) out[i] = -1;
}

cudaError_t launch_topk(const TopkArgs &a, cudaStream_t stream) {
    if (a.total_q == 0) return cudaSuccess;
    topk_kernel<<<a.total_q, kTopkThreads, 0, stream>>>(a);
    return cudaGetLastError();
}

}  // namespace dsa
