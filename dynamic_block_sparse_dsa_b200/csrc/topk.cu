// topk.cu -- per-query Top-K block selection from a score matrix.
//
// "Day-0 Adaptation for Massive LLMs: Overcoming Sparse Attention and MXFP4
// Expert Weights", section 4(1) "Scalable Top-K": the candidate count grows
// with the context, so no full sort -- an exact partial selection instead.
// "Day-0 Readiness for Trillion-Parameter Models ...", section "Index
// Selection Path": the indices follow the gather's semantics; here they are
// logical block ids, ascending, -1 padded.
//
// One CTA of 256 threads per query (several resident per SM), a radix
// select: the threshold key -- the (K-1)-th largest -- is found digit by
// digit, eight bits at a time from the highest bit where the candidates
// differ, with a shared-memory histogram per digit of the candidates still
// tied with the threshold so far; the search stops as soon as the threshold's
// bucket is taken whole.  Candidates above the threshold are taken, and of
// those equal to it the ones of lowest block id (the total order score
// descending, block id ascending).  A last pass over the candidates in id
// order writes the winners ascending, then the own block.  About 130
// instructions per candidate over all passes (measured at 4096 queries x 2111
// candidates), against about 240 for sorting networks on 64-bit keys.
#include "dsa_kernels.h"

namespace dsa {

namespace {
constexpr int kTopkThreads = 256;
constexpr int kTopkWarps = kTopkThreads / 32;

// larger score -> larger unsigned key
__device__ __forceinline__ uint32_t order_key(int32_t s) { return static_cast<uint32_t>(s) ^ 0x80000000u; }
}  // namespace

__global__ void __launch_bounds__(kTopkThreads) topk_kernel(TopkArgs a) {
    __shared__ uint32_t s_hist[256];
    __shared__ uint32_t s_warp[2][kTopkWarps];
    __shared__ uint32_t s_state[3];   // threshold digit, still needed, bucket taken whole
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
    const int kk = K - 1;      // of which kk are taken
    for (int i = K + tid; i < a.k_max; i += kTopkThreads) out[i] = -1;
    if (tid == 0) {
        out[kk] = n;   // the own block, the largest visible id
        a.cnt[t] = K;
    }
    if (kk == 0) return;
    const int32_t *row = a.scores + (size_t)t * a.max_blocks;

    // ---- the threshold: keys agree on every bit above the highest bit where
    // any two differ, so the digits start there
    uint32_t diff = 0;
    {
        const uint32_t u0 = order_key(__ldg(row));
        for (int i = tid; i < n; i += kTopkThreads) diff |= order_key(__ldg(row + i)) ^ u0;
        diff = __reduce_or_sync(0xffffffffu, diff);
        if (lane == 0) s_warp[0][warp] = diff;
        __syncthreads();
        diff = 0;
#pragma unroll
        for (int w = 0; w < kTopkWarps; ++w) diff |= s_warp[0][w];
    }
    // candidates whose masked key equals prefix are still tied with the
    // threshold; need of them are still to be taken
    uint32_t prefix = 0, mask = 0, need = (uint32_t)kk;
    bool whole = false;
    for (int hi = diff ? 31 - __clz(diff) : -1; hi >= 0;) {
        const int sh = hi >= 7 ? hi - 7 : 0;
        const uint32_t dmask = (2u << (hi - sh)) - 1u;   // the digit: bits sh..hi
        s_hist[tid] = 0u;
        __syncthreads();   // (also: the previous digit's state has been read by all)
        for (int i = tid; i < n; i += kTopkThreads) {
            const uint32_t u = order_key(__ldg(row + i));
            if ((u & mask) == prefix) atomicAdd(&s_hist[(u >> sh) & dmask], 1u);
        }
        __syncthreads();
        if (warp == 0) {
            // bins from the top: lane l holds bins 255 - 8l down to 248 - 8l
            uint32_t c[8], sum = 0;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                c[j] = s_hist[255 - 8 * lane - j];
                sum += c[j];
            }
            uint32_t incl = sum;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += v;
            }
            const uint32_t excl = incl - sum;
            if (excl < need && need <= incl) {   // exactly one lane holds the threshold's bin
                uint32_t above = excl, bin = 0, cb = 0;
                bool found = false;
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    if (!found) {
                        if (above + c[j] >= need) {
                            found = true;
                            bin = (uint32_t)(255 - 8 * lane - j);
                            cb = c[j];
                        } else {
                            above += c[j];
                        }
                    }
                }
                s_state[0] = bin;
                s_state[1] = need - above;
                s_state[2] = cb == need - above ? 1u : 0u;
            }
        }
        __syncthreads();
        prefix |= s_state[0] << sh;
        mask |= dmask << sh;
        need = s_state[1];
        whole = s_state[2] != 0u;
        if (whole) break;
        hi = sh - 1;
    }

    // ---- the winners in id order: each warp takes a contiguous id range,
    // counts, then writes at its offset
    const int per_warp = (n + kTopkThreads - 1) / kTopkThreads * 32;
    const int i_begin = warp * per_warp, i_end = min(n, i_begin + per_warp);
    uint32_t n_above = 0, n_tied = 0;
    for (int i0 = i_begin; i0 < i_end; i0 += 32) {
        const int i = i0 + lane;
        const uint32_t u = i < i_end ? order_key(__ldg(row + i)) & mask : 0u;
        n_above += __popc(__ballot_sync(0xffffffffu, i < i_end && u > prefix));
        n_tied += __popc(__ballot_sync(0xffffffffu, i < i_end && u == prefix));
    }
    if (lane == 0) {
        s_warp[0][warp] = n_above;
        s_warp[1][warp] = n_tied;
    }
    __syncthreads();
    uint32_t at = 0, tied_before = 0;
    for (int w = 0; w < warp; ++w) {
        const uint32_t tw = s_warp[1][w];
        const uint32_t take = whole ? tw : (need > tied_before ? min(tw, need - tied_before) : 0u);
        at += s_warp[0][w] + take;
        tied_before += tw;
    }
    const uint32_t lt = (1u << lane) - 1u;
    for (int i0 = i_begin; i0 < i_end; i0 += 32) {
        const int i = i0 + lane;
        const uint32_t u = i < i_end ? order_key(__ldg(row + i)) & mask : 0u;
        const bool tied = i < i_end && u == prefix;
        const uint32_t mt = __ballot_sync(0xffffffffu, tied);
        const bool take = (i < i_end && u > prefix) || (tied && (whole || tied_before + __popc(mt & lt) < need));
        const uint32_t ms = __ballot_sync(0xffffffffu, take);
        if (take) out[at + __popc(ms & lt)] = i;
        at += __popc(ms);
        tied_before += __popc(mt);
    }
}

int topk_max_blocks() { return 1 << 20; }

cudaError_t launch_topk(const TopkArgs &a, cudaStream_t stream) {
    if (a.total_q == 0) return cudaSuccess;
    if (a.k_max > 64) return cudaErrorInvalidValue;   // the host rejects these first
    return launch_pdl(topk_kernel, dim3(a.total_q), dim3(kTopkThreads), 0, stream, a);
}

}  // namespace dsa
