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
// Grid: (query, chunk of 512*G candidate blocks).  Each CTA scores its chunk
// with the int8 indexer on the tensor cores (mma.m16n8k32 s8, coarse keys as
// the M operand loaded straight into fragments, 64 blocks per warp step, the
// warps' groups interleaved; a CUDA-core dp4a version measured ALU-bound at
// the 1M-token decode shape) into unique 64-bit keys, and finds the chunk's
// Top-(K-1): warp bitonic Top-64 lists and a merge tree for decode chunks, a
// CTA-wide radix select over the keys in registers (radix_select.cuh) for the
// larger chunks of many-query batches.  It writes them to the workspace; the
// last CTA of the query -- elected with an atomic counter, nothing waits --
// selects over the chunks' lists, appends the query's own block and writes
// the ascending selection.  Result is identical to dsa_index_score followed
// by dsa_topk_blocks.
#include "dsa_kernels.h"
#include "dsa_tma.cuh"
#include "indexer_core.cuh"
#include "kv_append.cuh"
#include "radix_select.cuh"
#include "warp_topk.cuh"

namespace dsa {

namespace {
constexpr int kSelThreads = 256;
constexpr int kSelWarps = kSelThreads / 32;
constexpr int kCuqCache = 1024;   // cu_q entries staged in shared memory
constexpr long long kSelBusyCtas = 8 * 148;   // a grid this large keeps every SM of a B200 busy
// How a CTA finds its Top-(K-1).  With few candidates per thread (decode
// chunks of 512 blocks, G = 1) each warp sorts its 64 candidates with a
// bitonic network and a merge tree combines the warps; with more (G >= 2, the
// many-query prefill shapes) the candidates stay in registers and one CTA-wide
// radix select finds the winners.  The last CTA of a split query selects over
// the chunks' lists by radix select when kFinalRadix (or when the chunks used
// it: their lists are unordered), else by a merge tree of the sorted lists.
// Measured back to back on one B200, the radix select everywhere against this
// split: decode_1m step 29.13 / 28.96 us, decode_128k select 10.30 / 8.97 us,
// batched GQA select 11.09 / 9.30 us, chunked prefill select 189.9 / 189.7 us.
constexpr int kRadixMinGroups = 2;
constexpr bool kFinalRadix = false;
}  // namespace

// 64-block groups per warp: a chunk is kSelWarps * 64 * G blocks.  Chunks of
// G >= 2 (many-query batches) run three CTAs per SM: measured faster than two
// despite a few spilled registers (chunked prefill 189 -> 169 us), and than
// keeping the keys in shared memory instead (198 us).
template <int G>
__global__ void __launch_bounds__(kSelThreads, G >= 2 ? 3 : 2) select_blocks_kernel(SelectArgs a) {
    __shared__ int4 s_q[kMaxIdxHeads][kIdxDim / 16];
    __shared__ int s_w[kMaxIdxHeads];
    __shared__ int s_cuq[kCuqCache + 1];
    __shared__ RadixScratch s_rx;
    __shared__ key64 s_lists[kSelWarps * 64];
    __shared__ uint32_t s_ids[kSelMaxK];
    __shared__ int s_last, s_nsel[2];
    constexpr int CH = kSelWarps * 64 * G;
    constexpr bool kChunkRadix = G >= kRadixMinGroups;
    constexpr bool kMergeRadix = kFinalRadix || kChunkRadix;
    const int t = blockIdx.x, c = blockIdx.y, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g = lane >> 2, cq = lane & 3;
    const int H = a.num_idx_heads;

    pdl_trigger();
    if ((int)blockIdx.y >= a.sel_rows) {
        // an append CTA: one new token per CTA, overlapping the selection (which
        // never reads the rows written here -- see SelectArgs::cu_new)
        const int i = t + ((int)blockIdx.y - a.sel_rows) * (int)gridDim.x;
        if (i < a.app.total_new) append_token(a.app, i, tid, kSelThreads);
        return;
    }
    // ---- query facts.  The position and cu_q travel together; then, once the
    // sequence is known, its length, Top-K and the first group's page ids
    // travel together: two round trips before the coarse keys
    const int p = __ldg(a.q_pos + t);
    // a decode batch has one query per sequence (query t in sequence t): the
    // sequence's facts and first page ids are loaded with the position on that
    // guess, and reloaded below only if cu_q says otherwise
    const bool guess = t < a.num_seqs;
    int len = 0, K = 0, pg0[4][2];
    auto load_seq_facts = [&](int sq) {
        len = __ldg(a.seq_lens + sq);
        K = __ldg(a.k_per_seq + sq);
        // page ids of this warp's first group, before the facts are checked
        // (rows end at max_blocks; ids past the own block are never used)
        const int32_t *row = a.block_table + (size_t)sq * a.max_blocks;
        const int base = c * CH + warp * 64;
#pragma unroll
        for (int mt = 0; mt < 4; ++mt)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int b = base + 16 * mt + g + 8 * h;
                pg0[mt][h] = b < a.max_blocks ? __ldg(row + b) : -1;
            }
    };
    if (guess) load_seq_facts(t);
    const bool cached = a.num_seqs + 1 <= kCuqCache;
    if (cached)
        for (int i = tid; i <= a.num_seqs; i += kSelThreads) s_cuq[i] = __ldg(a.cu_q + i);
    for (int e = tid; e < kMaxIdxHeads * 4; e += kSelThreads)   // heads past H read as zero
        s_q[e >> 2][e & 3] = (e >> 2) < H
            ? __ldg(reinterpret_cast<const int4 *>(a.q_idx + (size_t)t * H * kIdxDim) + e) : make_int4(0, 0, 0, 0);
    if (tid < kMaxIdxHeads) s_w[tid] = tid < H ? __ldg(a.w + (size_t)t * H + tid) : 0;
    if (tid < 2) s_nsel[tid] = 0;
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
    if (!guess || s != t) load_seq_facts(s);
    const int n_vis = (p >> a.block_shift) + 1;
    const int32_t *table = a.block_table + (size_t)s * a.max_blocks;
    int32_t *out = a.sel + (size_t)t * a.k_max;
    bool bad_pos = p < 0 || p >= len || n_vis > a.max_blocks;
    if (a.cu_new && !bad_pos) {
        // an append follows and overlaps this kernel: no candidate block may be appended to
        const int n_new = __ldg(a.cu_new + s + 1) - __ldg(a.cu_new + s);
        if (n_new > len || (n_new > 0 && n_vis - 1 > ((len - n_new) >> a.block_shift))) bad_pos = true;
    }
    const bool bad_k = K < 1 || K > a.k_max;
    if (bad_pos || bad_k) {
        pdl_wait();
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
        pdl_wait();
        if (c == 0) {
            const int n = n_vis <= K ? n_vis : 1;
            for (int i = tid; i < a.k_max; i += kSelThreads) out[i] = i < n ? (n == 1 ? own : i) : -1;
            if (tid == 0) a.cnt[t] = n;
        }
        return;
    }
    const int n_chunks = (own + CH - 1) / CH;   // candidates: blocks 0 .. own-1
    if (c >= n_chunks) return;

    // ---- score this chunk on the int8 tensor cores, 64 blocks per warp step
    int qb[2][2][2], wl[2][2];
    {
        const int *qi = reinterpret_cast<const int *>(s_q);
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
            for (int ks = 0; ks < 2; ++ks) {
                qb[nt][ks][0] = qi[(8 * nt + g) * 16 + 8 * ks + cq];
                qb[nt][ks][1] = qi[(8 * nt + g) * 16 + 8 * ks + 4 + cq];
            }
            wl[nt][0] = s_w[8 * nt + 2 * cq];
            wl[nt][1] = s_w[8 * nt + 2 * cq + 1];
        }
    }
    // radix select: this thread's candidates (per group, blocks 16cq+g and
    // 16cq+g+8 of it); sort: the warp's running Top-64
    key64 keys[kChunkRadix ? 2 * G : 1];
    key64 acc[2] = {0ull, 0ull};
    uint32_t err_bits = 0;
#pragma unroll
    for (int gi = 0; gi < G; ++gi) {
        const int base = c * CH + (gi * kSelWarps + warp) * 64;
        key64 v[2] = {0ull, 0ull};
        if (base < own) {
            // all of the group's page ids, then all of its coarse-key fragments,
            // in flight before the first tensor-core op
            int pg[4][2];
#pragma unroll
            for (int mt = 0; mt < 4; ++mt)
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int b = base + 16 * mt + g + 8 * h;
                    int page = b < own ? (gi == 0 ? pg0[mt][h] : __ldg(table + b)) : -1;
                    if (b < own && (page < 0 || page >= a.num_pages)) { err_bits |= DSA_DEV_ERR_PAGE; page = -1; }
                    pg[mt][h] = page;
                }
            if (gi == 0) pdl_wait();   // coarse keys may come from the preceding append
            Tile16 f[4];
#pragma unroll
            for (int mt = 0; mt < 4; ++mt) tile16_load(a.kc_pool, pg[mt][0], pg[mt][1], f[mt]);
#pragma unroll
            for (int mt = 0; mt < 4; ++mt) {
                int s_g, s_g8;
                tile16_scores(f[mt], qb, wl, s_g, s_g8);
                if (mt == cq) {   // lane (g, cq) keeps blocks 16*cq + g and 16*cq + g + 8
                    const int b = base + 16 * mt + g;
                    v[0] = pg[mt][0] >= 0 ? make_key64(s_g, (uint32_t)b) : 0ull;
                    v[1] = pg[mt][1] >= 0 ? make_key64(s_g8, (uint32_t)(b + 8)) : 0ull;
                }
            }
        } else if (gi == 0) {
            pdl_wait();
        }
        if constexpr (kChunkRadix) {
            keys[2 * gi] = v[0];
            keys[2 * gi + 1] = v[1];
        } else if (gi == 0) {   // the first group: sorted, it is the warp's list (nothing to merge with)
            warp_sort64_desc(v);
            acc[0] = v[0];
            acc[1] = v[1];
        } else {
            warp_fold_topk(acc, v, kk);
        }
    }
    if (err_bits) set_err(a.dev_err, err_bits);

    // ---- the chunk's Top-(K-1) (the query's, when it has one chunk)
    key64 prefix = 0ull, mask = 0ull;
    int n_real = 0;
    if constexpr (kChunkRadix) {
        n_real = cta_radix_threshold<kSelThreads, 2 * G>(keys, (uint32_t)kk, s_rx, prefix, mask);
    } else {
        cta_merge_top64<kSelWarps>(acc, s_lists);   // sorted, in warp 0
    }
    bool from_ids = kChunkRadix;   // the winners' ids are in s_ids (else sorted in warp 0's acc)
    if (n_chunks > 1) {
        key64 *cand = a.cand + ((size_t)t * kSelMaxChunks + c) * (kSelMaxK - 1);
        if constexpr (kChunkRadix) {
            // in any order; slots past the chunk's winners are zeroed
            const int n_win = min(n_real, kk);
#pragma unroll
            for (int i = 0; i < 2 * G; ++i)
                if (keys[i] != 0ull && (keys[i] & mask) >= prefix) cand[atomicAdd(&s_nsel[0], 1)] = keys[i];
            for (int i = n_win + tid; i < kk; i += kSelThreads) cand[i] = 0ull;
        } else if (warp == 0) {   // sorted (zeros past the chunk's candidates)
            if (lane < kk) cand[lane] = acc[0];
            if (32 + lane < kk) cand[32 + lane] = acc[1];
        }
        // ---- the last chunk CTA of this query selects over the chunks'
        // lists: the barrier orders every list store before tid 0's
        // release-add, and the last adder's acquire (then the barrier) orders
        // every list before the loads below
        __syncthreads();
        if (tid == 0) {
            const int old = atomic_add_acq_rel_gpu(a.counters + t, 1);
            s_last = (old == n_chunks - 1);
        }
        __syncthreads();
        if (!s_last) return;
        if constexpr (kMergeRadix) {
            constexpr int kLoad = (kSelMaxChunks * (kSelMaxK - 1) + kSelThreads - 1) / kSelThreads;
            key64 lk[kLoad];
            const int n_slots = n_chunks * kk;
#pragma unroll
            for (int j = 0; j < kLoad; ++j) {   // every load in flight before the selection
                const int e = tid + j * kSelThreads;
                const int ci = e / kk, ei = e - ci * kk;
                lk[j] = e < n_slots ? __ldcg(a.cand + ((size_t)t * kSelMaxChunks + ci) * (kSelMaxK - 1) + ei)
                                    : 0ull;
            }
            cta_radix_threshold<kSelThreads, kLoad>(lk, (uint32_t)kk, s_rx, prefix, mask);
#pragma unroll
            for (int j = 0; j < kLoad; ++j)
                if (lk[j] != 0ull && (lk[j] & mask) >= prefix) s_ids[atomicAdd(&s_nsel[1], 1)] = key64_id(lk[j]);
            __syncthreads();
            from_ids = true;
        } else {
            constexpr int kPer = (kSelMaxChunks + kSelWarps - 1) / kSelWarps;   // lists per warp
            key64 lists[kPer][2];
#pragma unroll
            for (int k = 0; k < kPer; ++k) {   // every load in flight before the first merge
                const int ci = warp + k * kSelWarps;
                const key64 *src = a.cand + ((size_t)t * kSelMaxChunks + ci) * (kSelMaxK - 1);
                const bool in = ci < n_chunks;
                lists[k][0] = in && lane < kk ? __ldcg(src + lane) : 0ull;
                lists[k][1] = in && 32 + lane < kk ? __ldcg(src + 32 + lane) : 0ull;
            }
            acc[0] = lists[0][0];
            acc[1] = lists[0][1];
#pragma unroll
            for (int k = 1; k < kPer; ++k)
                if (warp + k * kSelWarps < n_chunks) warp_merge64_desc(acc, lists[k]);
            cta_merge_top64<kSelWarps>(acc, s_lists);
            from_ids = false;
        }
    } else if constexpr (kChunkRadix) {
#pragma unroll
        for (int i = 0; i < 2 * G; ++i)
            if (keys[i] != 0ull && (keys[i] & mask) >= prefix) s_ids[atomicAdd(&s_nsel[1], 1)] = key64_id(keys[i]);
        __syncthreads();
    }
    if (warp == 0) {
        // the winners in ascending block order (non-zero keys: candidates with a valid page)
        int km;
        uint32_t ids[2];
        if (from_ids) {
            km = s_nsel[1];
            ids[0] = lane < km ? s_ids[lane] : 0xffffffffu;
            ids[1] = 32 + lane < km ? s_ids[32 + lane] : 0xffffffffu;
        } else {
            const bool w0 = lane < kk && acc[0] != 0ull, w1 = 32 + lane < kk && acc[1] != 0ull;
            km = __popc(__ballot_sync(0xffffffffu, w0)) + __popc(__ballot_sync(0xffffffffu, w1));
            ids[0] = w0 ? key64_id(acc[0]) : 0xffffffffu;
            ids[1] = w1 ? key64_id(acc[1]) : 0xffffffffu;
        }
        warp_sort64_asc_u32(ids);
        const bool v0 = lane < km, v1 = 32 + lane < km;
        if (v0) out[lane] = (int32_t)ids[0];
        if (v1) out[32 + lane] = (int32_t)ids[1];
        if (lane == 0) {
            out[km] = own;              // the own block: the largest visible id, last in order
            a.cnt[t] = km + 1;
            a.counters[t] = 0;          // ready for the next call
        }
        for (int i = km + 1 + lane; i < a.k_max; i += 32) out[i] = -1;
        // the attention that follows looks these blocks' pages up first: warm
        // their block-table lines in L2 (a prefetch, no value is read)
        const int32_t *row = a.block_table + (size_t)s * a.max_blocks;
        if (v0) prefetch_l2_line(row + ids[0]);
        if (v1) prefetch_l2_line(row + ids[1]);
    }
}

cudaError_t launch_select_blocks(const SelectArgs &a, cudaStream_t stream) {
    if (a.total_q == 0) return cudaSuccess;
    // the chunk size keeps every query at <= kSelMaxChunks chunks
    const int need = (a.max_blocks + kSelMaxChunks - 1) / kSelMaxChunks;   // blocks per chunk
    int gr = (need + kSelWarps * 64 - 1) / (kSelWarps * 64);
    // with many queries (prefill) the grid fills the GPU anyway: larger chunks,
    // down to one per query, leave fewer candidate lists to merge (none with
    // one chunk: the query's only CTA writes its selection directly)
    auto chunks = [&](int g) { return (a.max_blocks + kSelWarps * 64 * g - 1) / (kSelWarps * 64 * g); };
    while (gr < 8 && chunks(gr) > 1 && (long long)a.total_q * chunks(2 * gr) >= kSelBusyCtas) gr *= 2;
    auto go = [&](auto kern, int G) {
        SelectArgs b = a;
        b.sel_rows = (a.max_blocks + kSelWarps * 64 * G - 1) / (kSelWarps * 64 * G);   // chunks
        const int app_rows = a.app.total_new > 0 ? (a.app.total_new + a.total_q - 1) / a.total_q : 0;
        if (b.sel_rows + app_rows > 65535) return cudaErrorInvalidValue;
        const dim3 grid(a.total_q, b.sel_rows + app_rows);
        if (a.cu_new) {
            // with the append in its grid: an ordinary launch, which starts once
            // everything before it has finished (measured faster at 1M-token
            // decode than a programmatic dependent of the attention before it)
            kern<<<grid, dim3(kSelThreads), 0, stream>>>(b);
            return cudaGetLastError();
        }
        return launch_pdl(kern, grid, dim3(kSelThreads), 0, stream, b);
    };
    if (gr <= 1) return go(select_blocks_kernel<1>, 1);
    if (gr <= 2) return go(select_blocks_kernel<2>, 2);
    if (gr <= 4) return go(select_blocks_kernel<4>, 4);
    if (gr <= 8) return go(select_blocks_kernel<8>, 8);
    return cudaErrorInvalidValue;   // the host rejects contexts this long first
}

}  // namespace dsa
