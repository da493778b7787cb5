// decode_fused.cuh -- the append and selection phases of the single-launch
// decode step (the attention phase is sparse_attn.cu's persistent loop).
//
// "Day-0 Readiness for Trillion-Parameter Models: Engineering Sparse Attention
// and Expert Weight Compression", section "Differentiated Adaptation of
// Prefill and Decode": in decode, fuse index selection, the gather and
// attention to cut launches and write-backs.  "Day-0 Adaptation for Massive
// LLMs: Overcoming Sparse Attention and MXFP4 Expert Weights", section 4(1):
// block-wise scoring and partial selection instead of a full sort.
//
// One persistent CTA per SM runs three phases:
//   1. select: the (query, 64-candidate group) list is split evenly over the
//      CTAs.  A CTA stages the page ids, the coarse keys (cp.async into its
//      idle TMA ring) and the query rows of up to kRoundGroups groups at once,
//      scores them on the int8 tensor cores and folds each group's 64 keys
//      into per-warp Top-64 lists.  A query wholly inside the CTA is finalised
//      there; a split query leaves the CTA's Top-(K-1) in the workspace and the
//      CTA completing its group count (acq_rel atomic, no waiting) merges the
//      lists.  The finaliser writes the ascending selection and releases the
//      query's ready flag;
//   2. append: CTA c copies new tokens c, c + C, ... into their page slots and
//      releases a count of appended tokens (after the selection, which never
//      reads them, so the copies stay off the selection's critical path);
//   3. attention: the producer warp acquires the ready flag of each query
//      before reading its selection, and the appended-token count before its
//      first TMA (a decode query's own block holds the new token).
// Phases 1 and 2 never wait on another CTA, so with every CTA resident (a
// cooperative launch) the waits of phase 3 always end; they are bounded all
// the same.  Flags carry an epoch tag that the last CTA to finish advances,
// so the workspace needs no clearing between calls.
//
// The selection never reads a coarse key written by this call's append: the
// host and device checks require every appended block of a sequence to lie at
// or after the own block of each of its queries (true for decode, where the
// one new token is the query itself), and the own block is always selected
// without being scored.
#pragma once

#include <climits>

#include "dsa_kernels.h"
#include "dsa_tma.cuh"
#include "indexer_core.cuh"
#include "warp_topk.cuh"

namespace dsa {

namespace fused {

constexpr int kThreads = 160;           // the attention kernel's 5 warps
constexpr int kWarps = kThreads / 32;
constexpr int kRoundGroups = 24;        // 64-block groups staged per round
// byte offsets inside the (idle) TMA ring during the select phase
constexpr int kOffKc = 0;                                           // [kRoundGroups*64][64] int8, chunk-swizzled
constexpr int kOffPages = kOffKc + kRoundGroups * 64 * 64;          // [kRoundGroups*64] int32
constexpr int kOffGq = kOffPages + kRoundGroups * 64 * 4;           // [kRoundGroups] query of each group
constexpr int kOffGqs = kOffGq + kRoundGroups * 4;                  // [kRoundGroups] its staged-query slot
constexpr int kOffQlist = kOffGqs + kRoundGroups * 4;               // [kRoundGroups] query of each slot
constexpr int kOffQi = kOffQlist + kRoundGroups * 4;                // [kRoundGroups][16][64] int8 query rows
constexpr int kOffW = kOffQi + kRoundGroups * kMaxIdxHeads * kIdxDim;   // [kRoundGroups][16] int32
constexpr int kOffLists = (kOffW + kRoundGroups * kMaxIdxHeads * 4 + 15) / 16 * 16;   // [kWarps*64] u64
constexpr int kOffGstart = kOffLists + kWarps * 64 * 8;             // [kFusedMaxQ+1] int32
constexpr int kOffFact = (kOffGstart + (kFusedMaxQ + 1) * 4 + 15) / 16 * 16;   // [kFusedMaxQ] int4
constexpr int kCuqCache = 1024;                                     // cu_q entries staged
constexpr int kOffCuq = kOffFact + kFusedMaxQ * 16;                 // [kCuqCache+1] int32
constexpr int kScratchBytes = kOffCuq + (kCuqCache + 1) * 4;

__device__ __forceinline__ int ld_acquire(const int32_t *p) {
    int v;
    asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void st_release(int32_t *p, int v) {
    asm volatile("st.release.gpu.global.s32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
// order this thread's generic-proxy global writes before later TMA reads of them
__device__ __forceinline__ void fence_proxy_async_global() {
    asm volatile("fence.proxy.async.global;" ::: "memory");
}

__device__ __forceinline__ int ld_relaxed(const int32_t *p) {
    int v;
    asm volatile("ld.relaxed.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void fence_acquire_gpu() { asm volatile("fence.acq_rel.gpu;" ::: "memory"); }

// wait until *p == v; false on timeout.  Polls are relaxed loads with a back
// off (a grid of acquire loads would crowd out the stores they wait for);
// the acquire is one fence once the value is seen.
__device__ __forceinline__ bool wait_flag(const int32_t *p, int v) {
    const long long t0 = clock64();
#pragma unroll 1
    while (ld_relaxed(p) != v) {
        if (clock64() - t0 > kWaitLimitCycles) return false;
        __nanosleep(128);
    }
    fence_acquire_gpu();
    return true;
}

// first group of CTA c in the even split of `total` groups over C CTAs (32-bit
// arithmetic: c <= 256 and total <= kFusedMaxQ * 2048 keep c * total < 2^31;
// 64-bit divisions are long dependent chains on the GPU)
__device__ __forceinline__ int group_begin(int c, int total, int C) {
    return (int)((unsigned)c * (unsigned)total / (unsigned)C);
}
// the CTA whose range holds group x (ranges are contiguous and ascending)
__device__ __forceinline__ int cta_of_group(int x, int total, int C) {
    int c = (int)((unsigned)x * (unsigned)C / (unsigned)total);
    while (c + 1 < C && group_begin(c + 1, total, C) <= x) ++c;
    while (c > 0 && group_begin(c, total, C) > x) --c;
    return c;
}

// query facts packed for shared memory
struct Fact {
    int s, p, n_vis, k;   // k < 0 marks an error query
};

// The query's ascending selection from the winners in warp 0's registers
// (acc sorted descending, the first kk valid), then the ready flag.  Warp 0 only.
__device__ __forceinline__ void finalize(const AttnArgs &a, const FusedArgs &f, int t, const Fact &q,
                                         const key64 (&acc)[2], int tag) {
    const int lane = threadIdx.x & 31;
    const int kk = q.k - 1, own = q.n_vis - 1;
    const bool v0 = lane < kk && acc[0] != 0ull, v1 = 32 + lane < kk && acc[1] != 0ull;
    const int km = __popc(__ballot_sync(0xffffffffu, v0)) + __popc(__ballot_sync(0xffffffffu, v1));
    uint32_t ids[2] = {v0 ? key64_id(acc[0]) : 0xffffffffu, v1 ? key64_id(acc[1]) : 0xffffffffu};
    warp_sort64_asc_u32(ids);
    int32_t *out = f.sel + (size_t)t * a.k_max;
    if (lane < km) out[lane] = (int32_t)ids[0];
    if (32 + lane < km) out[32 + lane] = (int32_t)ids[1];
    if (lane == 0) {
        out[km] = own;   // the own block: the largest visible id, last in order
        f.cnt[t] = km + 1;
    }
    for (int i = km + 1 + lane; i < a.k_max; i += 32) out[i] = -1;
    // the warp barrier orders every lane's stores before lane 0's release,
    // which carries them to whoever acquires the flag
    __syncwarp();
    if (lane == 0) st_release(f.flags + t, tag);
}

// Phase 2: CTA c copies new tokens c, c + C, ... into their page slots (K, V
// and, for the last new token of a block, the coarse key) and adds the count
// to the workspace.  Run after the selection: no selection reads these rows.
__device__ __forceinline__ void append_tokens(const AttnArgs &a, const FusedArgs &f) {
    const int tid = threadIdx.x;
    const int c = blockIdx.x, C = gridDim.x;
    if (f.total_new > 0) {
        const int row16 = a.num_kv_heads * (kHeadDim * 2 / 16);   // 16-byte vectors per token row
        int done = 0;
        for (int i = c; i < f.total_new; i += C) {
            const int s = find_seq(f.cu_new, a.num_seqs, i);
            const int first = __ldg(f.cu_new + s), last = __ldg(f.cu_new + s + 1);
            const int len = __ldg(a.seq_lens + s);
            const int n = last - first;
            const int pos = len - n + (i - first);
            const int blk = pos / kBlockSize, slot = pos % kBlockSize;
            bool ok = i >= first && i < last && n <= len && pos >= 0 && blk < a.max_blocks;
            int page = -1;
            if (ok) {
                page = __ldg(a.block_table + (size_t)s * a.max_blocks + blk);
                if (page < 0 || page >= a.num_pages) {
                    if (tid == 0) set_err(a.dev_err, DSA_DEV_ERR_PAGE);
                    ok = false;
                }
            } else if (tid == 0) {
                set_err(a.dev_err, DSA_DEV_ERR_POS);
            }
            if (ok) {
                const size_t dst = ((size_t)page * kBlockSize + slot) * row16;
                const uint4 *ks = reinterpret_cast<const uint4 *>(f.k_new) + (size_t)i * row16;
                const uint4 *vs = reinterpret_cast<const uint4 *>(f.v_new) + (size_t)i * row16;
                uint4 *kd = reinterpret_cast<uint4 *>(f.k_pool) + dst;
                uint4 *vd = reinterpret_cast<uint4 *>(f.v_pool) + dst;
                for (int e = tid; e < row16; e += kThreads) {
                    kd[e] = __ldg(ks + e);
                    vd[e] = __ldg(vs + e);
                }
                const bool last_in_block = (i == last - 1) || (slot == kBlockSize - 1);
                if (f.kc_new && last_in_block && tid < kIdxDim / 16) {
                    const uint4 *cs = reinterpret_cast<const uint4 *>(f.kc_new) + (size_t)i * (kIdxDim / 16);
                    uint4 *cd = reinterpret_cast<uint4 *>(f.kc_pool) + (size_t)page * (kIdxDim / 16);
                    cd[tid] = __ldg(cs + tid);
                }
            }
            ++done;   // counted even when skipped: the waiters count tokens, not successes
        }
        if (done > 0) {
            fence_proxy_async_global();   // the attention phase reads these rows with TMA
            __syncthreads();               // ordered before tid 0's release (cumulative)
            if (tid == 0) atomic_add_acq_rel_gpu(f.hdr + kHdrAppended, done);
        }
    }

}

// Phase 1.  Every thread of the CTA calls it; `scratch` is the idle TMA ring
// (generic pointer, 16-byte aligned, kScratchBytes long).
__device__ __forceinline__ void select_blocks_phase(const AttnArgs &a, const FusedArgs &f, uint8_t *scratch,
                                                  int tag, volatile int *s_last) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int c = blockIdx.x, C = gridDim.x;
    const int T = a.total_q;

    // ------------------------------------------------------------ B. select
    int *s_gstart = reinterpret_cast<int *>(scratch + kOffGstart);
    Fact *s_fact = reinterpret_cast<Fact *>(scratch + kOffFact);
    int *s_pages = reinterpret_cast<int *>(scratch + kOffPages);
    int *s_gq = reinterpret_cast<int *>(scratch + kOffGq);
    int *s_gqs = reinterpret_cast<int *>(scratch + kOffGqs);
    int *s_qlist = reinterpret_cast<int *>(scratch + kOffQlist);
    int4 *s_qi = reinterpret_cast<int4 *>(scratch + kOffQi);   // [group slot][16 heads][4]
    int *s_w = reinterpret_cast<int *>(scratch + kOffW);        // [group slot][16]
    key64 *s_lists = reinterpret_cast<key64 *>(scratch + kOffLists);
    const uint32_t s_kc = smem_u32(scratch + kOffKc);
    int *s_cnt = s_pages;   // group counts of the queries, before the first round

    // facts and candidate-group counts of every query: cu_q and the positions
    // first (one round trip), then the per-sequence facts (a second one)
    int *s_cuq = reinterpret_cast<int *>(scratch + kOffCuq);
    const bool cuq_cached = a.num_seqs + 1 <= kCuqCache + 1;
    if (cuq_cached)
        for (int i = tid; i <= a.num_seqs; i += kThreads) s_cuq[i] = __ldg(a.cu_q + i);
    for (int t = tid; t < T; t += kThreads) s_fact[t].p = __ldg(a.q_pos + t);
    __syncthreads();
    uint32_t err_bits = 0;
    for (int t = tid; t < T; t += kThreads) {
        int s;
        if (cuq_cached) {
            int lo = 0, hi = a.num_seqs - 1;
            while (lo < hi) {
                const int mid = (lo + hi + 1) >> 1;
                if (s_cuq[mid] <= t) lo = mid; else hi = mid - 1;
            }
            s = lo;
        } else {
            s = find_seq(a.cu_q, a.num_seqs, t);
        }
        const int p = s_fact[t].p;
        const int len = __ldg(a.seq_lens + s);
        int k = __ldg(f.k_per_seq + s);
        const int n_vis = p / kBlockSize + 1;
        bool bad_pos = p < 0 || p >= len || n_vis > a.max_blocks;
        if (f.total_new > 0 && !bad_pos) {
            // every appended block must lie at or after the query's own block
            const int n_new = __ldg(f.cu_new + s + 1) - __ldg(f.cu_new + s);
            if (n_new > len || (n_new > 0 && n_vis - 1 > (len - n_new) / kBlockSize)) bad_pos = true;
        }
        const bool bad_k = k < 1 || k > a.k_max;
        if (bad_pos || bad_k) {
            err_bits |= bad_k ? DSA_DEV_ERR_K : DSA_DEV_ERR_POS;
            k = -1;
        }
        s_fact[t] = Fact{s, p, n_vis, k};
        const int own = n_vis - 1;
        s_cnt[t] = (k > 1 && n_vis > k) ? (own + 63) / 64 : 0;
    }
    if (c == 0 && err_bits) set_err(a.dev_err, err_bits);
    __syncthreads();
    if (warp == 0) {   // exclusive scan of the group counts
        const int per = (T + 31) / 32;
        const int lo = min(T, lane * per), hi = min(T, lo + per);
        int sum = 0;
        for (int t = lo; t < hi; ++t) sum += s_cnt[t];
        int incl = sum;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, d);
            if (lane >= d) incl += y;
        }
        int run = incl - sum;
        for (int t = lo; t < hi; ++t) {
            s_gstart[t] = run;
            run += s_cnt[t];
        }
        if (lane == 31) s_gstart[T] = incl;
    }
    __syncthreads();
    const int total = s_gstart[T];

    // queries with nothing to score: written by CTA t % C, one warp each
    for (int t = c + warp * C; t < T; t += kWarps * C) {
        const Fact q = s_fact[t];
        if (q.k > 1 && q.n_vis > q.k) continue;
        int32_t *out = f.sel + (size_t)t * a.k_max;
        int n = 0;
        if (q.k > 0) n = q.n_vis <= q.k ? q.n_vis : 1;
        for (int i = lane; i < a.k_max; i += 32) out[i] = i < n ? (n == 1 ? q.n_vis - 1 : i) : -1;
        if (lane == 0) f.cnt[t] = n;
        __syncwarp();
        if (lane == 0) st_release(f.flags + t, tag);
    }
    if (total == 0) return;

    const int gb = group_begin(c, total, C), ge = group_begin(c + 1, total, C);
    const int H = f.num_idx_heads;
    const int g = lane >> 2, cq = lane & 3;
    key64 acc[2] = {0ull, 0ull};
    for (int r0 = gb; r0 < ge; r0 += kRoundGroups) {
        const int ng = min(kRoundGroups, ge - r0);
        if (tid < ng) {   // query of each staged group: last t with s_gstart[t] <= group
            const int x = r0 + tid;
            int lo = 0, hi = T - 1;
            while (lo < hi) {
                const int mid = (lo + hi + 1) >> 1;
                if (s_gstart[mid] <= x) lo = mid; else hi = mid - 1;
            }
            s_gq[tid] = lo;
        }
        __syncthreads();
        if (tid < ng) {   // distinct queries of the round (ascending), and each group's slot among them
            int slot = 0;
            for (int j = 1; j <= tid; ++j) slot += s_gq[j] != s_gq[j - 1];
            s_gqs[tid] = slot;
            if (tid == 0 || s_gq[tid] != s_gq[tid - 1]) s_qlist[slot] = s_gq[tid];
        }
        __syncthreads();
        const int nq = s_gqs[ng - 1] + 1;
        // page ids of the staged candidates (-1: past the candidates or a bad
        // page), the round's query rows and head weights: every load in
        // registers first, so they all travel in one round trip
        constexpr int kRowsPT = (kRoundGroups * 64 + kThreads - 1) / kThreads;
        int pg[kRowsPT];
#pragma unroll
        for (int k = 0; k < kRowsPT; ++k) {
            const int e = tid + k * kThreads;
            pg[k] = INT_MIN;   // not a candidate
            if (e < ng * 64) {
                const int t = s_gq[e >> 6];
                const Fact q = s_fact[t];
                const int b = 64 * (r0 + (e >> 6) - s_gstart[t]) + (e & 63);
                if (b < q.n_vis - 1) pg[k] = __ldg(a.block_table + (size_t)q.s * a.max_blocks + b);
            }
        }
        int4 qv[kRowsPT];
#pragma unroll
        for (int k = 0; k < kRowsPT; ++k) {   // nq * 16 heads * 4 int4 <= kRoundGroups * 64
            const int e = tid + k * kThreads;
            qv[k] = make_int4(0, 0, 0, 0);
            const int qq = e / (kMaxIdxHeads * 4), h = (e >> 2) & (kMaxIdxHeads - 1);
            if (e < nq * kMaxIdxHeads * 4 && h < H)
                qv[k] = __ldg(reinterpret_cast<const int4 *>(f.q_idx + ((size_t)s_qlist[qq] * H + h) * kIdxDim) +
                              (e & 3));
        }
        int wv[2];
#pragma unroll
        for (int k = 0; k < 2; ++k) {   // nq * 16 <= 384 <= 2 * kThreads + 64: the rest below
            const int e = tid + k * kThreads;
            const int qq = e / kMaxIdxHeads, h = e % kMaxIdxHeads;
            wv[k] = (e < nq * kMaxIdxHeads && h < H) ? __ldg(f.w + (size_t)s_qlist[qq] * H + h) : 0;
        }
        for (int e = tid + 2 * kThreads; e < nq * kMaxIdxHeads; e += kThreads) {
            const int qq = e / kMaxIdxHeads, h = e % kMaxIdxHeads;
            s_w[e] = h < H ? __ldg(f.w + (size_t)s_qlist[qq] * H + h) : 0;
        }
#pragma unroll
        for (int k = 0; k < 2; ++k) {
            const int e = tid + k * kThreads;
            if (e < nq * kMaxIdxHeads) s_w[e] = wv[k];
        }
#pragma unroll
        for (int k = 0; k < kRowsPT; ++k) {
            const int e = tid + k * kThreads;
            if (e < nq * kMaxIdxHeads * 4) s_qi[e] = qv[k];
        }
        // coarse keys straight from the page registers: 4 x 16 B per row,
        // chunks swizzled by (row / 2) % 4 against bank conflicts
#pragma unroll
        for (int k = 0; k < kRowsPT; ++k) {
            const int row = tid + k * kThreads;
            if (row >= ng * 64) continue;
            int page = pg[k];
            if (page == INT_MIN) {
                page = -1;
            } else if (page < 0 || page >= a.num_pages) {
                err_bits |= DSA_DEV_ERR_PAGE;
                page = -1;
            }
            s_pages[row] = page;
#pragma unroll
            for (int part = 0; part < 4; ++part) {
                const uint32_t dst = s_kc + row * 64 + ((part ^ ((row >> 1) & 3)) << 4);
                if (page >= 0) cp_async_16(dst, f.kc_pool + (size_t)page * kIdxDim + part * 16);
                else cp_async_16_zero(dst, f.kc_pool);
            }
        }
        cp_async_commit();
        cp_async_wait<0>();
        __syncthreads();

        // score, one query segment of the round at a time
        for (int i = 0; i < ng;) {
            const int t = s_gq[i];
            const int seg_hi = min(ge, s_gstart[t + 1]);   // end of t's groups in this CTA
            const int i_end = min(ng, seg_hi - r0);
            const Fact q = s_fact[t];
            const int qs = s_gqs[i];
            int qb[2][2][2], wl[2][2];
            {
                const int *qi = reinterpret_cast<const int *>(s_qi + qs * kMaxIdxHeads * 4);
#pragma unroll
                for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
                    for (int ks = 0; ks < 2; ++ks) {
                        qb[nt][ks][0] = qi[(8 * nt + g) * 16 + 8 * ks + cq];
                        qb[nt][ks][1] = qi[(8 * nt + g) * 16 + 8 * ks + 4 + cq];
                    }
                    wl[nt][0] = s_w[qs * kMaxIdxHeads + 8 * nt + 2 * cq];
                    wl[nt][1] = s_w[qs * kMaxIdxHeads + 8 * nt + 2 * cq + 1];
                }
            }
            for (int gi = i + warp; gi < i_end; gi += kWarps) {
                const int base = 64 * (r0 + gi - s_gstart[t]);   // first block of the group
                key64 v[2] = {0ull, 0ull};
#pragma unroll
                for (int mt = 0; mt < 4; ++mt) {
                    Tile16 fr;
                    const int r_g = gi * 64 + 16 * mt + g, r_g8 = r_g + 8;
#pragma unroll
                    for (int ks = 0; ks < 2; ++ks) {
                        // int (8*ks + c) of a row is word c of chunk 2*ks; (8*ks + 4 + c) of chunk 2*ks+1
                        fr.a[ks][0] = *reinterpret_cast<const int *>(scratch + kOffKc + r_g * 64 +
                                                                     (((2 * ks) ^ ((r_g >> 1) & 3)) << 4) + 4 * cq);
                        fr.a[ks][1] = *reinterpret_cast<const int *>(scratch + kOffKc + r_g8 * 64 +
                                                                     (((2 * ks) ^ ((r_g8 >> 1) & 3)) << 4) + 4 * cq);
                        fr.a[ks][2] = *reinterpret_cast<const int *>(scratch + kOffKc + r_g * 64 +
                                                                     (((2 * ks + 1) ^ ((r_g >> 1) & 3)) << 4) + 4 * cq);
                        fr.a[ks][3] = *reinterpret_cast<const int *>(scratch + kOffKc + r_g8 * 64 +
                                                                     (((2 * ks + 1) ^ ((r_g8 >> 1) & 3)) << 4) + 4 * cq);
                    }
                    int s_g, s_g8;
                    tile16_scores(fr, qb, wl, s_g, s_g8);
                    if (mt == cq) {   // lane (g, cq) keeps blocks 16*cq + g and 16*cq + g + 8
                        const int b = base + 16 * mt + g;
                        v[0] = s_pages[r_g] >= 0 ? make_key64(s_g, (uint32_t)b) : 0ull;
                        v[1] = s_pages[r_g8] >= 0 ? make_key64(s_g8, (uint32_t)(b + 8)) : 0ull;
                    }
                }
                warp_fold_topk(acc, v, q.k - 1);
            }
            if (seg_hi <= r0 + ng) {
                // ---- t's groups in this CTA are done: the CTA's Top-64 of t
                cta_merge_top64<kWarps>(acc, s_lists);
                const int g_lo = s_gstart[t], g_hi = s_gstart[t + 1];
                if (g_lo >= gb && g_hi <= ge) {
                    if (warp == 0) finalize(a, f, t, q, acc, tag);
                } else {
                    const int kk = q.k - 1;
                    const int slot = g_lo < gb ? 0 : 1;
                    key64 *cand = f.cand + ((size_t)c * 2 + slot) * (kSelMaxK - 1);
                    if (warp == 0) {
                        if (lane < kk) cand[lane] = acc[0];
                        if (32 + lane < kk) cand[32 + lane] = acc[1];
                        __syncwarp();   // ordered before lane 0's acq_rel add (cumulative)
                        if (lane == 0) {
                            const int covered = min(g_hi, ge) - max(g_lo, gb);
                            const int old = atomic_add_acq_rel_gpu(f.sel_count + t, covered);
                            *s_last = (old + covered == g_hi - g_lo);
                        }
                    }
                    __syncthreads();
                    if (*s_last) {
                        // merge the lists of the CTAs covering t (contiguous, non-empty ranges)
                        const int cf = cta_of_group(g_lo, total, C), cl = cta_of_group(g_hi - 1, total, C);
                        key64 m[2] = {0ull, 0ull};
                        constexpr int kBatch = 4;   // lists in flight per warp
                        for (int c0 = cf + warp; c0 <= cl; c0 += kBatch * kWarps) {
                            key64 lst[kBatch][2];
#pragma unroll
                            for (int j = 0; j < kBatch; ++j) {
                                const int cc = c0 + j * kWarps;
                                lst[j][0] = lst[j][1] = 0ull;
                                if (cc > cl) continue;
                                const int cb = group_begin(cc, total, C);
                                if (cb == group_begin(cc + 1, total, C)) continue;   // empty range: no list
                                const int sl = g_lo < cb ? 0 : 1;
                                const key64 *src = f.cand + ((size_t)cc * 2 + sl) * (kSelMaxK - 1);
                                if (lane < kk) lst[j][0] = __ldcg(src + lane);
                                if (32 + lane < kk) lst[j][1] = __ldcg(src + 32 + lane);
                            }
#pragma unroll
                            for (int j = 0; j < kBatch; ++j) warp_merge64_desc(m, lst[j]);
                        }
                        cta_merge_top64<kWarps>(m, s_lists);
                        if (warp == 0) {
                            if (lane == 0) f.sel_count[t] = 0;   // ready for the next call
                            finalize(a, f, t, q, m, tag);
                        }
                    }
                    __syncthreads();
                }
                acc[0] = acc[1] = 0ull;
            }
            i = i_end;
        }
        __syncthreads();   // the staging buffers are reused by the next round
    }
    if (err_bits) set_err(a.dev_err, err_bits);
}

}  // namespace fused
}  // namespace dsa
