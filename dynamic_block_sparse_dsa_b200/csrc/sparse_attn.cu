// sparse_attn.cu -- exact attention over the selected KV blocks only.
//
// "Day-0 Adaptation for Massive LLMs: Overcoming Sparse Attention and MXFP4
// Expert Weights", section 4(3): decode gathers the selected KV blocks on chip
// by their indices and attends under a valid mask; its cost is the gather of
// non-contiguous blocks.  "Day-0 Adaptation for Trillion-Parameter Models:
// Engineering Practices and Technical Breakdown", section 4.3: decode needs a
// dedicated gather kernel.  "Day-0 Readiness ...", section "KV Cache Layout":
// read whole blocks by block id, never token by token.
//
// Design (B200): a persistent grid of one CTA per SM.  The work is the list of
// units u = (query t, KV head, selection slot j) -- one 64-token page slice of
// K and of V (16 KiB each) -- and CTA c takes the contiguous range
// [c*U/C, (c+1)*U/C), so every SM streams the same number of bytes whatever
// the batch looks like.  When every CTA takes whole (query, KV head) pairs
// (prefill, and decode batches with many pairs) the pairs instead run
// KV-head-major and interleaved over the CTAs -- CTA c takes pairs c, c + C,
// ... of the order kvh * T + t -- so all CTAs read one KV head's slice of the
// pool at a time and the queries that select the same block find it in L2.
// Inside the CTA:
//   * a producer warp walks the range and, for each selected block, issues four
//     boxes of a 3-D TMA tensor map over the pool (K and V, two 128-byte halves
//     each, SWIZZLE_128B, no multicast) into a 6-stage (5 for 16-head groups)
//     shared-memory ring
//     guarded by full/empty mbarriers; it also TMA-loads the 16-row query tile
//     of each (query, KV head) pair into a 2-slot ring;
//   * four consumer warps take whole blocks round-robin.  Each runs its 64
//     tokens against the GQA group of query heads on the tensor cores with
//     mma.m16n8k16 bf16/fp32 in swap-AB form (the keys are the M dimension,
//     the <= 8 or 16 query heads N): S^T = K Q^T, online softmax in fp32 with
//     base-2 exponents and the causal mask of the own block, then
//     O^T += V^T P^T with P^T built from the score fragments by movmatrix;
//   * at the end of each pair the four warps' softmax states are merged in a
//     fixed order through shared memory.  A pair that lies wholly inside the
//     CTA is written straight out; a pair split across CTAs leaves a partial
//     (m, l, unnormalised O) in the workspace and the CTA completing its units
//     -- counted with an atomic, no waiting -- merges the partials;
//   * decode batches with between C/4 and C/2 pairs run one 2-CTA cluster per
//     pair instead: each rank takes half of the pair's blocks, and rank 1 hands
//     its merged state to rank 0 with st.async stores that complete their
//     bytes on rank 0's inbox mbarrier (armed with the full count before the
//     start-of-kernel cluster barrier); rank 0 combines and writes the output.
// All waits are bounded (DSA_DEV_ERR_WAIT on timeout, no hang).
#include <mutex>

#include "dsa_kernels.h"
#include "dsa_tma.cuh"
#include "decode_fused.cuh"

namespace dsa {

namespace {
constexpr int kConsumerWarps = 4;
constexpr int kAttnThreads = (kConsumerWarps + 1) * 32;
constexpr int kHalf = kBlockSize * 128;            // 8 KiB: 64 rows x 128 B (one swizzled half)
constexpr int kStageBytes = 4 * kHalf;             // K lo, K hi, V lo, V hi
constexpr int kQHalf = 16 * 128;                   // 16 query rows x 128 B
constexpr int kQSlotBytes = 2 * kQHalf;
constexpr int kSegSlots = 2;                       // query tile + pair facts, double buffered
constexpr int kMergeStride = 132;                  // floats per merge row (padded against bank conflicts)
constexpr int kMaxSmemSeqs = 256;                  // cu_q entries cached in shared memory
// int words after the barriers
constexpr int kWAbort = 0, kWLast = 1, kWNever = 2, kWTag = 3;
constexpr int kWFill = 4;                           // [kMaxStages] item index the stage was last armed for
constexpr int kMaxStages = 8;
constexpr int kWItemBlk = kWFill + kMaxStages;      // [kMaxStages] logical block of that item
constexpr int kWItemSeg = kWItemBlk + kMaxStages;   // [kMaxStages] segment of that item
constexpr int kWSegEndCnt = kWItemSeg + kMaxStages; // [kSegSlots] items issued when the segment ended
constexpr int kWSegEndTag = kWSegEndCnt + kSegSlots;  // [kSegSlots] which segment that count belongs to
constexpr int kWSegInfo = kWSegEndTag + kSegSlots;  // [kSegSlots][4]: t, kvh, p, n_vis
constexpr int kWSelLast = kWSegInfo + 4 * kSegSlots;   // fused select: this CTA merges
constexpr int kNumWords = kWSelLast + 1;
constexpr float kLn2 = 0.6931471805599453f;
// most CTAs whose ranges can cover one pair (the host caps the split at 60)
constexpr int kMaxSplitSlots = 63;
// bytes rank 1 sends per head row in 2-CTA cluster mode: o[128] then (m, l)
constexpr uint32_t kInboxRowBytes = 128 * 4 + 2 * 4;

// shared-memory plan for NT head tiles: a group of <= 8 heads leaves room for
// a sixth ring stage; 16-head groups need the larger merge buffer
template <int NT>
struct Plan {
    static constexpr int kStages = NT == 1 ? 6 : 5;
    static constexpr int kMergeRows = 8 * NT;
    static constexpr int kOffQ = kStages * kStageBytes;
    static constexpr int kOffMergeO = kOffQ + kSegSlots * kQSlotBytes;
    static constexpr int kOffMergeML = kOffMergeO + kConsumerWarps * kMergeRows * kMergeStride * 4;
    static constexpr int kOffCuq = kOffMergeML + kConsumerWarps * 16 * 2 * 4;
    static constexpr int kOffRb = (kOffCuq + (kMaxSmemSeqs + 1) * 4 + 4 + 7) / 8 * 8;
    static constexpr int kOffBars = kOffRb + (kAttnMaxCtas + 1) * 8;
    static constexpr int kNumBars = 2 * kStages + 2 * kSegSlots + 1;   // + the cluster inbox
    static constexpr int kOffWords = kOffBars + kNumBars * 8;
    // 2-CTA cluster mode: the partner's merged state (kMergeRows x (o[128], m, l))
    static constexpr int kOffInbox = (kOffWords + kNumWords * 4 + 15) / 16 * 16;
    static constexpr int kSmemBytes = kOffInbox + kMergeRows * kAttnPartStride * 4 + 1024;   // + base alignment slack
    static_assert(kStages <= kMaxStages, "stage words");
    static_assert(fused::kScratchBytes <= kStages * kStageBytes, "fused select scratch fits the ring");
    static_assert(kSmemBytes <= 227 * 1024, "shared memory");
};

template <int NT>
struct Smem {
    using P = Plan<NT>;
    uint32_t base;   // 1 KiB aligned shared address
    __device__ uint32_t stage(int s) const { return base + s * kStageBytes; }
    __device__ uint32_t qslot(int s) const { return base + P::kOffQ + s * kQSlotBytes; }
    __device__ uint32_t full(int s) const { return base + P::kOffBars + 8 * s; }
    __device__ uint32_t empty(int s) const { return base + P::kOffBars + 8 * (P::kStages + s); }
    __device__ uint32_t qfull(int s) const { return base + P::kOffBars + 8 * (2 * P::kStages + s); }
    __device__ uint32_t qempty(int s) const { return base + P::kOffBars + 8 * (2 * P::kStages + kSegSlots + s); }
    __device__ uint32_t inbox_full() const { return base + P::kOffBars + 8 * (2 * P::kStages + 2 * kSegSlots); }
    __device__ uint32_t inbox() const { return base + P::kOffInbox; }
};

// Unit indices are 32-bit (the host keeps total_units below 2^31): the hot
// loops divide them by the Top-K and the KV-head count, and 64-bit integer
// division is a long dependent instruction chain on the GPU.
using unit_t = uint32_t;

// first unit of CTA c (64-bit products; computed once per CTA)
__device__ __forceinline__ unit_t range_begin(const AttnArgs &a, int c) {
    if (a.pair_aligned) {
        const unsigned up = (unsigned)a.k_max << a.tile_shift;   // units per pair
        const unsigned long long pairs = (unsigned long long)a.total_units / up;
        return (unit_t)((unsigned long long)c * pairs / (unsigned)a.num_ctas * up);
    }
    return (unit_t)((unsigned long long)c * (unsigned long long)a.total_units / (unsigned)a.num_ctas);
}

// sequence of query t: last s with cu_q[s] <= t, from the shared-memory copy when it fits
__device__ __forceinline__ int seq_of(const AttnArgs &a, const int *s_cuq, int t) {
    if (a.num_seqs + 1 > kMaxSmemSeqs) return find_seq(a.cu_q, a.num_seqs, t);
    int lo = 0, hi = a.num_seqs - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (s_cuq[mid] <= t) lo = mid; else hi = mid - 1;
    }
    return lo;
}
}  // namespace

// NT: query-head n-tiles of 8 (the GQA group is <= 8 * NT).  kFused: the
// single-launch decode step -- the select and append phases of
// decode_fused.cuh run first, and the producer waits for each query's
// selection before reading it.
template <int NT, bool kFused>
__global__ void __launch_bounds__(kAttnThreads, 1)
sparse_attn_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                   const __grid_constant__ CUtensorMap tm_q, AttnArgs a, FusedArgs f) {
    using P = Plan<NT>;
    constexpr int kStages = P::kStages;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    Smem<NT> sm{(raw + 1023u) & ~1023u};
    uint8_t *gbase = smem_raw + (sm.base - raw);   // generic pointer of the aligned base
    volatile int *W = reinterpret_cast<volatile int *>(gbase + P::kOffWords);
    volatile int *s_abort = W + kWAbort;
    const volatile int *s_never = W + kWNever;      // stays 0: a wait that ignores the abort flag
    int *s_cuq = reinterpret_cast<int *>(gbase + P::kOffCuq);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int c = blockIdx.x;
    // every CTA's range start, once (64-bit divisions are slow; lookups are not)
    unit_t *s_rb = reinterpret_cast<unit_t *>(gbase + P::kOffRb);
    for (int i = tid; i <= a.num_ctas; i += kAttnThreads) s_rb[i] = range_begin(a, i);
    unit_t u0, u1;
    // units per (query, KV head) pair: every selection slot's 64-token tiles
    const unit_t K = (unit_t)a.k_max << a.tile_shift;
    if (a.cluster2) {   // half of pair c/2: units [0, h0) for rank 0, [h0, K) for rank 1
        const unit_t p0 = (unit_t)(c >> 1) * K;
        const unit_t h0 = (K + 1) / 2;
        u0 = p0 + ((c & 1) ? h0 : 0);
        u1 = p0 + ((c & 1) ? K : h0);
    } else if (!kFused && a.interleave) {
        // pairs c, c + C, c + 2C, ... of the KV-head-major order: local pair i
        // of this CTA is r = i * C + c (r = kvh * T + t)
        const unit_t P = (unit_t)a.total_q * (unit_t)a.num_kv_heads, C = (unit_t)a.num_ctas;
        u0 = 0;
        u1 = ((unit_t)c < P ? (P - 1 - (unit_t)c) / C + 1 : 0) * K;
    } else {
        u0 = range_begin(a, c);
        u1 = range_begin(a, c + 1);
    }
    const int G = a.group;
    const unit_t Hkv = (unit_t)a.num_kv_heads;

    if (tid == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(sm.full(s), 1);
            mbar_init(sm.empty(s), 1);
        }
        for (int s = 0; s < kSegSlots; ++s) {
            mbar_init(sm.qfull(s), 1);
            mbar_init(sm.qempty(s), 1);
        }
        mbar_init(sm.inbox_full(), 1);
        for (int k = 0; k < kNumWords; ++k) W[k] = 0;
        for (int s = 0; s < kStages; ++s) W[kWFill + s] = -1;
        for (int s = 0; s < kSegSlots; ++s) W[kWSegEndTag + s] = -1;
        if (kFused) W[kWTag] = fused::ld_acquire(f.hdr + kHdrEpoch) + 1;
        fence_barrier_init();
        // 2-CTA cluster mode: rank 0's inbox expects the partner's merged state
        // (G rows of o[128], m, l) before the cluster barrier below lets the
        // partner send it
        if (a.cluster2 && !(blockIdx.x & 1)) mbar_arrive_expect_tx(sm.inbox_full(), (uint32_t)a.group * kInboxRowBytes);
    }
    pdl_trigger();
    __syncthreads();
    if (a.cluster2) cluster_sync_all();   // the partner's inbox barrier is initialised before any remote arrive
    const int tag = W[kWTag];
    if constexpr (kFused) {
        fused::select_blocks_phase(a, f, gbase, tag, W + kWSelLast);
        fused::append_tokens(a, f);
        // the ring's generic-proxy use ends before TMA writes into it
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncthreads();
    }

    if (warp == kConsumerWarps) {
        // ================================================================ producer warp
        // The warp resolves 32 units per round trip (one lane per unit: pair
        // facts, selected block, page), then lane 0 publishes them in order:
        // a segment header (pair facts + TMA of the query tile) when a
        // (query, KV head) pair starts, one stage fill per usable block, and a
        // segment end marker (item count) when the pair's units are done.
        if (a.num_seqs + 1 <= kMaxSmemSeqs)
            for (int k = lane; k <= a.num_seqs; k += 32) s_cuq[k] = __ldg(a.cu_q + k);
        __syncwarp();
        if (lane == 0) {
            prefetch_tensormap(&tm_k);
            prefetch_tensormap(&tm_v);
            prefetch_tensormap(&tm_q);
        }
        // the selection and the appended tokens come from the kernels before:
        // pdl_wait() below, once the positions (inputs of the whole step) are
        // already on their way
        uint32_t err_bits = 0;
        bool sel_ready = true;
        if (kFused && lane == 0 && u0 < u1) {
            // the selections of the queries this CTA attends to (one poller
            // per CTA), then every append: a query's own block holds its new
            // token and the first TMA may read it
            const int t_first = (int)((u0 / K) / Hkv), t_last = (int)(((u1 - 1) / K) / Hkv);
            for (int t = t_first; t <= t_last && sel_ready; ++t) sel_ready = fused::wait_flag(f.flags + t, tag);
            if (f.total_new > 0) {
                const long long t0 = clock64();
                while (fused::ld_relaxed(f.hdr + kHdrAppended) < f.total_new) {
                    if (clock64() - t0 > kWaitLimitCycles) { sel_ready = false; break; }
                    __nanosleep(128);
                }
                fused::fence_acquire_gpu();
                fused::fence_proxy_async_global();
            }
            if (!sel_ready) err_bits |= DSA_DEV_ERR_WAIT;
        }
        sel_ready = __shfl_sync(0xffffffffu, (int)sel_ready, 0) != 0;
        int item = 0, seg = 0;
        bool stop = false;
        for (unit_t base = u0; base < u1 && !stop; base += 32) {
            const unit_t uu = base + lane;
            const bool in = uu < u1;
            // per unit: its pair's facts, the 64-token tile index within the
            // sequence (blk) and the tile's first pool row (page); n_vis counts
            // the query's visible 64-token tiles
            int t = 0, kvh = 0, s = 0, p = 0, n_vis = 0, blk = -1, page = -1;
            if (in) {
                const unit_t pair = uu / K;
                const int ju = (int)(uu - pair * K);
                const int j = ju >> a.tile_shift, sub = ju & ((1 << a.tile_shift) - 1);
                if (!kFused && a.interleave) {
                    const unit_t r = pair * (unit_t)a.num_ctas + (unit_t)c;
                    kvh = (int)(r / (unit_t)a.total_q);
                    t = (int)(r - (unit_t)kvh * (unit_t)a.total_q);
                } else {
                    t = (int)(pair / Hkv);
                    kvh = (int)(pair - (unit_t)t * Hkv);
                }
                s = seq_of(a, s_cuq, t);
                p = __ldg(a.q_pos + t);
                const int len = __ldg(a.seq_lens + s);
                pdl_wait();   // returns at once after the first time
                // the selection may have been written during this launch: read it through L2
                int n_sel = sel_ready ? __ldcg(a.cnt + t) : 0;
                const int b = sel_ready ? __ldcg(a.sel + (size_t)t * a.k_max + j) : -1;
                const int n_vis_blocks = (p >> a.block_shift) + 1;
                n_vis = (p >> 6) + 1;
                if (p < 0 || p >= len || n_vis_blocks > a.max_blocks || n_sel < 0 || n_sel > a.k_max) n_sel = 0;
                if (j < n_sel) {
                    if (b < 0 || b >= n_vis_blocks) {
                        err_bits |= DSA_DEV_ERR_SEL;
                    } else {
                        const int pg = __ldg(a.block_table + (size_t)s * a.max_blocks + b);
                        const int tile = (b << a.tile_shift) + sub;
                        if (pg < 0 || pg >= a.num_pages) err_bits |= DSA_DEV_ERR_PAGE;
                        else if (tile < n_vis) { blk = tile; page = (pg << a.block_shift) + (sub << 6); }
                        // tiles past the query's position (own block only) hold no visible token
                    }
                }
            }
            const unit_t chunk_end = min(u1, base + 32);
            unit_t v = base;
            while (v < chunk_end) {
                const int lf = (int)(v - base);
                const unit_t pair = v / K;
                const unit_t seg_stop = min(u1, (pair + 1) * K);
                const unit_t run_end = min(chunk_end, seg_stop);
                const int ll = (int)(run_end - 1 - base);
                const int pt = __shfl_sync(0xffffffffu, t, lf);
                const int pkvh = __shfl_sync(0xffffffffu, kvh, lf);
                const int pp = __shfl_sync(0xffffffffu, p, lf);
                const int pnv = __shfl_sync(0xffffffffu, n_vis, lf);
                if (v == u0 || v == pair * K) {
                    // ---- segment header: pair facts + query tile into slot seg % 2
                    const int qs = seg % kSegSlots;
                    if (lane == 0) {
                        bool ok = !*s_abort &&
                                  (seg < kSegSlots || mbar_wait(sm.qempty(qs), ((seg / kSegSlots) - 1) & 1, s_abort));
                        if (ok) {
                            W[kWSegInfo + 4 * qs + 0] = pt;
                            W[kWSegInfo + 4 * qs + 1] = pkvh;
                            W[kWSegInfo + 4 * qs + 2] = pp;
                            W[kWSegInfo + 4 * qs + 3] = pnv;
                            __threadfence_block();
                            mbar_arrive_expect_tx(sm.qfull(qs), kQSlotBytes);
                            const int qrow = pt * a.num_q_heads + pkvh * G;
                            tma_load_2d(sm.qslot(qs), &tm_q, 0, qrow, sm.qfull(qs));
                            tma_load_2d(sm.qslot(qs) + kQHalf, &tm_q, 64, qrow, sm.qfull(qs));
                        } else {
                            *s_abort = 1;
                        }
                    }
                    __syncwarp();
                }
                // ---- the run's usable blocks, in unit order
                unsigned todo = __ballot_sync(0xffffffffu, in && lane >= lf && lane <= ll && blk >= 0);
                while (todo) {
                    const int src = __ffs(todo) - 1;
                    todo &= todo - 1;
                    const int ib = __shfl_sync(0xffffffffu, blk, src);
                    const int ipg = __shfl_sync(0xffffffffu, page, src);
                    if (lane == 0 && !*s_abort) {
                        const int st = item % kStages;
                        if (item >= kStages && !mbar_wait(sm.empty(st), ((item / kStages) - 1) & 1, s_abort)) {
                            *s_abort = 1;
                        } else {
                            W[kWItemBlk + st] = ib;
                            W[kWItemSeg + st] = seg;
                            __threadfence_block();
                            W[kWFill + st] = item;
                            const uint32_t dst = sm.stage(st);
                            mbar_arrive_expect_tx(sm.full(st), kStageBytes);
                            const int z = ipg;   // the tile's first row in the pool
                            tma_load_3d(dst, &tm_k, 0, pkvh, z, sm.full(st));
                            tma_load_3d(dst + kHalf, &tm_k, 64, pkvh, z, sm.full(st));
                            tma_load_3d(dst + 2 * kHalf, &tm_v, 0, pkvh, z, sm.full(st));
                            tma_load_3d(dst + 3 * kHalf, &tm_v, 64, pkvh, z, sm.full(st));
                        }
                    }
                    ++item;
                    __syncwarp();
                }
                if (run_end == seg_stop) {
                    // ---- segment end marker
                    if (lane == 0) {
                        const int qs = seg % kSegSlots;
                        W[kWSegEndCnt + qs] = item;
                        __threadfence_block();
                        W[kWSegEndTag + qs] = seg;
                    }
                    ++seg;
                }
                v = run_end;
            }
            stop = __shfl_sync(0xffffffffu, (int)*s_abort, 0) != 0;
        }
        err_bits = __reduce_or_sync(0xffffffffu, err_bits);
        if (lane == 0) {
            if (err_bits) set_err(a.dev_err, err_bits);
            if (*s_abort) {
                set_err(a.dev_err, DSA_DEV_ERR_WAIT);
                // let the copies already issued land before the CTA exits: the
                // last fill of each stage is the only one that can be in flight
                for (int st = 0; st < kStages; ++st) {
                    const int k = W[kWFill + st];
                    if (k >= 0) mbar_wait(sm.full(st), (k / kStages) & 1, s_never);
                }
            }
        }
        return;
    }

    // ==================================================================== consumer warps
    pdl_wait();
    const int g = lane >> 2, cq = lane & 3;
    float *s_mo = reinterpret_cast<float *>(gbase + P::kOffMergeO);   // [4][kMergeRows][kMergeStride]
    float *s_ml = reinterpret_cast<float *>(gbase + P::kOffMergeML);  // [4][16][2]

    unit_t u = u0;
    unit_t pair = u0 / K;
    int cursor = 0, seg = 0;
    while (u < u1) {
        const unit_t seg_begin = u;
        const unit_t seg_end = min(u1, (pair + 1) * K);
        const int qs = seg % kSegSlots;
        bool ok = !*s_abort && mbar_wait(sm.qfull(qs), (seg / kSegSlots) & 1, s_abort);
        if (!ok) *s_abort = 1;
        const int pt = W[kWSegInfo + 4 * qs + 0];
        const int pkvh = W[kWSegInfo + 4 * qs + 1];
        const int pp = W[kWSegInfo + 4 * qs + 2];
        const int pnv = W[kWSegInfo + 4 * qs + 3];

        // Q^T fragments (B operand of S^T = K Q^T): k = dims, n = query heads
        uint32_t qb[8][NT][2];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int kp = 0; kp < 4; ++kp) {
                qb[2 * kp][nt][0] = qb[2 * kp][nt][1] = qb[2 * kp + 1][nt][0] = qb[2 * kp + 1][nt][1] = 0u;
                if (ok) {
                    const int r = 8 * nt + (lane & 7);
                    const int ch = 4 * kp + (lane >> 3);
                    ldmatrix_x4(sm.qslot(qs) + (ch >> 3) * kQHalf + swz128(r, ch & 7), qb[2 * kp][nt][0],
                                qb[2 * kp][nt][1], qb[2 * kp + 1][nt][0], qb[2 * kp + 1][nt][1]);
                }
            }
        // O^T accumulators: dims 16*dm + g (+8) x heads 8*nt + 2*cq (+1)
        float o[8][NT][4];
        float m_run[NT][2], l_run[NT][2];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            m_run[nt][0] = m_run[nt][1] = -INFINITY;
            l_run[nt][0] = l_run[nt][1] = 0.f;
#pragma unroll
            for (int dm = 0; dm < 8; ++dm) o[dm][nt][0] = o[dm][nt][1] = o[dm][nt][2] = o[dm][nt][3] = 0.f;
        }

        // this warp's items of the segment: indices cursor.. with index % 4 == warp
        int ui = cursor + ((warp - cursor % kConsumerWarps) + kConsumerWarps) % kConsumerWarps;
        while (true) {
            const int st = ui % kStages;
            // wait for item ui to be armed, or for this segment to end before it
            bool done = false;
            const long long t0 = clock64();
            while (true) {
                if (W[kWFill + st] == ui) {
                    __threadfence_block();
                    done = W[kWItemSeg + st] != seg;   // armed for a later segment: this one is over
                    break;
                }
                if (W[kWSegEndTag + qs] == seg) {
                    __threadfence_block();
                    if (ui >= W[kWSegEndCnt + qs]) { done = true; break; }
                }
                if (*s_abort || clock64() - t0 > kWaitLimitCycles) { *s_abort = 1; done = true; break; }
            }
            __syncwarp();
            if (done) break;
            if (!mbar_wait(sm.full(st), (ui / kStages) & 1, s_abort)) {
                *s_abort = 1;
                break;
            }
            __syncwarp();
            const int blk = W[kWItemBlk + st];
            const uint32_t tk = sm.stage(st), tv = tk + 2 * kHalf;
            // the last visible token of this tile (only the query's own tile is partial)
            const int lim = (blk == pnv - 1) ? pp - blk * kBlockSize : kBlockSize - 1;
            if (lim < kBlockSize - 1) {
                // the slots past the query's position hold whatever the cache had
                // there (nothing appended yet); a zero softmax weight times a NaN
                // or infinite value is still NaN, so their value rows are cleared
                // (both 128-byte halves, 16-byte chunks at their swizzled place)
                for (int e = lane; e < (kBlockSize - 1 - lim) * 16; e += 32) {
                    const int r = lim + 1 + (e >> 4), cc = e & 15;
                    st_shared_zero16(tv + (cc >> 3) * kHalf + swz128(r, cc & 7));
                }
                __syncwarp();
            }
            // ---- S^T = K Q^T: 4 m-tiles of 16 tokens x NT n-tiles of 8 heads
            float sc[4][NT][4];
#pragma unroll
            for (int mt = 0; mt < 4; ++mt)
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) sc[mt][nt][0] = sc[mt][nt][1] = sc[mt][nt][2] = sc[mt][nt][3] = 0.f;
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                const int ch = 2 * kk + (lane >> 4);
                const uint32_t half = tk + (ch >> 3) * kHalf;
#pragma unroll
                for (int mt = 0; mt < 4; ++mt) {
                    const int r = 16 * mt + (lane & 7) + 8 * ((lane >> 3) & 1);
                    uint32_t ka[4];
                    ldmatrix_x4(half + swz128(r, ch & 7), ka[0], ka[1], ka[2], ka[3]);
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) mma_bf16_16816(sc[mt][nt], ka, qb[kk][nt][0], qb[kk][nt][1]);
                }
            }
            // ---- causal mask (own block only), scale, online softmax per head column
            float alpha[NT][2];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
                for (int mt = 0; mt < 4; ++mt)
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const int tok = 16 * mt + g + 8 * (k >> 1);
                        const float x = tok <= lim ? sc[mt][nt][k] * a.scale_log2 : -INFINITY;
                        sc[mt][nt][k] = x;
                        mx[k & 1] = fmaxf(mx[k & 1], x);
                    }
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 4));
                    mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 8));
                    mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 16));
                    const float m_new = fmaxf(m_run[nt][h], mx[h]);
                    alpha[nt][h] = (m_new == -INFINITY) ? 1.f : exp2f(m_run[nt][h] - m_new);
                    m_run[nt][h] = m_new;
                }
                float rs[2] = {0.f, 0.f};
#pragma unroll
                for (int mt = 0; mt < 4; ++mt)
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const float mr = m_run[nt][k & 1];
                        const float pv = (mr == -INFINITY) ? 0.f : exp2f(sc[mt][nt][k] - mr);
                        sc[mt][nt][k] = pv;
                        rs[k & 1] += pv;
                    }
                l_run[nt][0] = l_run[nt][0] * alpha[nt][0] + rs[0];
                l_run[nt][1] = l_run[nt][1] * alpha[nt][1] + rs[1];
#pragma unroll
                for (int dm = 0; dm < 8; ++dm) {
                    o[dm][nt][0] *= alpha[nt][0]; o[dm][nt][1] *= alpha[nt][1];
                    o[dm][nt][2] *= alpha[nt][0]; o[dm][nt][3] *= alpha[nt][1];
                }
            }
            // ---- O^T += V^T P^T: k-steps of 16 tokens; P^T fragments by movmatrix
#pragma unroll
            for (int mt = 0; mt < 4; ++mt) {
                uint32_t pb[NT][2];
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    pb[nt][0] = movmatrix_trans(pack_bf16x2(sc[mt][nt][0], sc[mt][nt][1]));
                    pb[nt][1] = movmatrix_trans(pack_bf16x2(sc[mt][nt][2], sc[mt][nt][3]));
                }
                const int r = 16 * mt + (lane & 7) + 8 * (lane >> 4);
#pragma unroll
                for (int dm = 0; dm < 8; ++dm) {
                    const int ch = 2 * dm + ((lane >> 3) & 1);
                    uint32_t va[4];
                    ldmatrix_x4_trans(tv + (ch >> 3) * kHalf + swz128(r, ch & 7), va[0], va[1], va[2], va[3]);
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) mma_bf16_16816(o[dm][nt], va, pb[nt][0], pb[nt][1]);
                }
            }
            // generic-proxy stores (the cleared rows) before the TMA refills the stage
            if (lim < kBlockSize - 1) asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            __syncwarp();
            if (lane == 0) mbar_arrive(sm.empty(st));
            ui += kConsumerWarps;
        }
        // the segment's item count (published by the producer before it moves on)
        {
            const long long t0 = clock64();
            while (W[kWSegEndTag + qs] != seg) {
                if (*s_abort || clock64() - t0 > kWaitLimitCycles) { *s_abort = 1; break; }
            }
            __threadfence_block();
        }
        const int next_cursor = W[kWSegEndTag + qs] == seg ? W[kWSegEndCnt + qs] : cursor;

        // ---- end of this pair's units in the CTA: merge the four warps' states
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                l_run[nt][h] += __shfl_xor_sync(0xffffffffu, l_run[nt][h], 4);
                l_run[nt][h] += __shfl_xor_sync(0xffffffffu, l_run[nt][h], 8);
                l_run[nt][h] += __shfl_xor_sync(0xffffffffu, l_run[nt][h], 16);
            }
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const int h0 = 8 * nt + 2 * cq;
            float *row0 = s_mo + (warp * P::kMergeRows + h0) * kMergeStride;
            float *row1 = row0 + kMergeStride;
#pragma unroll
            for (int dm = 0; dm < 8; ++dm) {
                const int d = 16 * dm + g;
                row0[d] = o[dm][nt][0];
                row1[d] = o[dm][nt][1];
                row0[d + 8] = o[dm][nt][2];
                row1[d + 8] = o[dm][nt][3];
            }
            if (g == 0) {
                s_ml[(warp * 16 + h0) * 2] = m_run[nt][0];
                s_ml[(warp * 16 + h0) * 2 + 1] = l_run[nt][0];
                s_ml[(warp * 16 + h0 + 1) * 2] = m_run[nt][1];
                s_ml[(warp * 16 + h0 + 1) * 2 + 1] = l_run[nt][1];
            }
        }
        __syncwarp();
        named_barrier(1, kConsumerWarps * 32);
        // every warp has read this slot's query tile, pair facts and end count
        if (tid == 0) mbar_arrive(sm.qempty(qs));

        const bool whole = seg_begin == pair * K && seg_end == (pair + 1) * K;
        const size_t out_row = (size_t)pt * a.num_q_heads + (size_t)pkvh * G;
        const int slot = 2 * c + (seg == 0 ? 0 : 1);
        if (a.cluster2) {
            // the two halves of the pair meet in rank 0's shared memory: rank 1
            // stores its merged state there and arrives on rank 0's inbox
            // barrier; rank 0 combines it with its own and writes the output
            constexpr int kRowsPT = 2 * NT;
            float Mo[kRowsPT], Lo[kRowsPT], Ao[kRowsPT][4];
#pragma unroll
            for (int i = 0; i < kRowsPT; ++i) {
                const int e = tid + i * kConsumerWarps * 32;
                const int r = (e >> 5) < G ? (e >> 5) : 0, d0 = (e & 31) * 4;
                float M = -INFINITY;
#pragma unroll
                for (int w = 0; w < kConsumerWarps; ++w) M = fmaxf(M, s_ml[(w * 16 + r) * 2]);
                float L = 0.f, acc[4] = {0.f, 0.f, 0.f, 0.f};
                if (M != -INFINITY) {
#pragma unroll
                    for (int w = 0; w < kConsumerWarps; ++w) {
                        const float f = exp2f(s_ml[(w * 16 + r) * 2] - M);
                        L += s_ml[(w * 16 + r) * 2 + 1] * f;
                        const float4 v =
                            *reinterpret_cast<const float4 *>(s_mo + (w * P::kMergeRows + r) * kMergeStride + d0);
                        acc[0] += v.x * f; acc[1] += v.y * f; acc[2] += v.z * f; acc[3] += v.w * f;
                    }
                }
                Mo[i] = M; Lo[i] = L;
                Ao[i][0] = acc[0]; Ao[i][1] = acc[1]; Ao[i][2] = acc[2]; Ao[i][3] = acc[3];
            }
            if (c & 1) {
                // asynchronous stores that complete their bytes on rank 0's inbox
                // barrier (armed with the full count before the cluster barrier)
                const uint32_t remote = mapa_shared(sm.inbox(), 0);
                const uint32_t remote_bar = mapa_shared(sm.inbox_full(), 0);
#pragma unroll
                for (int i = 0; i < kRowsPT; ++i) {
                    const int e = tid + i * kConsumerWarps * 32;
                    if (e >= G * 32) break;
                    const int r = e >> 5, d0 = (e & 31) * 4;
                    const uint32_t row = remote + (uint32_t)(r * kAttnPartStride * 4);
                    st_async_f32x4(row + d0 * 4, Ao[i][0], Ao[i][1], Ao[i][2], Ao[i][3], remote_bar);
                    if (d0 == 0) st_async_f32x2(row + 128 * 4, Mo[i], Lo[i], remote_bar);
                }
            } else {
                // the partner's state; the wait outlasts any bounded stall of the partner
                bool got = mbar_try_wait_cluster(sm.inbox_full(), 0);
                const long long t0 = clock64();
                while (!got && clock64() - t0 < 4 * kWaitLimitCycles) got = mbar_try_wait_cluster(sm.inbox_full(), 0);
                if (!got && tid == 0) {
                    *s_abort = 1;
                    set_err(a.dev_err, DSA_DEV_ERR_WAIT);
                }
                const float *inbox = reinterpret_cast<const float *>(gbase + P::kOffInbox);
#pragma unroll
                for (int i = 0; i < kRowsPT; ++i) {
                    const int e = tid + i * kConsumerWarps * 32;
                    if (e >= G * 32) break;
                    const int r = e >> 5, d0 = (e & 31) * 4;
                    float Mp = -INFINITY, Lp = 0.f;
                    float4 ap = make_float4(0.f, 0.f, 0.f, 0.f);
                    if (got) {
                        Mp = inbox[r * kAttnPartStride + 128];
                        Lp = inbox[r * kAttnPartStride + 129];
                        ap = *reinterpret_cast<const float4 *>(inbox + r * kAttnPartStride + d0);
                    }
                    const float Mn = fmaxf(Mo[i], Mp);
                    float L = 0.f, o0 = 0.f, o1 = 0.f, o2 = 0.f, o3 = 0.f;
                    if (Mn != -INFINITY) {
                        const float f0 = Mo[i] == -INFINITY ? 0.f : exp2f(Mo[i] - Mn);
                        const float f1 = Mp == -INFINITY ? 0.f : exp2f(Mp - Mn);
                        L = Lo[i] * f0 + Lp * f1;
                        o0 = Ao[i][0] * f0 + ap.x * f1; o1 = Ao[i][1] * f0 + ap.y * f1;
                        o2 = Ao[i][2] * f0 + ap.z * f1; o3 = Ao[i][3] * f0 + ap.w * f1;
                    }
                    const float inv = L > 0.f ? 1.f / L : 0.f;
                    *reinterpret_cast<uint2 *>(a.out + (out_row + r) * kHeadDim + d0) =
                        make_uint2(pack_bf16x2(o0 * inv, o1 * inv), pack_bf16x2(o2 * inv, o3 * inv));
                    if (a.lse && d0 == 0) a.lse[out_row + r] = L > 0.f ? (Mn + log2f(L)) * kLn2 : -INFINITY;
                }
            }
            __syncwarp();
            named_barrier(1, kConsumerWarps * 32);   // merge buffers free again
            cursor = next_cursor;
            u = seg_end;
            ++pair;
            ++seg;
            continue;
        }
        for (int e = tid; e < G * 32; e += kConsumerWarps * 32) {
            const int r = e >> 5, d0 = (e & 31) * 4;
            float M = -INFINITY;
#pragma unroll
            for (int w = 0; w < kConsumerWarps; ++w) M = fmaxf(M, s_ml[(w * 16 + r) * 2]);
            float L = 0.f, acc[4] = {0.f, 0.f, 0.f, 0.f};
            if (M != -INFINITY) {
#pragma unroll
                for (int w = 0; w < kConsumerWarps; ++w) {
                    const float f = exp2f(s_ml[(w * 16 + r) * 2] - M);
                    L += s_ml[(w * 16 + r) * 2 + 1] * f;
                    const float4 v = *reinterpret_cast<const float4 *>(s_mo + (w * P::kMergeRows + r) * kMergeStride + d0);
                    acc[0] += v.x * f; acc[1] += v.y * f; acc[2] += v.z * f; acc[3] += v.w * f;
                }
            }
            if (whole) {
                const float inv = L > 0.f ? 1.f / L : 0.f;
                *reinterpret_cast<uint2 *>(a.out + (out_row + r) * kHeadDim + d0) =
                    make_uint2(pack_bf16x2(acc[0] * inv, acc[1] * inv), pack_bf16x2(acc[2] * inv, acc[3] * inv));
                if (a.lse && d0 == 0) a.lse[out_row + r] = L > 0.f ? (M + log2f(L)) * kLn2 : -INFINITY;
            } else {
                float *dst = a.part + ((size_t)slot * G + r) * kAttnPartStride;
                *reinterpret_cast<float4 *>(dst + d0) = make_float4(acc[0], acc[1], acc[2], acc[3]);
                if (d0 == 0) { dst[128] = M; dst[129] = L; }
            }
        }
        if (!whole) {
            // publish the partial: the barrier orders every thread's stores
            // before thread 0's release-add on the pair's counter; the CTA that
            // completes the count acquires them all and merges.
            __syncwarp();
            named_barrier(1, kConsumerWarps * 32);
            if (tid == 0) {
                const int covered = (int)(seg_end - seg_begin);
                const int old = atomic_add_acq_rel_gpu(a.counters + pair, covered);
                W[kWLast] = (old + covered == (int)K);
            }
            __syncwarp();
            named_barrier(1, kConsumerWarps * 32);
            if (W[kWLast]) {
                // CTAs covering the pair: closed form from the split, then a
                // fix-up step in case of rounding
                // the pair's CTAs are this CTA's neighbours (ranges are contiguous)
                const unit_t p_lo = pair * K, p_hi = p_lo + K;
                int cf = c, cl = c;
                while (cf > 0 && s_rb[cf] > p_lo) --cf;
                while (cl + 1 < a.num_ctas && s_rb[cl + 1] < p_hi) ++cl;
                const int n_slots = min(cl - cf + 1, kMaxSplitSlots);
                // each thread owns kRowsPT (row, 4-column) pieces; the loads of
                // all of them and of a batch of slots are issued before any is
                // used, so the merge costs one L2 round trip per batch
                constexpr int kRowsPT = 2 * NT;                 // 8 * NT rows * 32 pieces / 128 threads
                constexpr int kBatch = NT == 1 ? 4 : 2;         // slots per round trip
                float M[kRowsPT], L[kRowsPT], acc[kRowsPT][4];
#pragma unroll
                for (int i = 0; i < kRowsPT; ++i) {
                    M[i] = -INFINITY;
                    L[i] = 0.f;
                    acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
                }
                for (int k0 = 0; k0 < n_slots; k0 += kBatch) {
                    float2 ml[kRowsPT][kBatch];
                    float4 ov[kRowsPT][kBatch];
#pragma unroll
                    for (int i = 0; i < kRowsPT; ++i) {
                        const int e = tid + i * kConsumerWarps * 32;
                        const int r = e >> 5, d0 = (e & 31) * 4;
#pragma unroll
                        for (int k = 0; k < kBatch; ++k) {
                            const int cc = cf + k0 + k;
                            if (e < G * 32 && k0 + k < n_slots) {
                                const int sl = 2 * cc + (s_rb[cc] >= p_lo ? 0 : 1);
                                const float *src = a.part + ((size_t)sl * G + r) * kAttnPartStride;
                                ml[i][k] = __ldcg(reinterpret_cast<const float2 *>(src + 128));
                                ov[i][k] = __ldcg(reinterpret_cast<const float4 *>(src + d0));
                            } else {
                                ml[i][k] = make_float2(-INFINITY, 0.f);
                                ov[i][k] = make_float4(0.f, 0.f, 0.f, 0.f);
                            }
                        }
                    }
#pragma unroll
                    for (int i = 0; i < kRowsPT; ++i) {
                        float Mn = M[i];
#pragma unroll
                        for (int k = 0; k < kBatch; ++k) Mn = fmaxf(Mn, ml[i][k].x);
                        if (Mn != -INFINITY) {
                            const float fo = M[i] == -INFINITY ? 0.f : exp2f(M[i] - Mn);   // rescale what we have
                            L[i] *= fo;
                            acc[i][0] *= fo; acc[i][1] *= fo; acc[i][2] *= fo; acc[i][3] *= fo;
#pragma unroll
                            for (int k = 0; k < kBatch; ++k) {
                                const float f = ml[i][k].x == -INFINITY ? 0.f : exp2f(ml[i][k].x - Mn);
                                L[i] += ml[i][k].y * f;
                                acc[i][0] += ov[i][k].x * f; acc[i][1] += ov[i][k].y * f;
                                acc[i][2] += ov[i][k].z * f; acc[i][3] += ov[i][k].w * f;
                            }
                            M[i] = Mn;
                        }
                    }
                }
#pragma unroll
                for (int i = 0; i < kRowsPT; ++i) {
                    const int e = tid + i * kConsumerWarps * 32;
                    if (e >= G * 32) break;
                    const int r = e >> 5, d0 = (e & 31) * 4;
                    const float inv = L[i] > 0.f ? 1.f / L[i] : 0.f;
                    *reinterpret_cast<uint2 *>(a.out + (out_row + r) * kHeadDim + d0) =
                        make_uint2(pack_bf16x2(acc[i][0] * inv, acc[i][1] * inv),
                                   pack_bf16x2(acc[i][2] * inv, acc[i][3] * inv));
                    if (a.lse && d0 == 0) a.lse[out_row + r] = L[i] > 0.f ? (M[i] + log2f(L[i])) * kLn2 : -INFINITY;
                }
                if (tid == 0) a.counters[pair] = 0;
            }
        }
        __syncwarp();
        named_barrier(1, kConsumerWarps * 32);   // merge buffers free again
        cursor = next_cursor;
        u = seg_end;
        ++pair;
        ++seg;
    }
    if constexpr (kFused) {
        // the last CTA to finish clears the per-call counters and advances the
        // epoch, which retires this call's ready flags
        named_barrier(1, kConsumerWarps * 32);
        if (tid == 0) {
            const int old = atomic_add_acq_rel_gpu(f.hdr + kHdrDone, 1);
            if (old == (int)gridDim.x - 1) {
                f.hdr[kHdrAppended] = 0;
                f.hdr[kHdrDone] = 0;
                fused::st_release(f.hdr + kHdrEpoch, tag);
            }
        }
    }
}

namespace {

using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                   const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

}  // namespace

namespace {
struct AttnMaps {
    CUtensorMap k, v, q;
};

cudaError_t encode_maps(const AttnArgs &a, AttnMaps &m);

// Encoded maps of the last few (pools, queries) a launch used: a decode loop
// calls with the same buffers every step, and encoding three maps costs host
// time on every call otherwise.  The key is everything the maps encode.
struct MapKey {
    int dev;
    const void *k, *v, *q;
    int num_pages, num_kv_heads, block_shift, total_q, num_q_heads;
    bool operator==(const MapKey &o) const {
        return dev == o.dev && k == o.k && v == o.v && q == o.q && num_pages == o.num_pages &&
               num_kv_heads == o.num_kv_heads && block_shift == o.block_shift && total_q == o.total_q &&
               num_q_heads == o.num_q_heads;
    }
};
constexpr int kMapCache = 16;
std::mutex g_map_mu;
MapKey g_map_keys[kMapCache];
AttnMaps g_map_vals[kMapCache];
int g_map_n = 0, g_map_next = 0;

cudaError_t make_maps(const AttnArgs &a, AttnMaps &m) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) dev = -1;
    const MapKey key{dev, a.k_pool, a.v_pool, a.q, a.num_pages, a.num_kv_heads, a.block_shift, a.total_q,
                     a.num_q_heads};
    {
        std::lock_guard<std::mutex> lock(g_map_mu);
        for (int i = 0; i < g_map_n; ++i)
            if (g_map_keys[i] == key) {
                m = g_map_vals[i];
                return cudaSuccess;
            }
    }
    const cudaError_t e = encode_maps(a, m);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lock(g_map_mu);
    g_map_keys[g_map_next] = key;
    g_map_vals[g_map_next] = m;
    g_map_next = (g_map_next + 1) % kMapCache;
    if (g_map_n < kMapCache) ++g_map_n;
    return cudaSuccess;
}

cudaError_t encode_maps(const AttnArgs &a, AttnMaps &m) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return cudaErrorNotSupported;
    // K / V pool: dims (head_dim, kv_head, page*B+token), boxes of 64 dims x 1 head x 64 tokens (one tile)
    const cuuint64_t dims[3] = {(cuuint64_t)kHeadDim, (cuuint64_t)a.num_kv_heads,
                                (cuuint64_t)a.num_pages << a.block_shift};
    const cuuint64_t strides[2] = {(cuuint64_t)kHeadDim * 2, (cuuint64_t)a.num_kv_heads * kHeadDim * 2};
    const cuuint32_t box[3] = {64, 1, kBlockSize};
    const cuuint32_t estr[3] = {1, 1, 1};
    if (enc(&m.k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<__nv_bfloat16 *>(a.k_pool), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    if (enc(&m.v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<__nv_bfloat16 *>(a.v_pool), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    // Q: rows (query, head), boxes of 64 dims x 16 rows; rows past the end read as zero
    const cuuint64_t qdims[2] = {(cuuint64_t)kHeadDim, (cuuint64_t)a.total_q * a.num_q_heads};
    const cuuint64_t qstr[1] = {(cuuint64_t)kHeadDim * 2};
    const cuuint32_t qbox[2] = {64, 16};
    if (enc(&m.q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<__nv_bfloat16 *>(a.q), qdims, qstr, qbox, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    return cudaSuccess;
}

// the shared-memory opt-in of every instantiation, once per device
cudaError_t set_smem_attrs() {
    static unsigned long long attr_done = 0;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 64 && (attr_done & (1ull << dev))) return cudaSuccess;
    e = cudaFuncSetAttribute(sparse_attn_kernel<1, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             Plan<1>::kSmemBytes);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(sparse_attn_kernel<2, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 Plan<2>::kSmemBytes);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(sparse_attn_kernel<1, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 Plan<1>::kSmemBytes);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(sparse_attn_kernel<2, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 Plan<2>::kSmemBytes);
    if (e != cudaSuccess) return e;
    if (dev < 64) attr_done |= 1ull << dev;
    return cudaSuccess;
}
}  // namespace

cudaError_t launch_sparse_attn(const AttnArgs &a, cudaStream_t stream) {
    if (a.total_q == 0 || a.num_ctas == 0) return cudaSuccess;
    AttnMaps m;
    cudaError_t e = make_maps(a, m);
    if (e == cudaSuccess) e = set_smem_attrs();
    if (e != cudaSuccess) return e;
    const FusedArgs none{};
    if (a.cluster2) {   // pairs of CTAs on one GPC, merging through distributed shared memory
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(a.num_ctas);
        cfg.blockDim = dim3(kAttnThreads);
        cfg.stream = stream;
        cudaLaunchAttribute attr[2];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        attr[1].id = cudaLaunchAttributeClusterDimension;
        attr[1].val.clusterDim.x = 2;
        attr[1].val.clusterDim.y = 1;
        attr[1].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 2;
        if (a.group <= 8) {
            cfg.dynamicSmemBytes = Plan<1>::kSmemBytes;
            return cudaLaunchKernelEx(&cfg, sparse_attn_kernel<1, false>, m.k, m.v, m.q, a, none);
        }
        cfg.dynamicSmemBytes = Plan<2>::kSmemBytes;
        return cudaLaunchKernelEx(&cfg, sparse_attn_kernel<2, false>, m.k, m.v, m.q, a, none);
    }
    if (a.group <= 8)
        return launch_pdl(sparse_attn_kernel<1, false>, dim3(a.num_ctas), dim3(kAttnThreads), Plan<1>::kSmemBytes,
                          stream, m.k, m.v, m.q, a, none);
    return launch_pdl(sparse_attn_kernel<2, false>, dim3(a.num_ctas), dim3(kAttnThreads), Plan<2>::kSmemBytes,
                      stream, m.k, m.v, m.q, a, none);
}

cudaError_t launch_decode_fused(const AttnArgs &a, const FusedArgs &f, cudaStream_t stream) {
    if (a.total_q == 0 || a.num_ctas == 0) return cudaSuccess;
    AttnMaps m;
    cudaError_t e = make_maps(a, m);
    if (e == cudaSuccess) e = set_smem_attrs();
    if (e != cudaSuccess) return e;
    // every CTA resident at once: the attention phase waits on selections
    // that other CTAs publish
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(a.num_ctas);
    cfg.blockDim = dim3(kAttnThreads);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (a.group <= 8) {
        cfg.dynamicSmemBytes = Plan<1>::kSmemBytes;
        return cudaLaunchKernelEx(&cfg, sparse_attn_kernel<1, true>, m.k, m.v, m.q, a, f);
    }
    cfg.dynamicSmemBytes = Plan<2>::kSmemBytes;
    return cudaLaunchKernelEx(&cfg, sparse_attn_kernel<2, true>, m.k, m.v, m.q, a, f);
}

}  // namespace dsa
