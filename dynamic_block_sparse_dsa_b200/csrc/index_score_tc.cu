// index_score_tc.cu -- block scores of the int8 indexer on the 5th-generation
// tensor cores (prefill: many queries per sequence).
//
// "Day-0 Adaptation for Massive LLMs: Overcoming Sparse Attention and MXFP4
// Expert Weights", section 4(1): score the compressed per-block representation
// against each query in one kernel, writing nothing but the scores;
// section 4(3): prefill is the compute-heavy phase.  "Day-0 Readiness for
// Trillion-Parameter Models ...", section "Index Selection Path": low-precision
// (int8) scoring.  The score is
//     S[t][b] = sum_h w[t][h] * max(0, q_idx[t][h] . kc[page(s,b)])
// exactly in int32 (the host checks the range bound).
//
// The dot products of a tile of 128 blocks and 16 queries x 16 indexer heads
// are one int8 contraction D[block][(query, head)] (M = 128, N = 256, K = 64),
// run with tcgen05.mma kind::i8 into a tensor-memory accumulator; the relu,
// head weights and head sum then happen in the epilogue, one block row per
// thread, straight from tensor memory.
//
// Work items are (128-block tile, 16-query tile) pairs in block-tile-major
// order, split evenly over one persistent CTA per SM, so a CTA keeps the same
// 128 coarse keys (the MMA's A operand, gathered through the block table) for
// many query tiles.  Per item only asynchronous copies remain: one 3-D TMA box
// of the 16 queries' rows (heads past H zero-filled) and one 2-D box of their
// head weights.  The CTA runs two independent pipelines, each on half of its
// items with its own ring, A buffers and one 256-column accumulator, because
// one loader warp's per-item chain (decide, wait for a stage, publish, issue
// the copies) paced a single pipeline.  Warps of pipeline p:
//   2p    loader.  It works through its items 32 at a time: the batch's query
//         positions arrive in shared memory a batch ahead (cp.async), every
//         lane then decides one item (its sequences, whether any of its blocks
//         is visible), and a short loop publishes the visible items into a
//         4-stage ring.  When the (sequence, block tile) changes it gathers the
//         new tile (64-byte swizzle) into one of two A buffers, once the items
//         still reading that buffer have finished;
//   2p+1  MMA issuer (one thread): two K = 32 MMAs per item into the
//         pipeline's 256-column accumulator;
//   4+8p .. 11+8p  epilogue: the two warps of each SM sub-partition take that
//         sub-partition's 32 rows and half of the queries each, in two rounds
//         of four queries: tcgen05.ld, after the second of which the
//         accumulator goes back to the MMA, then relu * w summed over heads and
//         one coalesced 128-byte store per (query, warp).  The other
//         pipeline's MMA and loads overlap this arithmetic.
// A query tile spanning several sequences runs once per sequence with the
// other queries masked; items past every query's own block are skipped.  All
// waits are bounded.
#include <cstddef>
#include <cstdint>

#include "dsa_kernels.h"
#include "dsa_tcgen05.cuh"

namespace dsa {

namespace {
constexpr int kPipes = 2;                          // independent pipelines per CTA
constexpr int kEpiWarps = 16;                      // four per SM sub-partition, eight per pipeline
constexpr int kPipeEpi = kEpiWarps / kPipes;
constexpr int kEpiWarp0 = 2 * kPipes;              // warps 2p and 2p + 1: pipeline p's loader and MMA
constexpr int kTcThreads = 32 * (2 * kPipes + kEpiWarps);
constexpr int kTcStages = 4;
constexpr int kBT = 128;                 // blocks per tile (MMA M)
constexpr int kQT = 16;                  // queries per tile (MMA N = 16 x 16 heads)
constexpr int kN = kQT * kMaxIdxHeads;   // 256
constexpr int kABytes = kBT * kIdxDim;   // 8 KiB
constexpr int kBBytes = kN * kIdxDim;    // 16 KiB
// stage: [B 16 KiB][weights 16 x 16 int32][info]
struct StageInfo {
    int bt, y;                           // block tile (-1: the end marker), query tile
    int abw;                             // A buffer | its fill number << 1
    int mask;                            // queries of the tile in this item's sequence (bit q)
    uint32_t vbits[kBT / 32];            // rows of the A tile with a usable page, per 32-row quarter
    int own_off, pad[3];                 // the queries' own blocks: int offset into the batch own buffer
};
constexpr int kOffW = kBBytes;
constexpr int kOffInfo = kOffW + kQT * kMaxIdxHeads * 4;
constexpr int kStageBytes = (kOffInfo + (int)sizeof(StageInfo) + 1023) / 1024 * 1024;
constexpr int kOffA = kTcStages * kStageBytes;           // [2][kABytes], 1 KiB aligned
constexpr int kOffBars = kOffA + 2 * kABytes;
// barriers: full[S], empty[S], tfull[2], tempty[2], afull[2]
constexpr int kNumBars = 2 * kTcStages + 6;
constexpr int kOffMisc = kOffBars + kNumBars * 8;   // tmem base, abort, never
constexpr int kSeqCache = 1024;                      // cu_q and seq_lens entries staged in shared memory
constexpr int kOffCuq = kOffMisc + 16;               // [kSeqCache] cu_q, then [kSeqCache] seq_lens
constexpr int kBatch = 32;                           // items decided together, one per lane
constexpr int kOffPos = kOffCuq + 2 * kSeqCache * 4; // [2][kBatch][kQT] int32 query positions
constexpr int kOffOwn = kOffPos + 2 * kBatch * kQT * 4;   // [2][kBatch][kQT] int32 own blocks
constexpr int kWBytes = kQT * kMaxIdxHeads * 4;      // one tile's head weights
// + alignment slack; at least 116 KiB so that two CTAs never share an SM (each
// holds all 512 tensor-memory columns)
// one such layout per pipeline, kPipeBytes apart (the shared words of kOffMisc
// are pipeline 0's)
constexpr int kPipeBytes = (kOffOwn + 2 * kBatch * kQT * 4 + 1023) / 1024 * 1024;
constexpr int kSmemUsed = kPipes * kPipeBytes + 1024;
constexpr int kSmemBytes = kSmemUsed > 116 * 1024 ? kSmemUsed : 116 * 1024;
// full barrier: the loader's arrival with the TMA bytes, plus 32 cp.async
// arrivals when the weights are copied by cp.async (H not a multiple of 4)
constexpr int kFullCountTma = 1;
constexpr int kFullCountCpAsync = 33;
constexpr int kAFullCount = 33;                      // the loader: 32 cp.async arrivals + one
constexpr int kEmptyCount = 1 + kPipeEpi;            // MMA commit + the pipeline's epilogue warps
constexpr uint32_t kTmemCols = 512;                  // one 256-column accumulator per pipeline
static_assert(kSmemBytes <= 227 * 1024, "shared memory");
static_assert(kOffA % 1024 == 0, "A buffers keep the 64-byte swizzle's 512-byte alignment");
static_assert(kOffPos % 16 == 0 && kOffOwn % 16 == 0, "positions and own blocks move in 16-byte pieces");
static_assert(kOffInfo % 16 == 0, "the stage info is written and read in 16-byte pieces");

struct Bars {
    uint32_t base;
    __device__ uint32_t full(int s) const { return base + kOffBars + 8 * s; }
    __device__ uint32_t empty(int s) const { return base + kOffBars + 8 * (kTcStages + s); }
    __device__ uint32_t tfull(int b) const { return base + kOffBars + 8 * (2 * kTcStages + b); }
    __device__ uint32_t tempty(int b) const { return base + kOffBars + 8 * (2 * kTcStages + 2 + b); }
    __device__ uint32_t afull(int b) const { return base + kOffBars + 8 * (2 * kTcStages + 4 + b); }
};

__device__ __forceinline__ int seq_of_query(const IndexScoreArgs &a, int t) { return find_seq(a.cu_q, a.num_seqs, t); }

// 4-byte asynchronous copy global -> shared (zero-filled when !valid)
__device__ __forceinline__ void cp_async_4(uint32_t dst, const void *src, bool valid) {
    if (valid) asm volatile("cp.async.ca.shared.global [%0], [%1], 4;\n" ::"r"(dst), "l"(src) : "memory");
    else asm volatile("cp.async.ca.shared.global [%0], [%1], 4, 0;\n" ::"r"(dst), "l"(src) : "memory");
}
// 16-byte asynchronous copy of which the first `nbytes` are read, the rest zero-filled
__device__ __forceinline__ void cp_async_16_n(uint32_t dst, const void *src, int nbytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src), "r"(nbytes) : "memory");
}
}  // namespace

__global__ void __launch_bounds__(kTcThreads, 1)
index_score_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_w,
                      IndexScoreArgs a, int n_bt, int n_qt, int w_tma) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t *g = smem_raw + (base - raw);
    // [0] tmem base, [1] abort, [2] never set (shared by both pipelines)
    volatile int *misc = reinterpret_cast<volatile int *>(g + kOffMisc);
    volatile int *s_abort = misc + 1;
    const volatile int *s_never = misc + 2;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    if (tid == 0) {
        for (int p = 0; p < kPipes; ++p) {
            const Bars bp{base + (uint32_t)(p * kPipeBytes)};
            for (int s = 0; s < kTcStages; ++s) {
                mbar_init(bp.full(s), w_tma ? kFullCountTma : kFullCountCpAsync);
                mbar_init(bp.empty(s), kEmptyCount);
            }
            mbar_init(bp.tfull(0), 1);
            mbar_init(bp.tempty(0), kPipeEpi);
            for (int b = 0; b < 2; ++b) mbar_init(bp.afull(b), kAFullCount);
        }
        misc[1] = 0;
        misc[2] = 0;
        fence_barrier_init();
    }
    if (warp == 1) {   // pipeline 0's MMA warp holds tensor memory for both
        tc::tmem_alloc(smem_u32(g + kOffMisc), kTmemCols);
        tc::tmem_relinquish();
    }
    pdl_trigger();
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = (uint32_t)misc[0];

    // item indices fit 32 bits (the host checks); only this split uses 64-bit products
    const unsigned n_items = (unsigned)n_bt * (unsigned)n_qt;
    const unsigned c0 = (unsigned)((unsigned long long)n_items * blockIdx.x / gridDim.x);
    const unsigned c1 = (unsigned)((unsigned long long)n_items * (blockIdx.x + 1) / gridDim.x);
    const int H = a.num_idx_heads;
    // the pipeline of this warp: the first or the second half of the CTA's items
    const int pipe = warp < kEpiWarp0 ? (warp >> 1) : (warp - kEpiWarp0) / kPipeEpi;
    const unsigned cmid = c0 + (c1 - c0 + 1) / 2;
    const unsigned i0 = pipe == 0 ? c0 : cmid, i1 = pipe == 0 ? cmid : c1;
    const uint32_t pbase = base + (uint32_t)(pipe * kPipeBytes);
    uint8_t *gp = g + pipe * kPipeBytes;
    const Bars bars{pbase};

    if (warp < kEpiWarp0 && !(warp & 1)) {
        // ============================================================ loader
        if (lane == 0) {
            prefetch_tensormap(&tm_q);
            if (w_tma) prefetch_tensormap(&tm_w);
        }
        int *s_cuq = reinterpret_cast<int *>(gp + kOffCuq);
        int *s_len = s_cuq + kSeqCache;
        const bool cached = a.num_seqs + 1 <= kSeqCache;
        if (cached) {
            for (int i = lane; i <= a.num_seqs; i += 32) s_cuq[i] = __ldg(a.cu_q + i);
            for (int i = lane; i < a.num_seqs; i += 32) s_len[i] = __ldg(a.seq_lens + i);
        }
        __syncwarp();
        auto seq_of = [&](int t) {
            if (!cached) return seq_of_query(a, t);
            int lo = 0, hi = a.num_seqs - 1;
            while (lo < hi) {
                const int mid = (lo + hi + 1) >> 1;
                if (s_cuq[mid] <= t) lo = mid; else hi = mid - 1;
            }
            return lo;
        };
        auto cu = [&](int s) { return cached ? s_cuq[s] : __ldg(a.cu_q + s); };
        auto seq_len = [&](int s) { return cached ? s_len[s] : __ldg(a.seq_lens + s); };
        // the query positions of items b0 .. b0+31 into buffer `buf` (16 bytes
        // per copy, zero past the last query); one commit group per batch
        int *s_posb = reinterpret_cast<int *>(gp + kOffPos);
        const uint32_t s_posb_u32 = smem_u32(s_posb);
        auto fetch_batch = [&](unsigned b0, int buf) {
#pragma unroll
            for (int c = lane; c < kBatch * 4; c += 32) {
                const unsigned j = b0 + (unsigned)(c >> 2);
                if (j < i1) {
                    const unsigned bt = j / (unsigned)n_qt;
                    const int t = kQT * (int)(j - bt * (unsigned)n_qt) + 4 * (c & 3);
                    const int n = min(max(a.total_q - t, 0), 4);
                    cp_async_16_n(s_posb_u32 + (uint32_t)(((buf * kBatch + (c >> 2)) * kQT + 4 * (c & 3)) * 4),
                                  a.q_pos + (n > 0 ? t : 0), 4 * n);
                }
            }
            cp_async_commit();
        };
        {
            // warm the L2 with what the first items read while a preceding kernel
            // may still run (prefetches only: nothing is read before the wait):
            // the first batch's positions, the first query tiles and weights, and
            // the first block tile's table entries
            const unsigned j = i0 + (unsigned)lane;
            if (j < i1) {
                const unsigned bt = j / (unsigned)n_qt;
                const int y = (int)(j - bt * (unsigned)n_qt);
                prefetch_l2_line(a.q_pos + kQT * y);
                if (lane < kTcStages) {
                    tma_prefetch_3d(&tm_q, 0, 0, kQT * y);
                    if (w_tma) tma_prefetch_2d(&tm_w, 0, kQT * y);
                }
            }
            const unsigned bt0 = i0 / (unsigned)n_qt;
            const int s0 = seq_of(kQT * (int)(i0 - bt0 * (unsigned)n_qt));
            if (lane < kBT * 4 / 128 && (int)bt0 * kBT + 32 * lane < a.max_blocks)
                prefetch_l2_line(a.block_table + (size_t)s0 * a.max_blocks + bt0 * kBT + 32 * lane);
        }
        pdl_wait();   // coarse keys may come from the preceding append
        fetch_batch(i0, 0);
        fetch_batch(i0 + kBatch, 1);
        int *s_own = reinterpret_cast<int *>(gp + kOffOwn);
        int k = 0;          // items published
        int a_s = -1, a_bt = -1, ab = 1;
        int agen0 = 0, agen1 = 0, alast0 = -1, alast1 = -1;   // per A buffer: fill number, last item
        uint32_t vb0[kBT / 32] = {0, 0, 0, 0}, vb1[kBT / 32] = {0, 0, 0, 0};   // per A buffer: valid rows
        int olast0 = 0, olast1 = 0;   // per own buffer: items published from it so far (exclusive end)
        uint32_t err_bits = 0;
        bool stop = false;
        int pbuf = 0;
        // Until the items before `end` are finished (false on abort).  Item j is
        // finished when its stage's empty barrier completes the phase of j: the
        // epilogue warps take items in order, so every earlier item is finished
        // too.  Only items already published are asked for; a phase of item j
        // cannot be confused with item j + 4's, which waits for this very
        // barrier before it is published (j < k - 4 is known finished already).
        int k_seen = -1;   // the latest item known to be finished
        // The pipeline's epilogue warps take its items in order, so item j
        // finished means every item before it is (the wait on j - 1 as well
        // costs nothing then).  When item k is published, item k - 5 is known
        // finished (the wait for item k - 1's stage), so neither wait below can
        // meet a reused stage's later phase.
        auto wait_done = [&](int end) {
            const int j = end - 1;
            if (j <= k_seen) return true;
            if (!mbar_wait(bars.empty(j & (kTcStages - 1)), (j / kTcStages) & 1, s_abort) ||
                (j - 1 > k_seen && j >= 1 &&
                 !mbar_wait(bars.empty((j - 1) & (kTcStages - 1)), ((j - 1) / kTcStages) & 1, s_abort))) {
                *s_abort = 1;
                return false;
            }
            k_seen = j;
            return true;
        };
        for (unsigned b0 = i0; b0 < i1 && !stop; b0 += kBatch, pbuf ^= 1) {
            cp_async_wait<1>();   // this batch's positions (the next batch may still be in flight)
            __syncwarp();
            const int *posb = s_posb + pbuf * kBatch * kQT;
            int *ownb = s_own + pbuf * kBatch * kQT;
            // the own buffer is free once the items published from it two batches ago are done
            if (!wait_done(pbuf ? olast1 : olast0)) break;
            // ---- decisions: lane L takes item b0 + L
            int d_bt = 0, d_y = 0, d_slo = 0, d_shi = -1, d_len = 0, d_vis = 0;
            {
                const unsigned my = b0 + (unsigned)lane;
                if (my < i1) {
                    d_bt = (int)(my / (unsigned)n_qt);
                    d_y = (int)(my - (unsigned)d_bt * (unsigned)n_qt);
                    const int t0 = kQT * d_y, tn = min(t0 + kQT, a.total_q);
                    d_slo = seq_of(t0);
                    d_shi = seq_of(tn - 1);
                    if (d_slo == d_shi) {
                        // one sequence: visible when a member's own block reaches the tile
                        d_len = seq_len(d_slo);
                        const int4 *pp = reinterpret_cast<const int4 *>(posb + lane * kQT);
                        int4 *po = reinterpret_cast<int4 *>(ownb + lane * kQT);
                        int mx = -1;
                        bool bad = false;
                        auto take = [&](int pos, int t) {
                            int own = -1;
                            if (t < tn) {
                                own = pos >> a.block_shift;
                                if (pos < 0 || pos >= d_len || own >= a.max_blocks) {
                                    bad = true;
                                    own = -1;
                                }
                                mx = max(mx, own);
                            }
                            return own;
                        };
#pragma unroll
                        for (int v = 0; v < 4; ++v) {
                            const int4 p = pp[v];
                            int4 o;
                            o.x = take(p.x, t0 + 4 * v);
                            o.y = take(p.y, t0 + 4 * v + 1);
                            o.z = take(p.z, t0 + 4 * v + 2);
                            o.w = take(p.w, t0 + 4 * v + 3);
                            po[v] = o;
                        }
                        if (bad) err_bits |= DSA_DEV_ERR_POS;
                        d_vis = mx >= d_bt * kBT;
                    } else {
                        d_vis = 1;   // several sequences: decided per sequence below
                    }
                }
            }
            // ---- publish the batch's visible items in order
            const int n_here = (int)min((unsigned)kBatch, i1 - b0);
            for (int i = 0; i < n_here && !stop; ++i) {
                if (!__shfl_sync(0xffffffffu, d_vis, i)) continue;
                const int bt = __shfl_sync(0xffffffffu, d_bt, i);
                const int y = __shfl_sync(0xffffffffu, d_y, i);
                const int s_lo = __shfl_sync(0xffffffffu, d_slo, i);
                const int s_hi = __shfl_sync(0xffffffffu, d_shi, i);
                const bool single = s_lo == s_hi;
                const int t0 = kQT * y;
                for (int s = s_lo; s <= s_hi; ++s) {
                    int mask = 0xffff;
                    if (!single) {
                        // several sequences: this sequence's queries, their own blocks
                        const int t = t0 + (lane & (kQT - 1));
                        const int pos = posb[i * kQT + (lane & (kQT - 1))];
                        const int len = seq_len(s);
                        const bool member = lane < kQT && t < a.total_q && cu(s) <= t && t < cu(s + 1);
                        int own = -1;
                        if (member) {
                            own = pos >> a.block_shift;
                            if (pos < 0 || pos >= len || own >= a.max_blocks) {
                                err_bits |= DSA_DEV_ERR_POS;
                                own = -1;
                            }
                            ownb[i * kQT + lane] = own;
                        }
                        mask = (int)__ballot_sync(0xffffffffu, member);
                        if (__reduce_max_sync(0xffffffffu, own) < bt * kBT) continue;   // nothing visible
                    }
                    if (s != a_s || bt != a_bt) {
                        // a new block tile: into the other A buffer once the items
                        // still reading it have all finished
                        a_s = s;
                        a_bt = bt;
                        ab ^= 1;
                        if (!wait_done((ab ? alast1 : alast0) + 1)) {
                            stop = true;
                            break;
                        }
                        if (ab) ++agen1; else ++agen0;
                        const int len = single ? __shfl_sync(0xffffffffu, d_len, i) : seq_len(s);
                        const int n_blocks = (len + (1 << a.block_shift) - 1) >> a.block_shift;
                        const int32_t *row = a.block_table + (size_t)s * a.max_blocks;
                        int page[kBT / 32];
#pragma unroll
                        for (int j = 0; j < kBT / 32; ++j) {   // rows 32 j + lane
                            const int b = bt * kBT + 32 * j + lane;
                            page[j] = b < n_blocks && b < a.max_blocks ? __ldg(row + b) : -1;
                        }
                        const uint32_t sa = pbase + kOffA + ab * kABytes;
#pragma unroll
                        for (int j = 0; j < kBT / 32; ++j) {
                            const int b = bt * kBT + 32 * j + lane;
                            if (b < n_blocks && b < a.max_blocks && (page[j] < 0 || page[j] >= a.num_pages)) {
                                err_bits |= DSA_DEV_ERR_PAGE;
                                page[j] = -1;
                            }
                            const uint32_t bits = __ballot_sync(0xffffffffu, page[j] >= 0);
                            if (ab) vb1[j] = bits; else vb0[j] = bits;
                            const int r = 32 * j + lane;
                            const int8_t *src = a.kc_pool + (size_t)max(page[j], 0) * kIdxDim;
#pragma unroll
                            for (int c = 0; c < 4; ++c) {
                                const uint32_t dst = sa + r * 64 + ((c ^ ((r >> 1) & 3)) << 4);
                                if (page[j] >= 0) cp_async_16(dst, src + 16 * c);
                                else cp_async_16_zero(dst, a.kc_pool);
                            }
                        }
                        tc::cp_async_arrive_noinc(bars.afull(ab));
                        __syncwarp();
                        if (lane == 0) mbar_arrive(bars.afull(ab));
                    }
                    if (ab) alast1 = k; else alast0 = k;
                    const int st = k & (kTcStages - 1);
                    if (k >= kTcStages && !wait_done(k - kTcStages + 1)) {   // the stage's previous item
                        stop = true;
                        break;
                    }
                    const uint32_t sb = pbase + st * kStageBytes;
                    if (!w_tma) {
                        // the tile's head weights (16 queries x 16 heads, zero past H and the last query)
#pragma unroll
                        for (int j = 0; j < 8; ++j) {
                            const int e = lane + 32 * j, qi = e / kMaxIdxHeads, h = e % kMaxIdxHeads;
                            const bool ok = t0 + qi < a.total_q && h < H;
                            cp_async_4(sb + kOffW + 4 * e, a.w + (ok ? (size_t)(t0 + qi) * H + h : 0), ok);
                        }
                        tc::cp_async_arrive_noinc(bars.full(st));
                    }
                    __syncwarp();   // the own blocks written above, before the release arrival
                    if (lane == 0) {
                        int4 *info = reinterpret_cast<int4 *>(gp + st * kStageBytes + kOffInfo);
                        info[0] = make_int4(bt, y, ab | ((ab ? agen1 : agen0) << 1), mask);
                        info[1] = ab ? make_int4((int)vb1[0], (int)vb1[1], (int)vb1[2], (int)vb1[3])
                                     : make_int4((int)vb0[0], (int)vb0[1], (int)vb0[2], (int)vb0[3]);
                        info[2].x = (pbuf * kBatch + i) * kQT;
                        // the queries' rows: box (64 B, 16 heads, 16 queries) at query t0, and
                        // their weights: box (16 heads, 16 queries), zero past H and the last query
                        mbar_arrive_expect_tx(bars.full(st), kBBytes + (w_tma ? kWBytes : 0));
                        tma_load_3d(sb, &tm_q, 0, 0, t0, bars.full(st));
                        if (w_tma) tma_load_2d(sb + kOffW, &tm_w, 0, t0, bars.full(st));
                    }
                    ++k;
                }
            }
            if (pbuf) olast1 = k; else olast0 = k;
            // every lane is done with this batch's positions: refill the buffer
            __syncwarp();
            fetch_batch(b0 + 2 * kBatch, pbuf);
            if (*s_abort) stop = true;
        }
        // the end marker (the pipeline's epilogue warps all read every item)
        for (int e = 0; e < 1 && !stop && !*s_abort; ++e) {
            const int st = k & (kTcStages - 1);
            if (k >= kTcStages && !mbar_wait(bars.empty(st), ((k / kTcStages) - 1) & 1, s_abort)) {
                *s_abort = 1;
            } else {
                StageInfo *info = reinterpret_cast<StageInfo *>(gp + st * kStageBytes + kOffInfo);
                if (lane == 0) info->bt = -1;
                if (!w_tma) tc::cp_async_arrive_noinc(bars.full(st));
                __syncwarp();
                if (lane == 0) mbar_arrive(bars.full(st));
                ++k;
            }
        }
        err_bits = __reduce_or_sync(0xffffffffu, err_bits);
        if (lane == 0 && err_bits) set_err(a.dev_err, err_bits);
        cp_async_commit();
        cp_async_wait<0>();
        if (*s_abort && lane == 0) {
            set_err(a.dev_err, DSA_DEV_ERR_WAIT);
            for (int j = max(0, k - kTcStages); j < k; ++j)
                mbar_wait(bars.full(j % kTcStages), (j / kTcStages) & 1, s_never);
        }
    } else if (warp < kEpiWarp0) {
        // ============================================================ MMA issuer
        constexpr uint32_t idesc = tc::idesc_i8(kBT, kN);
        int k = 0;
        while (true) {
            const int st = k % kTcStages;
            bool ok = mbar_wait(bars.full(st), (k / kTcStages) & 1, s_abort);
            const StageInfo *info = reinterpret_cast<const StageInfo *>(gp + st * kStageBytes + kOffInfo);
            const bool end = ok && info->bt < 0;
            const int abw = ok ? info->abw : 0;
            if (ok && !end) ok = mbar_wait(bars.afull(abw & 1), ((abw >> 1) - 1) & 1, s_abort);
            // the accumulator's previous item has been read (the end marker's
            // arrival on tfull must not run two phases ahead of the epilogue)
            if (ok && k >= 1) ok = mbar_wait(bars.tempty(0), (k - 1) & 1, s_abort);
            if (!ok) {
                if (lane == 0) *s_abort = 1;
                break;
            }
            if (lane == 0) {
                if (end) {
                    mbar_arrive(bars.tfull(0));   // wake the epilogue to see the end marker
                } else {
                    tc::fence_proxy_async_smem();   // the cp.async-written keys, for the tensor core
                    tc::fence_after_sync();
                    const uint32_t sa = pbase + kOffA + (abw & 1) * kABytes;
                    const uint32_t sb = pbase + st * kStageBytes;
                    const uint32_t d = tmem + (uint32_t)(pipe * kN);
                    const uint64_t da = tc::smem_desc_k64_sw64(sa), db = tc::smem_desc_k64_sw64(sb);
                    tc::mma_i8(d, da, db, idesc, false);
                    tc::mma_i8(d, da + (32 >> 4), db + (32 >> 4), idesc, true);   // K bytes 32..63
                    tc::commit(bars.empty(st));
                    tc::commit(bars.tfull(0));
                }
            }
            __syncwarp();
            ++k;
            if (end) break;
        }
        // the last MMAs have completed before the accumulator is released
        if (lane == 0 && k > 0) {
            const int j = k - 1;
            mbar_wait(bars.tfull(0), j & 1, s_never);
        }
    } else {
        // ============================================================ epilogue
        // the pipeline's 8 warps take each of its items; the two warps of a
        // sub-partition take the 32 rows that sub-partition can read and half
        // of the 16 queries each, in two rounds of 4 queries (64 accumulator
        // columns of the pipeline's accumulator)
        const int ew = warp - kEpiWarp0;
        const int quarter = warp & 3;            // TMEM lanes 32*quarter .. +31
        const int half = (ew >> 2) & 1;          // queries 8*half .. +7
        const int row = quarter * 32 + lane;     // block row of the tile
        const int *s_own_e = reinterpret_cast<const int *>(gp + kOffOwn);
        int k = 0;
        while (true) {
            const int st = k % kTcStages;
            bool ok = mbar_wait(bars.tfull(0), k & 1, s_abort) &&
                      mbar_wait(bars.full(st), (k / kTcStages) & 1, s_abort);   // acquire the info words
            if (!ok) {
                if (lane == 0) *s_abort = 1;
                break;
            }
            tc::fence_after_sync();
            const StageInfo *info = reinterpret_cast<const StageInfo *>(gp + st * kStageBytes + kOffInfo);
            const int4 i0w = *reinterpret_cast<const int4 *>(info);
            if (i0w.x < 0) break;   // the end marker
            const int bt = i0w.x, y = i0w.y, mask = i0w.w;
            const int b = bt * kBT + row;
            const bool row_ok = (info->vbits[quarter] >> lane) & 1u;
            uint32_t v[2][32];
#pragma unroll
            for (int rnd = 0; rnd < 2; ++rnd) {
                const int qgrp = 2 * half + rnd;   // queries 4*qgrp .. +3 (columns 64*qgrp ..)
                const uint32_t taddr =
                    tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(pipe * kN + qgrp * 64);
                tc::ld_32x32b_x32(taddr, v[0]);
                tc::ld_32x32b_x32(taddr + 32, v[1]);
                tc::wait_ld();
                if (rnd == 1) {
                    // the accumulator is all in registers: release it to the next MMA
                    tc::fence_before_sync();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(bars.tempty(0));
                }
                const int4 o4 = *reinterpret_cast<const int4 *>(s_own_e + info->own_off + 4 * qgrp);
                const int own4[4] = {(mask >> (4 * qgrp)) & 1 ? o4.x : -1, (mask >> (4 * qgrp + 1)) & 1 ? o4.y : -1,
                                     (mask >> (4 * qgrp + 2)) & 1 ? o4.z : -1, (mask >> (4 * qgrp + 3)) & 1 ? o4.w : -1};
                const int4 *w4 = reinterpret_cast<const int4 *>(gp + st * kStageBytes + kOffW) + qgrp * kMaxIdxHeads;
#pragma unroll
                for (int u = 0; u < 4; ++u) {   // query 4*qgrp + u: columns 16u .. 16u+15 of these 64
                    const uint32_t *x = v[u >> 1] + 16 * (u & 1);
                    int part[4];
#pragma unroll
                    for (int h4 = 0; h4 < 4; ++h4) {   // four independent chains
                        const int4 wv = w4[u * (kMaxIdxHeads / 4) + h4];
                        part[h4] = wv.x * max((int)x[4 * h4 + 0], 0) + wv.y * max((int)x[4 * h4 + 1], 0) +
                                   wv.z * max((int)x[4 * h4 + 2], 0) + wv.w * max((int)x[4 * h4 + 3], 0);
                    }
                    const int sum = (part[0] + part[1]) + (part[2] + part[3]);
                    if (row_ok && b <= own4[u])
                        a.scores[(size_t)(kQT * y + 4 * qgrp + u) * a.max_blocks + b] = sum;
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(bars.empty(st));   // the stage (info, weights, own blocks) is read
            ++k;
        }
    }

    tc::fence_before_sync();
    __syncthreads();
    if (warp == 1) {
        tc::fence_after_sync();
        tc::tmem_dealloc(tmem, kTmemCols);
    }
}

namespace {
using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                   const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn tc_encode_fn() {
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

int index_score_tc_min_queries_per_seq() { return 16; }

cudaError_t launch_index_score_tc(const IndexScoreArgs &a, int num_sms, cudaStream_t stream) {
    if (a.total_q == 0 || a.num_seqs == 0) return cudaSuccess;
    EncodeTiledFn enc = tc_encode_fn();
    if (!enc) return cudaErrorNotSupported;
    // q_idx as (64 bytes, head, query); boxes of 64 B x 16 heads x 16 queries,
    // zero-filled past H heads and past the last query
    CUtensorMap tq;
    const cuuint64_t dims[3] = {(cuuint64_t)kIdxDim, (cuuint64_t)a.num_idx_heads, (cuuint64_t)a.total_q};
    const cuuint64_t strides[2] = {(cuuint64_t)kIdxDim, (cuuint64_t)a.num_idx_heads * kIdxDim};
    const cuuint32_t box[3] = {kIdxDim, kMaxIdxHeads, kQT};
    const cuuint32_t estr[3] = {1, 1, 1};
    if (enc(&tq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<int8_t *>(a.q_idx), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    // head weights as (head, query) int32 boxes of 16 x 16 when a row is a whole
    // number of 16-byte units (H % 4 == 0) and the base is 16-byte aligned;
    // otherwise the kernel copies them with cp.async
    CUtensorMap tw = tq;
    int w_tma = 0;
    if (a.num_idx_heads % 4 == 0 && (reinterpret_cast<uintptr_t>(a.w) & 15) == 0) {
        const cuuint64_t wdims[2] = {(cuuint64_t)a.num_idx_heads, (cuuint64_t)a.total_q};
        const cuuint64_t wstrides[1] = {(cuuint64_t)a.num_idx_heads * 4};
        const cuuint32_t wbox[2] = {kMaxIdxHeads, kQT};
        const cuuint32_t westr[2] = {1, 1};
        if (enc(&tw, CU_TENSOR_MAP_DATA_TYPE_INT32, 2, const_cast<int32_t *>(a.w), wdims, wstrides, wbox, westr,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS)
            w_tma = 1;
    }
    static unsigned long long attr_done = 0;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev >= 64 || !(attr_done & (1ull << dev))) {
        e = cudaFuncSetAttribute(index_score_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
        if (e != cudaSuccess) return e;
        if (dev < 64) attr_done |= 1ull << dev;
    }
    const int n_bt = (a.max_blocks + kBT - 1) / kBT;
    const int n_qt = (a.total_q + kQT - 1) / kQT;   // items (bt, y), block-tile-major
    const long long items = (long long)n_bt * n_qt;
    if (items >= (1LL << 31)) return cudaErrorInvalidValue;   // item indices are 32-bit in the kernel
    const int grid = (int)(items < num_sms ? items : num_sms);
    return launch_pdl(index_score_tc_kernel, dim3(grid), dim3(kTcThreads), (size_t)kSmemBytes, stream, tq, tw, a, n_bt,
                      n_qt, w_tma);
}

}  // namespace dsa
