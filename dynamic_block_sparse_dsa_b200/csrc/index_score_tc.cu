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
// thread, straight from tensor memory.  One persistent CTA per SM, 6 warps:
//   warp 0   loader: the tile's 128 coarse keys gathered through the block
//            table (cp.async, 64-byte swizzle; the page ids themselves
//            copied a few tiles ahead) and the 16 queries' rows (one 3-D TMA
//            box, heads past H zero-filled), plus the queries' own blocks and
//            weights, into a 4-stage ring;
//   warp 1   MMA issuer (one thread): two K=32 MMAs per tile into one of two
//            256-column accumulators;
//   warps 2-17 epilogue (four per SM sub-partition: a quarter of the rows and
//            a quarter of the queries each): tcgen05.ld of the accumulator rows,
//            relu * w summed over heads, one coalesced 128-byte store per
//            (query, warp).
// Tiles are (16-query tile, 128-block tile) pairs in query-tile-major order,
// split evenly over the CTAs; a tile whose queries belong to several
// sequences is run once per sequence with the other queries masked.  Tiles
// past every query's own block are skipped.  All waits are bounded.
#include <cstddef>

#include "dsa_kernels.h"
#include "dsa_tcgen05.cuh"

namespace dsa {

namespace {
constexpr int kEpiWarps = 16;                      // four per SM sub-partition
constexpr int kLoadWarps = 4;                      // one gathered row per lane
constexpr int kMmaWarp = kLoadWarps;
constexpr int kEpiWarp0 = kLoadWarps + 1;
constexpr int kTcThreads = 32 * (kLoadWarps + 1 + kEpiWarps);   // loaders, MMA, epilogue
constexpr int kTcStages = 4;
constexpr int kBT = 128;                 // blocks per tile (MMA M)
constexpr int kQT = 16;                  // queries per tile (MMA N = 16 x 16 heads)
constexpr int kN = kQT * kMaxIdxHeads;   // 256
constexpr int kABytes = kBT * kIdxDim;   // 8 KiB
constexpr int kBBytes = kN * kIdxDim;    // 16 KiB
// stage: [A 8 KiB][B 16 KiB][info]
struct StageInfo {
    int bt, y, qslot, end;               // block tile, query tile, its facts slot; end marker
    uint32_t valid[kBT / 32];            // rows with a usable page
};
// facts of a (query tile, sequence): written once per change into a ring of
// kQSlots (a slot is rewritten only after every tile using it has finished)
struct QueryFacts {
    int own[kQT];                        // own block of each query of the tile in the sequence, else -1
    int w[kQT][kMaxIdxHeads];            // head weights (0 past H)
};
constexpr int kQSlots = 5;               // > kTcStages: see the loader
constexpr int kOffB = kABytes;
constexpr int kOffInfo = kABytes + kBBytes;
constexpr int kStageBytes = (kOffInfo + (int)sizeof(StageInfo) + 1023) / 1024 * 1024;
constexpr int kOffBars = kTcStages * kStageBytes;
// barriers: full[S], empty[S], tfull[2], tempty[2]
constexpr int kNumBars = 2 * kTcStages + 4;
constexpr int kOffMisc = kOffBars + kNumBars * 8;   // tmem base, abort flag
constexpr int kCuqCache = 1024;                      // cu_q entries staged in shared memory
constexpr int kOffCuq = kOffMisc + 16;
constexpr int kOffFacts = kOffCuq + kCuqCache * 4;   // [kQSlots] QueryFacts (16-byte aligned)
constexpr int kPidDepth = 4;                         // block tiles of page ids in flight
// + alignment slack; at least 116 KiB so that two CTAs never share an SM (each
// holds all 512 tensor-memory columns)
constexpr int kSmemUsed = kOffFacts + kQSlots * (int)sizeof(QueryFacts) + 1024;
constexpr int kSmemBytes = kSmemUsed > 116 * 1024 ? kSmemUsed : 116 * 1024;
constexpr int kFullCount = kLoadWarps * 33;          // per loader warp: 32 cp.async arrivals + its info arrival
constexpr int kEmptyCount = 1 + kEpiWarps;           // MMA commit + the epilogue warps
constexpr uint32_t kTmemCols = 512;                  // two 256-column accumulators
static_assert(kSmemBytes <= 227 * 1024, "shared memory");

struct Bars {
    uint32_t base;
    __device__ uint32_t full(int s) const { return base + kOffBars + 8 * s; }
    __device__ uint32_t empty(int s) const { return base + kOffBars + 8 * (kTcStages + s); }
    __device__ uint32_t tfull(int b) const { return base + kOffBars + 8 * (2 * kTcStages + b); }
    __device__ uint32_t tempty(int b) const { return base + kOffBars + 8 * (2 * kTcStages + 2 + b); }
};

__device__ __forceinline__ int seq_of_query(const IndexScoreArgs &a, int t) { return find_seq(a.cu_q, a.num_seqs, t); }
}  // namespace

__global__ void __launch_bounds__(kTcThreads, 1)
index_score_tc_kernel(const __grid_constant__ CUtensorMap tm_q, IndexScoreArgs a, int n_bt, int n_qt) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t *g = smem_raw + (base - raw);
    Bars bars{base};
    volatile int *misc = reinterpret_cast<volatile int *>(g + kOffMisc);   // [0] tmem base, [1] abort, [2] never
    volatile int *s_abort = misc + 1;
    const volatile int *s_never = misc + 2;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    if (tid == 0) {
        for (int s = 0; s < kTcStages; ++s) {
            mbar_init(bars.full(s), kFullCount);
            mbar_init(bars.empty(s), kEmptyCount);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(bars.tfull(b), 1);
            mbar_init(bars.tempty(b), kEpiWarps);
        }
        misc[1] = 0;
        misc[2] = 0;
        fence_barrier_init();
    }
    if (warp == kMmaWarp) {
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
    const unsigned i0 = (unsigned)((unsigned long long)n_items * blockIdx.x / gridDim.x);
    const unsigned i1 = (unsigned)((unsigned long long)n_items * (blockIdx.x + 1) / gridDim.x);
    const int H = a.num_idx_heads;

    if (warp < kLoadWarps) {
        // ============================================================ loaders
        const int lw = warp;   // rows 32*lw .. 32*lw+31 of every tile
        // Items are (query tile y, block tile bt), y-major: the queries'
        // positions and weights change once per query tile, the coarse keys
        // every item.  The page ids of item j are loaded into a register ring
        // kPidDepth items ahead, so the gather of item j never waits on a
        // global load; its keys then land through the stage's full barrier.
        if (lw == 0 && lane == 0) prefetch_tensormap(&tm_q);
        int *s_cuq = reinterpret_cast<int *>(g + kOffCuq);
        const bool cuq_cached = a.num_seqs + 1 <= kCuqCache;
        if (cuq_cached)
            for (int i = lane + 32 * lw; i <= a.num_seqs; i += 32 * kLoadWarps) s_cuq[i] = __ldg(a.cu_q + i);
        named_barrier(1, 32 * kLoadWarps);
        auto seq_of = [&](int t) {
            if (!cuq_cached) return seq_of_query(a, t);
            int lo = 0, hi = a.num_seqs - 1;
            while (lo < hi) {
                const int mid = (lo + hi + 1) >> 1;
                if (s_cuq[mid] <= t) lo = mid; else hi = mid - 1;
            }
            return lo;
        };
        auto cu = [&](int s) { return cuq_cached ? s_cuq[s] : __ldg(a.cu_q + s); };
        // page id of this lane's row of item j (first sequence of its tile)
        auto load_pid = [&](unsigned j) {
            const int y = (int)(j / (unsigned)n_bt), bt = (int)(j - (unsigned)y * (unsigned)n_bt);
            const int s0 = seq_of(kQT * y);
            const int b = bt * kBT + 32 * lw + lane;
            return b < a.max_blocks ? __ldg(a.block_table + (size_t)s0 * a.max_blocks + b) : -1;
        };
        pdl_wait();   // coarse keys may come from the preceding append
        int ring[kPidDepth];
#pragma unroll
        for (int d = 0; d < kPidDepth; ++d) ring[d] = i0 + d < i1 ? load_pid(i0 + d) : -1;
        int k = 0;    // stages published
        int cur_y = -1;
        int pos = -1, s_lo = 0, s_hi = -1, len_lo = 0;
        int wv[8];
        // facts of the current (query tile, sequence): own block of query
        // lane % 16, the largest of them, and their slot
        int fy = -1, fs = -1, f_own = -1, f_max = -1, f_len = 0, n_slots = 0, qslot = 0;
        bool slot_due = false;
        uint32_t err_bits = 0;
        // one item: its sub-items (one per sequence of the query tile) into the ring
        auto process = [&](unsigned it, int pg_pre) {
            const int y = (int)(it / (unsigned)n_bt), bt = (int)(it - (unsigned)y * (unsigned)n_bt);
            const int t0 = kQT * y;
            if (y != cur_y) {   // a new query tile: positions, weights, sequences
                cur_y = y;
                const int t = t0 + (lane & (kQT - 1));
                pos = t < a.total_q ? __ldg(a.q_pos + t) : -1;
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const int e = lane + 32 * j, qi = e / kMaxIdxHeads, h = e % kMaxIdxHeads;
                    wv[j] = (t0 + qi < a.total_q && h < H) ? __ldg(a.w + (size_t)(t0 + qi) * H + h) : 0;
                }
                s_lo = seq_of(t0);
                s_hi = seq_of(min(t0 + kQT, a.total_q) - 1);
                len_lo = __ldg(a.seq_lens + s_lo);
            }
            for (int s = s_lo; s <= s_hi && !*s_abort; ++s) {
                if (y != fy || s != fs) {   // facts of this (query tile, sequence)
                    fy = y;
                    fs = s;
                    f_len = s == s_lo ? len_lo : __ldg(a.seq_lens + s);
                    const int t = t0 + (lane & (kQT - 1));
                    f_own = -1;
                    if (t < a.total_q && cu(s) <= t && t < cu(s + 1)) {
                        f_own = pos / kBlockSize;
                        if (pos < 0 || pos >= f_len || f_own >= a.max_blocks) {
                            err_bits |= DSA_DEV_ERR_POS;
                            f_own = -1;
                        }
                    }
                    f_max = __reduce_max_sync(0xffffffffu, f_own);
                    slot_due = true;
                }
                if (f_max < bt * kBT) continue;   // nothing visible in this tile
                const int st = k % kTcStages;
                if (k >= kTcStages && !mbar_wait(bars.empty(st), ((k / kTcStages) - 1) & 1, s_abort)) {
                    *s_abort = 1;
                    break;
                }
                if (slot_due) {
                    // slot n_slots % kQSlots was last used by a tile published at
                    // least kQSlots tiles ago; the empty wait above completed every
                    // tile up to kTcStages < kQSlots before this one
                    qslot = n_slots % kQSlots;
                    ++n_slots;
                    slot_due = false;
                    if (lw == 0) {
                        QueryFacts *qf = reinterpret_cast<QueryFacts *>(g + kOffFacts) + qslot;
                        if (lane < kQT) qf->own[lane] = f_own;
#pragma unroll
                        for (int j = 0; j < 8; ++j) (&qf->w[0][0])[lane + 32 * j] = wv[j];
                    }
                }
                uint8_t *stage = g + st * kStageBytes;
                StageInfo *info = reinterpret_cast<StageInfo *>(stage + kOffInfo);
                const uint32_t sa = base + st * kStageBytes;
                if (lw == 0 && lane == 0) { info->end = 0; info->bt = bt; info->y = y; info->qslot = qslot; }
                // this lane's coarse key: 4 x 16 B, swizzled
                {
                    const int n_blocks = (f_len + kBlockSize - 1) / kBlockSize;
                    const int r = 32 * lw + lane;
                    const int b = bt * kBT + r;
                    int page = -1;
                    if (b < n_blocks && b < a.max_blocks && b <= f_max) {
                        page = s == s_lo ? pg_pre : __ldg(a.block_table + (size_t)s * a.max_blocks + b);
                        if (page < 0 || page >= a.num_pages) {
                            err_bits |= DSA_DEV_ERR_PAGE;
                            page = -1;
                        }
                    }
                    const uint32_t bits = __ballot_sync(0xffffffffu, page >= 0);
                    if (lane == 0) info->valid[lw] = bits;
                    const int8_t *src = a.kc_pool + (size_t)max(page, 0) * kIdxDim;
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        const uint32_t dst = sa + r * 64 + ((c ^ ((r >> 1) & 3)) << 4);
                        if (page >= 0) cp_async_16(dst, src + 16 * c);
                        else cp_async_16_zero(dst, a.kc_pool);
                    }
                }
                // the queries' rows: box (64 B, 16 heads, 16 queries) at query t0
                if (lw == 0 && lane == 0) {
                    tc::mbar_expect_tx(bars.full(st), kBBytes);
                    tma_load_3d(sa + kOffB, &tm_q, 0, 0, t0, bars.full(st));
                }
                tc::cp_async_arrive_noinc(bars.full(st));
                __syncwarp();
                if (lane == 0) mbar_arrive(bars.full(st));   // the info words above
                ++k;
            }
        };
        // the item loop, unrolled by the ring depth so that every ring slot is a
        // fixed register: slot d is read for item base + d and refilled with
        // the page id of item base + d + kPidDepth, which is read kPidDepth
        // items later -- no register copy ever waits on a load in flight
        for (unsigned base0 = i0; base0 < i1 && !*s_abort; base0 += kPidDepth) {
#pragma unroll
            for (int d = 0; d < kPidDepth; ++d) {
                const unsigned it = base0 + d;
                if (it < i1 && !*s_abort) {
                    const int pg_pre = ring[d];
                    ring[d] = it + kPidDepth < i1 ? load_pid(it + kPidDepth) : -1;
                    process(it, pg_pre);
                }
            }
        }
        // the end marker
        if (!*s_abort) {
            const int st = k % kTcStages;
            if (k >= kTcStages && !mbar_wait(bars.empty(st), ((k / kTcStages) - 1) & 1, s_abort)) {
                *s_abort = 1;
            } else {
                StageInfo *info = reinterpret_cast<StageInfo *>(g + st * kStageBytes + kOffInfo);
                if (lw == 0 && lane == 0) info->end = 1;
                tc::cp_async_arrive_noinc(bars.full(st));
                __syncwarp();
                if (lane == 0) mbar_arrive(bars.full(st));
                ++k;
            }
        }
        err_bits = __reduce_or_sync(0xffffffffu, err_bits);
        if (lane == 0 && err_bits) set_err(a.dev_err, err_bits);
        cp_async_commit();
        cp_async_wait<0>();
        if (*s_abort && lw == 0 && lane == 0) {
            set_err(a.dev_err, DSA_DEV_ERR_WAIT);
            for (int j = max(0, k - kTcStages); j < k; ++j)
                mbar_wait(bars.full(j % kTcStages), (j / kTcStages) & 1, s_never);
        }
    } else if (warp == kMmaWarp) {
        // ============================================================ MMA issuer
        constexpr uint32_t idesc = tc::idesc_i8(kBT, kN);
        int k = 0;
        while (true) {
            const int st = k % kTcStages, buf = k & 1;
            bool ok = mbar_wait(bars.full(st), (k / kTcStages) & 1, s_abort);
            if (ok && k >= 2) ok = mbar_wait(bars.tempty(buf), ((k >> 1) - 1) & 1, s_abort);
            if (!ok) {
                if (lane == 0) *s_abort = 1;
                break;
            }
            const StageInfo *info = reinterpret_cast<const StageInfo *>(g + st * kStageBytes + kOffInfo);
            const bool end = info->end != 0;
            if (lane == 0) {
                if (end) {
                    mbar_arrive(bars.tfull(buf));   // wake the epilogue to see the end marker
                } else {
                    tc::fence_proxy_async_smem();   // the cp.async-written keys, for the tensor core
                    tc::fence_after_sync();
                    const uint32_t sa = base + st * kStageBytes;
                    const uint32_t d = tmem + (uint32_t)(buf * kN);
                    const uint64_t da = tc::smem_desc_k64_sw64(sa), db = tc::smem_desc_k64_sw64(sa + kOffB);
                    tc::mma_i8(d, da, db, idesc, false);
                    tc::mma_i8(d, da + (32 >> 4), db + (32 >> 4), idesc, true);   // K bytes 32..63
                    tc::commit(bars.empty(st));
                    tc::commit(bars.tfull(buf));
                }
            }
            __syncwarp();
            ++k;
            if (end) break;
        }
        // the last MMAs have completed before the accumulator is released
        if (lane == 0 && k > 0) {
            const int j = k - 1;
            mbar_wait(bars.tfull(j & 1), (j >> 1) & 1, s_never);
        }
    } else {
        // ============================================================ epilogue
        const int ew = warp - kEpiWarp0;
        const int quarter = warp & 3;            // TMEM lanes 32*quarter .. +31
        const int qgrp = ew >> 2;                // queries 4*qgrp .. +3 (columns 64*qgrp ..)
        const int row = quarter * 32 + lane;     // block row of the tile
        int k = 0;
        while (true) {
            const int st = k % kTcStages, buf = k & 1;
            bool ok = mbar_wait(bars.tfull(buf), (k >> 1) & 1, s_abort) &&
                      mbar_wait(bars.full(st), (k / kTcStages) & 1, s_abort);   // acquire the info words
            if (!ok) {
                if (lane == 0) *s_abort = 1;
                break;
            }
            tc::fence_after_sync();
            const StageInfo *info = reinterpret_cast<const StageInfo *>(g + st * kStageBytes + kOffInfo);
            if (info->end) break;
            const int bt = info->bt, y = info->y;
            const QueryFacts *qf = reinterpret_cast<const QueryFacts *>(g + kOffFacts) + info->qslot;
            const int b = bt * kBT + row;
            const bool row_ok = (info->valid[row >> 5] >> (row & 31)) & 1u;
            const uint32_t taddr =
                tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(buf * kN + qgrp * 64);
            // weights and own blocks of this warp's 4 queries, read as shared-space vectors
            const uint32_t s_w = base + kOffFacts + (uint32_t)(info->qslot * (int)sizeof(QueryFacts)) +
                                 (uint32_t)offsetof(QueryFacts, w) + (uint32_t)(4 * qgrp * kMaxIdxHeads * 4);
            int own4[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) own4[u] = qf->own[4 * qgrp + u];
            uint32_t v[2][32];
            tc::ld_32x32b_x32(taddr, v[0]);
            tc::ld_32x32b_x32(taddr + 32, v[1]);
            tc::wait_ld();
#pragma unroll
            for (int u = 0; u < 4; ++u) {   // query 4*qgrp + u: columns 16u .. 16u+15 of this warp's 64
                const uint32_t *x = v[u >> 1] + 16 * (u & 1);
                int part[4];
#pragma unroll
                for (int h4 = 0; h4 < 4; ++h4) {   // four independent chains
                    int4 wv;
                    asm volatile("ld.shared.v4.s32 {%0,%1,%2,%3}, [%4];"
                                 : "=r"(wv.x), "=r"(wv.y), "=r"(wv.z), "=r"(wv.w)
                                 : "r"(s_w + (uint32_t)((u * kMaxIdxHeads + 4 * h4) * 4)));
                    part[h4] = wv.x * max((int)x[4 * h4 + 0], 0) + wv.y * max((int)x[4 * h4 + 1], 0) +
                               wv.z * max((int)x[4 * h4 + 2], 0) + wv.w * max((int)x[4 * h4 + 3], 0);
                }
                const int sum = (part[0] + part[1]) + (part[2] + part[3]);
                if (row_ok && b <= own4[u])
                    a.scores[(size_t)(kQT * y + 4 * qgrp + u) * a.max_blocks + b] = sum;
            }
            tc::fence_before_sync();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(bars.tempty(buf));
                mbar_arrive(bars.empty(st));
            }
            ++k;
        }
    }

    tc::fence_before_sync();
    __syncthreads();
    if (warp == kMmaWarp) {
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
    const int n_qt = (a.total_q + kQT - 1) / kQT;   // items (y, bt), y-major
    const long long items = (long long)n_bt * n_qt;
    if (items >= (1LL << 31)) return cudaErrorInvalidValue;   // item indices are 32-bit in the kernel
    const int grid = (int)(items < num_sms ? items : num_sms);
    return launch_pdl(index_score_tc_kernel, dim3(grid), dim3(kTcThreads), (size_t)kSmemBytes, stream, tq, a, n_bt,
                      n_qt);
}

}  // namespace dsa
