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
// Grid: one thread-block cluster of CL CTAs per query (CL = 1..16, chosen
// from the longest block table), CTA r of the cluster taking the candidate
// blocks [r*512*G, (r+1)*512*G) of its query.  Each warp scores 64 blocks at a
// time with the int8 indexer on the tensor cores (mma.m16n8k32 s8, coarse keys
// as the M operand loaded straight into fragments; a CUDA-core dp4a version
// measured ALU-bound at the 1M-token decode shape) and folds them into its
// running Top-64 (warp-level bitonic networks on unique 64-bit keys); a merge
// tree over the 8 warps gives the CTA's list.  The cluster then meets on chip:
// every CTA stores its list into the leader CTA's shared memory with st.async
// (each store completes its bytes on the leader's mbarrier, armed with the
// exact count before the cluster barrier that orders it before any store),
// the leader merges the CL lists, appends the query's own block and writes
// the ascending selection.  No workspace, no global atomics, no second pass.
// A closing cluster barrier keeps every CTA resident until the leader is done
// with its shared memory.  When the call also appends tokens
// (dsa_select_blocks_append), the copies run in the non-leader CTAs (in every
// CTA when CL = 1) after their lists are sent.  Result is identical to
// dsa_index_score followed by dsa_topk_blocks.
#include "dsa_kernels.h"
#include "dsa_tma.cuh"
#include "indexer_core.cuh"
#include "kv_append.cuh"
#include "warp_topk.cuh"

namespace dsa {

namespace {
constexpr int kSelThreads = 256;
constexpr int kSelWarps = kSelThreads / 32;
constexpr int kCuqCache = 1024;   // cu_q entries staged in shared memory
constexpr int kGroupBlocks = kSelWarps * 64;   // blocks a CTA covers per group step

__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ void cluster_arrive() { asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory"); }
__device__ __forceinline__ void cluster_wait() { asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory"); }
// start moving [p, p + bytes) into L2 (16-byte aligned, a multiple of 16 bytes)
__device__ __forceinline__ void bulk_prefetch_l2(const void *p, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}
// 8-byte asynchronous store into another CTA's shared memory, completing on its mbarrier
__device__ __forceinline__ void st_async_b64(uint32_t addr, unsigned long long v, uint32_t bar) {
    asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.b64 [%0], %1, [%2];" ::"r"(addr), "l"(v),
                 "r"(bar)
                 : "memory");
}
}  // namespace

template <int G>   // 64-block groups per warp: a CTA covers kSelWarps * 64 * G candidate blocks
__global__ void __launch_bounds__(kSelThreads) select_blocks_kernel(SelectArgs a) {
    __shared__ int4 s_q[kMaxIdxHeads][kIdxDim / 16];
    __shared__ int s_w[kMaxIdxHeads];
    __shared__ int s_cuq[kCuqCache + 1];
    __shared__ key64 s_lists[kSelWarps * 64];
    __shared__ __align__(16) key64 s_inbox[kSelMaxCluster][64];   // leader: every CTA's Top-(K-1)
    __shared__ __align__(8) unsigned long long s_bar;              // leader: inbox barrier
    constexpr int CH = kGroupBlocks * G;
    const int CL = a.cluster;
    const int r = (int)cluster_ctarank();
    const int t = (int)blockIdx.x / CL;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g = lane >> 2, cq = lane & 3;
    const int H = a.num_idx_heads;
    const uint32_t bar = smem_u32(&s_bar);

    pdl_trigger();
    if (r == 0 && tid == 0) {
        mbar_init(bar, 1);
        fence_barrier_init();
    }
    // ---- query facts.  The position and cu_q travel together with, on the
    // guess that query t is sequence t (a decode batch), that sequence's
    // length, Top-K and this CTA's first page ids; they are reloaded only if
    // cu_q says otherwise: one round trip before the coarse keys
    // groups whose page ids and coarse keys are in flight together
    constexpr int GB = G < 2 ? G : 2;
    const int p = __ldg(a.q_pos + t);
    const bool guess = t < a.num_seqs;
    int len = 0, K = 0, pg[GB][4][2];
    // page ids of this warp's groups g0 .. g0+GB-1 (rows end at max_blocks; ids
    // past the own block are never used)
    auto load_pages = [&](int sq, int g0) {
        const int32_t *row = a.block_table + (size_t)sq * a.max_blocks;
#pragma unroll
        for (int j = 0; j < GB; ++j) {
            const int base = r * CH + ((g0 + j) * kSelWarps + warp) * 64;
#pragma unroll
            for (int mt = 0; mt < 4; ++mt)
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int b = base + 16 * mt + g + 8 * h;
                    pg[j][mt][h] = b < a.max_blocks ? __ldg(row + b) : -1;
                }
        }
    };
    auto load_seq_facts = [&](int sq) {
        len = __ldg(a.seq_lens + sq);
        K = __ldg(a.k_per_seq + sq);
        load_pages(sq, 0);
    };
    if (guess) load_seq_facts(t);
    const bool cached = a.num_seqs + 1 <= kCuqCache;
    if (cached)
        for (int i = tid; i <= a.num_seqs; i += kSelThreads) s_cuq[i] = __ldg(a.cu_q + i);
    for (int e = tid; e < kMaxIdxHeads * 4; e += kSelThreads)   // heads past H read as zero
        s_q[e >> 2][e & 3] = (e >> 2) < H
            ? __ldg(reinterpret_cast<const int4 *>(a.q_idx + (size_t)t * H * kIdxDim) + e) : make_int4(0, 0, 0, 0);
    if (tid < kMaxIdxHeads) s_w[tid] = tid < H ? __ldg(a.w + (size_t)t * H + tid) : 0;
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
    const int n_vis = p / kBlockSize + 1;
    int32_t *out = a.sel + (size_t)t * a.k_max;
    bool bad_pos = p < 0 || p >= len || n_vis > a.max_blocks;
    if (a.cu_new && !bad_pos) {
        // an append follows and overlaps this kernel: no candidate block may be appended to
        const int n_new = __ldg(a.cu_new + s + 1) - __ldg(a.cu_new + s);
        if (n_new > len || (n_new > 0 && n_vis - 1 > (len - n_new) / kBlockSize)) bad_pos = true;
    }
    const bool bad_k = K < 1 || K > a.k_max;
    const int own = n_vis - 1;
    const int kk = K - 1;
    // every CTA of the cluster reads the same facts and so takes the same branch
    const bool scored = !bad_pos && !bad_k && n_vis > K && kk > 0;
    const int n_active = scored ? (own + CH - 1) / CH : 0;   // CTAs holding candidates (blocks 0 .. own-1)
    const bool mine = r < n_active;
    if (r == 0 && tid == 0 && n_active > 1)   // the other active CTAs' lists, in bytes
        mbar_arrive_expect_tx(bar, (uint32_t)((n_active - 1) * kk * sizeof(key64)));
    __syncwarp();
    cluster_arrive();   // phase 1: the leader's barrier is initialised and armed

    key64 acc[2] = {0ull, 0ull};
    if (mine) {
        // ---- score the CTA's candidates on the int8 tensor cores, 64 blocks per warp step
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
        uint32_t err_bits = 0;
        // GB groups at a time: their page ids, then their coarse-key fragments,
        // all in flight before the first tensor-core op
#pragma unroll 1
        for (int g0 = 0; g0 < G; g0 += GB) {
            if (g0 > 0) load_pages(s, g0);
#pragma unroll
            for (int j = 0; j < GB; ++j)
#pragma unroll
                for (int mt = 0; mt < 4; ++mt)
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const int b = r * CH + ((g0 + j) * kSelWarps + warp) * 64 + 16 * mt + g + 8 * h;
                        int page = b < own ? pg[j][mt][h] : -1;
                        if (b < own && (page < 0 || page >= a.num_pages)) { err_bits |= DSA_DEV_ERR_PAGE; page = -1; }
                        pg[j][mt][h] = page;
                    }
            if (g0 == 0) pdl_wait();   // coarse keys may come from the preceding append
            Tile16 f[GB][4];
#pragma unroll
            for (int j = 0; j < GB; ++j)
#pragma unroll
                for (int mt = 0; mt < 4; ++mt) tile16_load(a.kc_pool, pg[j][mt][0], pg[j][mt][1], f[j][mt]);
#pragma unroll
            for (int j = 0; j < GB; ++j) {
                const int base = r * CH + ((g0 + j) * kSelWarps + warp) * 64;
                key64 v[2] = {0ull, 0ull};
#pragma unroll
                for (int mt = 0; mt < 4; ++mt) {
                    int s_g, s_g8;
                    tile16_scores(f[j][mt], qb, wl, s_g, s_g8);
                    if (mt == cq) {   // lane (g, cq) keeps blocks 16*cq + g and 16*cq + g + 8
                        const int b = base + 16 * mt + g;
                        v[0] = pg[j][mt][0] >= 0 ? make_key64(s_g, (uint32_t)b) : 0ull;
                        v[1] = pg[j][mt][1] >= 0 ? make_key64(s_g8, (uint32_t)(b + 8)) : 0ull;
                    }
                }
                warp_fold_topk(acc, v, kk);
            }
        }
        if (err_bits) set_err(a.dev_err, err_bits);
        // ---- the CTA's Top-64 over its warps (warp 0 holds it)
        cta_merge_top64<kSelWarps>(acc, s_lists);
    } else if (scored) {
        pdl_wait();
    }
    cluster_wait();     // phase 1 complete: the leader expects the lists
    if (mine && r > 0 && warp == 0) {
        // send the first kk keys to the leader's inbox row r
        const uint32_t dst = mapa_shared(smem_u32(&s_inbox[r][0]), 0);
        const uint32_t rbar = mapa_shared(bar, 0);
        if (lane < kk) st_async_b64(dst + 8u * lane, acc[0], rbar);
        if (32 + lane < kk) st_async_b64(dst + 8u * (32 + lane), acc[1], rbar);
    }

    if (r == 0) {
        pdl_wait();   // the outputs below may be read by the kernel before this one
        if (!scored) {
            if (tid == 0) {
                if (bad_pos || bad_k) set_err(a.dev_err, bad_k ? DSA_DEV_ERR_K : DSA_DEV_ERR_POS);
                a.cnt[t] = (bad_pos || bad_k) ? 0 : (n_vis <= K ? n_vis : 1);
            }
            const int n = (bad_pos || bad_k) ? 0 : (n_vis <= K ? n_vis : 1);
            for (int i = tid; i < a.k_max; i += kSelThreads) out[i] = i < n ? (n == 1 ? own : i) : -1;
        } else {
            // the other CTAs' lists; the wait outlasts any bounded stall of theirs
            bool got = n_active <= 1 || mbar_try_wait_cluster(bar, 0);
            const long long t0 = clock64();
            while (!got && clock64() - t0 < 2 * kWaitLimitCycles) got = mbar_try_wait_cluster(bar, 0);
            got = __syncthreads_and(got) != 0;   // one decision for the whole CTA
            if (!got) {
                if (tid == 0) {
                    set_err(a.dev_err, DSA_DEV_ERR_WAIT);
                    a.cnt[t] = 0;
                }
                for (int i = tid; i < a.k_max; i += kSelThreads) out[i] = -1;
            } else {
                // warp w merges the lists of ranks w, w + 8 (its own CTA's list is rank 0's)
                key64 m[2] = {0ull, 0ull};
                if (warp == 0) {
                    m[0] = lane < kk ? acc[0] : 0ull;
                    m[1] = 32 + lane < kk ? acc[1] : 0ull;
                } else if (warp < n_active) {
                    m[0] = lane < kk ? s_inbox[warp][lane] : 0ull;
                    m[1] = 32 + lane < kk ? s_inbox[warp][32 + lane] : 0ull;
                }
                if (warp + kSelWarps < n_active) {
                    const key64 b[2] = {lane < kk ? s_inbox[warp + kSelWarps][lane] : 0ull,
                                        32 + lane < kk ? s_inbox[warp + kSelWarps][32 + lane] : 0ull};
                    warp_merge64_desc(m, b);
                }
                cta_merge_top64<kSelWarps>(m, s_lists);
                if (warp == 0) {
                    // the winners (non-zero keys among the first kk) in ascending block order
                    const bool v0 = lane < kk && m[0] != 0ull, v1 = 32 + lane < kk && m[1] != 0ull;
                    const int km = __popc(__ballot_sync(0xffffffffu, v0)) + __popc(__ballot_sync(0xffffffffu, v1));
                    uint32_t ids[2] = {v0 ? key64_id(m[0]) : 0xffffffffu, v1 ? key64_id(m[1]) : 0xffffffffu};
                    warp_sort64_asc_u32(ids);
                    if (lane < km) out[lane] = (int32_t)ids[0];
                    if (32 + lane < km) out[32 + lane] = (int32_t)ids[1];
                    if (lane == 0) {
                        out[km] = own;              // the own block: the largest visible id, last in order
                        a.cnt[t] = km + 1;
                    }
                    for (int i = km + 1 + lane; i < a.k_max; i += 32) out[i] = -1;
                    const int32_t *row = a.block_table + (size_t)s * a.max_blocks;
                    if (a.prefetch_kv) {
                        // the attention that follows gathers exactly these pages: start
                        // streaming them into L2 now, while it launches and looks them up
                        // (a hint; the host enables it only when every call's selected
                        // pages fit in L2 together)
                        const int pg0 = v0 ? __ldg(row + ids[0]) : -1;
                        const int pg1 = v1 ? __ldg(row + ids[1]) : -1;
                        const int pgo = lane == 0 ? __ldg(row + own) : -1;
                        const size_t pb = (size_t)a.kv_page_bytes;
                        auto fetch = [&](int page) {
                            if (page < 0 || page >= a.num_pages) return;
                            bulk_prefetch_l2(static_cast<const char *>(a.k_pool) + (size_t)page * pb, (uint32_t)pb);
                            bulk_prefetch_l2(static_cast<const char *>(a.v_pool) + (size_t)page * pb, (uint32_t)pb);
                        };
                        fetch(pg0);
                        fetch(pg1);
                        fetch(pgo);
                    } else {
                        // warm the block-table lines the attention looks up first
                        if (v0) prefetch_l2_line(row + ids[0]);
                        if (v1) prefetch_l2_line(row + ids[1]);
                    }
                }
            }
        }
    }
    if (a.app.total_new > 0 && (CL == 1 || r > 0)) {
        // the token copies of an append that overlaps this selection (which
        // never reads the rows written here -- see SelectArgs::cu_new); they
        // wait for the kernel before this one like every other write
        pdl_wait();
        const int per = CL == 1 ? 1 : CL - 1;
        const int n_app = (int)(gridDim.x / CL) * per;
        for (int i = t * per + (CL == 1 ? 0 : r - 1); i < a.app.total_new; i += n_app)
            append_token(a.app, i, tid, kSelThreads);
    }
    // every CTA stays until the leader is done with its inbox
    cluster_arrive();
    cluster_wait();
}

namespace {
template <int G>
cudaError_t launch_g(const SelectArgs &a, int CL, cudaStream_t stream) {
    SelectArgs b = a;
    b.cluster = CL;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)a.total_q * CL);
    cfg.blockDim = dim3(kSelThreads);
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    int n = 0;
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = CL;
    attr[n].val.clusterDim.y = 1;
    attr[n].val.clusterDim.z = 1;
    ++n;
    if (!a.cu_new) {   // the overlapping append relies on nothing earlier still running
        attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[n].val.programmaticStreamSerializationAllowed = 1;
        ++n;
    }
    cfg.attrs = attr;
    cfg.numAttrs = n;
    if (CL > 8) {   // the non-portable cluster size, opted into once per device
        static unsigned long long done = 0;
        int dev = 0;
        cudaError_t e = cudaGetDevice(&dev);
        if (e != cudaSuccess) return e;
        if (dev >= 64 || !(done & (1ull << dev))) {
            e = cudaFuncSetAttribute(select_blocks_kernel<G>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
            if (e != cudaSuccess) return e;
            if (dev < 64) done |= 1ull << dev;
        }
    }
    return cudaLaunchKernelEx(&cfg, select_blocks_kernel<G>, b);
}

// largest cluster the selection may use on the current device: 16 where the
// device can place such clusters (a non-portable size), else the portable 8
int max_cluster() {
    static int cached[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 8;
    if (cached[dev]) return cached[dev];
    int best = 8;
    if (cudaFuncSetAttribute(select_blocks_kernel<1>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) ==
        cudaSuccess) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(kSelMaxCluster);
        cfg.blockDim = dim3(kSelThreads);
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = kSelMaxCluster;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int n = 0;
        if (cudaOccupancyMaxActiveClusters(&n, select_blocks_kernel<1>, &cfg) == cudaSuccess && n >= 1)
            best = kSelMaxCluster;
    }
    (void)cudaGetLastError();
    cached[dev] = best;
    return best;
}
}  // namespace

cudaError_t launch_select_blocks(const SelectArgs &a, cudaStream_t stream) {
    if (a.total_q == 0) return cudaSuccess;
    // CTAs per query: one per kGroupBlocks candidate blocks up to the largest
    // cluster, then more blocks per CTA (G groups per warp)
    const int cmax = max_cluster();
    const int groups = (a.max_blocks + kGroupBlocks - 1) / kGroupBlocks;
    int CL = 1;
    while (CL < cmax && CL < groups) CL <<= 1;
    const int need = (groups + CL - 1) / CL;
    if ((long long)a.total_q * CL > 0x7fffffffLL) return cudaErrorInvalidValue;
    if (need <= 1) return launch_g<1>(a, CL, stream);
    if (need <= 2) return launch_g<2>(a, CL, stream);
    if (need <= 4) return launch_g<4>(a, CL, stream);
    if (need <= 8) return launch_g<8>(a, CL, stream);
    if (need <= 16) return launch_g<16>(a, CL, stream);
    return cudaErrorInvalidValue;   // the host rejects contexts this long first
}

}  // namespace dsa
