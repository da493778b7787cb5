// sparse_attn.cu -- exact attention over the selected KV blocks only.
//
// "Day-0 Adaptation for Massive LLMs: Overcoming Sparse Attention and MXFP4
// Expert Weights", section 4(3): decode gathers the selected KV blocks on chip
// by their indices and attends under a valid mask; the cost is the gather of
// non-contiguous blocks.  "Day-0 Adaptation for Trillion-Parameter Models:
// Engineering Practices and Technical Breakdown", section 4.3: decode needs a
// dedicated gather kernel.  "Day-0 Readiness ...", section "KV Cache Layout":
// read whole blocks by block id, never per token.
//
// One CTA = (split of the selection, KV head, query).  The CTA streams its
// selected blocks' K and V page slices -- 64 tokens x 256 bytes each, token
// stride num_kv_heads*256 bytes -- through a 3-stage cp.async ring of 16-byte
// copies into XOR-swizzled shared memory, and runs the GQA group of query
// heads (rows of an m16 tile) against them on the tensor cores with
// mma.m16n8k16 bf16 / fp32 accumulate:
//   S = Q K^T  (A = Q from registers, B = K via ldmatrix),
//   online softmax in fp32 (base-2 exponent, causal mask inside the own block),
//   O += P V   (P re-used from the S accumulators as the A operand, B = V via
//               ldmatrix.trans).
// Each of the 4 warps takes 16 of the 64 tokens of every block; their softmax
// states are merged through shared memory at the end.  With n_splits > 1 the
// CTA writes its partial state (m, l, unnormalised O) to the workspace and the
// last CTA of the (query, KV head) -- elected by an atomic counter, no waiting
// -- merges the partials and resets the counter.
#include "dsa_kernels.h"

namespace dsa {

namespace {
constexpr int kAttnThreads = 128;
constexpr int kStages = 3;
constexpr int kTileBytes = kBlockSize * kHeadDim * 2;       // 16 KiB: one K or V page slice
constexpr int kQBytes = 16 * kHeadDim * 2;                  // 4 KiB: 16 padded query rows
constexpr int kSmemBytes = kQBytes + kStages * 2 * kTileBytes;
constexpr float kLn2 = 0.6931471805599453f;

// byte offset of 16-byte chunk c of row r in a [rows][256 B] tile, XOR-swizzled
__device__ __forceinline__ uint32_t swz(int r, int c) { return r * 256 + ((c ^ (r & 7)) << 4); }

struct BlockRef {
    int blk;        // logical block id, -1 if unusable
    int page;
    uint32_t err;   // DSA_DEV_ERR_* bit explaining an unusable block
};

__device__ __forceinline__ BlockRef block_ref(const AttnArgs &a, int t, int s, int j, int n_vis) {
    BlockRef r{-1, -1, 0u};
    const int b = __ldg(a.sel + (size_t)t * a.k_max + j);
    if (b < 0 || b >= n_vis) { r.err = DSA_DEV_ERR_SEL; return r; }
    const int page = __ldg(a.block_table + (size_t)s * a.max_blocks + b);
    if (page < 0 || page >= a.num_pages) { r.err = DSA_DEV_ERR_PAGE; return r; }
    r.blk = b;
    r.page = page;
    return r;
}
}  // namespace

__global__ void __launch_bounds__(kAttnThreads) sparse_attn_kernel(AttnArgs a) {
    extern __shared__ __align__(128) uint8_t smem[];
    __shared__ int s_last;

    const int t = blockIdx.x, kvh = blockIdx.y, split = blockIdx.z;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, c = lane & 3;
    const int G = a.group;
    const int h0 = kvh * G;

    const int s = find_seq(a.cu_q, a.num_seqs, t);
    const int p = __ldg(a.q_pos + t);
    const int len = __ldg(a.seq_lens + s);
    int n_sel = __ldg(a.cnt + t);
    const int n_vis = p / kBlockSize + 1;
    bool bad_query = (p < 0 || p >= len || n_vis > a.max_blocks);
    if (n_sel < 0 || n_sel > a.k_max) {
        if (tid == 0 && split == 0 && kvh == 0) set_err(a.dev_err, DSA_DEV_ERR_SEL);
        n_sel = 0;
    }
    if (bad_query) {
        if (tid == 0 && split == 0 && kvh == 0) set_err(a.dev_err, DSA_DEV_ERR_POS);
        n_sel = 0;
    }
    const int j0 = split * a.blocks_per_split;
    const int j1 = min(n_sel, j0 + a.blocks_per_split);

    const uint32_t sQ = smem_u32(smem);
    const uint32_t sKV = sQ + kQBytes;
    const size_t row_elems = (size_t)a.num_kv_heads * kHeadDim;   // one token row of the pool

    // ---- query tile: rows 0..G-1 real, the rest zero
    for (int e = tid; e < 16 * 16; e += kAttnThreads) {
        const int r = e >> 4, ch = e & 15;
        const __nv_bfloat16 *src = a.q + ((size_t)t * a.num_q_heads + h0 + min(r, G - 1)) * kHeadDim + ch * 8;
        if (r < G) cp_async_16(sQ + swz(r, ch), src);
        else cp_async_16_zero(sQ + swz(r, ch), src);
    }

    auto load_block = [&](int j, int stage) {
        const BlockRef br = block_ref(a, t, s, j, n_vis);
        const uint32_t dk = sKV + stage * 2 * kTileBytes;
        const uint32_t dv = dk + kTileBytes;
        if (br.blk < 0) {
            // unusable block: flag it and zero the stage so that the masked
            // products see finite values (0 * stale NaN would poison O)
            if (tid == 0) set_err(a.dev_err, br.err);
#pragma unroll
            for (int i = 0; i < (kBlockSize * 16) / kAttnThreads; ++i) {
                const int e = tid + i * kAttnThreads;
                cp_async_16_zero(dk + swz(e >> 4, e & 15), a.k_pool);
                cp_async_16_zero(dv + swz(e >> 4, e & 15), a.v_pool);
            }
            return;
        }
        const __nv_bfloat16 *kb = a.k_pool + ((size_t)br.page * kBlockSize * a.num_kv_heads + kvh) * kHeadDim;
        const __nv_bfloat16 *vb = a.v_pool + ((size_t)br.page * kBlockSize * a.num_kv_heads + kvh) * kHeadDim;
#pragma unroll
        for (int i = 0; i < (kBlockSize * 16) / kAttnThreads; ++i) {
            const int e = tid + i * kAttnThreads;
            const int r = e >> 4, ch = e & 15;
            const size_t off = (size_t)r * row_elems + ch * 8;
            cp_async_16(dk + swz(r, ch), kb + off);
            cp_async_16(dv + swz(r, ch), vb + off);
        }
    };

#pragma unroll
    for (int i = 0; i < kStages - 1; ++i) {
        if (j0 + i < j1) load_block(j0 + i, i);
        cp_async_commit();
    }

    // Q fragments stay in registers for the whole CTA
    uint32_t qa[8][4];
    float o[16][4];
    float m_run[2] = {-INFINITY, -INFINITY};
    float l_run[2] = {0.f, 0.f};
#pragma unroll
    for (int n = 0; n < 16; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;

    bool q_loaded = false;
    for (int j = j0; j < j1; ++j) {
        cp_async_wait<kStages - 2>();
        __syncthreads();
        {
            const int jn = j + kStages - 1;
            if (jn < j1) load_block(jn, (jn - j0) % kStages);
            cp_async_commit();
        }
        if (!q_loaded) {
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                const int r = (lane & 7) + 8 * ((lane >> 3) & 1);
                const int ch = 2 * kk + (lane >> 4);
                ldmatrix_x4(sQ + swz(r, ch), qa[kk][0], qa[kk][1], qa[kk][2], qa[kk][3]);
            }
            q_loaded = true;
        }
        const BlockRef br = block_ref(a, t, s, j, n_vis);
        const int stage = (j - j0) % kStages;
        const uint32_t tk = sKV + stage * 2 * kTileBytes;
        const uint32_t tv = tk + kTileBytes;
        const int tok0 = warp * 16;

        // ---- S = Q K^T for this warp's 16 tokens (two n8 tiles)
        float sc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
            const int r = tok0 + (lane & 7) + 8 * (lane >> 4);
            const int ch = 2 * kk + ((lane >> 3) & 1);
            uint32_t b0, b1, b2, b3;
            ldmatrix_x4(tk + swz(r, ch), b0, b1, b2, b3);
            mma_bf16_16816(sc[0], qa[kk], b0, b1);
            mma_bf16_16816(sc[1], qa[kk], b2, b3);
        }
        // ---- mask, scale, online softmax (rows g and g+8 of the head tile)
        float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int pos = br.blk * kBlockSize + tok0 + nt * 8 + 2 * c + (e & 1);
                const bool ok = br.blk >= 0 && pos <= p;
                const float x = ok ? sc[nt][e] * a.scale_log2 : -INFINITY;
                sc[nt][e] = x;
                mx[e >> 1] = fmaxf(mx[e >> 1], x);
            }
        float alpha[2];
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 1));
            mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 2));
            const float m_new = fmaxf(m_run[r], mx[r]);
            // all tokens so far masked: keep zero state, avoid (-inf) - (-inf)
            alpha[r] = (m_new == -INFINITY) ? 1.f : exp2f(m_run[r] - m_new);
            m_run[r] = m_new;
        }
        float rs[2] = {0.f, 0.f};
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float mr = m_run[e >> 1];
                const float pv = (mr == -INFINITY) ? 0.f : exp2f(sc[nt][e] - mr);
                sc[nt][e] = pv;
                rs[e >> 1] += pv;
            }
#pragma unroll
        for (int r = 0; r < 2; ++r) l_run[r] = l_run[r] * alpha[r] + rs[r];
#pragma unroll
        for (int n = 0; n < 16; ++n) {
            o[n][0] *= alpha[0]; o[n][1] *= alpha[0];
            o[n][2] *= alpha[1]; o[n][3] *= alpha[1];
        }
        // ---- O += P V
        uint32_t pa[4];
        pa[0] = pack_bf16x2(sc[0][0], sc[0][1]);
        pa[1] = pack_bf16x2(sc[0][2], sc[0][3]);
        pa[2] = pack_bf16x2(sc[1][0], sc[1][1]);
        pa[3] = pack_bf16x2(sc[1][2], sc[1][3]);
#pragma unroll
        for (int n = 0; n < 8; ++n) {
            const int r = tok0 + (lane & 7) + 8 * ((lane >> 3) & 1);
            const int ch = 2 * n + (lane >> 4);
            uint32_t b0, b1, b2, b3;
            ldmatrix_x4_trans(tv + swz(r, ch), b0, b1, b2, b3);
            mma_bf16_16816(o[2 * n], pa, b0, b1);
            mma_bf16_16816(o[2 * n + 1], pa, b2, b3);
        }
    }
    cp_async_wait<0>();
    __syncthreads();

    // ---- merge the 4 warps' softmax states through shared memory
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        l_run[r] += __shfl_xor_sync(0xffffffffu, l_run[r], 1);
        l_run[r] += __shfl_xor_sync(0xffffffffu, l_run[r], 2);
    }
    float *s_o = reinterpret_cast<float *>(smem + kQBytes);      // [4][16][128]
    float *s_m = s_o + 4 * 16 * kHeadDim;                          // [4][16]
    float *s_l = s_m + 4 * 16;                                     // [4][16]
#pragma unroll
    for (int n = 0; n < 16; ++n) {
        float *row0 = s_o + (warp * 16 + g) * kHeadDim + n * 8 + 2 * c;
        float *row1 = s_o + (warp * 16 + g + 8) * kHeadDim + n * 8 + 2 * c;
        row0[0] = o[n][0]; row0[1] = o[n][1];
        row1[0] = o[n][2]; row1[1] = o[n][3];
    }
    if (c == 0) {
        s_m[warp * 16 + g] = m_run[0];
        s_m[warp * 16 + g + 8] = m_run[1];
        s_l[warp * 16 + g] = l_run[0];
        s_l[warp * 16 + g + 8] = l_run[1];
    }
    __syncthreads();

    // thread -> (row r, 4 consecutive dims); G rows x 32 dim-quads
    const size_t unit = (size_t)t * a.num_q_heads + h0;   // first head row of this CTA
    for (int e = tid; e < G * 32; e += kAttnThreads) {
        const int r = e >> 5, d0 = (e & 31) * 4;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < 4; ++w) M = fmaxf(M, s_m[w * 16 + r]);
        float L = 0.f, acc[4] = {0.f, 0.f, 0.f, 0.f};
        if (M != -INFINITY) {
#pragma unroll
            for (int w = 0; w < 4; ++w) {
                const float f = exp2f(s_m[w * 16 + r] - M);
                L += s_l[w * 16 + r] * f;
#pragma unroll
                for (int k = 0; k < 4; ++k) acc[k] += s_o[(w * 16 + r) * kHeadDim + d0 + k] * f;
            }
        }
        if (a.n_splits == 1) {
            const float inv = L > 0.f ? 1.f / L : 0.f;
            __nv_bfloat16 *dst = a.out + (unit + r) * kHeadDim + d0;
            *reinterpret_cast<uint2 *>(dst) =
                make_uint2(pack_bf16x2(acc[0] * inv, acc[1] * inv), pack_bf16x2(acc[2] * inv, acc[3] * inv));
            if (a.lse && d0 == 0) a.lse[unit + r] = L > 0.f ? (M + log2f(L)) * kLn2 : -INFINITY;
        } else {
            const size_t pi = (unit + r) * a.n_splits + split;
            *reinterpret_cast<float4 *>(a.part_o + pi * kHeadDim + d0) = make_float4(acc[0], acc[1], acc[2], acc[3]);
            if (d0 == 0) *reinterpret_cast<float2 *>(a.part_ml + pi * 2) = make_float2(M, L);
        }
    }
    if (a.n_splits == 1) return;

    // ---- the last CTA of this (query, KV head) merges the splits
    __threadfence();
    __syncthreads();
    if (tid == 0) {
        const int old = atomicAdd(a.counters + (size_t)t * a.num_kv_heads + kvh, 1);
        s_last = (old == a.n_splits - 1);
    }
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    for (int e = tid; e < G * 32; e += kAttnThreads) {
        const int r = e >> 5, d0 = (e & 31) * 4;
        const size_t pb = (unit + r) * a.n_splits;
        float M = -INFINITY;
        for (int sp = 0; sp < a.n_splits; ++sp) M = fmaxf(M, __ldcg(a.part_ml + (pb + sp) * 2));
        float L = 0.f, acc[4] = {0.f, 0.f, 0.f, 0.f};
        if (M != -INFINITY) {
            for (int sp = 0; sp < a.n_splits; ++sp) {
                const float2 ml = __ldcg(reinterpret_cast<const float2 *>(a.part_ml + (pb + sp) * 2));
                if (ml.x == -INFINITY) continue;
                const float f = exp2f(ml.x - M);
                L += ml.y * f;
                const float4 ov = __ldcg(reinterpret_cast<const float4 *>(a.part_o + (pb + sp) * kHeadDim + d0));
                acc[0] += ov.x * f; acc[1] += ov.y * f; acc[2] += ov.z * f; acc[3] += ov.w * f;
            }
        }
        const float inv = L > 0.f ? 1.f / L : 0.f;
        __nv_bfloat16 *dst = a.out + (unit + r) * kHeadDim + d0;
        *reinterpret_cast<uint2 *>(dst) =
            make_uint2(pack_bf16x2(acc[0] * inv, acc[1] * inv), pack_bf16x2(acc[2] * inv, acc[3] * inv));
        if (a.lse && d0 == 0) a.lse[unit + r] = L > 0.f ? (M + log2f(L)) * kLn2 : -INFINITY;
    }
    if (tid == 0) a.counters[(size_t)t * a.num_kv_heads + kvh] = 0;
}

cudaError_t launch_sparse_attn(const AttnArgs &a, cudaStream_t stream) {
    if (a.total_q == 0) return cudaSuccess;
    // the shared-memory opt-in is a per-device function attribute
    static unsigned long long attr_done = 0;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev >= 64 || !(attr_done & (1ull << dev))) {
        e = cudaFuncSetAttribute(sparse_attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
        if (e != cudaSuccess) return e;
        if (dev < 64) attr_done |= 1ull << dev;
    }
    dim3 grid(a.total_q, a.num_kv_heads, a.n_splits);
    sparse_attn_kernel<<<grid, kAttnThreads, kSmemBytes, stream>>>(a);
    return cudaGetLastError();
}

}  // namespace dsa
