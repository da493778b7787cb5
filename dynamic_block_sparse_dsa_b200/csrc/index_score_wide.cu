// index_score_wide.cu -- block scores in int64: the int8 indexer without the
// int32 bound, and the FP8 (E4M3) indexer, both exact.
//
// "Day-0 Readiness for Trillion-Parameter Models: Engineering Sparse Attention
// and Expert Weight Compression", section "Index Selection Path": the scoring
// operator takes low-precision inputs; "Day-0 Adaptation for Massive LLMs ...",
// section 4(1): score the compressed per-block representation against each
// query.  The score is S[t][b] = sum_h w[t][h] * max(0, q_idx[t][h] . kc[b]).
//
//  * int8 inputs, any int32 weights: the dot products are exact in int32
//    (|dot| <= 64 * 128 * 128), the weighted sum is accumulated in int64.
//  * FP8 E4M3 inputs (OCP 8-bit float: bias 7, 3 mantissa bits, subnormals,
//    codes 0x7F / 0xFF are NaN): every finite E4M3 value times 2^9 is an
//    integer of magnitude <= 448 * 2^9 < 2^18, so each product is an exact
//    integer times 2^-18 and the dot product is exact in int64.  The kernel
//    returns S * 2^18 (an int64; the host checks the range), so the selection
//    made from it is exact and independent of summation order.  A NaN code is
//    read as 0 and flagged with DSA_DEV_ERR_VALUE.
//
// Layout as in the dp4a kernel: grid (256-block chunk, sequence), one thread
// per block, the queries of the sequence in batches staged in shared memory.
#include <cuda_fp8.h>

#include "dsa_kernels.h"
#include "indexer_core.cuh"

namespace dsa {

namespace {
constexpr int kWideThreads = 256;
constexpr int kWideQBatch = 8;

// value * 2^9 of an E4M3 code, by the hardware conversion to half (exact for
// every E4M3 value); a NaN code gives 0 and sets *bad
__device__ __forceinline__ int e4m3_scaled(uint32_t code, bool &bad) {
    const __half_raw hr = __nv_cvt_fp8_to_halfraw((__nv_fp8_storage_t)code, __NV_E4M3);
    const float f = __half2float(__half(hr));
    if (f != f) {
        bad = true;
        return 0;
    }
    return __float2int_rn(f * 512.0f);
}
}  // namespace

template <bool kFp8>
__global__ void __launch_bounds__(kWideThreads) index_score_wide_kernel(IndexScoreArgs a, int64_t *scores) {
    // int8: query rows as packed int4; FP8: query values times 2^9
    __shared__ int4 s_q8[kFp8 ? 1 : kWideQBatch][kMaxIdxHeads][kIdxDim / 16];
    __shared__ int s_qf[kFp8 ? kWideQBatch : 1][kMaxIdxHeads][kFp8 ? kIdxDim : 1];
    __shared__ int s_w[kWideQBatch][kMaxIdxHeads];
    __shared__ int s_own[kWideQBatch];

    pdl_trigger();
    pdl_wait();   // coarse keys may come from the preceding append
    const int s = blockIdx.y;
    const int q0 = __ldg(a.cu_q + s), q1 = __ldg(a.cu_q + s + 1);
    if (q1 <= q0) return;
    if (q0 < 0 || q1 > a.total_q) {
        if (blockIdx.x == 0 && threadIdx.x == 0) set_err(a.dev_err, DSA_DEV_ERR_POS);
        return;
    }
    const int len = __ldg(a.seq_lens + s);
    const int b = blockIdx.x * kWideThreads + threadIdx.x;
    const int H = a.num_idx_heads;
    const int n_blocks = (len + (1 << a.block_shift) - 1) >> a.block_shift;
    if (blockIdx.x * kWideThreads >= n_blocks) return;
    bool have = false, bad_value = false;
    int kc8[16];                    // int8: the key packed
    int kcf[kFp8 ? kIdxDim : 1];    // FP8: the key's values times 2^9
    if (b < n_blocks && b < a.max_blocks) {
        const int page = __ldg(a.block_table + (size_t)s * a.max_blocks + b);
        if (page >= 0 && page < a.num_pages) {
            load_coarse_key(a.kc_pool, page, kc8);
            if constexpr (kFp8) {
#pragma unroll
                for (int i = 0; i < 16; ++i)
#pragma unroll
                    for (int j = 0; j < 4; ++j) kcf[4 * i + j] = e4m3_scaled(((uint32_t)kc8[i] >> (8 * j)) & 0xffu, bad_value);
            }
            have = true;
        } else {
            set_err(a.dev_err, DSA_DEV_ERR_PAGE);
        }
    }
    for (int qb = q0; qb < q1; qb += kWideQBatch) {
        const int nq = min(kWideQBatch, q1 - qb);
        __syncthreads();
        if constexpr (kFp8) {
            const uint8_t *src = reinterpret_cast<const uint8_t *>(a.q_idx) + (size_t)qb * H * kIdxDim;
            for (int e = threadIdx.x; e < nq * H * kIdxDim; e += kWideThreads) {
                bool bad = false;
                const int v = e4m3_scaled(__ldg(src + e), bad);
                if (bad) bad_value = true;
                s_qf[e / (H * kIdxDim)][(e / kIdxDim) % H][e % kIdxDim] = v;
            }
        } else {
            for (int e = threadIdx.x; e < nq * H * (kIdxDim / 16); e += kWideThreads) {
                const int qi = e / (H * 4), rest = e % (H * 4);
                s_q8[qi][rest / 4][rest % 4] =
                    __ldg(reinterpret_cast<const int4 *>(a.q_idx + ((size_t)(qb + qi) * H) * kIdxDim) + rest);
            }
        }
        for (int e = threadIdx.x; e < nq * H; e += kWideThreads)
            s_w[e / H][e % H] = __ldg(a.w + (size_t)(qb + e / H) * H + e % H);
        if (threadIdx.x < nq) {
            const int p = __ldg(a.q_pos + qb + threadIdx.x);
            int own = p >> a.block_shift;
            if (p < 0 || p >= len || own >= a.max_blocks) {
                if (blockIdx.x == 0) set_err(a.dev_err, DSA_DEV_ERR_POS);
                own = -1;
            }
            s_own[threadIdx.x] = own;
        }
        __syncthreads();
        if (!have) continue;
        for (int qi = 0; qi < nq; ++qi) {
            if (b > s_own[qi]) continue;
            long long total = 0;
            for (int h = 0; h < H; ++h) {
                long long dot;
                if constexpr (kFp8) {
                    dot = 0;
#pragma unroll
                    for (int d = 0; d < kIdxDim; ++d) dot += (long long)s_qf[qi][h][d] * kcf[d];
                } else {
                    int d32 = 0;
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int4 qv = s_q8[qi][h][i];
                        d32 = __dp4a(kc8[4 * i + 0], qv.x, d32);
                        d32 = __dp4a(kc8[4 * i + 1], qv.y, d32);
                        d32 = __dp4a(kc8[4 * i + 2], qv.z, d32);
                        d32 = __dp4a(kc8[4 * i + 3], qv.w, d32);
                    }
                    dot = d32;
                }
                total += (long long)s_w[qi][h] * (dot > 0 ? dot : 0);
            }
            scores[(size_t)(qb + qi) * a.max_blocks + b] = total;
        }
    }
    if (bad_value) set_err(a.dev_err, DSA_DEV_ERR_VALUE);
}

cudaError_t launch_index_score_wide(const IndexScoreArgs &a, bool fp8, int64_t *scores, cudaStream_t stream) {
    if (a.total_q == 0 || a.num_seqs == 0) return cudaSuccess;
    dim3 grid((a.max_blocks + kWideThreads - 1) / kWideThreads, a.num_seqs);
    if (fp8) return launch_pdl(index_score_wide_kernel<true>, grid, dim3(kWideThreads), 0, stream, a, scores);
    return launch_pdl(index_score_wide_kernel<false>, grid, dim3(kWideThreads), 0, stream, a, scores);
}

}  // namespace dsa
