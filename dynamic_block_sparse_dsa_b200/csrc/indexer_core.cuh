// indexer_core.cuh -- the CUDA-core block score of the int8 indexer.
//
// S = sum_h w[h] * max(0, q_idx[h] . kc) for one 64-byte coarse key kc held in
// 16 registers; the query rows sit in shared memory and are read as
// broadcasts.  16 dp4a per head, exact in int32 under the host's range check.
#pragma once

#include "dsa_common.cuh"

namespace dsa {

// 64-byte coarse key of a page as 16 packed int8x4 words
__device__ __forceinline__ void load_coarse_key(const int8_t *kc_pool, int page, int (&kc)[16]) {
    const int4 *src = reinterpret_cast<const int4 *>(kc_pool + (size_t)page * kIdxDim);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int4 v = __ldg(src + i);
        kc[4 * i + 0] = v.x; kc[4 * i + 1] = v.y; kc[4 * i + 2] = v.z; kc[4 * i + 3] = v.w;
    }
}

// q: [heads][4] int4 rows of one query in shared memory; w: [heads] weights
__device__ __forceinline__ int block_score(const int (&kc)[16], const int4 (*q)[4], const int *w, int heads) {
    int total = 0;
    for (int h = 0; h < heads; ++h) {
        int dot = 0;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int4 qv = q[h][i];
            dot = __dp4a(kc[4 * i + 0], qv.x, dot);
            dot = __dp4a(kc[4 * i + 1], qv.y, dot);
            dot = __dp4a(kc[4 * i + 2], qv.z, dot);
            dot = __dp4a(kc[4 * i + 3], qv.w, dot);
        }
        total += w[h] * max(dot, 0);
    }
    return total;
}

// Scores of 16 blocks (one m16 tile) for one query on the int8 tensor cores:
// S^T[block][head] = kc[block] . q_idx[head] with mma.m16n8k32 s8 (coarse keys
// as the M operand, straight from global memory into the A fragment; the query
// as B).  Lane (g, c) holds bytes 4c.., 16+4c.., 32+4c.., 48+4c.. of blocks g
// and g+8 (tile16_load); qb holds the lane's B fragments for 2 k-steps x 2
// head tiles.  The epilogue applies max(0, .) and the head weights to the
// lane's four heads and sums over the quad: every lane of quad g ends with
// S[g] and S[g+8].  Heads past the query's head count carry zero weight.
struct Tile16 {
    int a[2][4];
};

__device__ __forceinline__ void tile16_load(const int8_t *kc_pool, int page_g, int page_g8, Tile16 &f) {
    const int c = threadIdx.x & 3;
    const int *row_g = reinterpret_cast<const int *>(kc_pool + (size_t)max(page_g, 0) * kIdxDim);
    const int *row_g8 = reinterpret_cast<const int *>(kc_pool + (size_t)max(page_g8, 0) * kIdxDim);
#pragma unroll
    for (int ks = 0; ks < 2; ++ks) {
        f.a[ks][0] = page_g >= 0 ? __ldg(row_g + 8 * ks + c) : 0;
        f.a[ks][1] = page_g8 >= 0 ? __ldg(row_g8 + 8 * ks + c) : 0;
        f.a[ks][2] = page_g >= 0 ? __ldg(row_g + 8 * ks + 4 + c) : 0;
        f.a[ks][3] = page_g8 >= 0 ? __ldg(row_g8 + 8 * ks + 4 + c) : 0;
    }
}

__device__ __forceinline__ void tile16_scores(const Tile16 &f, const int (&qb)[2][2][2], const int (&wl)[2][2],
                                              int &s_g, int &s_g8) {
    int acc[2][4] = {{0, 0, 0, 0}, {0, 0, 0, 0}};
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int ks = 0; ks < 2; ++ks) mma_s8_16832(acc[nt], f.a[ks], qb[nt][ks][0], qb[nt][ks][1]);
    // lane holds heads 8nt+2c, 8nt+2c+1 of blocks g (acc[.][0..1]) and g+8 (acc[.][2..3])
    int sg = 0, sg8 = 0;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
        sg += wl[nt][0] * max(acc[nt][0], 0) + wl[nt][1] * max(acc[nt][1], 0);
        sg8 += wl[nt][0] * max(acc[nt][2], 0) + wl[nt][1] * max(acc[nt][3], 0);
    }
    sg += __shfl_xor_sync(0xffffffffu, sg, 1);
    sg += __shfl_xor_sync(0xffffffffu, sg, 2);
    sg8 += __shfl_xor_sync(0xffffffffu, sg8, 1);
    sg8 += __shfl_xor_sync(0xffffffffu, sg8, 2);
    s_g = sg;
    s_g8 = sg8;
}

}  // namespace dsa
