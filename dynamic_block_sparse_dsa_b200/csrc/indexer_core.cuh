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

}  // namespace dsa
