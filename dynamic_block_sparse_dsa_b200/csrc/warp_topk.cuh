// warp_topk.cuh -- exact Top-64 with warp-level bitonic networks.
//
// A candidate is one 64-bit key, (order key of the score << 32) | ~block id:
// larger keys win, so the total order (score descending, block id ascending)
// of the selection is plain unsigned comparison and no two keys tie.  Zero is
// below every real key and pads empty slots.
//
// A warp holds a 64-key list in two registers per lane, element i in lane
// i % 32, register i / 32.  Lists are kept sorted descending: a new batch of
// 64 keys is sorted with a bitonic network (shuffles for strides < 32, an
// in-lane exchange for stride 32) and folded into the running Top-64 by the
// bitonic merge trick -- max(A[i], reverse(B)[i]) holds the 64 largest of
// A and B as a bitonic sequence, which one merge network sorts again.  No
// shared memory, no barriers; CTA-wide results come from a tree of such
// merges through a small shared-memory buffer.
#pragma once

#include "dsa_common.cuh"

namespace dsa {

using key64 = unsigned long long;

__device__ __forceinline__ key64 make_key64(int32_t score, uint32_t id) {
    return ((key64)(static_cast<uint32_t>(score) ^ 0x80000000u) << 32) | (key64)(~id);
}
__device__ __forceinline__ uint32_t key64_id(key64 k) { return ~static_cast<uint32_t>(k); }

// one compare-exchange stage of a descending network at stride j (< 32)
__device__ __forceinline__ key64 cx_lanes(key64 v, int j, bool keep_max) {
    const key64 w = __shfl_xor_sync(0xffffffffu, v, j);
    return keep_max ? (v > w ? v : w) : (v < w ? v : w);
}

// sort the warp's 64 keys descending
__device__ __forceinline__ void warp_sort64_desc(key64 (&v)[2]) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int k = 2; k <= 64; k <<= 1) {
#pragma unroll
        for (int j = k >> 1; j > 0; j >>= 1) {
            if (j == 32) {   // partner is the other register of the same lane (k == 64)
                const key64 hi = v[0] > v[1] ? v[0] : v[1];
                const key64 lo = v[0] > v[1] ? v[1] : v[0];
                v[0] = hi;
                v[1] = lo;
            } else {
#pragma unroll
                for (int r = 0; r < 2; ++r) {
                    const int i = r * 32 + lane;
                    const bool lower = (lane & j) == 0;
                    const bool desc = (i & k) == 0;
                    v[r] = cx_lanes(v[r], j, lower == desc);
                }
            }
        }
    }
}

// sort a bitonic 64-key sequence descending
__device__ __forceinline__ void warp_bitonic_merge64_desc(key64 (&v)[2]) {
    const int lane = threadIdx.x & 31;
    {
        const key64 hi = v[0] > v[1] ? v[0] : v[1];
        const key64 lo = v[0] > v[1] ? v[1] : v[0];
        v[0] = hi;
        v[1] = lo;
    }
#pragma unroll
    for (int j = 16; j > 0; j >>= 1) {
        const bool lower = (lane & j) == 0;
        v[0] = cx_lanes(v[0], j, lower);
        v[1] = cx_lanes(v[1], j, lower);
    }
}

// a <- Top-64 of (a, b), both sorted descending; a stays sorted descending
__device__ __forceinline__ void warp_merge64_desc(key64 (&a)[2], const key64 (&b)[2]) {
    const int lane = threadIdx.x & 31;
    // reverse(b)[i] = b[63 - i]: lane l, register r <- lane 31 - l, register 1 - r
    const key64 r0 = __shfl_sync(0xffffffffu, b[1], 31 - lane);
    const key64 r1 = __shfl_sync(0xffffffffu, b[0], 31 - lane);
    a[0] = a[0] > r0 ? a[0] : r0;
    a[1] = a[1] > r1 ? a[1] : r1;
    warp_bitonic_merge64_desc(a);
}

// Fold a batch of 64 keys (any order, zeros for empty slots) into a running
// descending list whose first kk (1..63) entries are the kk largest keys seen
// so far.  Keys not above the current kk-th largest can never reach those kk,
// so they are dropped first; a batch with none left costs one vote, which is
// the common case once the list has filled (the entries past kk are then only
// a partial record and must not be used).
__device__ __forceinline__ void warp_fold_topk(key64 (&acc)[2], key64 (&v)[2], int kk) {
    const int i = kk - 1;
    const key64 thr = __shfl_sync(0xffffffffu, i < 32 ? acc[0] : acc[1], i & 31);
    const bool p0 = v[0] > thr, p1 = v[1] > thr;
    if (!__any_sync(0xffffffffu, p0 || p1)) return;
    v[0] = p0 ? v[0] : 0ull;
    v[1] = p1 ? v[1] : 0ull;
    warp_sort64_desc(v);
    warp_merge64_desc(acc, v);
}

// sort 64 unsigned 32-bit values ascending (used to order selected block ids)
__device__ __forceinline__ void warp_sort64_asc_u32(uint32_t (&v)[2]) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int k = 2; k <= 64; k <<= 1) {
#pragma unroll
        for (int j = k >> 1; j > 0; j >>= 1) {
            if (j == 32) {
                const uint32_t lo = min(v[0], v[1]), hi = max(v[0], v[1]);
                v[0] = lo;
                v[1] = hi;
            } else {
#pragma unroll
                for (int r = 0; r < 2; ++r) {
                    const int i = r * 32 + lane;
                    const bool lower = (lane & j) == 0;
                    const bool asc = (i & k) == 0;
                    const uint32_t w = __shfl_xor_sync(0xffffffffu, v[r], j);
                    v[r] = (lower == asc) ? min(v[r], w) : max(v[r], w);
                }
            }
        }
    }
}

// Top-64 over all warps of the CTA: every warp passes its sorted list; the
// result (sorted descending) is returned in warp 0's registers.  s_lists holds
// NW * 64 keys.  Every thread of the CTA must call it.
template <int NW>
__device__ __forceinline__ void cta_merge_top64(key64 (&v)[2], key64 *s_lists) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int step = 1; step < NW; step <<= 1) {
        if ((warp & (2 * step - 1)) == step) {   // this warp hands its list to warp - step
            s_lists[warp * 64 + lane] = v[0];
            s_lists[warp * 64 + 32 + lane] = v[1];
        }
        __syncthreads();
        if ((warp & (2 * step - 1)) == 0 && warp + step < NW) {
            const key64 b[2] = {s_lists[(warp + step) * 64 + lane], s_lists[(warp + step) * 64 + 32 + lane]};
            warp_merge64_desc(v, b);
        }
        __syncthreads();
    }
}

}  // namespace dsa
