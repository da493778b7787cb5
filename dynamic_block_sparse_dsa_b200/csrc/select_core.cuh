// select_core.cuh -- CTA-level exact Top-k selection on register-resident keys.
//
// Candidates are (key, id) pairs held E per thread, in id order across the CTA
// (thread i holds list positions i*E .. i*E+E-1, ids ascending along the list).
// cta_select marks exactly `kk` of them: every key above the kk-th largest key
// T, plus the keys equal to T that come first in list order -- i.e. the total
// order (key descending, id ascending) of the block selection.  T is found by
// an MSB-first radix select over four 8-bit digits with a shared-memory
// histogram (lanes holding the same digit are aggregated with match.any); the
// ties are ranked by a CTA-wide prefix count.  Keys are the order-preserving
// unsigned image of the int32 scores.
#pragma once

#include "dsa_common.cuh"

namespace dsa {

__device__ __forceinline__ uint32_t order_key(int32_t v) { return static_cast<uint32_t>(v) ^ 0x80000000u; }

struct SelectSmem {
    uint32_t hist[256];
    uint32_t digit, rem;
    int warp_sum[33];
};

// exclusive prefix sum over the CTA (NT threads); *total = sum of all v
template <int NT>
__device__ __forceinline__ int cta_exclusive_scan(int v, SelectSmem &sh, int *total) {
    constexpr int kWarps = NT / 32;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) sh.warp_sum[warp] = x;
    __syncthreads();
    if (warp == 0) {
        const int w = lane < kWarps ? sh.warp_sum[lane] : 0;
        int incl = w;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        if (lane < kWarps) sh.warp_sum[lane] = incl - w;
        if (lane == 31) sh.warp_sum[32] = incl;
    }
    __syncthreads();
    const int res = sh.warp_sum[warp] + x - v;
    *total = sh.warp_sum[32];
    __syncthreads();
    return res;
}

// Mark exactly kk (0 <= kk <= number of valid candidates) winners in `take`.
// Every thread of the CTA must call it.
template <int NT, int E>
__device__ __forceinline__ void cta_select(const uint32_t (&key)[E], const bool (&valid)[E], int kk,
                                           bool (&take)[E], SelectSmem &sh) {
    const int lane = threadIdx.x & 31;
    uint32_t prefix = 0, mask = 0, remaining = (uint32_t)kk;
    if (kk > 0) {
#pragma unroll 1
        for (int pass = 0; pass < 4; ++pass) {
            const int shift = 24 - 8 * pass;
            for (int i = threadIdx.x; i < 256; i += NT) sh.hist[i] = 0;
            __syncthreads();
#pragma unroll
            for (int e = 0; e < E; ++e) {
                const bool in = valid[e] && (key[e] & mask) == prefix;
                const uint32_t d = in ? (key[e] >> shift) & 255u : 256u + lane;
                const uint32_t peers = __match_any_sync(0xffffffffu, d);
                if (in && lane == __ffs(peers) - 1) atomicAdd(&sh.hist[d], __popc(peers));
            }
            __syncthreads();
            if (threadIdx.x < 32) {
                // lane l owns digits 8l..8l+7; find the digit holding the kk-th largest
                uint32_t c[8], sum = 0;
#pragma unroll
                for (int j = 0; j < 8; ++j) { c[j] = sh.hist[8 * lane + j]; sum += c[j]; }
                uint32_t x = sum;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const uint32_t y = __shfl_down_sync(0xffffffffu, x, o);
                    if (lane + o < 32) x += y;
                }
                const uint32_t above = x - sum;   // keys in the digits of higher lanes
                if (above < remaining && remaining <= above + sum) {
                    uint32_t acc = above;
                    for (int j = 7; j >= 0; --j) {
                        if (acc + c[j] >= remaining) {
                            sh.digit = 8 * lane + j;
                            sh.rem = remaining - acc;
                            break;
                        }
                        acc += c[j];
                    }
                }
            }
            __syncthreads();
            prefix |= sh.digit << shift;
            mask |= 255u << shift;
            remaining = sh.rem;
            __syncthreads();
        }
    }
    // winners: key > T, then the first `remaining` keys == T in list order
    const uint32_t T = prefix;
    int n_eq = 0;
#pragma unroll
    for (int e = 0; e < E; ++e) n_eq += (kk > 0 && valid[e] && key[e] == T);
    int tot;
    const int eq_before = cta_exclusive_scan<NT>(n_eq, sh, &tot);
    int seen = 0;
#pragma unroll
    for (int e = 0; e < E; ++e) {
        bool t = false;
        if (kk > 0 && valid[e]) {
            if (key[e] > T) {
                t = true;
            } else if (key[e] == T) {
                t = eq_before + seen < (int)remaining;
                ++seen;
            }
        }
        take[e] = t;
    }
}

}  // namespace dsa
