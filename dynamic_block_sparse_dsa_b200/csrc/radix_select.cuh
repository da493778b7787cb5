// radix_select.cuh -- CTA-wide exact selection of the `need` largest of a set
// of unique 64-bit keys held in registers (key = order key of the score << 32
// | ~block id, so "larger" is the order score descending, block id ascending
// and no two keys tie; 0 marks an empty slot and is never selected).
//
// The threshold is found digit by digit, eight bits at a time from the
// highest bit where the keys differ: a shared-memory histogram of the digit
// over the keys still tied with the threshold, then one warp finds the bin
// where the count from the top reaches `need`.  The walk stops as soon as that
// bin is taken whole, which unique keys guarantee by the last digit at the
// latest.  Two barriers per digit; typically two or three digits.
#pragma once

#include "dsa_common.cuh"

namespace dsa {

struct RadixScratch {
    uint32_t hist[256];
    uint32_t state[4];                    // digit, still needed, taken whole
    unsigned long long ored[32], anded[32];   // per-warp OR / AND of the keys
    int count[32];                        // per-warp number of keys
};

// On return, in every thread: a non-zero key k is among the `need` largest
// non-zero keys of the CTA iff (k & mask) >= prefix.  If the CTA holds at
// most `need` non-zero keys, prefix = mask = 0 (every non-zero key is taken).
// Returns the number of non-zero keys.  Every thread of the CTA must call it
// with the same `need` (>= 1).
template <int kThreads, int kPer>
__device__ __forceinline__ int cta_radix_threshold(const unsigned long long (&k)[kPer], uint32_t need,
                                                   RadixScratch &s, unsigned long long &prefix,
                                                   unsigned long long &mask) {
    constexpr int kWarps = kThreads / 32;
    static_assert(kThreads >= 256 && kWarps <= 32, "one histogram bin per thread");
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    // the bits where the non-zero keys differ, and how many there are
    unsigned long long o = 0ull, a = ~0ull;
    int cnt = 0;
#pragma unroll
    for (int i = 0; i < kPer; ++i)
        if (k[i] != 0ull) {
            o |= k[i];
            a &= k[i];
            ++cnt;
        }
#pragma unroll
    for (int d = 16; d > 0; d >>= 1) {
        o |= __shfl_xor_sync(0xffffffffu, o, d);
        a &= __shfl_xor_sync(0xffffffffu, a, d);
    }
    cnt = __reduce_add_sync(0xffffffffu, cnt);
    if (lane == 0) {
        s.ored[warp] = o;
        s.anded[warp] = a;
        s.count[warp] = cnt;
    }
    if (tid < 256) s.hist[tid] = 0u;
    __syncthreads();
    o = 0ull;
    a = ~0ull;
    int total = 0;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
        o |= s.ored[w];
        a &= s.anded[w];
        total += s.count[w];
    }
    prefix = 0ull;
    mask = 0ull;
    if ((uint32_t)total <= need) return total;
    const unsigned long long diff = o & ~a;   // total > need >= 1: at least two keys, so diff != 0
    for (int hi = 63 - __clzll((long long)diff); hi >= 0;) {
        const int sh = hi >= 7 ? hi - 7 : 0;
        const uint32_t dmask = (2u << (hi - sh)) - 1u;
#pragma unroll
        for (int i = 0; i < kPer; ++i)
            if (k[i] != 0ull && (k[i] & mask) == prefix) atomicAdd(&s.hist[(uint32_t)(k[i] >> sh) & dmask], 1u);
        __syncthreads();
        if (warp == 0) {
            // bins from the top: lane l holds bins 255 - 8l down to 248 - 8l
            uint32_t c[8], sum = 0;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                c[j] = s.hist[255 - 8 * lane - j];
                s.hist[255 - 8 * lane - j] = 0u;   // cleared for the next digit
                sum += c[j];
            }
            uint32_t incl = sum;
#pragma unroll
            for (int d = 1; d < 32; d <<= 1) {
                const uint32_t v = __shfl_up_sync(0xffffffffu, incl, d);
                if (lane >= d) incl += v;
            }
            const uint32_t excl = incl - sum;
            if (excl < need && need <= incl) {   // exactly one lane holds the threshold's bin
                uint32_t above = excl, bin = 0, cb = 0;
                bool found = false;
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    if (!found) {
                        if (above + c[j] >= need) {
                            found = true;
                            bin = (uint32_t)(255 - 8 * lane - j);
                            cb = c[j];
                        } else {
                            above += c[j];
                        }
                    }
                }
                s.state[0] = bin;
                s.state[1] = need - above;
                s.state[2] = cb == need - above ? 1u : 0u;
            }
        }
        __syncthreads();
        prefix |= (unsigned long long)s.state[0] << sh;
        mask |= (unsigned long long)dmask << sh;
        need = s.state[1];
        if (s.state[2] != 0u) break;
        hi = sh - 1;
        // the next digit's adds follow the state reads of every thread: the
        // barrier after them (before warp 0 writes the state again) orders both
    }
    return total;
}

}  // namespace dsa
