// select_core.cuh -- radix-select helpers shared by the split and fused paths.
#pragma once

#include "tri_internal.cuh"

namespace tri {

struct SelState {
    uint32_t prefix;  // digits fixed so far
    uint32_t k;       // rank still to find among keys matching the prefix (1-based)
    uint32_t gt;      // keys strictly above the prefix range
    int keep_all;     // n_valid <= B: every valid key is kept
};

// Digit p of the 32-bit key: bits [pass_shift(p), pass_shift(p) + pass_bits(p)).
__host__ __device__ __forceinline__ int pass_bits(int p) { return p < 2 ? 11 : 10; }
__host__ __device__ __forceinline__ int pass_shift(int p) { return p == 0 ? 21 : (p == 1 ? 10 : 0); }

// Descending search in one histogram by a single warp: the bin b* such that
// (sum of bins above b*) < k <= (sum of bins >= b*).  Returns b* and the sum
// above it.
__device__ __forceinline__ void warp_find_bin(const uint32_t* hist, int nbins, uint32_t k,
                                              uint32_t& bin, uint32_t& above) {
    const int lane = threadIdx.x & 31;
    const int per = nbins / 32;
    // Lane 0 owns the highest bins.
    const int hi = nbins - lane * per;  // exclusive
    uint32_t sum = 0;
    for (int b = hi - 1; b >= hi - per; --b) sum += hist[b];
    uint32_t excl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t v = __shfl_up_sync(0xffffffffu, excl, o);
        if (lane >= o) excl += v;
    }
    excl -= sum;  // exclusive prefix (bins above this lane's slice)
    const bool mine = (excl < k) && (k <= excl + sum);
    const uint32_t who = __ballot_sync(0xffffffffu, mine);
    const int src = who ? (__ffs(who) - 1) : 31;
    uint32_t b_out = 0, a_out = 0;
    if (lane == src) {
        uint32_t acc = excl;
        int b = hi - 1;
        for (; b > hi - per; --b) {
            if (acc + hist[b] >= k) break;
            acc += hist[b];
        }
        b_out = static_cast<uint32_t>(b);
        a_out = acc;
    }
    bin = __shfl_sync(0xffffffffu, b_out, src);
    above = __shfl_sync(0xffffffffu, a_out, src);
}

}  // namespace tri
