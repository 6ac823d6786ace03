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

// Linear bin of a standardised score: 2048 bins of width 1/64 over
// [-16, 16), both ends open, NaN in the lowest bin.  Non-decreasing in the
// selection order (NaN lowest, -0 = +0), so the keys above the bin of the
// B-th key are all kept; at the thresholds z-scores reach (|z| of a few
// units) a bin holds far fewer keys than a bin of the key's top 11 bits.
constexpr int kZBins = 2048;
__device__ __forceinline__ uint32_t zbin(float z) {
    if (!(z == z)) return 0u;
    const float t = floorf((z + 16.0f) * 64.0f);
    return t < 0.f ? 0u : (t > 2047.f ? 2047u : static_cast<uint32_t>(t));
}

// Digit p of the 32-bit key: bits [pass_shift(p), pass_shift(p) + pass_bits(p)).
__host__ __device__ __forceinline__ int pass_bits(int p) { return p < 2 ? 11 : 10; }
__host__ __device__ __forceinline__ int pass_shift(int p) { return p == 0 ? 21 : (p == 1 ? 10 : 0); }

// Descending search in one histogram by a single warp: the bin b* such that
// (sum of bins above b*) < k <= (sum of bins >= b*).  Returns b* and the sum
// above it.  Lane l owns the l-th highest slice of nbins / 32 bins (read with
// 16-byte loads; hist must be 16-byte aligned); after a warp scan of the slice
// sums, all lanes scan the slice that holds b* together.
__device__ __forceinline__ void warp_find_bin(const uint32_t* hist, int nbins, uint32_t k,
                                              uint32_t& bin, uint32_t& above) {
    const int lane = threadIdx.x & 31;
    const int per = nbins / 32;                 // 64 or 32
    const int hi = nbins - lane * per;          // exclusive top of this lane's slice
    const uint4* h4 = reinterpret_cast<const uint4*>(hist + (hi - per));
    uint32_t sum = 0;
#pragma unroll 4
    for (int i = 0; i < per / 4; ++i) {
        const uint4 v = h4[i];
        sum += (v.x + v.y) + (v.z + v.w);
    }
    uint32_t incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
    }
    const uint32_t excl = incl - sum;           // bins above this lane's slice
    const bool mine = (excl < k) && (k <= incl);
    const uint32_t who = __ballot_sync(0xffffffffu, mine);
    const int src = who ? (__ffs(who) - 1) : 31;
    const uint32_t base = __shfl_sync(0xffffffffu, excl, src);
    // Slice of lane src, top bin first: lane l takes q consecutive bins.
    const int q = per / 32;                     // 2 or 1
    const int top = nbins - src * per - 1;
    const int i0 = top - lane * q;               // >= 0 for every lane
    const uint32_t v0 = hist[i0];
    const uint32_t v1 = q > 1 ? hist[i0 - 1] : 0u;  // i0 >= 1 whenever q == 2
    const uint32_t loc = v0 + v1;
    uint32_t inc2 = loc;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t v = __shfl_up_sync(0xffffffffu, inc2, o);
        if (lane >= o) inc2 += v;
    }
    const uint32_t exc2 = inc2 - loc;
    const bool hit = (base + exc2 < k) && (k <= base + inc2);
    const uint32_t who2 = __ballot_sync(0xffffffffu, hit);
    const int t = who2 ? (__ffs(who2) - 1) : 31;
    uint32_t b_out = 0, a_out = 0;
    if (lane == t) {
        if (base + exc2 + v0 >= k || q == 1) {
            b_out = static_cast<uint32_t>(top - lane * q);
            a_out = base + exc2;
        } else {
            b_out = static_cast<uint32_t>(top - lane * q - 1);
            a_out = base + exc2 + v0;
        }
    }
    bin = __shfl_sync(0xffffffffu, b_out, t);
    above = __shfl_sync(0xffffffffu, a_out, t);
}

}  // namespace tri
