// compact.cu -- order-preserving gather of kept K/V/position rows, and the
// append of newly generated rows used by the windowed streaming driver.
//
// Gather: K_dst[u][r] = K[u][kept[u][r]], same for V and positions, r < n_kept
// (jaedaily.cn KV-compression tutorial, eviction step: keys[idx], values[idx]
// with idx sorted so the temporal order is kept).  Rows are bit copies moved
// as 16-byte vectors: 16 lanes per 256-byte bf16 row (32 per float32 row),
// so each warp moves two (or one) whole rows per instruction.
#include "tri_internal.cuh"
#include "tri_launch.h"

namespace tri {

// One 16-byte lane per vector; a row has kVec vectors.  Grid-stride over all
// (unit, kept row) pairs; 4 rows per lane in flight for memory parallelism.
// Four CTAs per SM (at most 64 registers a thread) instead of the three that
// an unbounded register count allows: 128 KB of loads in flight per SM, and
// 1.03 -> 0.83 ms for the long-prefill workload's 3.3 GB of kept rows.
template <int kVec>
__global__ void __launch_bounds__(256, 4)
gather_kernel(const uint4* __restrict__ k_src, const uint4* __restrict__ v_src,
              const int32_t* __restrict__ pos_src, int64_t n_units, int64_t cap_src,
              const int32_t* __restrict__ kept, const int32_t* __restrict__ n_kept, int64_t B,
              uint4* __restrict__ k_dst, uint4* __restrict__ v_dst, int32_t* __restrict__ pos_dst,
              int64_t cap_dst, uint32_t* flag) {
    constexpr int kRowsPerBlock = 256 / kVec;
    constexpr int kUnroll = 4;
    const int lane = threadIdx.x % kVec;
    const int rsub = threadIdx.x / kVec;
    const int64_t total = n_units * B;
    for (int64_t base = static_cast<int64_t>(blockIdx.x) * kRowsPerBlock * kUnroll; base < total;
         base += static_cast<int64_t>(gridDim.x) * kRowsPerBlock * kUnroll) {
        uint4 kv[kUnroll], vv[kUnroll];
        int64_t src[kUnroll], dst[kUnroll];
#pragma unroll
        for (int q = 0; q < kUnroll; ++q) {
            const int64_t g = base + q * kRowsPerBlock + rsub;
            src[q] = -1;
            if (g < total) {
                const int64_t u = g / B;
                const int64_t r = g - u * B;
                int64_t nk = n_kept[u];
                const int64_t lim = B < cap_dst ? B : cap_dst;
                if (nk > lim || nk < 0) {
                    if (lane == 0 && r == 0) raise_flag(flag, TRI_FLAG_INDEX_RANGE);
                    nk = nk < 0 ? 0 : lim;
                }
                if (r < nk) {
                    const int32_t j = kept[g];
                    if (j >= 0 && j < cap_src) {
                        src[q] = u * cap_src + j;
                        dst[q] = u * cap_dst + r;
                    } else if (lane == 0) {
                        raise_flag(flag, TRI_FLAG_INDEX_RANGE);
                    }
                }
            }
        }
#pragma unroll
        for (int q = 0; q < kUnroll; ++q) {
            if (src[q] >= 0) {
                kv[q] = ld_stream(k_src + src[q] * kVec + lane);
                if (v_src) vv[q] = ld_stream(v_src + src[q] * kVec + lane);
            }
        }
#pragma unroll
        for (int q = 0; q < kUnroll; ++q) {
            if (src[q] >= 0) {
                st_stream(k_dst + dst[q] * kVec + lane, kv[q]);
                if (v_dst) st_stream(v_dst + dst[q] * kVec + lane, vv[q]);
                if (pos_dst && lane == 0) pos_dst[dst[q]] = pos_src[src[q]];
            }
        }
    }
}

cudaError_t launch_gather(tri_dtype dt, const void* k_src, const void* v_src,
                          const int32_t* pos_src, int64_t n_units, int64_t cap_src,
                          const int32_t* kept, const int32_t* n_kept, int64_t B, void* k_dst,
                          void* v_dst, int32_t* pos_dst, int64_t cap_dst, uint32_t* flag,
                          int n_blocks, cudaStream_t s) {
    const int64_t total = n_units * B;
    if (total == 0) return cudaSuccess;
    if (dt == TRI_BF16) {
        constexpr int kVec = kD * 2 / 16;
        const int64_t need = (total + (256 / kVec) * 4 - 1) / ((256 / kVec) * 4);
        const int grid = static_cast<int>(need < n_blocks ? need : n_blocks);
        gather_kernel<kVec><<<grid, 256, 0, s>>>(
            static_cast<const uint4*>(k_src), static_cast<const uint4*>(v_src), pos_src, n_units,
            cap_src, kept, n_kept, B, static_cast<uint4*>(k_dst), static_cast<uint4*>(v_dst),
            pos_dst, cap_dst, flag);
        note_launch(s);
    } else {
        constexpr int kVec = kD * 4 / 16;
        const int64_t need = (total + (256 / kVec) * 4 - 1) / ((256 / kVec) * 4);
        const int grid = static_cast<int>(need < n_blocks ? need : n_blocks);
        gather_kernel<kVec><<<grid, 256, 0, s>>>(
            static_cast<const uint4*>(k_src), static_cast<const uint4*>(v_src), pos_src, n_units,
            cap_src, kept, n_kept, B, static_cast<uint4*>(k_dst), static_cast<uint4*>(v_dst),
            pos_dst, cap_dst, flag);
        note_launch(s);
    }
    return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// In-place compaction: row kept[u][r] moves to row r of the same buffer, for
// r < n_kept[u] (the same bit copies as the gather, without a second cache).
// A kept list is ascending, so kept[r] >= r and rows only move towards the
// front.  Each CTA walks one unit's rows in rounds of kRows destinations: a
// round loads every source row it needs into registers, passes a CTA
// barrier (loads requested before it are performed for every thread of the
// CTA), then stores.  A round's sources lie at or after its first
// destination row and its destinations before the next round's first one,
// so no store lands on a row that a later round still has to read; rows
// whose source is outside [r, cap) are skipped and flagged.  A round in
// which every row stays where it is (the prefix before the first dropped
// row) moves nothing.
// ---------------------------------------------------------------------------
template <int kVec>
__global__ void __launch_bounds__(256)
compact_inplace_kernel(uint4* __restrict__ k, uint4* __restrict__ v, int32_t* __restrict__ pos,
                       int64_t n_units, int64_t cap, const int32_t* __restrict__ kept,
                       const int32_t* __restrict__ n_kept, int64_t B, uint32_t* flag,
                       const PageMap pm) {
    constexpr int kThreads = 256;
    constexpr int kRows = 64;                        // destination rows per round
    constexpr int kPer = kRows * kVec / kThreads;    // vectors per thread per array
    static_assert(kRows * kVec % kThreads == 0, "round must split evenly");
    const int tid = threadIdx.x;
    const int64_t lim = B < cap ? B : cap;
    for (int64_t u = blockIdx.x; u < n_units; u += gridDim.x) {
        int64_t nk = n_kept[u];
        if (nk > lim || nk < 0) {
            if (tid == 0) raise_flag(flag, TRI_FLAG_INDEX_RANGE);
            nk = nk < 0 ? 0 : lim;
        }
        const int32_t* ku = kept + u * B;
        for (int64_t r0 = 0; r0 < nk; r0 += kRows) {
            // Source row of each destination row this thread moves (-1: none),
            // and the physical rows of both (a paged pool maps them).
            int64_t src[kPer], ps[kPer], pd[kPer];
            bool still = true;
#pragma unroll
            for (int q = 0; q < kPer; ++q) {
                const int64_t r = r0 + (tid + q * kThreads) / kVec;
                src[q] = -1;
                if (r < nk) {
                    const int64_t j = ku[r];
                    const int64_t pj = (j >= r && j < cap) ? phys_row(pm, u, cap, j) : -1;
                    const int64_t pr = pj >= 0 ? phys_row(pm, u, cap, r) : -1;
                    if (pr >= 0) {
                        src[q] = j;
                        ps[q] = pj;
                        pd[q] = pr;
                        still = still && j == r;
                    } else if ((tid + q * kThreads) % kVec == 0) {
                        raise_flag(flag, TRI_FLAG_INDEX_RANGE);
                    }
                }
            }
            if (__syncthreads_and(still)) continue;
            const int lane = tid % kVec;
            uint4 kv[kPer], vv[kPer];
            int32_t pv[kPer];
#pragma unroll
            for (int q = 0; q < kPer; ++q) {
                if (src[q] >= 0) {
                    kv[q] = k[ps[q] * kVec + lane];
                    if (v) vv[q] = v[ps[q] * kVec + lane];
                    if (pos && lane == 0) pv[q] = pos[u * cap + src[q]];
                }
            }
            __syncthreads();
#pragma unroll
            for (int q = 0; q < kPer; ++q) {
                if (src[q] >= 0) {
                    const int64_t r = r0 + (tid + q * kThreads) / kVec;
                    k[pd[q] * kVec + lane] = kv[q];
                    if (v) v[pd[q] * kVec + lane] = vv[q];
                    if (pos && lane == 0) pos[u * cap + r] = pv[q];
                }
            }
        }
        __syncthreads();
    }
}

cudaError_t launch_compact_inplace(tri_dtype dt, void* k, void* v, int32_t* pos, int64_t n_units,
                                   int64_t cap, const int32_t* kept, const int32_t* n_kept,
                                   int64_t B, uint32_t* flag, int n_blocks, cudaStream_t s,
                                   const PageMap& pm) {
    if (n_units == 0) return cudaSuccess;
    const int grid = static_cast<int>(n_units < n_blocks ? n_units : n_blocks);
    if (dt == TRI_BF16) {
        compact_inplace_kernel<kD * 2 / 16><<<grid, 256, 0, s>>>(
            static_cast<uint4*>(k), static_cast<uint4*>(v), pos, n_units, cap, kept, n_kept, B,
            flag, pm);
    } else {
        compact_inplace_kernel<kD * 4 / 16><<<grid, 256, 0, s>>>(
            static_cast<uint4*>(k), static_cast<uint4*>(v), pos, n_units, cap, kept, n_kept, B,
            flag, pm);
    }
    note_launch(s);
    return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Append n_new rows per unit at rows n_valid[u] .. n_valid[u] + n_new - 1.
// One CTA per unit; the new position count and p_cur are written by thread 0
// after every thread has read n_valid.
// ---------------------------------------------------------------------------
template <int kVec>
__global__ void __launch_bounds__(256)
append_kernel(uint4* __restrict__ k_cache, uint4* __restrict__ v_cache, int32_t* __restrict__ pos_cache,
              int64_t cap, int32_t* __restrict__ n_valid, const uint4* __restrict__ k_new,
              const uint4* __restrict__ v_new, const int32_t* __restrict__ pos_new, int64_t n_new,
              uint32_t* flag) {
    const int64_t u = blockIdx.x;
    __shared__ int n0;
    if (threadIdx.x == 0) n0 = n_valid[u];
    __syncthreads();
    const int n = n0;
    if (n < 0 || n + n_new > cap) {
        if (threadIdx.x == 0) raise_flag(flag, TRI_FLAG_NVALID_RANGE);
        return;
    }
    const int64_t vecs = n_new * kVec;
    for (int64_t e = threadIdx.x; e < vecs; e += blockDim.x) {
        const int64_t r = e / kVec, l = e % kVec;
        const int64_t dst = (u * cap + n + r) * kVec + l;
        const int64_t src = (u * n_new + r) * kVec + l;
        k_cache[dst] = k_new[src];
        if (v_cache) v_cache[dst] = v_new[src];
    }
    if (pos_cache)
        for (int64_t r = threadIdx.x; r < n_new; r += blockDim.x)
            pos_cache[u * cap + n + r] = pos_new[u * n_new + r];
    __syncthreads();
    if (threadIdx.x == 0) n_valid[u] = static_cast<int32_t>(n + n_new);
}

// p_cur[seq] = 1 + max appended position over the sequence's units.
__global__ void __launch_bounds__(256)
append_pcur_kernel(int64_t* __restrict__ p_cur, int64_t units_per_seq,
                   const int32_t* __restrict__ pos_new, int64_t n_new) {
    const int64_t seq = blockIdx.x;
    int32_t best = INT32_MIN;
    const int64_t m = units_per_seq * n_new;
    for (int64_t e = threadIdx.x; e < m; e += blockDim.x)
        best = max(best, pos_new[seq * m + e]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) best = max(best, __shfl_xor_sync(0xffffffffu, best, o));
    __shared__ int32_t red[8];
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = best;
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int w = 1; w < 8; ++w) best = max(best, red[w]);
        p_cur[seq] = static_cast<int64_t>(red[0] > best ? red[0] : best) + 1;
    }
}

cudaError_t launch_append(tri_dtype dt, void* k_cache, void* v_cache, int32_t* pos_cache,
                          int64_t n_seq, int64_t n_units, int64_t cap, int32_t* n_valid,
                          int64_t* p_cur, const void* k_new, const void* v_new,
                          const int32_t* pos_new, int64_t n_new, uint32_t* flag, cudaStream_t s) {
    if (dt == TRI_BF16) {
        append_kernel<kD * 2 / 16><<<static_cast<unsigned>(n_units), 256, 0, s>>>(
            static_cast<uint4*>(k_cache), static_cast<uint4*>(v_cache), pos_cache, cap, n_valid,
            static_cast<const uint4*>(k_new), static_cast<const uint4*>(v_new), pos_new, n_new, flag);
        note_launch(s);
    } else {
        append_kernel<kD * 4 / 16><<<static_cast<unsigned>(n_units), 256, 0, s>>>(
            static_cast<uint4*>(k_cache), static_cast<uint4*>(v_cache), pos_cache, cap, n_valid,
            static_cast<const uint4*>(k_new), static_cast<const uint4*>(v_new), pos_new, n_new, flag);
        note_launch(s);
    }
    if (p_cur && pos_new && n_new > 0) {
        append_pcur_kernel<<<static_cast<unsigned>(n_seq), 256, 0, s>>>(p_cur, n_units / n_seq,
                                                                         pos_new, n_new);
        note_launch(s);
    }
    return cudaGetLastError();
}

}  // namespace tri
