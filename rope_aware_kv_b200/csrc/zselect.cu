// zselect.cu -- top-B selection of the split prune path by z-bins.
//
// Keep the B keys with the highest final score, in ascending index order
// (B per unit when a per-unit budget array is given: per-layer budgets)
// (talk page: keep only the top-B; jaedaily.cn tutorial, eviction step:
// top-k then sort to keep the temporal order).  Ranking: score descending,
// NaN lowest, -0.0 == +0.0, equal scores by ascending index.
//
// The final scores here are z-scores (maxima over the GQA group of per-head
// standardised scores), so a linear histogram of z (2048 bins of width 1/64
// over [-16, 16), built by the z-max kernel) places the B-th key in a bin
// that holds few keys.  Four kernels then finish the selection with two
// passes over the final scores (instead of two radix passes, a count and a
// compaction):
//   bin      per unit (one warp): the B-th key's bin b0 and the keys above it;
//   collect  per chunk of kZChunk keys: the keys above the B-th key's bin b0
//            are counted, the keys inside b0 (the candidates) are listed per
//            unit (up to kCandMax).
//   rank     per unit: the threshold key T (the B-th key's ordered 32-bit
//            key) and the number kt of keys equal to T that are kept, by a
//            radix select over the candidates (or, if they overflowed the
//            list, over the unit's keys in b0); then every chunk's base rank:
//            keys above T before the chunk plus min(ties before it, kt).
//   compact  per chunk: the kept indices in order from the chunk's base.
#include "tri_internal.cuh"
#include "tri_launch.h"
#include "select_core.cuh"

namespace tri {

// Per-unit selection state: the B-th key's z-bin b0 and the keys above it
// (bin kernel), then the threshold key T and the ties of T kept (rank kernel).
struct ZSelState {
    uint32_t b0;
    uint32_t above;
    uint32_t T;   // ordered key of the B-th key
    uint32_t kt;  // keys equal to T that are kept
};

// ---------------------------------------------------------------------------
// bin: the z-bin of each unit's B-th key, once per unit (grid U, one warp).
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(32)
zsel_bin_kernel(int64_t cap, const int32_t* __restrict__ n_valid, int64_t B,
                const int32_t* __restrict__ ub, const uint32_t* __restrict__ zhist,
                ZSelState* __restrict__ st) {
    const int64_t u = blockIdx.x;
    const int n = clamp_nvalid(n_valid, u, cap, nullptr);
    const int64_t Bu = unit_budget(ub, u, B);
    if (n <= Bu || Bu == 0) return;
    uint32_t bin, above;
    warp_find_bin(zhist + u * kZBins, kZBins, static_cast<uint32_t>(Bu), bin, above);
    if (threadIdx.x == 0) {
        st[u].b0 = bin;
        st[u].above = above;
    }
}

__device__ __forceinline__ uint32_t block_sum_256(uint32_t v, uint32_t* red8) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (lane == 0) red8[warp] = v;
    __syncthreads();
    uint32_t t = 0;
#pragma unroll
    for (int w = 0; w < 8; ++w) t += red8[w];
    __syncthreads();
    return t;
}

// ---------------------------------------------------------------------------
// collect: keys above b0 per chunk, candidates in b0 per unit.
// grid (chunks, U), 256 threads; each thread keeps its 8 keys' loads in flight.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256)
zsel_collect_kernel(const float* __restrict__ fin, int64_t cap, const int32_t* __restrict__ n_valid,
                    int64_t B, const int32_t* __restrict__ ub, const uint32_t* __restrict__ zhist,
                    uint2* __restrict__ counts, int2* __restrict__ cand,
                    uint32_t* __restrict__ cand_count, const ZSelState* __restrict__ st) {
    __shared__ uint32_t red8[8];
    const int64_t u = blockIdx.y;
    const int n = clamp_nvalid(n_valid, u, cap, nullptr);
    const int64_t Bu = unit_budget(ub, u, B);
    if (n <= Bu || Bu == 0) return;
    (void)zhist;
    const uint32_t b0 = __ldg(&st[u].b0);
    const int j0 = blockIdx.x * kZChunk;
    constexpr int kPer = kZChunk / 256;
    float f[kPer];
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
        const int j = j0 + threadIdx.x + 256 * i;
        f[i] = j < n ? fin[u * cap + j] : 0.f;
    }
    uint32_t above = 0;
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
        const int j = j0 + threadIdx.x + 256 * i;
        if (j < n) {
            const uint32_t zb = zbin(f[i]);
            above += zb > b0;
            if (zb == b0) {
                const uint32_t r = atomicAdd(&cand_count[u], 1u);
                if (r < static_cast<uint32_t>(kCandMax))
                    cand[u * kCandMax + r] = make_int2(static_cast<int>(ordered_key(f[i])), j);
            }
        }
    }
    above = block_sum_256(above, red8);
    if (threadIdx.x == 0) counts[u * gridDim.x + blockIdx.x] = make_uint2(above, 0u);
}

// Exclusive prefix sum over the block's 256 threads; returns this thread's
// prefix and writes the block total into *total.
__device__ __forceinline__ uint32_t block_excl_scan_256(uint32_t v, uint32_t* red8, uint32_t* total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint32_t incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t t = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += t;
    }
    if (lane == 31) red8[warp] = incl;
    __syncthreads();
    uint32_t before = 0, all = 0;
#pragma unroll
    for (int w = 0; w < 8; ++w) {
        before += w < warp ? red8[w] : 0u;
        all += red8[w];
    }
    __syncthreads();
    *total = all;
    return before + incl - v;
}

// ---------------------------------------------------------------------------
// rank: the threshold key and the chunks' base ranks of one unit.
// grid U, 256 threads, dynamic shared memory: the unit's candidate list.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256)
zsel_rank_kernel(const float* __restrict__ fin, int64_t cap, const int32_t* __restrict__ n_valid,
                 int64_t B, const int32_t* __restrict__ ub, const uint32_t* __restrict__ zhist,
                 uint2* __restrict__ counts, int n_chunks, const int2* __restrict__ cand,
                 const uint32_t* __restrict__ cand_count, ZSelState* __restrict__ st) {
    extern __shared__ int2 sc[];  // [kCandMax]
    __shared__ uint32_t hist[kHistBins0];
    __shared__ uint32_t sb0, sk, sprefix;
    __shared__ uint32_t red8[8];
    const int64_t u = blockIdx.x;
    const int n = clamp_nvalid(n_valid, u, cap, nullptr);
    const int64_t Bu = unit_budget(ub, u, B);
    if (n <= Bu || Bu == 0) return;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    if (tid == 0) {
        sb0 = st[u].b0;
        sk = static_cast<uint32_t>(Bu) - st[u].above;  // rank of the Bu-th key inside bin b0
        sprefix = 0;
    }
    (void)zhist;
    const uint32_t nc_all = cand_count[u];
    const bool listed = nc_all <= static_cast<uint32_t>(kCandMax);
    const int nc = listed ? static_cast<int>(nc_all) : 0;
    for (int i = tid; i < nc; i += 256) sc[i] = cand[u * kCandMax + i];
    __syncthreads();
    const uint32_t b0 = sb0;
    // Three-digit radix select of the sk-th largest key among the keys of b0.
    for (int p = 0; p < 3; ++p) {
        const int nb = 1 << pass_bits(p);
        for (int b = tid; b < nb; b += 256) hist[b] = 0;
        __syncthreads();
        const uint32_t prefix = sprefix;
        const int shift = pass_shift(p);
        const int hi_shift = shift + pass_bits(p);
        if (listed) {
            for (int i = tid; i < nc; i += 256) {
                const uint32_t key = static_cast<uint32_t>(sc[i].x);
                if (p == 0 || (key >> hi_shift) == prefix) atomicAdd(&hist[(key >> shift) & (nb - 1)], 1u);
            }
        } else {
            for (int j = tid; j < n; j += 256) {
                const float f = fin[u * cap + j];
                const uint32_t key = ordered_key(f);
                if (zbin(f) == b0 && (p == 0 || (key >> hi_shift) == prefix))
                    atomicAdd(&hist[(key >> shift) & (nb - 1)], 1u);
            }
        }
        __syncthreads();
        if (warp == 0) {
            uint32_t bin, above;
            warp_find_bin(hist, nb, sk, bin, above);
            if (lane == 0) {
                sprefix = (prefix << pass_bits(p)) | bin;
                sk -= above;
            }
        }
        __syncthreads();
    }
    const uint32_t T = sprefix, kt = sk;
    // Each chunk's keys above T and ties of T (its keys above b0 are already
    // counted): from the list, or from the unit's keys in b0.
    uint2* cu = counts + u * n_chunks;
    if (listed) {
        for (int i = tid; i < nc; i += 256) {
            const int2 e = sc[i];
            const uint32_t key = static_cast<uint32_t>(e.x);
            const int c = e.y / kZChunk;
            if (key > T) atomicAdd(&cu[c].x, 1u);
            if (key == T) atomicAdd(&cu[c].y, 1u);
        }
    } else {
        for (int j = tid; j < n; j += 256) {
            const float f = fin[u * cap + j];
            if (zbin(f) != b0) continue;
            const uint32_t key = ordered_key(f);
            if (key > T) atomicAdd(&cu[j / kZChunk].x, 1u);
            if (key == T) atomicAdd(&cu[j / kZChunk].y, 1u);
        }
    }
    __syncthreads();
    // Base ranks: keys above T in earlier chunks plus the ties of T taken in
    // index order before the chunk (at most kt).
    uint32_t gt_run = 0, eq_run = 0;
    for (int c0 = 0; c0 < n_chunks; c0 += 256) {
        const int c = c0 + tid;
        const uint2 v = c < n_chunks ? __ldcg(&cu[c]) : make_uint2(0u, 0u);
        uint32_t gt_tot, eq_tot;
        const uint32_t gt_b = block_excl_scan_256(v.x, red8, &gt_tot);
        const uint32_t eq_b = block_excl_scan_256(v.y, red8, &eq_tot);
        if (c < n_chunks) {
            const uint32_t ties = eq_run + eq_b;
            cu[c] = make_uint2(gt_run + gt_b + min(ties, kt), ties);
        }
        gt_run += gt_tot;
        eq_run += eq_tot;
    }
    if (tid == 0) {
        st[u].T = T;
        st[u].kt = kt;
    }
}

// ---------------------------------------------------------------------------
// compact: the kept indices of one chunk, in order.  grid (chunks, U), 256
// threads; warp w walks keys j0 + 256 w + 32 i + lane, i = 0..7; ballots
// give each kept key its rank.  Units with n_valid <= B keep every key.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256)
zsel_compact_kernel(const float* __restrict__ fin, int64_t cap, const int32_t* __restrict__ n_valid,
                    int64_t B, const int32_t* __restrict__ ub, const uint2* __restrict__ counts,
                    const ZSelState* __restrict__ st, int32_t* __restrict__ kept,
                    int32_t* __restrict__ n_kept) {
    __shared__ uint32_t wgt[8], weq[8];
    const int64_t u = blockIdx.y;
    const int n = clamp_nvalid(n_valid, u, cap, nullptr);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t Bu = unit_budget(ub, u, B);
    const int64_t m = n < Bu ? n : Bu;
    int32_t* out = kept + u * B;
    const int j0 = blockIdx.x * kZChunk + warp * 256;
    if (n <= Bu) {
        for (int i = 0; i < 8; ++i) {
            const int j = j0 + 32 * i + lane;
            if (j < n) out[j] = j;
        }
    } else if (Bu > 0) {
        // Every score load of the thread is issued before the first use of
        // the unit's state (and before the first ballot).
        float fv[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int j = j0 + 32 * i + lane;
            fv[i] = j < n ? __ldcs(&fin[u * cap + j]) : 0.f;
        }
        const ZSelState s = st[u];
        const uint2 base = counts[u * gridDim.x + blockIdx.x];
        uint32_t key[8];
        uint32_t gt = 0, eq = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int j = j0 + 32 * i + lane;
            const bool valid = j < n;
            key[i] = valid ? ordered_key(fv[i]) : 0u;
            gt += __popc(__ballot_sync(0xffffffffu, valid && key[i] > s.T));
            eq += __popc(__ballot_sync(0xffffffffu, valid && key[i] == s.T));
        }
        if (lane == 0) {
            wgt[warp] = gt;
            weq[warp] = eq;
        }
        __syncthreads();
        uint32_t pos = base.x, ties = base.y;
        for (int w = 0; w < warp; ++w) {
            const uint32_t take = ties < s.kt ? min(weq[w], s.kt - ties) : 0u;
            pos += wgt[w] + take;
            ties += weq[w];
        }
        const uint32_t lt = (1u << lane) - 1u;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int j = j0 + 32 * i + lane;
            const bool valid = j < n;
            const bool is_eq = valid && key[i] == s.T;
            const uint32_t beq = __ballot_sync(0xffffffffu, is_eq);
            const uint32_t my_tie = ties + __popc(beq & lt);
            const bool keep = valid && (key[i] > s.T || (is_eq && my_tie < s.kt));
            const uint32_t bk = __ballot_sync(0xffffffffu, keep);
            if (keep) {
                const uint32_t r = pos + __popc(bk & lt);
                if (r < static_cast<uint32_t>(Bu)) out[r] = j;
            }
            pos += __popc(bk);
            ties += __popc(beq);
        }
    }
    if (blockIdx.x == 0) {
        if (threadIdx.x == 0) n_kept[u] = static_cast<int32_t>(m);
        for (int64_t r = m + threadIdx.x; r < B; r += blockDim.x) out[r] = -1;
    }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
size_t zsel_state_bytes() { return sizeof(ZSelState); }

cudaError_t launch_zselect(const float* fin, int64_t n_units, int64_t cap, const int32_t* n_valid,
                           int64_t B, const int32_t* ub, const uint32_t* zhist, uint2* counts,
                           int2* cand, uint32_t* cand_count, void* state, int32_t* kept,
                           int32_t* n_kept, cudaStream_t s) {
    const int n_chunks = static_cast<int>((cap + kZChunk - 1) / kZChunk);
    dim3 grid(static_cast<unsigned>(n_chunks), static_cast<unsigned>(n_units));
    ZSelState* st = static_cast<ZSelState*>(state);
    zsel_bin_kernel<<<static_cast<unsigned>(n_units), 32, 0, s>>>(cap, n_valid, B, ub, zhist, st);
    note_launch(s);
    zsel_collect_kernel<<<grid, 256, 0, s>>>(fin, cap, n_valid, B, ub, zhist, counts, cand,
                                             cand_count, st);
    note_launch(s);
    const size_t smem = static_cast<size_t>(kCandMax) * sizeof(int2);
    cudaError_t e = cudaFuncSetAttribute(zsel_rank_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    zsel_rank_kernel<<<static_cast<unsigned>(n_units), 256, smem, s>>>(
        fin, cap, n_valid, B, ub, zhist, counts, n_chunks, cand, cand_count, st);
    note_launch(s);
    zsel_compact_kernel<<<grid, 256, 0, s>>>(fin, cap, n_valid, B, ub, counts, st, kept, n_kept);
    note_launch(s);
    return cudaGetLastError();
}

}  // namespace tri
