// score.cu -- fold, fused score and GQA z-max kernels.
//
// Score of key k for query head h (talk page: S_trig, S_norm and the
// offset-averaged S~; hyper.ai summary, Method section):
//   S~(k) = mean_{delta in D} sum_f |E q_f| |k_f| cos(w_f (p_cur+delta-p_k) + phi_f)
//         + sum_f (1 - R_f) E|q_f| |k_f|.
// With k_f = k'_f e^{-i w_f p_k} (the key de-rotated by its position) every
// trigonometric term is Re(E[q_f] conj(k'_f) e^{i w_f (p_cur+delta)}), so the
// key position cancels and the mean over D is Re(A_f conj(k'_f)) with
//   A_f = E[q_f] e^{i w_f p_cur} C_f,   C_f = (1/|D|) sum_delta e^{i w_f delta}.
// fold_kernel computes A_f (float64, rounded once to float32) and the norm
// weights c_f = (1 - R_f) E|q_f| per query head; the score kernel then needs,
// per key and head, one 128-wide dot product with (Re A_f, Im A_f) pairs and
// one 64-wide dot product of c with the band norms |k'_f| = |k_f|.
//
// Data path: keys stream HBM -> shared memory by TMA (128-byte swizzle, one
// box per 128-byte part of a row) into a ring of half tiles kept full by a
// producer lane; seven math warps each score whole 128-key tiles (4 keys per
// lane, all heads), the tiles of a CTA's range taken round robin within each
// unit.  Each tile's float64 moment partial (a warp reduction) is merged in
// tile order by moment_merge_kernel (or, with TRI_SCORE_DEFER_MERGE 0, by the
// warp that finishes the unit's last tile, through a fence and an atomic
// counter), so mu and sigma are bitwise reproducible.
#include "tri_internal.cuh"
#include "tri_launch.h"
#include "score_core.cuh"
#include "select_core.cuh"

// How many key tiles ahead of its shared-memory ring the score kernel asks
// L2 to fetch (0: no prefetch), and the L2 policy of those requests (0
// evict-first, 1 evict-normal, 2 evict-last).  Off by default: with six
// tiles ahead the kernel read about 10 % more DRAM bytes than the keys (the
// same time within noise); with none it reads each key once.
#ifndef TRI_PREFETCH_TILES
#define TRI_PREFETCH_TILES 0
#endif
#ifndef TRI_PREFETCH_POLICY
#define TRI_PREFETCH_POLICY 0
#endif
// 1: the score kernel only writes each tile's moment partial and a separate
// kernel merges a unit's partials in tile order (no fence and atomic per
// tile: 5 % faster on the long-prefill workload); 0: the warp that finishes
// a unit's last tile merges them.
#ifndef TRI_SCORE_DEFER_MERGE
#define TRI_SCORE_DEFER_MERGE 1
#endif

namespace tri {

// ---------------------------------------------------------------------------
// Fold: per (seq, layer, query head) weights, chunk-major for the score loop.
// Record layout per query head: 16 chunks x 12 floats; chunk c covers bands
// 4c..4c+3: [ReA_4c, ReA_4c+1, ImA_4c, ImA_4c+1, ReA_4c+2, ReA_4c+3, ImA_4c+2,
// ImA_4c+3, c_4c, ..., c_4c+3] (wrec_re / wrec_im / wrec_c).
// One block per (sequence, group of kFoldHeads query heads): the block first
// forms C_f = mean_delta e^{i w_f delta} (256 threads, each a quarter of the
// offsets of one band, merged in a fixed order) and e^{i w_f p_cur}, then
// A_f = E[q_f] e^{i w_f p_cur} C_f for every head of its group, in float64.
// ---------------------------------------------------------------------------
constexpr int kFoldHeads = 64;

__global__ void __launch_bounds__(256)
fold_kernel(const float* __restrict__ stats, const int64_t* __restrict__ p_cur, int64_t n_layers,
            int64_t n_qheads, double theta, FoldOffsets off, int variant, float* __restrict__ wts) {
    __shared__ double part[4][kF][2];
    __shared__ double cf[kF][2], ef[kF][2];
    const int t = threadIdx.x;
    const int64_t seq = blockIdx.x;
    {
        const int f = t & (kF - 1), q = t >> 6;
        const double w = pow(theta, -2.0 * static_cast<double>(f) / static_cast<double>(kD));
        double cre = 0.0, cim = 0.0;
        for (int i = q; i < off.n; i += 4) {
            double sn, cs;
            sincos(w * static_cast<double>(off.v[i]), &sn, &cs);
            cre += cs;
            cim += sn;
        }
        part[q][f][0] = cre;
        part[q][f][1] = cim;
        if (q == 0) {
            double ps, pc;
            sincos(w * static_cast<double>(p_cur[seq]), &ps, &pc);
            ef[f][0] = pc;
            ef[f][1] = ps;
        }
    }
    __syncthreads();
    if (t < kF) {
        const double inv = 1.0 / off.n;
        cf[t][0] = (((part[0][t][0] + part[1][t][0]) + part[2][t][0]) + part[3][t][0]) * inv;
        cf[t][1] = (((part[0][t][1] + part[1][t][1]) + part[2][t][1]) + part[3][t][1]) * inv;
    }
    __syncthreads();
    const int64_t LH = n_layers * n_qheads;
    const int64_t h0 = static_cast<int64_t>(blockIdx.y) * kFoldHeads;
    const int64_t h1 = h0 + kFoldHeads < LH ? h0 + kFoldHeads : LH;
    for (int64_t e = h0 * kF + t; e < h1 * kF; e += blockDim.x) {
        const int64_t lh = e / kF;  // layer * Hq + qh
        const int f = static_cast<int>(e % kF);
        const float* st = stats + (lh * kF + f) * 4;
        const double mre = st[0], mim = st[1];
        const double tre = mre * ef[f][0] - mim * ef[f][1];  // E[q_f] e^{i w p_cur}
        const double tim = mre * ef[f][1] + mim * ef[f][0];
        const bool trig = (variant & TRI_VAR_NO_TRIG) == 0;
        const double are = trig ? tre * cf[f][0] - tim * cf[f][1] : 0.0;  // ... * C_f
        const double aim = trig ? tre * cf[f][1] + tim * cf[f][0] : 0.0;
        const double rw = (variant & TRI_VAR_NO_R) ? 1.0 : 1.0 - static_cast<double>(st[3]);
        const double cw = rw * static_cast<double>(st[2]);
        const int64_t q = seq * LH + lh;  // (seq * L + layer) * Hq + qh
        float* rec = wts + q * kWHead;
        rec[wrec_re(f)] = static_cast<float>(are);
        rec[wrec_im(f)] = static_cast<float>(aim);
        rec[wrec_c(f)] = static_cast<float>(cw);
    }
}

// ---------------------------------------------------------------------------
// Score kernel
// ---------------------------------------------------------------------------
template <typename T>
struct ScoreShape {
    static constexpr int kRowBytes = kD * static_cast<int>(sizeof(T));  // 256 / 512
    static constexpr int kBoxes = kRowBytes / 128;                      // 2 / 4
    static constexpr int kKPT = sizeof(T) == 2 ? 4 : 2;                 // keys per lane
    static constexpr int kTile = 32 * kKPT;                             // keys per tile
    static constexpr int kBoxBytes = kTile * 128;
    static constexpr int kStageBytes = kTile * kRowBytes;               // 32 KB
    static constexpr int kHalfBoxes = kBoxes / 2;
    static constexpr int kHalfBytes = kStageBytes / 2;                  // 16 KB
    static constexpr int kHalfChunks = kHalfBoxes * 8;
    static constexpr int kHSlots = 12;                                  // 192 KB ring
    static constexpr int kMathWarps = 7;
    static constexpr int kMath = 32 * kMathWarps;
    static constexpr int kThreads = kMath + 32;
    // Half-landed barriers indexed by the running half count (a warp takes
    // every kMathWarps-th tile of a unit and skips phases of a slot's
    // barrier).  A warp waiting for a half of tile t has finished tile
    // t - kMathWarps of the same unit, or (its first tile of a unit) every
    // tile before the unit was consumed at the unit's CTA barrier; either
    // way the previous use of the barrier, kHalfBars halves earlier, was
    // consumed when kHalfBars >= 2 kMathWarps + 1 + kHSlots.
    static constexpr int kHalfBars = 32;
    static_assert(kHalfBars >= 2 * kMathWarps + 1 + kHSlots, "half barriers too few");
    static constexpr int kPrefetchTiles = TRI_PREFETCH_TILES;
};

template <typename T, int G>
struct ScoreSmem {
    using S = ScoreShape<T>;
    alignas(1024) uint8_t ring[S::kHSlots][S::kHalfBytes];
    alignas(16) float w[G * kWHead];
    uint64_t full[S::kHalfBars];
    uint64_t empty[S::kHSlots];
    int abort;  // a bounded wait gave up: every thread stops at the next unit
};

// Merge the per-tile moment partials of one unit, by one warp: lane l sums
// tiles l, l+32, ... in order, then a fixed shuffle tree; lane 0's result is
// used, so the merge is bitwise reproducible.
template <int G>
__device__ __forceinline__ void merge_unit_moments(const double* part, int tpu, int n,
                                                   float2* mom_u) {
    const int lane = threadIdx.x & 31;
    double s1[G], s2[G];
#pragma unroll
    for (int h = 0; h < G; ++h) s1[h] = s2[h] = 0.0;
    for (int i = lane; i < tpu; i += 32) {
#pragma unroll
        for (int h = 0; h < G; ++h) {
            s1[h] += part[(static_cast<int64_t>(i) * G + h) * 2];
            s2[h] += part[(static_cast<int64_t>(i) * G + h) * 2 + 1];
        }
    }
#pragma unroll
    for (int h = 0; h < G; ++h) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            s1[h] += __shfl_down_sync(0xffffffffu, s1[h], o);
            s2[h] += __shfl_down_sync(0xffffffffu, s2[h], o);
        }
    }
    if (lane == 0) {
#pragma unroll
        for (int h = 0; h < G; ++h) {
            float mu = 0.f, inv = 0.f;
            if (n > 0) {
                const double m = s1[h] / n;
                double var = s2[h] / n - m * m;
                if (var < 0.0) var = 0.0;
                const double sd = sqrt(var);
                mu = static_cast<float>(m);
                inv = sd > 0.0 ? static_cast<float>(1.0 / sd) : 0.f;
                if (!(sd == sd)) inv = __int_as_float(0x7fc00000);  // NaN propagates
            }
            mom_u[h] = make_float2(mu, inv);
        }
    }
}

template <typename T, int G>
__global__ void __launch_bounds__(ScoreShape<T>::kThreads, 1)
score_kernel(const __grid_constant__ CUtensorMap kmap, ScoreArgs a) {
    using S = ScoreShape<T>;
    extern __shared__ uint8_t smem_raw[];
    ScoreSmem<T, G>& sm = *reinterpret_cast<ScoreSmem<T, G>*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    // This CTA's tiles: a contiguous range of the flattened (unit, tile) list.
    const int64_t total = a.n_units * a.tpu;
    const int64_t t_begin = total * blockIdx.x / gridDim.x;
    const int64_t t_end = total * (blockIdx.x + 1) / gridDim.x;

    if (tid == S::kMath) {
        for (int i = 0; i < S::kHalfBars; ++i) mbar_init(&sm.full[i], 1);
        for (int i = 0; i < S::kHSlots; ++i) mbar_init(&sm.empty[i], 32);
        fence_barrier_init();
        prefetch_tensormap(&kmap);
        sm.abort = 0;
    }
    __syncthreads();

    // Units of the range in order; tiles i0 <= i < i1 of unit u, empty tiles
    // (beyond n_valid) skipped.  hbase counts the halves before the unit.
    const int64_t u_first = t_begin / a.tpu;
    const int64_t u_last = t_end > t_begin ? (t_end - 1) / a.tpu : u_first - 1;
    uint32_t hbase = 0;
    for (int64_t u = u_first; u <= u_last; ++u) {
        const int n = clamp_nvalid(a.n_valid, u, a.cap, tid == 0 ? a.flag : nullptr);
        const int64_t lo = u * a.tpu > t_begin ? u * a.tpu : t_begin;
        const int64_t hi = (u + 1) * a.tpu < t_end ? (u + 1) * a.tpu : t_end;
        const int i0 = static_cast<int>(lo - u * a.tpu);
        const int ntv = (n + S::kTile - 1) / S::kTile;  // tiles with keys
        const int i1 = min(static_cast<int>(hi - u * a.tpu), ntv);
        const int nt = i1 > i0 ? i1 - i0 : 0;
        if (nt == 0) continue;
        // Weights of the unit (every earlier tile is consumed past this barrier).
        __syncthreads();
        if (sm.abort) break;
        {
            const float4* src = reinterpret_cast<const float4*>(a.wts + u * G * kWHead);
            float4* dst = reinterpret_cast<float4*>(sm.w);
            for (int e = tid; e < G * kWHead / 4; e += S::kThreads) dst[e] = src[e];
        }
        __syncthreads();
        if (tid >= S::kMath) {
            if (tid == S::kMath) {
                // Tiles are also requested into L2 kPrefetchTiles ahead of
                // their load into the ring (TRI_PREFETCH_TILES, 0: none).
                const uint64_t pol = TRI_PREFETCH_POLICY == 2   ? policy_evict_last()
                                     : TRI_PREFETCH_POLICY == 1 ? policy_evict_normal()
                                                                : policy_evict_first();
                // First physical row of tile t of the unit (a page holds whole
                // tiles); -1: the tile's page is outside the pool (flagged; its
                // load lands zeros from beyond the tensor map).
                auto tile_row = [&](int t) -> int64_t {
                    return phys_row(a.pm, u, a.cap, static_cast<int64_t>(t) * S::kTile);
                };
                auto prefetch_tile = [&](int k) {
                    if (S::kPrefetchTiles == 0 || k >= nt) return;
                    const int t = i0 + k;
                    const int64_t r0 = tile_row(t);
                    if (r0 < 0) return;
                    const int rows = min(S::kTile, static_cast<int>(a.cap) - t * S::kTile);
                    prefetch_l2_bulk(static_cast<const char*>(a.keys) + r0 * S::kRowBytes,
                                     static_cast<uint32_t>(rows * S::kRowBytes), pol);
                };
                for (int k = S::kHSlots / 2; k < S::kHSlots / 2 + S::kPrefetchTiles; ++k)
                    prefetch_tile(k);
                for (int hh = 0; hh < 2 * nt; ++hh) {
                    if ((hh & 1) == 0 && hh >= S::kHSlots) prefetch_tile(hh / 2 + S::kPrefetchTiles);
                    const uint32_t hc = hbase + hh;
                    const int slot = hc % S::kHSlots;
                    if (sm.abort ||
                        !mbar_wait(&sm.empty[slot], ((hc / S::kHSlots) & 1) ^ 1, a.flag)) {
                        sm.abort = 1;
                        break;
                    }
                    uint64_t* landed = &sm.full[hc % S::kHalfBars];
                    mbar_arrive_expect_tx(landed, S::kHalfBytes);
                    int64_t r0 = tile_row(i0 + (hh >> 1));
                    if (r0 < 0) {
                        raise_flag(a.flag, TRI_FLAG_INDEX_RANGE);
                        r0 = INT32_MAX - S::kTile;  // past the map: zero fill
                    }
                    const int32_t y = static_cast<int32_t>(r0);
#pragma unroll
                    for (int b = 0; b < S::kHalfBoxes; ++b)
                        tma_load_2d(sm.ring[slot] + b * S::kBoxBytes, &kmap, landed,
                                    ((hh & 1) * S::kHalfBoxes + b) *
                                        (128 / static_cast<int>(sizeof(T))),
                                    y);
                }
            }
        } else {
            for (int k = warp; k < nt; k += S::kMathWarps) {
                const int i = i0 + k;
                float2 acc[S::kKPT][G];
                score_acc_zero<G, S::kKPT>(acc);
                bool ok = true;
#pragma unroll 1
                for (int half = 0; half < 2; ++half) {
                    const uint32_t hc = hbase + 2 * k + half;
                    const int slot = hc % S::kHSlots;
                    if (!mbar_wait(&sm.full[hc % S::kHalfBars], (hc / S::kHalfBars) & 1, a.flag)) {
                        ok = false;
                        break;
                    }
                    score_rows_acc<T, G, S::kKPT, S::kBoxBytes, 32>(
                        sm.ring[slot], half * S::kHalfChunks, (half + 1) * S::kHalfChunks, sm.w,
                        lane, acc);
                    __syncwarp();
                    mbar_arrive(&sm.empty[slot]);
                }
                if (!ok) {
                    sm.abort = 1;
                    break;
                }
                float s[S::kKPT][G];
                score_acc_final<G, S::kKPT>(acc, s);
                double m1[G], m2[G];
#pragma unroll
                for (int h = 0; h < G; ++h) m1[h] = m2[h] = 0.0;
#pragma unroll
                for (int kk = 0; kk < S::kKPT; ++kk) {
                    const int j = i * S::kTile + lane + 32 * kk;
                    if (j < n) {
#pragma unroll
                        for (int h = 0; h < G; ++h) {
                            a.raw[(u * G + h) * a.cap + j] = s[kk][h];
                            const double d = s[kk][h];
                            m1[h] += d;
                            m2[h] = fma(d, d, m2[h]);
                        }
                    }
                }
#pragma unroll
                for (int h = 0; h < G; ++h) {
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1) {
                        m1[h] += __shfl_xor_sync(0xffffffffu, m1[h], o);
                        m2[h] += __shfl_xor_sync(0xffffffffu, m2[h], o);
                    }
                }
                uint32_t done = 0;
                if (lane == 0) {
                    double* part = a.partial + (u * a.tpu + i) * G * 2;
#pragma unroll
                    for (int h = 0; h < G; ++h) {
                        part[2 * h] = m1[h];
                        part[2 * h + 1] = m2[h];
                    }
                    if (!TRI_SCORE_DEFER_MERGE) {
                        __threadfence();
                        done = atomicAdd(&a.counters[u], 1u);
                    }
                }
                if (TRI_SCORE_DEFER_MERGE) continue;
                done = __shfl_sync(0xffffffffu, done, 0);
                if (done == static_cast<uint32_t>(ntv) - 1u) {
                    // The last tile of the unit: merge every tile's partial.
                    __threadfence();
                    merge_unit_moments<G>(a.partial + u * a.tpu * G * 2, ntv, n, a.mom + u * G);
                    if (lane == 0) a.counters[u] = 0u;
                }
            }
        }
        hbase += 2 * nt;
    }
    // Every load issued has landed before the CTA may exit: the math warps
    // consumed them all, unless a wait gave up; then loads still in flight
    // are given time to land.
    __syncthreads();
    if (sm.abort && tid == 0) {
        const uint64_t t0 = globaltimer_ns();
        while (globaltimer_ns() - t0 < 100000) __nanosleep(1000);
    }
    __syncthreads();
}

// The deferred merge: one warp per unit sums the unit's tile partials in
// tile order (the same arithmetic as the in-kernel merge).
template <int G>
__global__ void __launch_bounds__(32)
moment_merge_kernel(const double* __restrict__ partial, int64_t tpu, int64_t cap, int tile,
                    const int32_t* __restrict__ n_valid, float2* __restrict__ mom) {
    const int64_t u = blockIdx.x;
    const int n = clamp_nvalid(n_valid, u, cap, nullptr);
    const int ntv = (n + tile - 1) / tile;
    merge_unit_moments<G>(partial + u * tpu * G * 2, ntv, n, mom + u * G);
}

// ---------------------------------------------------------------------------
// z-score per head, max over the group, optional first radix histogram.
// (hyper.ai summary, Method section: GQA normalise-then-aggregate.)
// ---------------------------------------------------------------------------
template <int G>
__global__ void __launch_bounds__(256)
zmax_kernel(const float* __restrict__ raw, int64_t cap, const int32_t* __restrict__ n_valid,
            const float2* __restrict__ mom, float* __restrict__ fin, uint32_t* __restrict__ hist0,
            int zbins, int64_t n_sink, int64_t n_recent, uint32_t* flag) {
    __shared__ uint32_t hist[kHistBins0];
    const int64_t u = blockIdx.y;
    const int n = clamp_nvalid(n_valid, u, cap, nullptr);
    const int j0 = blockIdx.x * kZChunk;
    if (hist0) {
        for (int b = threadIdx.x; b < kHistBins0; b += blockDim.x) hist[b] = 0;
        __syncthreads();
    }
    float mu[G], inv[G];
#pragma unroll
    for (int h = 0; h < G; ++h) {
        const float2 m = mom[u * G + h];
        mu[h] = m.x;
        inv[h] = m.y;
    }
    bool nonfinite = false;
    constexpr int kPer = kZChunk / 256;  // keys per thread
    float sv[kPer][G];
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
        const int j = j0 + threadIdx.x + 256 * i;
#pragma unroll
        for (int h = 0; h < G; ++h) sv[i][h] = (j < n) ? raw[(u * G + h) * cap + j] : 0.f;
    }
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
        const int j = j0 + threadIdx.x + 256 * i;
        if (j < n) {
            float best = 0.f;
#pragma unroll
            for (int h = 0; h < G; ++h) {
                const float z = (sv[i][h] - mu[h]) * inv[h];
                best = (h == 0) ? z : fmaxf(best, z);
            }
            if (best != best) nonfinite = true;
            // Protected sink / recent keys rank above every score.
            if (j < n_sink || j >= n - n_recent) best = INFINITY;
            fin[u * cap + j] = best;
            if (hist0) atomicAdd(&hist[zbins ? zbin(best) : (ordered_key(best) >> kShift0)], 1u);
        }
    }
    if (nonfinite) raise_flag(flag, TRI_FLAG_NONFINITE);
    if (hist0) {
        __syncthreads();
        uint32_t* g = hist0 + u * kHistBins0;
        for (int b = threadIdx.x; b < kHistBins0; b += blockDim.x)
            if (hist[b]) atomicAdd(&g[b], hist[b]);
    }
}

// ---------------------------------------------------------------------------
// Host launchers
// ---------------------------------------------------------------------------
template <typename T, int G>
static cudaError_t launch_score_t(const CUtensorMap& map, const ScoreArgs& a, int n_sm,
                                  cudaStream_t s) {
    const size_t smem = sizeof(ScoreSmem<T, G>) + 1024;
    auto kern = score_kernel<T, G>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    const int64_t total = a.n_units * a.tpu;
    const int grid = static_cast<int>(total < n_sm ? total : n_sm);
    kern<<<grid, ScoreShape<T>::kThreads, smem, s>>>(map, a);
    if (TRI_SCORE_DEFER_MERGE) {
        note_launch(s);
        moment_merge_kernel<G><<<static_cast<unsigned>(a.n_units), 32, 0, s>>>(
            a.partial, a.tpu, a.cap, ScoreShape<T>::kTile, a.n_valid, a.mom);
    }
    note_launch(s);
    return cudaGetLastError();
}

template <typename T>
static cudaError_t launch_score_g(int G, const CUtensorMap& map, const ScoreArgs& a, int n_sm,
                                  cudaStream_t s) {
    switch (G) {
        case 1: return launch_score_t<T, 1>(map, a, n_sm, s);
        case 2: return launch_score_t<T, 2>(map, a, n_sm, s);
        case 3: return launch_score_t<T, 3>(map, a, n_sm, s);
        case 4: return launch_score_t<T, 4>(map, a, n_sm, s);
        case 5: return launch_score_t<T, 5>(map, a, n_sm, s);
        case 6: return launch_score_t<T, 6>(map, a, n_sm, s);
        case 7: return launch_score_t<T, 7>(map, a, n_sm, s);
        case 8: return launch_score_t<T, 8>(map, a, n_sm, s);
    }
    return cudaErrorInvalidValue;
}

int score_tile_keys(tri_dtype dt) {
    return dt == TRI_BF16 ? ScoreShape<__nv_bfloat16>::kTile : ScoreShape<float>::kTile;
}

cudaError_t launch_fold(const float* stats, const int64_t* p_cur, int64_t n_seq, int64_t n_layers,
                        int64_t n_qheads, double theta, const FoldOffsets& off, int variant,
                        float* wts, cudaStream_t s) {
    const int64_t groups = (n_layers * n_qheads + kFoldHeads - 1) / kFoldHeads;
    dim3 grid(static_cast<unsigned>(n_seq), static_cast<unsigned>(groups));
    fold_kernel<<<grid, 256, 0, s>>>(stats, p_cur, n_layers, n_qheads, theta, off, variant, wts);
    note_launch(s);
    return cudaGetLastError();
}

cudaError_t launch_score(tri_dtype dt, int G, const CUtensorMap& map, const ScoreArgs& a,
                         int n_sm, cudaStream_t s) {
    if (dt == TRI_BF16) return launch_score_g<__nv_bfloat16>(G, map, a, n_sm, s);
    return launch_score_g<float>(G, map, a, n_sm, s);
}

cudaError_t launch_zmax(int G, const float* raw, int64_t n_units, int64_t cap,
                        const int32_t* n_valid, const float2* mom, float* fin, uint32_t* hist0,
                        int zbins, int64_t n_sink, int64_t n_recent, uint32_t* flag,
                        cudaStream_t s) {
    dim3 grid(static_cast<unsigned>((cap + kZChunk - 1) / kZChunk), static_cast<unsigned>(n_units));
    switch (G) {
#define TRI_ZCASE(g)                                                                              \
    case g:                                                                                       \
        zmax_kernel<g><<<grid, 256, 0, s>>>(raw, cap, n_valid, mom, fin, hist0, zbins, n_sink,    \
                                            n_recent, flag);                                      \
        break;
        TRI_ZCASE(1) TRI_ZCASE(2) TRI_ZCASE(3) TRI_ZCASE(4)
        TRI_ZCASE(5) TRI_ZCASE(6) TRI_ZCASE(7) TRI_ZCASE(8)
#undef TRI_ZCASE
        default: return cudaErrorInvalidValue;
    }
    note_launch(s);
    return cudaGetLastError();
}

}  // namespace tri
