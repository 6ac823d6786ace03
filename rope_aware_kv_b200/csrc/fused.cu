// fused.cu -- one prune step of a small cache in a single kernel, one CTA per
// unit: score -> z-score / max -> radix select -> ordered gather.
//
// Every phase follows the same definitions as the split kernels (score.cu,
// select.cu, compact.cu): the folded S~ per query head (talk page: S_trig,
// S_norm, S~), z-score per head and max over the GQA group (hyper.ai summary,
// Method section), top-B by (score desc, index asc) kept in temporal order
// (jaedaily.cn tutorial, eviction step).  Here the per-head scores of the unit
// stay in shared memory, the moments need no second launch, and the three
// radix passes run on shared-memory histograms.  Only the key reads, the kept
// V reads and the K/V/position writes touch HBM (the kept K rows are re-read,
// usually from L2).
//
// Shared memory: [key tiles][G weight records][G x cap scores][barriers ...].
// After scoring, the tile area is reused for the histogram and the kept list.
#include "select_core.cuh"
#include "score_core.cuh"
#include "tri_internal.cuh"
#include "tri_launch.h"

namespace tri {

template <typename T>
struct FusedShape {
    static constexpr int kRowBytes = kD * static_cast<int>(sizeof(T));
    static constexpr int kBoxes = kRowBytes / 128;
    static constexpr int kTile = 128;                      // keys per tile, one per consumer
    static constexpr int kBoxBytes = kTile * 128;
    static constexpr int kStageBytes = kTile * kRowBytes;  // 32 KB bf16 / 64 KB f32
    static constexpr int kStages = sizeof(T) == 2 ? 3 : 2;
    static constexpr int kTilesBytes = kStages * kStageBytes;
    static constexpr int kConsumers = 128;
    static constexpr int kThreads = kConsumers + 32;
    static constexpr int kWarps = kThreads / 32;
    static constexpr int kVec = kRowBytes / 16;            // 16-byte vectors per row
};

struct FusedLayout {
    size_t w, sc, bars, red, mom, misc, total;
};

template <typename T>
__host__ __device__ inline FusedLayout fused_layout(int G, int64_t cap) {
    using S = FusedShape<T>;
    FusedLayout L;
    const int64_t capP = (cap + 3) & ~int64_t(3);
    L.w = S::kTilesBytes;
    L.sc = L.w + static_cast<size_t>(G) * kWHead * 4;
    L.bars = L.sc + static_cast<size_t>(G) * capP * 4;
    L.bars = (L.bars + 15) & ~size_t(15);
    L.red = L.bars + 2 * S::kStages * 8;
    L.mom = L.red + static_cast<size_t>(4) * G * 2 * 8;
    L.misc = L.mom + static_cast<size_t>(G) * 8;
    L.total = L.misc + 128 + 1024;  // + state / warp counts, + alignment slack
    return L;
}

template <typename T, int G>
__global__ void __launch_bounds__(FusedShape<T>::kThreads, 1)
prune_fused_kernel(const __grid_constant__ CUtensorMap kmap, FusedArgs a) {
    using S = FusedShape<T>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const FusedLayout L = fused_layout<T>(G, a.cap);
    const int64_t capP = (a.cap + 3) & ~int64_t(3);
    uint8_t* tiles = base;
    float* w = reinterpret_cast<float*>(base + L.w);
    float* sc = reinterpret_cast<float*>(base + L.sc);
    uint64_t* full = reinterpret_cast<uint64_t*>(base + L.bars);
    uint64_t* empty = full + S::kStages;
    double* red = reinterpret_cast<double*>(base + L.red);      // [4][G][2]
    float2* mom = reinterpret_cast<float2*>(base + L.mom);       // [G]
    SelState* st = reinterpret_cast<SelState*>(base + L.misc);
    uint32_t* wcnt = reinterpret_cast<uint32_t*>(base + L.misc + 32);  // [kWarps][2]
    uint32_t* hist = reinterpret_cast<uint32_t*>(tiles);               // after scoring
    int32_t* kidx = reinterpret_cast<int32_t*>(tiles + kHistBins0 * 4);

    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int64_t u = blockIdx.x;
    const int n = clamp_nvalid(a.n_valid, u, a.cap, tid == 0 ? a.flag : nullptr);
    const int64_t B = a.B;
    const int m = static_cast<int>(n < B ? n : B);
    const bool keep_all = n <= B;

    if (!keep_all) {
        // ---------------- Phase A: scores into shared memory ----------------
        if (tid == S::kConsumers) {
            for (int i = 0; i < S::kStages; ++i) {
                mbar_init(&full[i], 1);
                mbar_init(&empty[i], S::kConsumers);
            }
            fence_barrier_init();
            prefetch_tensormap(&kmap);
        }
        {
            const float4* src = reinterpret_cast<const float4*>(a.wts + u * G * kWHead);
            float4* dst = reinterpret_cast<float4*>(w);
            for (int e = tid; e < G * kWHead / 4; e += S::kThreads) dst[e] = src[e];
        }
        __syncthreads();
        const int n_tiles = (n + S::kTile - 1) / S::kTile;
        if (tid >= S::kConsumers) {
            if (tid == S::kConsumers) {
                int stage = 0;
                uint32_t phase = 0;
                uint32_t issued[S::kStages] = {};
                for (int i = 0; i < n_tiles; ++i) {
                    if (!mbar_wait(&empty[stage], phase ^ 1, a.flag)) break;
                    mbar_arrive_expect_tx(&full[stage], S::kStageBytes);
                    const int32_t y = static_cast<int32_t>(u * a.cap + static_cast<int64_t>(i) * S::kTile);
#pragma unroll
                    for (int b = 0; b < S::kBoxes; ++b)
                        tma_load_2d(tiles + stage * S::kStageBytes + b * S::kBoxBytes, &kmap,
                                    &full[stage], b * (128 / static_cast<int>(sizeof(T))), y);
                    issued[stage]++;
                    if (++stage == S::kStages) {
                        stage = 0;
                        phase ^= 1;
                    }
                }
                for (int s2 = 0; s2 < S::kStages; ++s2)
                    if (issued[s2]) mbar_wait(&full[s2], (issued[s2] - 1) & 1, a.flag);
            }
        } else {
            double m1[G], m2[G];
#pragma unroll
            for (int h = 0; h < G; ++h) m1[h] = m2[h] = 0.0;
            int stage = 0;
            uint32_t phase = 0;
            for (int i = 0; i < n_tiles; ++i) {
                if (!mbar_wait(&full[stage], phase, a.flag)) break;
                float s[1][G];
                score_rows<T, G, 1, S::kBoxBytes>(tiles + stage * S::kStageBytes, w, tid, s);
                mbar_arrive(&empty[stage]);
                if (++stage == S::kStages) {
                    stage = 0;
                    phase ^= 1;
                }
                const int j = i * S::kTile + tid;
                if (j < n) {
#pragma unroll
                    for (int h = 0; h < G; ++h) {
                        sc[h * capP + j] = s[0][h];
                        const double d = s[0][h];
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
                if (lane == 0) {
                    red[(warp * G + h) * 2] = m1[h];
                    red[(warp * G + h) * 2 + 1] = m2[h];
                }
            }
        }
        __syncthreads();
        // ---------------- Phase B: moments (fixed order) ----------------
        if (tid < G) {
            const int h = tid;
            const double s1 = ((red[(0 * G + h) * 2] + red[(1 * G + h) * 2]) + red[(2 * G + h) * 2]) +
                              red[(3 * G + h) * 2];
            const double s2 = ((red[(0 * G + h) * 2 + 1] + red[(1 * G + h) * 2 + 1]) +
                               red[(2 * G + h) * 2 + 1]) + red[(3 * G + h) * 2 + 1];
            const double mu = s1 / n;
            double var = s2 / n - mu * mu;
            if (var < 0.0) var = 0.0;
            const double sd = sqrt(var);
            float inv = sd > 0.0 ? static_cast<float>(1.0 / sd) : 0.f;
            if (!(sd == sd)) inv = __int_as_float(0x7fc00000);
            mom[h] = make_float2(static_cast<float>(mu), inv);
        }
        for (int b = tid; b < kHistBins0; b += S::kThreads) hist[b] = 0;
        __syncthreads();
        // ---------------- Phase C: final score + first digit ----------------
        {
            float mu[G], inv[G];
#pragma unroll
            for (int h = 0; h < G; ++h) {
                mu[h] = mom[h].x;
                inv[h] = mom[h].y;
            }
            bool nonfinite = false;
            for (int j = tid; j < n; j += S::kThreads) {
                float best = 0.f;
#pragma unroll
                for (int h = 0; h < G; ++h) {
                    const float z = (sc[h * capP + j] - mu[h]) * inv[h];
                    best = (h == 0) ? z : fmaxf(best, z);
                }
                sc[j] = best;
                if (best != best) nonfinite = true;
                atomicAdd(&hist[ordered_key(best) >> pass_shift(0)], 1u);
            }
            if (nonfinite) raise_flag(a.flag, TRI_FLAG_NONFINITE);
        }
        __syncthreads();
        // ---------------- Phase D: radix passes 1 and 2 ----------------
        if (warp == 0) {
            uint32_t bin, above;
            warp_find_bin(hist, 1 << pass_bits(0), static_cast<uint32_t>(B), bin, above);
            if (lane == 0) {
                st->prefix = bin;
                st->k = static_cast<uint32_t>(B) - above;
                st->gt = above;
                st->keep_all = 0;
            }
        }
        __syncthreads();
        for (int p = 1; p < 3; ++p) {
            const int nb = 1 << pass_bits(p);
            for (int b = tid; b < nb; b += S::kThreads) hist[b] = 0;
            __syncthreads();
            const uint32_t prefix = st->prefix;
            const int shift = pass_shift(p);
            const int hi_shift = shift + pass_bits(p);
            for (int j = tid; j < n; j += S::kThreads) {
                const uint32_t key = ordered_key(sc[j]);
                if ((key >> hi_shift) == prefix) atomicAdd(&hist[(key >> shift) & (nb - 1)], 1u);
            }
            __syncthreads();
            if (warp == 0) {
                uint32_t bin, above;
                warp_find_bin(hist, nb, st->k, bin, above);
                if (lane == 0) {
                    st->prefix = (prefix << pass_bits(p)) | bin;
                    st->k -= above;
                    st->gt += above;
                }
            }
            __syncthreads();
        }
        // ---------------- Phase E: ordered compaction of indices ----------------
        {
            const uint32_t T = st->prefix, kt = st->k;
            const int seg = ((n + S::kWarps * 32 - 1) / (S::kWarps * 32)) * 32;
            const int j0 = warp * seg;
            const int j1 = min(j0 + seg, n);
            uint32_t gt = 0, eq = 0;
            for (int j = j0 + lane; j - lane < j1; j += 32) {
                const bool valid = j < j1;
                const uint32_t key = valid ? ordered_key(sc[j]) : 0u;
                gt += __popc(__ballot_sync(0xffffffffu, valid && key > T));
                eq += __popc(__ballot_sync(0xffffffffu, valid && key == T));
            }
            if (lane == 0) {
                wcnt[2 * warp] = gt;
                wcnt[2 * warp + 1] = eq;
            }
            __syncthreads();
            uint32_t pos = 0, ties = 0;
            for (int v = 0; v < warp; ++v) {
                const uint32_t take = ties < kt ? min(wcnt[2 * v + 1], kt - ties) : 0u;
                pos += wcnt[2 * v] + take;
                ties += wcnt[2 * v + 1];
            }
            const uint32_t lt = (1u << lane) - 1u;
            for (int j = j0 + lane; j - lane < j1; j += 32) {
                const bool valid = j < j1;
                const uint32_t key = valid ? ordered_key(sc[j]) : 0u;
                const bool is_eq = valid && key == T;
                const uint32_t beq = __ballot_sync(0xffffffffu, is_eq);
                const uint32_t my_tie = ties + __popc(beq & lt);
                const bool keep = valid && (key > T || (is_eq && my_tie < kt));
                const uint32_t bk = __ballot_sync(0xffffffffu, keep);
                if (keep) {
                    const uint32_t r = pos + __popc(bk & lt);
                    if (r < static_cast<uint32_t>(m)) kidx[r] = j;
                }
                pos += __popc(bk);
                ties += __popc(beq);
            }
        }
        __syncthreads();
    }

    // ---------------- Phase F: gather rows (and the kept list) ----------------
    if (a.kept) {
        int32_t* out = a.kept + u * B;
        for (int r = tid; r < B; r += S::kThreads)
            out[r] = r < m ? (keep_all ? r : kidx[r]) : -1;
    }
    if (tid == 0) a.n_kept[u] = m;
    {
        constexpr int kVec = S::kVec;
        constexpr int kRows = S::kThreads / kVec;  // rows per pass (10 bf16 / 5 f32)
        constexpr int kUnroll = 8;
        const int l = tid % kVec;
        const int rs = tid / kVec;
        const uint4* ks = static_cast<const uint4*>(a.k_src);
        const uint4* vs = static_cast<const uint4*>(a.v_src);
        uint4* kd = static_cast<uint4*>(a.k_dst);
        uint4* vd = static_cast<uint4*>(a.v_dst);
        for (int r0 = 0; r0 < m; r0 += kRows * kUnroll) {
            uint4 kv[kUnroll], vv[kUnroll];
            int src[kUnroll];
#pragma unroll
            for (int q = 0; q < kUnroll; ++q) {
                const int r = r0 + q * kRows + rs;
                src[q] = (rs < kRows && r < m) ? (keep_all ? r : kidx[r]) : -1;
                if (src[q] >= n) {  // cannot happen when the selection is consistent
                    raise_flag(a.flag, TRI_FLAG_INDEX_RANGE);
                    src[q] = -1;
                }
                if (src[q] >= 0) {
                    const int64_t row = u * a.cap + src[q];
                    kv[q] = ks[row * kVec + l];
                    if (vs) vv[q] = vs[row * kVec + l];
                }
            }
#pragma unroll
            for (int q = 0; q < kUnroll; ++q) {
                if (src[q] >= 0) {
                    const int r = r0 + q * kRows + rs;
                    const int64_t drow = u * a.cap_dst + r;
                    kd[drow * kVec + l] = kv[q];
                    if (vd) vd[drow * kVec + l] = vv[q];
                    if (a.pos_dst && l == 0) a.pos_dst[drow] = a.pos_src[u * a.cap + src[q]];
                }
            }
        }
    }
}

size_t fused_smem_bytes(tri_dtype dt, int G, int64_t cap) {
    return dt == TRI_BF16 ? fused_layout<__nv_bfloat16>(G, cap).total
                          : fused_layout<float>(G, cap).total;
}

size_t fused_smem_limit() {
    static int lim = 0;
    if (!lim) {
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&lim, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    }
    return static_cast<size_t>(lim);
}

template <typename T, int G>
static cudaError_t launch_fused_t(const CUtensorMap& map, const FusedArgs& a, int64_t n_units,
                                  cudaStream_t s) {
    const size_t smem = fused_layout<T>(G, a.cap).total;
    auto kern = prune_fused_kernel<T, G>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    kern<<<static_cast<unsigned>(n_units), FusedShape<T>::kThreads, smem, s>>>(map, a);
    note_launch(s);
    return cudaGetLastError();
}

template <typename T>
static cudaError_t launch_fused_g(int G, const CUtensorMap& map, const FusedArgs& a,
                                  int64_t n_units, cudaStream_t s) {
    switch (G) {
        case 1: return launch_fused_t<T, 1>(map, a, n_units, s);
        case 2: return launch_fused_t<T, 2>(map, a, n_units, s);
        case 3: return launch_fused_t<T, 3>(map, a, n_units, s);
        case 4: return launch_fused_t<T, 4>(map, a, n_units, s);
        case 5: return launch_fused_t<T, 5>(map, a, n_units, s);
        case 6: return launch_fused_t<T, 6>(map, a, n_units, s);
        case 7: return launch_fused_t<T, 7>(map, a, n_units, s);
        case 8: return launch_fused_t<T, 8>(map, a, n_units, s);
    }
    return cudaErrorInvalidValue;
}

cudaError_t launch_fused(tri_dtype dt, int G, const CUtensorMap& map, const FusedArgs& a,
                         int64_t n_units, cudaStream_t s) {
    if (dt == TRI_BF16) return launch_fused_g<__nv_bfloat16>(G, map, a, n_units, s);
    return launch_fused_g<float>(G, map, a, n_units, s);
}

}  // namespace tri
