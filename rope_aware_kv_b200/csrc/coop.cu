// coop.cu -- one prune step of a few large caches in a single kernel: every
// unit (one KV head's cache) is split over C consecutive CTAs, one per SM, and
// the CTAs of a unit meet at three unit-wide barriers.
//
// Same definitions as the other paths: the folded S~ per query head (talk
// page: S_trig, S_norm, S~), z-score per head and max over the GQA group
// (hyper.ai summary, Method section), top-B by (score desc, index asc) kept
// in temporal order (jaedaily.cn tutorial, eviction step).
//
//   phase 1  score the CTA's tiles (a TMA ring of half tiles; seven math
//            warps, each on whole 128-key tiles with all heads) into an
//            L2-resident per-CTA scratch; float64 moment partial per CTA
//                                                              -> barrier 1
//   phase 2  fixed-order merge of the unit's partials; final = max_h z_h of
//            the CTA's keys into shared memory; histogram of the linear
//            z-bins of final added to the unit's global one    -> barrier 2
//   phase 3  the z-bin b0 of the B-th key; the CTA's count of keys above b0
//            and its keys inside b0 (the candidates) appended to a unit-wide
//            list                                              -> barrier 3
//   phase 4  every CTA ranks all candidates itself (a three-digit radix
//            select of their full keys in shared memory) and derives how many
//            rows and ties the CTAs before it keep: no further barrier
//   phase 5  ordered compaction of the CTA's kept keys, gather of their
//            K / V / position rows.
// If more than kCandMax keys share b0 (many equal scores), phase 4 falls back
// to unit-wide histograms of the same three digits over the keys of b0 and
// per-CTA counts, with barriers 4 to 7.
//
// A barrier is an atomic arrival counter per unit (zeroed by the host before
// the launch) and a bounded spin on it; every CTA of the grid is resident (one
// per SM, grid <= SMs), and a spin that exceeds its time limit raises
// TRI_FLAG_TIMEOUT and makes the CTA skip the remaining phases, so a fault
// elsewhere cannot hang the GPU.
#include "select_core.cuh"
#include "fold_core.cuh"
#include "score_core.cuh"
#include "tri_internal.cuh"
#include "tri_launch.h"

namespace tri {

template <typename T>
struct CoopShape {
    static constexpr int kRowBytes = kD * static_cast<int>(sizeof(T));
    static constexpr int kBoxes = kRowBytes / 128;
    static constexpr int kKPT = sizeof(T) == 2 ? 4 : 2;
    static constexpr int kTile = 32 * kKPT;
    static constexpr int kBoxBytes = kTile * 128;
    static constexpr int kStageBytes = kTile * kRowBytes;  // 32 KB
    static constexpr int kMaxStages = 6;
    static constexpr int kMathWarps = 7;          // + one producer warp: 256 threads
    static constexpr int kMath = 32 * kMathWarps;
    static constexpr int kThreads = kMath + 32;
    static constexpr int kWarps = kThreads / 32;
    // The ring holds half tiles (one TMA box of bf16 rows, two of float32):
    // half h of the CTA's tile l is slot 2l + h, so a warp frees the first
    // half of its tile while it scores the second.
    static constexpr int kHalfBoxes = kBoxes / 2;
    static constexpr int kHalfBytes = kStageBytes / 2;
    static constexpr int kHalfChunks = kHalfBoxes * 8;
    static constexpr int kMaxHStages = 2 * kMaxStages;
    // Half-landed barriers indexed by the half number, not the ring slot (a
    // math warp takes every kMathWarps-th tile and so skips phases of a slot's
    // barrier): a warp waiting for a half of tile l has finished tile
    // l - kMathWarps, so every half up to 2 (l - kMathWarps) - slots has been
    // consumed, including the previous use of its barrier (kHalfBars halves
    // earlier).
    static constexpr int kHalfBars = 32;
    static_assert(kBoxes % 2 == 0, "a tile splits into two halves of whole boxes");
    static_assert(kHalfBars >= 2 * kMathWarps + 1 + kMaxHStages, "half barriers too few");
};

static_assert(static_cast<size_t>(kCandMax) * 8 <= 2 * CoopShape<float>::kStageBytes &&
                  static_cast<size_t>(kCandMax) * 8 <= 2 * CoopShape<__nv_bfloat16>::kStageBytes,
              "the candidate list must fit a two-stage TMA ring");

struct CoopLayout {
    size_t w, fin, list, bars, red, misc, total;
};

template <typename T>
__host__ __device__ inline CoopLayout coop_layout(int G, int64_t keys_max, int stages) {
    using S = CoopShape<T>;
    CoopLayout L;
    const int64_t kp = (keys_max + 3) & ~int64_t(3);
    L.w = static_cast<size_t>(stages) * S::kStageBytes;
    L.fin = L.w + static_cast<size_t>(G) * kWHead * 4;
    L.list = L.fin + static_cast<size_t>(kp) * 4;
    L.bars = L.list + static_cast<size_t>(kp) * 8;
    L.red = L.bars + (S::kHalfBars + S::kMaxHStages) * 8;
    L.misc = L.red + static_cast<size_t>(S::kMathWarps) * kMaxG * 2 * 8;
    // histogram, state; alignment slack; static shared memory (fold)
    L.total = L.misc + kHistBins0 * 4 + 512 + 1024 + kFoldStaticBytes;
    return L;
}

__device__ __forceinline__ uint32_t ld_acquire_u32(const uint32_t* p) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Unit-wide barrier: arrive on the unit's counter, wait (bounded) until
// `target` arrivals.  Returns false, for every thread of the CTA, if this or
// an earlier barrier gave up.  The CTA barrier orders every thread's writes
// before thread 0's device-scope fence and arrival (the fence is cumulative),
// and thread 0's fence after the wait orders the other CTAs' writes before
// everything that follows the second CTA barrier.
__device__ __forceinline__ bool unit_barrier(uint32_t* ctr, uint32_t target, uint32_t* flag,
                                             int* abort_flag, uint64_t limit_ns) {
    __syncthreads();
    if (threadIdx.x == 0 && !*abort_flag) {
        __threadfence();
        atomicAdd(ctr, 1u);
        const uint64_t t0 = globaltimer_ns();
        while (ld_acquire_u32(ctr) < target) {
            if (globaltimer_ns() - t0 > limit_ns) {
                raise_flag(flag, TRI_FLAG_TIMEOUT);
                *abort_flag = 1;
                break;
            }
            __nanosleep(64);
        }
        __threadfence();
    }
    __syncthreads();
    return !*abort_flag;
}

// Phase trace by CTA: lane 0 of every warp records %globaltimer at point i.
__device__ __forceinline__ void coop_trace(const CoopArgs& a, int i) {
    if (a.trace && (threadIdx.x & 31) == 0)
        a.trace[(static_cast<int64_t>(blockIdx.x) * kTracePoints + i) * kTraceWarps +
                (threadIdx.x >> 5)] = globaltimer_ns();
}

template <typename T, int G>
__global__ void __launch_bounds__(CoopShape<T>::kThreads, 1)
prune_coop_kernel(const __grid_constant__ CUtensorMap kmap, CoopArgs a) {
    using S = CoopShape<T>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const CoopLayout L = coop_layout<T>(G, a.keys_max, a.stages);
    uint8_t* ring = base;
    float* w = reinterpret_cast<float*>(base + L.w);
    float* fin = reinterpret_cast<float*>(base + L.fin);
    int2* list = reinterpret_cast<int2*>(base + L.list);
    uint64_t* full = reinterpret_cast<uint64_t*>(base + L.bars);  // [kHalfBars] half landed
    uint64_t* empty = full + S::kHalfBars;                         // [half slots] slot free
    double* red = reinterpret_cast<double*>(base + L.red);  // [math warps][kMaxG][2]
    uint32_t* hist = reinterpret_cast<uint32_t*>(base + L.misc);
    SelState* st = reinterpret_cast<SelState*>(base + L.misc + kHistBins0 * 4);
    float2* mom = reinterpret_cast<float2*>(base + L.misc + kHistBins0 * 4 + 16);   // [kMaxG]
    uint32_t* wcnt = reinterpret_cast<uint32_t*>(base + L.misc + kHistBins0 * 4 + 80);  // [kWarps][2]
    uint32_t* bases = wcnt + 16;                                            // [2]
    int* abort_flag = reinterpret_cast<int*>(bases + 4);
    int* nlist = abort_flag + 1;

    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int C = a.ctas_per_unit;
    const int64_t u = blockIdx.x / C;
    const int c = blockIdx.x % C;
    const int64_t B = a.B;
    const int n = clamp_nvalid(a.n_valid, u, a.cap, (tid == 0 && c == 0) ? a.flag : nullptr);
    const int m = static_cast<int>(n < B ? n : B);
    const bool keep_all = n <= B;
    const int T_u = (n + S::kTile - 1) / S::kTile;
    const int t0 = static_cast<int>(static_cast<int64_t>(c) * T_u / C);
    const int t1 = static_cast<int>(static_cast<int64_t>(c + 1) * T_u / C);
    const int j0 = t0 * S::kTile;                       // first key of this CTA
    const int j1 = min(t1 * S::kTile, n);               // one past the last
    const int nk = max(j1 - j0, 0);
    float* scratch = a.scratch + static_cast<int64_t>(blockIdx.x) * G * a.keys_max;
    uint32_t* ctr = a.bar + u;

    if (tid == 0) {
        *abort_flag = 0;
        *nlist = 0;
    }
    coop_trace(a, 0);
    if (keep_all) {
        // Every valid key is kept: rows j0..j1-1 go to the same rows.
        __syncthreads();
        if (a.kept) {
            for (int j = j0 + tid; j < j1; j += S::kThreads) a.kept[u * B + j] = j;
            if (c == C - 1)
                for (int64_t r = m + tid; r < B; r += S::kThreads) a.kept[u * B + r] = -1;
        }
        for (int j = tid; j < nk; j += S::kThreads) list[j] = make_int2(j0 + j, j0 + j);
        if (tid == 0) *nlist = nk;
        if (c == 0 && tid == 0) a.n_kept[u] = m;
    } else {
        // ---------------- phase 1: score ----------------
        if (tid == S::kMath) {
            for (int i = 0; i < S::kHalfBars; ++i) mbar_init(&full[i], 1);
            for (int i = 0; i < 2 * a.stages; ++i) mbar_init(&empty[i], 32);
            fence_barrier_init();
            prefetch_tensormap(&kmap);
        }
        __syncthreads();  // barriers initialised before the producer starts
        const int nt = t1 - t0;
        const int n_hslots = 2 * a.stages;
        const int n_halves = 2 * nt;
        const int pre = n_halves < n_hslots ? n_halves : n_hslots;
        __shared__ FoldShared fs;
        auto issue_half = [&](int hh) {
            uint64_t* landed = &full[hh % S::kHalfBars];
            mbar_arrive_expect_tx(landed, S::kHalfBytes);
            const int32_t y =
                static_cast<int32_t>(u * a.cap + static_cast<int64_t>(t0 + (hh >> 1)) * S::kTile);
#pragma unroll
            for (int b = 0; b < S::kHalfBoxes; ++b)
                tma_load_2d(ring + (hh % n_hslots) * S::kHalfBytes + b * S::kBoxBytes, &kmap, landed,
                            ((hh & 1) * S::kHalfBoxes + b) * (128 / static_cast<int>(sizeof(T))), y);
        };
        if (tid == S::kMath) {
            // Issue the first half tiles before the fold so they overlap it.
            for (int hh = 0; hh < pre; ++hh) issue_half(hh);
            // The CTA's other tiles are requested into L2 at once.
            const char* kunit = static_cast<const char*>(a.k_src) + u * a.cap * S::kRowBytes;
            const uint64_t pol = policy_evict_last();
            for (int l = pre / 2; l < nt; ++l) {
                const int t = t0 + l;
                const int rows = min(S::kTile, static_cast<int>(a.cap) - t * S::kTile);
                prefetch_l2_bulk(kunit + static_cast<int64_t>(t) * S::kStageBytes,
                                 static_cast<uint32_t>(rows * S::kRowBytes), pol);
            }
        }
        fold_unit<G>(fs, a.fc, w, a.stats, a.p_cur, u, a.n_layers, a.n_kvheads);
        if (tid >= S::kMath) {
            if (tid == S::kMath) {
                for (int hh = pre; hh < n_halves; ++hh) {  // the first slots were issued above
                    if (!mbar_wait(&empty[hh % n_hslots], ((hh / n_hslots) & 1) ^ 1, a.flag)) {
                        *abort_flag = 1;
                        break;
                    }
                    issue_half(hh);
                }
            }
        } else {
            double m1[G], m2[G];
#pragma unroll
            for (int h = 0; h < G; ++h) m1[h] = m2[h] = 0.0;
            for (int l = warp; l < nt; l += S::kMathWarps) {
                float2 acc[S::kKPT][G];
                score_acc_zero<G, S::kKPT>(acc);
                bool ok = true;
#pragma unroll 1
                for (int half = 0; half < 2; ++half) {
                    const int hh = 2 * l + half;
                    if (!mbar_wait(&full[hh % S::kHalfBars], (hh / S::kHalfBars) & 1, a.flag)) {
                        ok = false;
                        break;
                    }
                    score_rows_acc<T, G, S::kKPT, S::kBoxBytes, 32>(
                        ring + (hh % n_hslots) * S::kHalfBytes, half * S::kHalfChunks,
                        (half + 1) * S::kHalfChunks, w, lane, acc);
                    __syncwarp();
                    mbar_arrive(&empty[hh % n_hslots]);
                }
                if (!ok) {
                    *abort_flag = 1;
                    break;
                }
                float s[S::kKPT][G];
                score_acc_final<G, S::kKPT>(acc, s);
#pragma unroll
                for (int k = 0; k < S::kKPT; ++k) {
                    const int jl = l * S::kTile + lane + 32 * k;  // local key index
                    if (j0 + jl < n) {
#pragma unroll
                        for (int h = 0; h < G; ++h) {
                            scratch[static_cast<int64_t>(h) * a.keys_max + jl] = s[k][h];
                            const double d = s[k][h];
                            m1[h] += d;
                            m2[h] = fma(d, d, m2[h]);
                        }
                    }
                }
            }
#pragma unroll
            for (int h = 0; h < G; ++h) {
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) {
                    m1[h] += __shfl_down_sync(0xffffffffu, m1[h], o);
                    m2[h] += __shfl_down_sync(0xffffffffu, m2[h], o);
                }
                if (lane == 0) {
                    red[(warp * kMaxG + h) * 2] = m1[h];
                    red[(warp * kMaxG + h) * 2 + 1] = m2[h];
                }
            }
        }
        __syncthreads();
        if (tid < G) {
            const int h = tid;
            double* part = a.partial + ((u * C + c) * G + h) * 2;
            double s1 = 0.0, s2 = 0.0;  // fixed order: math warps 0, 1, ...
#pragma unroll
            for (int v = 0; v < S::kMathWarps; ++v) {
                s1 += red[(v * kMaxG + h) * 2];
                s2 += red[(v * kMaxG + h) * 2 + 1];
            }
            part[0] = s1;
            part[1] = s2;
        }
        coop_trace(a, 1);
        if (!unit_barrier(ctr, 1u * C, a.flag, abort_flag, a.barrier_wait_ns)) return;
        coop_trace(a, 2);

        // ---------------- phase 2: moments, final, digit 0 ----------------
        // Warp w merges heads w, w + 5, ...: lane l sums CTAs l, l + 32, ...
        // in order, then a fixed shuffle tree; lane 0's value is used.
        for (int h = warp; h < G; h += S::kWarps) {
            double s1 = 0.0, s2 = 0.0;
            double2 pv[kMaxCtasPerUnit / 32];
#pragma unroll
            for (int q = 0; q < kMaxCtasPerUnit / 32; ++q) {
                const int cc = lane + 32 * q;
                pv[q] = cc < C ? __ldcg(reinterpret_cast<const double2*>(
                                     a.partial + ((u * C + cc) * G + h) * 2))
                               : make_double2(0.0, 0.0);
            }
#pragma unroll
            for (int q = 0; q < kMaxCtasPerUnit / 32; ++q) {
                s1 += pv[q].x;
                s2 += pv[q].y;
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                s1 += __shfl_down_sync(0xffffffffu, s1, o);
                s2 += __shfl_down_sync(0xffffffffu, s2, o);
            }
            if (lane == 0) {
                const double mu = s1 / n;
                double var = s2 / n - mu * mu;
                if (var < 0.0) var = 0.0;
                const double sd = sqrt(var);
                float inv = sd > 0.0 ? static_cast<float>(1.0 / sd) : 0.f;
                if (!(sd == sd)) inv = __int_as_float(0x7fc00000);
                mom[h] = make_float2(static_cast<float>(mu), inv);
            }
        }
        for (int b = tid; b < kHistBins0; b += S::kThreads) hist[b] = 0;
        __syncthreads();
        {
            float mu[G], inv[G];
#pragma unroll
            for (int h = 0; h < G; ++h) {
                mu[h] = mom[h].x;
                inv[h] = mom[h].y;
            }
            bool nonfinite = false;
            constexpr int kU = 4;
            for (int j0l = tid; j0l < nk; j0l += S::kThreads * kU) {
                float sv[kU][G];
#pragma unroll
                for (int q = 0; q < kU; ++q) {
                    const int jl = j0l + q * S::kThreads;
#pragma unroll
                    for (int h = 0; h < G; ++h)
                        sv[q][h] = jl < nk ? scratch[static_cast<int64_t>(h) * a.keys_max + jl] : 0.f;
                }
#pragma unroll
                for (int q = 0; q < kU; ++q) {
                    const int jl = j0l + q * S::kThreads;
                    if (jl < nk) {
                        float best = 0.f;
#pragma unroll
                        for (int h = 0; h < G; ++h) {
                            const float z = (sv[q][h] - mu[h]) * inv[h];
                            best = (h == 0) ? z : fmaxf(best, z);
                        }
                        fin[jl] = best;
                        if (a.final_out) a.final_out[u * a.cap + j0 + jl] = best;
                        if (best != best) nonfinite = true;
                        atomicAdd(&hist[zbin(best)], 1u);
                    }
                }
            }
            if (nonfinite) raise_flag(a.flag, TRI_FLAG_NONFINITE);
        }
        __syncthreads();
        {
            uint32_t* g = a.hists + u * kHistBins0;
            for (int b = tid; b < kHistBins0; b += S::kThreads)
                if (hist[b]) atomicAdd(&g[b], hist[b]);
        }
        coop_trace(a, 3);
        if (!unit_barrier(ctr, 2u * C, a.flag, abort_flag, a.barrier_wait_ns)) return;
        coop_trace(a, 4);

        // ---------------- phase 3: threshold bin, candidates ----------------
        // Every CTA reads the unit's z-bin histogram and finds the bin b0 that
        // holds the B-th key.  Keys above b0 are kept; the keys in b0 (the
        // candidates) go to a unit-wide list in global memory, so that after
        // one more barrier every CTA can finish the selection on its own.
        copy_l2_to_shared(reinterpret_cast<uint4*>(hist),
                          reinterpret_cast<const uint4*>(a.hists + u * kHistBins0),
                          kHistBins0 / 4);
        __syncthreads();
        uint32_t* zb0 = bases + 2;  // the threshold z-bin
        if (warp == 0) {
            uint32_t bin, above;
            warp_find_bin(hist, kZBins, static_cast<uint32_t>(B), bin, above);
            if (lane == 0) {
                *zb0 = bin;
                st->prefix = 0;
                st->k = static_cast<uint32_t>(B) - above;  // to take from bin b0
                st->gt = above;
                st->keep_all = 0;
            }
        }
        // This CTA's share of the unit's three full-key digit histograms,
        // which only the overflow path accumulates into (after barrier 3).
        {
            const int z0 = (c * kHistBins0) / C, z1 = ((c + 1) * kHistBins0) / C;
            for (int p = 0; p < 3; ++p) {
                uint32_t* g = a.hists_key + (static_cast<int64_t>(p) * a.n_units + u) * kHistBins0;
                for (int b = z0 + tid; b < z1; b += S::kThreads) g[b] = 0u;
            }
        }
        __syncthreads();
        const uint32_t b0 = *zb0;
        // Warp w owns the contiguous keys [l0, l1) of this CTA (here and in
        // the ordered compaction).
        const int seg = ((nk + S::kWarps * 32 - 1) / (S::kWarps * 32)) * 32;
        const int l0 = warp * seg;
        const int l1 = min(l0 + seg, nk);
        const uint32_t lt = (1u << lane) - 1u;
        {
            uint32_t above = 0, cands = 0;
            for (int jl = l0 + lane; jl - lane < l1; jl += 32) {
                const bool valid = jl < l1;
                const uint32_t bin = valid ? zbin(fin[jl]) : 0u;
                above += __popc(__ballot_sync(0xffffffffu, valid && bin > b0));
                cands += __popc(__ballot_sync(0xffffffffu, valid && bin == b0));
            }
            if (lane == 0) {
                wcnt[2 * warp] = above;
                wcnt[2 * warp + 1] = cands;
            }
            __syncthreads();
            if (tid == 0) {
                uint32_t ab = 0, cn = 0;
                for (int v = 0; v < S::kWarps; ++v) {
                    ab += wcnt[2 * v];
                    cn += wcnt[2 * v + 1];
                }
                bases[0] = atomicAdd(&a.cand_count[u], cn);  // this CTA's first slot
                a.counts[u * C + c] = make_uint2(ab, cn);
            }
            __syncthreads();
            uint32_t slot = bases[0];
            for (int v = 0; v < warp; ++v) slot += wcnt[2 * v + 1];
            int2* out = a.cand + u * kCandMax;
            for (int jl = l0 + lane; jl - lane < l1; jl += 32) {
                const bool valid = jl < l1;
                const float f = valid ? fin[jl] : 0.f;
                const bool is_c = valid && zbin(f) == b0;
                const uint32_t bc = __ballot_sync(0xffffffffu, is_c);
                const uint32_t r = slot + __popc(bc & lt);
                if (is_c && r < static_cast<uint32_t>(kCandMax))
                    out[r] = make_int2(static_cast<int>(ordered_key(f)), j0 + jl);
                slot += __popc(bc);
            }
        }
        if (!unit_barrier(ctr, 3u * C, a.flag, abort_flag, a.barrier_wait_ns)) return;

        // ---------------- phase 4: the threshold key ----------------
        // Three radix digits of the full key (11, 11, 10 bits) find the
        // k-th largest key of bin b0 and how many of its ties are kept.
        const uint32_t n_cand = ld_acquire_u32(a.cand_count + u);
        if (n_cand <= static_cast<uint32_t>(kCandMax)) {
            // Over the candidates, by every CTA in its own shared memory (the
            // TMA ring is free after scoring).
            int2* cs = reinterpret_cast<int2*>(ring);
            const int nc = static_cast<int>(n_cand);
            // Pairs of entries; an odd count also copies the unused slot nc.
            copy_l2_to_shared(reinterpret_cast<uint4*>(cs),
                              reinterpret_cast<const uint4*>(a.cand + u * kCandMax), (nc + 1) / 2);
            if (nc <= S::kThreads) {
                // Few candidates: thread i ranks candidate i against all of
                // them by (key desc, index asc); rank k0 - 1 is the threshold.
                const uint32_t k0 = st->k;
                __syncthreads();  // the list is staged and k0 read before st changes
                const int2 me = tid < nc ? cs[tid] : make_int2(0, 0);
                const uint32_t mk = static_cast<uint32_t>(me.x);
                uint32_t above = 0, rank = 0;
                for (int i = 0; i < nc; ++i) {
                    const int2 e = cs[i];
                    const uint32_t ek = static_cast<uint32_t>(e.x);
                    above += ek > mk;
                    rank += (ek > mk) || (ek == mk && e.y < me.y);
                }
                if (tid < nc && rank == k0 - 1) {
                    st->prefix = mk;
                    st->k = k0 - above;  // ties of the threshold key that are kept
                }
                __syncthreads();
            } else {
                for (int p = 0; p < 3; ++p) {
                    const int nb = 1 << pass_bits(p);
                    for (int b = tid; b < nb; b += S::kThreads) hist[b] = 0;
                    __syncthreads();
                    const uint32_t prefix = st->prefix;
                    const int shift = pass_shift(p);
                    const int hi_shift = shift + pass_bits(p);
                    for (int i = tid; i < nc; i += S::kThreads) {
                        const uint32_t key = static_cast<uint32_t>(cs[i].x);
                        if (p == 0 || (key >> hi_shift) == prefix)
                            atomicAdd(&hist[(key >> shift) & (nb - 1)], 1u);
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
            }
            // Kept rows and threshold ties in the CTAs before this one: their
            // keys above b0 (the published counts), their candidates above the
            // threshold key, and their ties up to the number taken.
            const uint32_t Tk = st->prefix, kt = st->k;
            uint32_t gs = 0, es = 0;
            for (int i = tid; i < nc; i += S::kThreads) {
                const int2 e = cs[i];
                if (e.y < j0) {
                    gs += static_cast<uint32_t>(e.x) > Tk;
                    es += static_cast<uint32_t>(e.x) == Tk;
                }
            }
            for (int cc = tid; cc < c; cc += S::kThreads) gs += __ldcg(a.counts + u * C + cc).x;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                gs += __shfl_xor_sync(0xffffffffu, gs, o);
                es += __shfl_xor_sync(0xffffffffu, es, o);
            }
            if (lane == 0) {
                wcnt[2 * warp] = gs;
                wcnt[2 * warp + 1] = es;
            }
            __syncthreads();
            if (tid == 0) {
                uint32_t g2 = 0, e2 = 0;
                for (int v = 0; v < S::kWarps; ++v) {
                    g2 += wcnt[2 * v];
                    e2 += wcnt[2 * v + 1];
                }
                bases[0] = g2 + min(e2, kt);  // kept before this CTA
                bases[1] = e2;                // ties before this CTA
            }
        } else {
            // Overflow: more than kCandMax keys share bin b0 (many equal
            // scores).  The same digits as unit-wide histograms over the keys
            // of bin b0, then the CTAs' counts above / equal to the threshold.
            for (int p = 0; p < 3; ++p) {
                const int nb = 1 << pass_bits(p);
                for (int b = tid; b < nb; b += S::kThreads) hist[b] = 0;
                __syncthreads();
                const uint32_t prefix = st->prefix;
                const int shift = pass_shift(p);
                const int hi_shift = shift + pass_bits(p);
                for (int jl = tid; jl < nk; jl += S::kThreads) {
                    const float f = fin[jl];
                    const uint32_t key = ordered_key(f);
                    if (zbin(f) == b0 && (p == 0 || (key >> hi_shift) == prefix))
                        atomicAdd(&hist[(key >> shift) & (nb - 1)], 1u);
                }
                __syncthreads();
                uint32_t* g = a.hists_key + (static_cast<int64_t>(p) * a.n_units + u) * kHistBins0;
                for (int b = tid; b < nb; b += S::kThreads)
                    if (hist[b]) atomicAdd(&g[b], hist[b]);
                if (!unit_barrier(ctr, (4u + p) * C, a.flag, abort_flag, a.barrier_wait_ns)) return;
                copy_l2_to_shared(reinterpret_cast<uint4*>(hist),
                                  reinterpret_cast<const uint4*>(g), nb / 4);
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
            const uint32_t Tk = st->prefix, kt = st->k;
            {
                uint32_t gt = 0, eq = 0;
                for (int jl = tid; jl < nk; jl += S::kThreads) {
                    const uint32_t key = ordered_key(fin[jl]);
                    gt += key > Tk;
                    eq += key == Tk;
                }
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) {
                    gt += __shfl_xor_sync(0xffffffffu, gt, o);
                    eq += __shfl_xor_sync(0xffffffffu, eq, o);
                }
                if (lane == 0) {
                    wcnt[2 * warp] = gt;
                    wcnt[2 * warp + 1] = eq;
                }
                __syncthreads();
                if (tid == 0) {
                    uint32_t g2 = 0, e2 = 0;
                    for (int v = 0; v < S::kWarps; ++v) {
                        g2 += wcnt[2 * v];
                        e2 += wcnt[2 * v + 1];
                    }
                    a.counts[u * C + c] = make_uint2(g2, e2);
                }
            }
            if (!unit_barrier(ctr, 7u * C, a.flag, abort_flag, a.barrier_wait_ns)) return;
            if (warp == 0) {
                uint32_t gsum = 0, esum = 0;
                for (int cc = lane; cc < c; cc += 32) {
                    const uint2 v = __ldcg(a.counts + u * C + cc);
                    gsum += v.x;
                    esum += v.y;
                }
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) {
                    gsum += __shfl_xor_sync(0xffffffffu, gsum, o);
                    esum += __shfl_xor_sync(0xffffffffu, esum, o);
                }
                if (lane == 0) {
                    bases[0] = gsum + min(esum, kt);  // kept before this CTA
                    bases[1] = esum;                  // ties before this CTA
                }
            }
        }
        coop_trace(a, 5);
        const uint32_t Tk = st->prefix, kt = st->k;
        __syncthreads();

        // ---------------- phase 5: ordered compaction ----------------
        {
            uint32_t gt = 0, eq = 0;
            for (int jl = l0 + lane; jl - lane < l1; jl += 32) {
                const bool valid = jl < l1;
                const uint32_t key = valid ? ordered_key(fin[jl]) : 0u;
                gt += __popc(__ballot_sync(0xffffffffu, valid && key > Tk));
                eq += __popc(__ballot_sync(0xffffffffu, valid && key == Tk));
            }
            if (lane == 0) {
                wcnt[2 * warp] = gt;
                wcnt[2 * warp + 1] = eq;
            }
            __syncthreads();
            uint32_t pos = bases[0], ties = bases[1];
            uint32_t lpos = 0;  // kept before this warp within the CTA
            for (int v = 0; v < warp; ++v) {
                const uint32_t take = ties < kt ? min(wcnt[2 * v + 1], kt - ties) : 0u;
                lpos += wcnt[2 * v] + take;
                ties += wcnt[2 * v + 1];
            }
            pos += lpos;
            for (int jl = l0 + lane; jl - lane < l1; jl += 32) {
                const bool valid = jl < l1;
                const uint32_t key = valid ? ordered_key(fin[jl]) : 0u;
                const bool is_eq = valid && key == Tk;
                const uint32_t beq = __ballot_sync(0xffffffffu, is_eq);
                const uint32_t my_tie = ties + __popc(beq & lt);
                const bool keep = valid && (key > Tk || (is_eq && my_tie < kt));
                const uint32_t bk = __ballot_sync(0xffffffffu, keep);
                if (keep) {
                    const uint32_t r = pos + __popc(bk & lt);
                    const uint32_t lr = lpos + __popc(bk & lt);
                    if (r < static_cast<uint32_t>(m) && lr < static_cast<uint32_t>(nk)) {
                        list[lr] = make_int2(j0 + jl, static_cast<int>(r));
                        if (a.kept) a.kept[u * B + r] = j0 + jl;
                    }
                }
                pos += __popc(bk);
                lpos += __popc(bk);
                ties += __popc(beq);
            }
            if (warp == S::kWarps - 1 && lane == 0) *nlist = static_cast<int>(lpos);
        }
        if (c == 0 && tid == 0) a.n_kept[u] = m;
    }
    coop_trace(a, 6);
    __syncthreads();

    // ---------------- gather of this CTA's kept rows ----------------
    {
        constexpr int kVec = S::kRowBytes / 16;
        constexpr int kGroups = S::kThreads / kVec;
        constexpr int kBatch = 8;
        const int cnt = *nlist;
        const int l = tid % kVec;
        const int g = tid / kVec;
        const uint4* ks = static_cast<const uint4*>(a.k_src);
        const uint4* vs = static_cast<const uint4*>(a.v_src);
        uint4* kd = static_cast<uint4*>(a.k_dst);
        uint4* vd = static_cast<uint4*>(a.v_dst);
        if (g < kGroups) {
            for (int e0 = 0; e0 < cnt; e0 += kGroups * kBatch) {
                uint4 kv[kBatch], vv[kBatch];
                int2 jr[kBatch];
#pragma unroll
                for (int q = 0; q < kBatch; ++q) {
                    const int e = e0 + q * kGroups + g;
                    jr[q] = e < cnt ? list[e] : make_int2(-1, -1);
                    if (jr[q].x >= n || jr[q].y >= m) jr[q].x = -1;  // cannot happen
                }
#pragma unroll
                for (int q = 0; q < kBatch; ++q) {
                    if (jr[q].x >= 0) {
                        const int64_t srow = u * a.cap + jr[q].x;
                        kv[q] = ld_stream(ks + srow * kVec + l);
                        if (vs) vv[q] = ld_stream(vs + srow * kVec + l);
                    }
                }
#pragma unroll
                for (int q = 0; q < kBatch; ++q) {
                    if (jr[q].x >= 0) {
                        const int64_t drow = u * a.cap_dst + jr[q].y;
                        st_stream(kd + drow * kVec + l, kv[q]);
                        if (vd) st_stream(vd + drow * kVec + l, vv[q]);
                        if (a.pos_dst && l == 0) a.pos_dst[drow] = a.pos_src[u * a.cap + jr[q].x];
                    }
                }
            }
        }
    }
    coop_trace(a, 7);
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
size_t coop_smem_bytes(tri_dtype dt, int G, int64_t keys_max, int stages) {
    return dt == TRI_BF16 ? coop_layout<__nv_bfloat16>(G, keys_max, stages).total
                          : coop_layout<float>(G, keys_max, stages).total;
}

int coop_tile_keys(tri_dtype dt) {
    return dt == TRI_BF16 ? CoopShape<__nv_bfloat16>::kTile : CoopShape<float>::kTile;
}

int coop_max_stages() { return CoopShape<float>::kMaxStages; }

template <typename T, int G>
static cudaError_t launch_coop_t(const CUtensorMap& map, const CoopArgs& a, int n_ctas,
                                 cudaStream_t s) {
    // Dynamic part only; the static fold factors are within kFoldStaticBytes.
    const size_t smem = coop_layout<T>(G, a.keys_max, a.stages).total - kFoldStaticBytes;
    auto kern = prune_coop_kernel<T, G>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    // The CTAs of a unit wait for one another at unit barriers, so all of
    // them must be resident at once: a cooperative launch guarantees it or
    // fails here, instead of leaving CTAs to time out at the barriers.
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(n_ctas));
    cfg.blockDim = dim3(CoopShape<T>::kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, kern, map, a);
    note_launch(s);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

template <typename T>
static cudaError_t launch_coop_g(int G, const CUtensorMap& map, const CoopArgs& a, int n_ctas,
                                 cudaStream_t s) {
    switch (G) {
        case 1: return launch_coop_t<T, 1>(map, a, n_ctas, s);
        case 2: return launch_coop_t<T, 2>(map, a, n_ctas, s);
        case 3: return launch_coop_t<T, 3>(map, a, n_ctas, s);
        case 4: return launch_coop_t<T, 4>(map, a, n_ctas, s);
        case 5: return launch_coop_t<T, 5>(map, a, n_ctas, s);
        case 6: return launch_coop_t<T, 6>(map, a, n_ctas, s);
        case 7: return launch_coop_t<T, 7>(map, a, n_ctas, s);
        case 8: return launch_coop_t<T, 8>(map, a, n_ctas, s);
    }
    return cudaErrorInvalidValue;
}

cudaError_t launch_coop(tri_dtype dt, int G, const CUtensorMap& map, const CoopArgs& a,
                        int n_ctas, cudaStream_t s) {
    if (dt == TRI_BF16) return launch_coop_g<__nv_bfloat16>(G, map, a, n_ctas, s);
    return launch_coop_g<float>(G, map, a, n_ctas, s);
}

}  // namespace tri
