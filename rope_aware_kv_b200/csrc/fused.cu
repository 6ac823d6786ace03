// fused.cu -- one prune step of small caches in a single persistent kernel:
// each CTA takes whole units (one KV head's cache) in turn and runs
// score -> z-score / max -> radix select -> ordered gather on each.
//
// Every phase follows the same definitions as the split kernels (score.cu,
// select.cu, compact.cu): the folded S~ per query head (talk page: S_trig,
// S_norm, S~), z-score per head and max over the GQA group (hyper.ai summary,
// Method section), top-B by (score desc, index asc) kept in temporal order
// (jaedaily.cn tutorial, eviction step).
//
// Per unit:
//   score   a producer lane streams 128-key tiles (32 KB, as two 16 KB halves
//           of one TMA box each) into a ring of 8 to 12 half slots and asks L2
//           for the tiles after them; each of the seven math warps scores
//           whole tiles, every lane on 4 keys for all GQA heads (so one
//           broadcast weight load feeds 4 keys); per-head scores go to a
//           per-CTA float32 scratch that stays in L2, float64 moments stay in
//           registers.
//   z-max   fixed-order moment merge, final = max_h z_h into shared memory,
//           histogram of its linear z-bins.
//   select  the keys in the z-bin of the B-th key are listed and ranked
//           (directly, or by a three-digit radix of their full keys), then
//           the ordered compaction of kept indices (warp ballots).
//   gather  with most rows kept, 16 KB chunks of consecutive source rows are
//           bulk-loaded and each kept row stored at its rank; otherwise the
//           runs of kept rows fill 8 KB buffers of consecutive destination
//           rows (one cp.async.bulk per run).  The whole ring is in flight;
//           the math warps copy landed buffers out with 16-byte stores and
//           free each as soon as it is read.
// HBM traffic per unit is the compulsory bytes plus the re-read of kept K
// rows (mostly from L2) and, for chunks, the dropped rows among them.
#include "select_core.cuh"
#include "fold_core.cuh"
#include "score_core.cuh"
#include "tri_internal.cuh"
#include "tri_launch.h"

// How many key tiles ahead of its shared-memory ring the fused kernel asks
// L2 to fetch (0: no prefetch).
#ifndef TRI_PREFETCH_TILES
#define TRI_PREFETCH_TILES 6
#endif

namespace tri {

template <typename T>
struct FusedShape {
    static constexpr int kRowBytes = kD * static_cast<int>(sizeof(T));  // 256 / 512
    static constexpr int kBoxes = kRowBytes / 128;
    static constexpr int kKPT = sizeof(T) == 2 ? 4 : 2;                 // keys per lane
    static constexpr int kTile = 32 * kKPT;                             // keys per tile
    static constexpr int kBoxBytes = kTile * 128;
    static constexpr int kStageBytes = kTile * kRowBytes;               // 32 KB
    static constexpr int kMaxStages = 6;                                // TMA ring depth (runtime)
    static constexpr int kMathWarps = 7;  // + one producer / copy-engine warp: 256 threads
    static constexpr int kMath = 32 * kMathWarps;
    static constexpr int kThreads = kMath + 32;
    static constexpr int kWarps = kThreads / 32;
    static constexpr int kGStage = 8192;                                // gather piece buffer
    static constexpr int kMaxGStages = kMaxStages * kStageBytes / kGStage;
    static constexpr int kGRows = kGStage / kRowBytes;                  // rows per piece
    // The score ring holds half tiles (16 KB: one 128-byte TMA box of bf16
    // rows, two of float32 rows), so a warp frees the first half of its tile
    // while it scores the second.  Half h of tile t is ring slot 2t + h.
    static constexpr int kHalfBoxes = kBoxes / 2;
    static constexpr int kHalfBytes = kStageBytes / 2;
    static constexpr int kHalfChunks = kHalfBoxes * 8;                   // 16-byte chunks per half
    static constexpr int kMaxHStages = 2 * kMaxStages;
    static constexpr int kPrefetchTiles = TRI_PREFETCH_TILES;  // L2 prefetch distance, tiles
    // "Landed" barriers are indexed by the running half-tile / piece count,
    // not by the ring stage.  A math warp takes every kMathWarps-th tile, so
    // it skips phases of a stage's barrier; a parity wait on a barrier that is
    // more than one phase behind would pass at once.  When a warp waits for a
    // half of tile t it has finished tile t - kMathWarps, so every half up to
    // 2 (t - kMathWarps) - half stages has been consumed; with kHalfBars >=
    // 2 kMathWarps + 1 + kMaxHStages the previous use of the half's barrier
    // (kHalfBars halves earlier) is among them, and the wait is exact.  Same
    // for gather pieces with kPieceBars >= kMathWarps + 1 + kMaxGStages.
    static constexpr int kHalfBars = 32;
    static constexpr int kPieceBars = 32;
    static_assert(kBoxes % 2 == 0, "a tile splits into two halves of whole boxes");
    static_assert(kHalfBars >= 2 * kMathWarps + 1 + kMaxHStages, "half-tile barriers too few");
    static_assert(kPieceBars >= kMathWarps + 1 + kMaxGStages, "piece barriers too few");
    // Dense gather (most rows kept): 16 KB buffers of kDRows source rows.
    static constexpr int kDStage = 16384;
    static constexpr int kMaxDStages = kMaxStages * kStageBytes / kDStage;
    static constexpr int kDRows = kDStage / kRowBytes;  // 64 / 32, a multiple of 32
    static_assert(kDRows % 32 == 0, "dense chunks are whole 32-key groups");
    static_assert(kPieceBars >= kMathWarps + 1 + kMaxDStages, "dense barriers too few");
};

struct FusedLayout {
    size_t w, fin, kidx, bars, red, misc, total;
};

template <typename T>
__host__ __device__ inline FusedLayout fused_layout(int G, int64_t cap, int64_t B, int stages) {
    using S = FusedShape<T>;
    FusedLayout L;
    const int64_t capP = (cap + 4) & ~int64_t(3);
    const int64_t m = B < cap ? B : cap;
    L.w = static_cast<size_t>(stages) * S::kStageBytes;
    L.fin = L.w + static_cast<size_t>(G) * kWHead * 4;
    L.kidx = L.fin + static_cast<size_t>(capP) * 4;
    L.bars = L.kidx + ((static_cast<size_t>(m) * 4 + 15) & ~size_t(15));
    L.red = L.bars + (S::kHalfBars + S::kMaxHStages + 2 * S::kPieceBars + S::kMaxGStages +
                      S::kMaxDStages) * 8;
    L.misc = L.red + static_cast<size_t>(FusedShape<T>::kMathWarps) * kMaxG * 2 * 8;
    // state and warp counts; alignment slack; static shared memory (fold)
    L.total = L.misc + 256 + 1024 + kFoldStaticBytes;
    return L;
}

// Phase trace: lane 0 of every warp records %globaltimer just before the
// barrier that ends phase i of unit u (the phase ends at the latest warp);
// slot i = 0 marks the start of the unit.
__device__ __forceinline__ void trace_point(const FusedArgs& a, int64_t u, int i) {
    if (a.trace && (threadIdx.x & 31) == 0)
        a.trace[(u * kTracePoints + i) * kTraceWarps + (threadIdx.x >> 5)] = globaltimer_ns();
}

template <typename T, int G>
__global__ void __launch_bounds__(FusedShape<T>::kThreads, 1)
prune_fused_kernel(const __grid_constant__ CUtensorMap kmap, FusedArgs a) {
    using S = FusedShape<T>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int n_stages = a.stages;
    const int n_hstages = 2 * n_stages;  // half-tile slots of the score ring
    const int n_gstages = n_stages * S::kStageBytes / S::kGStage;
    const int n_dstages = n_stages * S::kStageBytes / S::kDStage;
    const FusedLayout L = fused_layout<T>(G, a.cap, a.B, n_stages);
    uint8_t* regA = base;
    float* w = reinterpret_cast<float*>(base + L.w);
    float* fin = reinterpret_cast<float*>(base + L.fin);
    int32_t* kidx = reinterpret_cast<int32_t*>(base + L.kidx);
    uint64_t* full = reinterpret_cast<uint64_t*>(base + L.bars);  // [kHalfBars] half landed
    uint64_t* empty = full + S::kHalfBars;                         // [half stages] stage free
    uint64_t* gfull = empty + S::kMaxHStages;                      // [kPieceBars] piece landed
    uint64_t* gempty = gfull + S::kPieceBars;                      // [gather stages] buffer free
    uint64_t* dfull = gempty + S::kMaxGStages;                     // dense: [kPieceBars] landed
    uint64_t* dempty = dfull + S::kPieceBars;                      // dense: [stages] free
    double* red = reinterpret_cast<double*>(base + L.red);  // [math warps][kMaxG][2]
    SelState* st = reinterpret_cast<SelState*>(base + L.misc);
    float2* mom = reinterpret_cast<float2*>(base + L.misc + 16);            // [kMaxG]
    uint32_t* wcnt = reinterpret_cast<uint32_t*>(base + L.misc + 16 + 64);  // [kWarps][2]
    int32_t* nchunks = reinterpret_cast<int32_t*>(base + L.misc + 16 + 64 + 8 * S::kWarps);
    int32_t* abort_flag = nchunks + 1;
    uint32_t* hist = reinterpret_cast<uint32_t*>(regA);  // between scoring and gathering
    int32_t* chunk_r = reinterpret_cast<int32_t*>(fin);  // after the compaction

    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int64_t B = a.B;
    float* scratch = a.scratch + static_cast<int64_t>(blockIdx.x) * G * a.cap;

    if (tid == S::kMath) {
        for (int i = 0; i < S::kHalfBars; ++i) mbar_init(&full[i], 1);
        for (int i = 0; i < n_hstages; ++i) mbar_init(&empty[i], 32);
        for (int i = 0; i < S::kPieceBars; ++i) mbar_init(&gfull[i], 1);
        for (int i = 0; i < n_gstages; ++i) mbar_init(&gempty[i], 32);
        for (int i = 0; i < S::kPieceBars; ++i) mbar_init(&dfull[i], 1);
        for (int i = 0; i < n_dstages; ++i) mbar_init(&dempty[i], 32);
        fence_barrier_init();
        prefetch_tensormap(&kmap);
        *abort_flag = 0;
    }
    __shared__ FoldShared fs;
    __syncthreads();  // barriers and the abort flag initialised before anyone reads them

    uint32_t tiles_done = 0;   // running tile count (TMA ring position) of this CTA
    uint32_t pieces_done = 0;  // running gather-piece count (gather ring position)
    uint32_t dense_done = 0;   // running dense-chunk count (dense ring position)

    for (int64_t u = blockIdx.x; u < a.n_units; u += gridDim.x) {
        if (*abort_flag) break;  // a bounded wait gave up: stop cleanly
        const int n = clamp_nvalid(a.n_valid, u, a.cap, tid == 0 ? a.flag : nullptr);
        const int m = static_cast<int>(n < B ? n : B);
        const bool keep_all = n <= B;
        const int n_tiles = keep_all ? 0 : (n + S::kTile - 1) / S::kTile;
        trace_point(a, u, 0);

        if (!keep_all) {
            // ---------------- score ----------------
            // The first half tiles of the unit are requested before the fold
            // so that their loads overlap it (every ring slot is free here).
            // Keys stay in L2 for the kept-row re-read of the gather.
            const int n_halves = 2 * n_tiles;
            const int pre = n_halves < n_hstages ? n_halves : n_hstages;
            auto issue_half = [&](int hh, uint64_t pol) {  // hh: half index within the unit
                const uint32_t hc = 2 * tiles_done + hh;
                uint64_t* landed = &full[hc % S::kHalfBars];
                mbar_arrive_expect_tx(landed, S::kHalfBytes);
                const int32_t y =
                    static_cast<int32_t>(u * a.cap + static_cast<int64_t>(hh >> 1) * S::kTile);
#pragma unroll
                for (int b = 0; b < S::kHalfBoxes; ++b)
                    tma_load_2d_hint(regA + (hc % n_hstages) * S::kHalfBytes + b * S::kBoxBytes,
                                     &kmap, landed,
                                     ((hh & 1) * S::kHalfBoxes + b) * (128 / static_cast<int>(sizeof(T))),
                                     y, pol);
            };
            // Tiles beyond the ring are requested into L2 kPrefetchTiles ahead
            // of their load into shared memory, so that far more bytes are in
            // flight than the ring holds (most of it is being scored).
            const char* kunit = static_cast<const char*>(a.k_src) + u * a.cap * S::kRowBytes;
            auto prefetch_tile = [&](int t, uint64_t pol) {
                if (S::kPrefetchTiles == 0 || t >= n_tiles) return;
                const int rows = min(S::kTile, static_cast<int>(a.cap) - t * S::kTile);
                prefetch_l2_bulk(kunit + static_cast<int64_t>(t) * S::kStageBytes,
                                 static_cast<uint32_t>(rows * S::kRowBytes), pol);
            };
            if (tid == S::kMath) {
                const uint64_t keep_pol = policy_evict_last();
                for (int hh = 0; hh < pre; ++hh) issue_half(hh, keep_pol);
                for (int t = pre / 2; t < pre / 2 + S::kPrefetchTiles; ++t) prefetch_tile(t, keep_pol);
            }
            fold_unit<G>(fs, a.fc, w, a.stats, a.p_cur, u, a.n_layers, a.n_kvheads);
            if (tid >= S::kMath) {
                if (tid == S::kMath) {
                    const uint64_t keep_pol = policy_evict_last();
                    for (int hh = pre; hh < n_halves; ++hh) {
                        const uint32_t hc = 2 * tiles_done + hh;
                        const int slot = hc % n_hstages;
                        if (!mbar_wait(&empty[slot], ((hc / n_hstages) & 1) ^ 1, a.flag)) {
                            *abort_flag = 1;
                            break;
                        }
                        issue_half(hh, keep_pol);
                        if ((hh & 1) == 0) prefetch_tile(hh / 2 + S::kPrefetchTiles, keep_pol);
                    }
                }
            } else {
                // Math warp w scores tiles w, w + kMathWarps, ... with all G heads.
                double m1[G], m2[G];
#pragma unroll
                for (int h = 0; h < G; ++h) m1[h] = m2[h] = 0.0;
                for (int i = warp; i < n_tiles; i += S::kMathWarps) {
                    float2 acc[S::kKPT][G];
                    score_acc_zero<G, S::kKPT>(acc);
                    bool ok = true;
#pragma unroll 1
                    for (int half = 0; half < 2; ++half) {
                        const uint32_t hc = 2 * (tiles_done + i) + half;
                        const int slot = hc % n_hstages;
                        if (!mbar_wait(&full[hc % S::kHalfBars], (hc / S::kHalfBars) & 1, a.flag)) {
                            ok = false;
                            break;
                        }
                        score_rows_acc<T, G, S::kKPT, S::kBoxBytes, 32>(
                            regA + slot * S::kHalfBytes, half * S::kHalfChunks,
                            (half + 1) * S::kHalfChunks, w, lane, acc);
                        __syncwarp();
                        mbar_arrive(&empty[slot]);
                    }
                    if (!ok) {
                        *abort_flag = 1;
                        break;
                    }
                    float s[S::kKPT][G];
                    score_acc_final<G, S::kKPT>(acc, s);
#pragma unroll
                    for (int k = 0; k < S::kKPT; ++k) {
                        const int j = i * S::kTile + lane + 32 * k;
                        if (j < n) {
#pragma unroll
                            for (int h = 0; h < G; ++h) {
                                scratch[static_cast<int64_t>(h) * a.cap + j] = s[k][h];
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
            trace_point(a, u, 1);
            __syncthreads();
            if (*abort_flag) break;
            // ---------------- moments (fixed order: math warps 0, 1, ...) ----------------
            if (tid < G) {
                const int h = tid;
                double s1 = 0.0, s2 = 0.0;
#pragma unroll
                for (int v = 0; v < S::kMathWarps; ++v) {
                    s1 += red[(v * kMaxG + h) * 2];
                    s2 += red[(v * kMaxG + h) * 2 + 1];
                }
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
            // ---------------- final score + first digit ----------------
            {
                float mu[G], inv[G];
#pragma unroll
                for (int h = 0; h < G; ++h) {
                    mu[h] = mom[h].x;
                    inv[h] = mom[h].y;
                }
                bool nonfinite = false;
                constexpr int kU = 4;
                for (int j0 = tid; j0 < n; j0 += S::kThreads * kU) {
                    float sv[kU][G];
#pragma unroll
                    for (int q = 0; q < kU; ++q) {
                        const int j = j0 + q * S::kThreads;
#pragma unroll
                        for (int h = 0; h < G; ++h)
                            sv[q][h] = j < n ? scratch[static_cast<int64_t>(h) * a.cap + j] : 0.f;
                    }
#pragma unroll
                    for (int q = 0; q < kU; ++q) {
                        const int j = j0 + q * S::kThreads;
                        if (j < n) {
                            float best = 0.f;
#pragma unroll
                            for (int h = 0; h < G; ++h) {
                                const float z = (sv[q][h] - mu[h]) * inv[h];
                                best = (h == 0) ? z : fmaxf(best, z);
                            }
                            fin[j] = best;
                            if (a.final_out) a.final_out[u * a.cap + j] = best;
                            if (best != best) nonfinite = true;
                            atomicAdd(&hist[zbin(best)], 1u);
                        }
                    }
                }
                if (nonfinite) raise_flag(a.flag, TRI_FLAG_NONFINITE);
            }
            trace_point(a, u, 2);
            __syncthreads();
            // ---------------- threshold ----------------
            // The z-bin b0 of the B-th key; the keys in b0 (the candidates)
            // go to a list in the free TMA ring, and the B-th key is found
            // among them: by direct ranking when there are at most one per
            // thread, else by a three-digit radix select of their full keys;
            // if they do not fit the list, by the same radix over the keys of
            // b0 in place.
            uint32_t* zb0 = reinterpret_cast<uint32_t*>(base + L.misc + 152);
            int32_t* ncand = reinterpret_cast<int32_t*>(base + L.misc + 156);
            if (warp == 0) {
                uint32_t bin, above;
                warp_find_bin(hist, kZBins, static_cast<uint32_t>(B), bin, above);
                if (lane == 0) {
                    *zb0 = bin;
                    *ncand = 0;
                    st->prefix = 0;
                    st->k = static_cast<uint32_t>(B) - above;  // to take from bin b0
                    st->gt = above;
                    st->keep_all = 0;
                }
            }
            __syncthreads();
            const uint32_t b0 = *zb0;
            int2* cand = reinterpret_cast<int2*>(regA + kHistBins0 * 4);
            const int cand_cap =
                static_cast<int>((static_cast<size_t>(n_stages) * S::kStageBytes - kHistBins0 * 4) / 8);
            {
                const uint32_t lt = (1u << lane) - 1u;
                for (int j0 = warp * 32; j0 < n; j0 += S::kWarps * 32) {
                    const int j = j0 + lane;
                    const float f = j < n ? fin[j] : 0.f;
                    const bool is_c = j < n && zbin(f) == b0;
                    const uint32_t bc = __ballot_sync(0xffffffffu, is_c);
                    if (bc == 0u) continue;
                    int slot = 0;
                    if (lane == 0) slot = atomicAdd(ncand, __popc(bc));
                    slot = __shfl_sync(0xffffffffu, slot, 0);
                    const int r = slot + __popc(bc & lt);
                    if (is_c && r < cand_cap) cand[r] = make_int2(static_cast<int>(ordered_key(f)), j);
                }
            }
            __syncthreads();
            const int nc = *ncand;
            if (nc <= S::kThreads) {
                const uint32_t k0 = st->k;
                __syncthreads();  // k0 read before st changes
                const int2 me = tid < nc ? cand[tid] : make_int2(0, 0);
                const uint32_t mk = static_cast<uint32_t>(me.x);
                uint32_t above = 0, rank = 0;
                for (int i = 0; i < nc; ++i) {
                    const int2 e = cand[i];
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
                const bool listed = nc <= cand_cap;
                for (int p = 0; p < 3; ++p) {
                    const int nb = 1 << pass_bits(p);
                    for (int b = tid; b < nb; b += S::kThreads) hist[b] = 0;
                    __syncthreads();
                    const uint32_t prefix = st->prefix;
                    const int shift = pass_shift(p);
                    const int hi_shift = shift + pass_bits(p);
                    const int cnt = listed ? nc : n;
                    for (int i = tid; i < cnt; i += S::kThreads) {
                        uint32_t key;
                        bool in_bin;
                        if (listed) {
                            key = static_cast<uint32_t>(cand[i].x);
                            in_bin = true;
                        } else {
                            const float f = fin[i];
                            key = ordered_key(f);
                            in_bin = zbin(f) == b0;
                        }
                        if (in_bin && (p == 0 || (key >> hi_shift) == prefix))
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
            // ---------------- ordered compaction of indices ----------------
            {
                const uint32_t Tk = st->prefix, kt = st->k;
                const int seg = ((n + S::kWarps * 32 - 1) / (S::kWarps * 32)) * 32;
                const int j0 = warp * seg;
                const int j1 = min(j0 + seg, n);
                uint32_t gt = 0, eq = 0;
                for (int j = j0 + lane; j - lane < j1; j += 32) {
                    const bool valid = j < j1;
                    const uint32_t key = valid ? ordered_key(fin[j]) : 0u;
                    gt += __popc(__ballot_sync(0xffffffffu, valid && key > Tk));
                    eq += __popc(__ballot_sync(0xffffffffu, valid && key == Tk));
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
                    const uint32_t key = valid ? ordered_key(fin[j]) : 0u;
                    const bool is_eq = valid && key == Tk;
                    const uint32_t beq = __ballot_sync(0xffffffffu, is_eq);
                    const uint32_t my_tie = ties + __popc(beq & lt);
                    const bool keep = valid && (key > Tk || (is_eq && my_tie < kt));
                    const uint32_t bk = __ballot_sync(0xffffffffu, keep);
                    if (keep) {
                        const uint32_t r = pos + __popc(bk & lt);
                        if (r < static_cast<uint32_t>(m)) kidx[r] = j;
                    }
                    pos += __popc(bk);
                    ties += __popc(beq);
                }
            }
        } else {
            for (int r = tid; r < m; r += S::kThreads) kidx[r] = r;
        }
        trace_point(a, u, 3);
        __syncthreads();

        // ---------------- gather ----------------
        // Two ways, chosen per unit.
        //  dense (at least 3/4 of the rows kept): the ring holds 16 KB chunks
        //    of kDRows consecutive source rows, one cp.async.bulk each (the
        //    few dropped rows are read too); the copying warp stores each
        //    kept row of a landed chunk at its destination rank, from a
        //    per-32-key keep mask and the rank of the group's first kept row.
        //  runs (otherwise): kept rows form runs of consecutive source rows;
        //    a piece is a run cut at destination rows that are multiples of
        //    kGRows.  Buffer q (8 KB) receives destination rows [q kGRows,
        //    (q + 1) kGRows): the engine warp issues one cp.async.bulk per
        //    piece inside it (lane l takes the l-th piece), all completing on
        //    the buffer's barrier, so every buffer in flight is full.
        // Either way, loads hold no registers or L1 miss slots, and math warp
        // (slot % kMathWarps) copies each landed buffer out with 16-byte
        // stores, freeing it as soon as it is read.
        const bool dense = 4 * static_cast<int64_t>(m) >= 3 * static_cast<int64_t>(n);
        const int n_groups = (n + 31) / 32;
        uint32_t* kmask = reinterpret_cast<uint32_t*>(fin);  // dense: after the compaction
        uint32_t* kbase = kmask + n_groups;
        if (dense) {
            for (int g = tid; g < n_groups; g += S::kThreads) kmask[g] = 0u;
            __syncthreads();
            for (int r = tid; r < m; r += S::kThreads) {
                const int32_t j = kidx[r];
                if (j < 0 || j >= n) continue;  // cannot happen
                atomicOr(&kmask[j >> 5], 1u << (j & 31));
                if (r == 0 || (kidx[r - 1] >> 5) != (j >> 5)) kbase[j >> 5] = static_cast<uint32_t>(r);
            }
        } else {
            {
                const int seg = ((m + S::kWarps * 32 - 1) / (S::kWarps * 32)) * 32;
                const int r0 = warp * seg;
                const int r1 = min(r0 + seg, m);
                uint32_t cnt = 0;
                for (int r = r0 + lane; r - lane < r1; r += 32) {
                    bool start = false;
                    if (r < r1) {
                        const int32_t j = kidx[r];
                        const int32_t jp = r > 0 ? kidx[r - 1] : -2;
                        start = (r % S::kGRows == 0) || j != jp + 1;
                    }
                    cnt += __popc(__ballot_sync(0xffffffffu, start));
                }
                if (lane == 0) wcnt[2 * warp] = cnt;
                __syncthreads();
                uint32_t pos = 0;
                for (int v = 0; v < warp; ++v) pos += wcnt[2 * v];
                if (warp == S::kWarps - 1 && lane == 0) *nchunks = static_cast<int>(pos + cnt);
                const uint32_t lt = (1u << lane) - 1u;
                for (int r = r0 + lane; r - lane < r1; r += 32) {
                    bool start = false;
                    if (r < r1) {
                        const int32_t j = kidx[r];
                        const int32_t jp = r > 0 ? kidx[r - 1] : -2;
                        start = (r % S::kGRows == 0) || j != jp + 1;
                    }
                    const uint32_t b = __ballot_sync(0xffffffffu, start);
                    if (start) chunk_r[pos + __popc(b & lt)] = r;
                    pos += __popc(b);
                }
            }
        }
        fence_proxy_async();
        __syncthreads();
        // Math warps copy the positions of the kept rows first (8 loads in
        // flight per thread).
        auto copy_positions = [&]() {
            if (!a.pos_dst) return;
            for (int r0 = tid; r0 < m; r0 += S::kMath * 8) {
                int32_t pv[8];
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    const int r = r0 + q * S::kMath;
                    const int32_t j = r < m ? kidx[r] : -1;
                    pv[q] = (j >= 0 && j < n) ? a.pos_src[u * a.cap + j] : 0;
                }
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    const int r = r0 + q * S::kMath;
                    if (r < m) a.pos_dst[u * a.cap_dst + r] = pv[q];
                }
            }
        };
        constexpr int kVec = S::kRowBytes / 16;
        uint4* kd = static_cast<uint4*>(a.k_dst);
        uint4* vd = static_cast<uint4*>(a.v_dst);
        int npc = 0;
        if (dense) {
            const int n_dchunks = (n + S::kDRows - 1) / S::kDRows;
            npc = a.v_src ? 2 * n_dchunks : n_dchunks;  // K (and V) slot per chunk
            if (tid == S::kMath) {
                const uint64_t last_use = policy_evict_first();
                for (int p = 0; p < npc; ++p) {
                    const uint32_t pc = dense_done + p;
                    const int sb = pc % n_dstages;
                    if (!mbar_wait(&dempty[sb], ((pc / n_dstages) & 1) ^ 1, a.flag)) {
                        *abort_flag = 1;
                        break;
                    }
                    const int c = a.v_src ? (p >> 1) : p;
                    const bool is_v = a.v_src && (p & 1);
                    const int row0 = c * S::kDRows;
                    const int rows = min(S::kDRows, n - row0);
                    bool any = false;
                    for (int g = row0 >> 5; g < ((row0 + rows + 31) >> 5); ++g) any |= kmask[g] != 0u;
                    const uint32_t bytes = any ? static_cast<uint32_t>(rows * S::kRowBytes) : 0u;
                    uint64_t* landed = &dfull[pc % S::kPieceBars];
                    mbar_arrive_expect_tx(landed, bytes);
                    if (bytes)
                        bulk_load_hint(regA + sb * S::kDStage,
                                       static_cast<const char*>(is_v ? a.v_src : a.k_src) +
                                           (u * a.cap + row0) * S::kRowBytes,
                                       bytes, landed, last_use);
                }
            } else if (tid < S::kMath) {
                copy_positions();
                for (int p = warp; p < npc; p += S::kMathWarps) {
                    const uint32_t pc = dense_done + p;
                    const int sb = pc % n_dstages;
                    if (!mbar_wait(&dfull[pc % S::kPieceBars], (pc / S::kPieceBars) & 1, a.flag)) {
                        *abort_flag = 1;
                        break;
                    }
                    const int c = a.v_src ? (p >> 1) : p;
                    const bool is_v = a.v_src && (p & 1);
                    const int row0 = c * S::kDRows;
                    const int nv = min(S::kDRows, n - row0) * kVec;
                    const uint4* buf = reinterpret_cast<const uint4*>(regA + sb * S::kDStage);
                    uint4* dst = (is_v ? vd : kd) + u * a.cap_dst * kVec;
                    // Rounds of 8 loads in flight per lane; the buffer is freed
                    // once its last round is read.
                    constexpr int kRound = 8;
                    constexpr int kRounds = S::kDStage / 16 / 32 / kRound;
#pragma unroll
                    for (int h = 0; h < kRounds; ++h) {
                        uint4 v[kRound];
#pragma unroll
                        for (int i = 0; i < kRound; ++i) {
                            const int e = lane + 32 * (h * kRound + i);
                            if (e < nv) v[i] = buf[e];
                        }
                        if (h == kRounds - 1) {
                            __syncwarp();
                            mbar_arrive(&dempty[sb]);
                        }
#pragma unroll
                        for (int i = 0; i < kRound; ++i) {
                            const int e = lane + 32 * (h * kRound + i);
                            if (e < nv) {
                                const int j = row0 + e / kVec;
                                const uint32_t mask = kmask[j >> 5];
                                const uint32_t bit = 1u << (j & 31);
                                if (mask & bit) {
                                    const uint32_t r = kbase[j >> 5] + __popc(mask & (bit - 1u));
                                    st_stream(dst + static_cast<int64_t>(r) * kVec + e % kVec, v[i]);
                                }
                            }
                        }
                    }
                }
            }
        } else {
            const int n_chunks = *nchunks;
            // A buffer holds kGRows consecutive destination rows, gathered from
            // the pieces (runs) that start inside them; K and V of buffer q are
            // slots 2q and 2q + 1.
            const int n_buf = (m + S::kGRows - 1) / S::kGRows;
            npc = a.v_src ? 2 * n_buf : n_buf;
            if (tid >= S::kMath) {
                // Engine warp: for each buffer, lane l issues the bulk loads of
                // the buffer's l-th piece (a buffer of kGRows rows holds at most
                // kGRows <= 32 pieces).  Last use of these rows: evict first.
                const uint64_t last_use = policy_evict_first();
                const char* ks = static_cast<const char*>(a.k_src);
                const char* vs = static_cast<const char*>(a.v_src);
                const int halves = a.v_src ? 2 : 1;
                int c0 = 0;  // first piece of the current buffer
                for (int q = 0; q < n_buf; ++q) {
                    const int rq0 = q * S::kGRows;
                    const int rq1 = min(rq0 + S::kGRows, m);
                    const int c = c0 + lane;
                    const bool mine = c < n_chunks && chunk_r[c] < rq1;
                    const int r = mine ? chunk_r[c] : 0;
                    const int rend = mine ? ((c + 1 < n_chunks) ? chunk_r[c + 1] : m) : 0;
                    const int32_t j = mine ? kidx[r] : 0;
                    const bool ok =
                        mine && r >= rq0 && rend <= rq1 && rend > r && j >= 0 && j + (rend - r) <= n;
                    if (mine && !ok) raise_flag(a.flag, TRI_FLAG_INDEX_RANGE);  // cannot happen
                    uint32_t bytes = ok ? static_cast<uint32_t>((rend - r) * S::kRowBytes) : 0u;
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1) bytes += __shfl_xor_sync(0xffffffffu, bytes, o);
                    const int n_mine = __popc(__ballot_sync(0xffffffffu, mine));
                    bool stop = false;
                    for (int half = 0; half < halves; ++half) {
                        const uint32_t pc = pieces_done + (a.v_src ? 2 * q + half : q);
                        const int sb = pc % n_gstages;
                        uint64_t* landed = &gfull[pc % S::kPieceBars];
                        if (lane == 0) {
                            if (!mbar_wait(&gempty[sb], ((pc / n_gstages) & 1) ^ 1, a.flag)) {
                                *abort_flag = 1;
                            } else {
                                mbar_arrive_expect_tx(landed, bytes);
                            }
                        }
                        __syncwarp();
                        if (*abort_flag) {
                            stop = true;
                            break;
                        }
                        if (ok)
                            bulk_load_hint(regA + sb * S::kGStage + (r - rq0) * S::kRowBytes,
                                           (half ? vs : ks) + (u * a.cap + j) * S::kRowBytes,
                                           static_cast<uint32_t>((rend - r) * S::kRowBytes), landed,
                                           last_use);
                    }
                    if (stop) break;
                    c0 += n_mine;
                }
            } else if (tid < S::kMath) {
                // Math warps: positions of the kept rows (8 loads in flight per
                // thread), then drain pieces warp, warp + kMathWarps, ... to global
                // memory.
                copy_positions();
                for (int p = warp; p < npc; p += S::kMathWarps) {
                    const uint32_t pc = pieces_done + p;
                    const int sb = pc % n_gstages;
                    if (!mbar_wait(&gfull[pc % S::kPieceBars], (pc / S::kPieceBars) & 1, a.flag)) {
                        *abort_flag = 1;
                        break;
                    }
                    const int q = a.v_src ? (p >> 1) : p;
                    const bool is_v = a.v_src && (p & 1);
                    const int rq0 = q * S::kGRows;
                    const int len = min(S::kGRows, m - rq0);
                    const uint4* buf = reinterpret_cast<const uint4*>(regA + sb * S::kGStage);
                    uint4* dst = (is_v ? vd : kd) + (u * a.cap_dst + rq0) * kVec;
                    const int nv = len * kVec;
                    // Two halves through registers (8 loads in flight per lane);
                    // the buffer is freed once its second half is read.
                    constexpr int kHalf = S::kGStage / 16 / 32 / 2;
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        uint4 v[kHalf];
#pragma unroll
                        for (int i = 0; i < kHalf; ++i) {
                            const int e = lane + 32 * (h * kHalf + i);
                            if (e < nv) v[i] = buf[e];
                        }
                        if (h == 1) {
                            __syncwarp();
                            mbar_arrive(&gempty[sb]);
                        }
#pragma unroll
                        for (int i = 0; i < kHalf; ++i) {
                            const int e = lane + 32 * (h * kHalf + i);
                            if (e < nv) st_stream(dst + e, v[i]);
                        }
                    }
                }
            }
        }
        if (a.kept)
            for (int r = tid; r < B; r += S::kThreads) a.kept[u * B + r] = r < m ? kidx[r] : -1;
        if (tid == 0) a.n_kept[u] = m;
        trace_point(a, u, 4);
        __syncthreads();
        tiles_done += n_tiles;
        if (dense)
            dense_done += static_cast<uint32_t>(npc);
        else
            pieces_done += static_cast<uint32_t>(npc);
        fence_proxy_async();
        __syncthreads();
    }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
size_t fused_smem_bytes(tri_dtype dt, int G, int64_t cap, int64_t B, int stages) {
    return dt == TRI_BF16 ? fused_layout<__nv_bfloat16>(G, cap, B, stages).total
                          : fused_layout<float>(G, cap, B, stages).total;
}

int fused_max_stages() { return FusedShape<float>::kMaxStages; }

size_t fused_smem_limit() {
    static int lim = 0;
    if (!lim) {
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&lim, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    }
    return static_cast<size_t>(lim);
}

int fused_tile_keys(tri_dtype dt) {
    return dt == TRI_BF16 ? FusedShape<__nv_bfloat16>::kTile : FusedShape<float>::kTile;
}

template <typename T, int G>
static cudaError_t launch_fused_t(const CUtensorMap& map, const FusedArgs& a, int n_ctas,
                                  cudaStream_t s) {
    // Dynamic part only; the static fold factors are within kFoldStaticBytes.
    const size_t smem = fused_layout<T>(G, a.cap, a.B, a.stages).total - kFoldStaticBytes;
    auto kern = prune_fused_kernel<T, G>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    kern<<<n_ctas, FusedShape<T>::kThreads, smem, s>>>(map, a);
    note_launch(s);
    return cudaGetLastError();
}

template <typename T>
static cudaError_t launch_fused_g(int G, const CUtensorMap& map, const FusedArgs& a, int n_ctas,
                                  cudaStream_t s) {
    switch (G) {
        case 1: return launch_fused_t<T, 1>(map, a, n_ctas, s);
        case 2: return launch_fused_t<T, 2>(map, a, n_ctas, s);
        case 3: return launch_fused_t<T, 3>(map, a, n_ctas, s);
        case 4: return launch_fused_t<T, 4>(map, a, n_ctas, s);
        case 5: return launch_fused_t<T, 5>(map, a, n_ctas, s);
        case 6: return launch_fused_t<T, 6>(map, a, n_ctas, s);
        case 7: return launch_fused_t<T, 7>(map, a, n_ctas, s);
        case 8: return launch_fused_t<T, 8>(map, a, n_ctas, s);
    }
    return cudaErrorInvalidValue;
}

cudaError_t launch_fused(tri_dtype dt, int G, const CUtensorMap& map, const FusedArgs& a,
                         int n_ctas, cudaStream_t s) {
    if (dt == TRI_BF16) return launch_fused_g<__nv_bfloat16>(G, map, a, n_ctas, s);
    return launch_fused_g<float>(G, map, a, n_ctas, s);
}

}  // namespace tri
