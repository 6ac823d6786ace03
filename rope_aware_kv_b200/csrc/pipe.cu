// pipe.cu -- one prune step in a single persistent, warp-specialised kernel
// whose gather of one unit overlaps the scoring of the next.
//
// The step is the same as the split kernels compute (score.cu, select.cu,
// compact.cu): the folded S~ per query head (talk page: S_trig, S_norm, S~),
// z-score per head and max over the GQA group (hyper.ai summary, Method
// section, "normalise then aggregate"), top-B by (score desc, index asc)
// kept in temporal order (jaedaily.cn tutorial, eviction step).
//
// One CTA per SM, 256 threads: six math warps and two gather engine warps
// (TRI_PIPE_ENGINE_WARPS; eight warps in all keep 255 registers a thread).
//
//   math warps   score, z-max and select, one unit (or one chunk of a unit)
//                at a time.  Warp w scores tiles w, w + 6, ... of the unit
//                (a tile is 128 bf16 or 64 float32 rows, every lane on 4 or 2
//                keys for all G heads).  Each warp streams its own tiles
//                through a private TMA ring (small units: four 4 KB slots,
//                one 32-byte column slice of the tile per slot, 32-byte
//                swizzle; large units: two 8 KB slots of 64-byte slices),
//                issues the next slice itself as soon as it frees a slot, and
//                asks L2 for its tiles two tiles ahead.  Per-head scores go
//                to a float32 scratch in global memory (it stays in L2),
//                float64 moments to registers.  After selecting, they write
//                kept / n_kept and copy the kept rows' positions.
//   engine warps gather the units the math warps have selected, in order:
//                a piece is 32 bf16 (16 float32) destination rows, its K and
//                V rows together in one 16 KB buffer; lane o issues the o-th
//                cp.async.bulk load (the K or V rows of one run of
//                consecutive kept rows), all completing on the buffer's
//                barrier, and two lanes store the landed buffer with one
//                cp.async.bulk store each.  Engine warp e takes pieces e,
//                e + 2, ...; in place, a piece is stored only after the
//                other engine's previous piece has landed.
//                They hold no data in registers, so the gather of unit u
//                runs while the math warps score unit u + 1.
//
// Hand-off: the math warps write the kept indices of a unit into one of two
// index buffers in shared memory and arrive on its "ready" barrier; the
// engine arrives on its "free" barrier once it has issued the unit's last
// load.  A sentinel unit (-1) ends the engine.
//
// Two modes.
//   small units (the whole unit's final scores fit in shared memory): CTA b
//     takes units b, b + grid, ...; the fold of each unit runs in the kernel.
//   large units: the work items are chunks of kChunkTiles tiles of a unit,
//     taken from an atomic queue in unit order, so all CTAs work on the same
//     few units and their per-head scores stay in L2; each chunk leaves a
//     float64 moment partial, and the CTA that completes a unit's last chunk
//     (an atomic counter) merges the partials in chunk order, computes the
//     final scores into global memory and selects; its engine gathers.  The
//     per-head weights come from the fold kernel (score.cu).
#include <type_traits>

#include "select_core.cuh"
#include "fold_core.cuh"
#include "score_core.cuh"
#include "tri_internal.cuh"
#include "tri_launch.h"

namespace tri {

#ifndef TRI_PIPE_ENGINE_WARPS
#define TRI_PIPE_ENGINE_WARPS 2
#endif
// Ring slots per math warp in the small-unit mode.
#ifndef TRI_PIPE_RING_SLOTS
#define TRI_PIPE_RING_SLOTS 4
#endif
// How many of its own tiles ahead a math warp asks L2 for its keys.
#ifndef TRI_PIPE_PF_AHEAD
#define TRI_PIPE_PF_AHEAD 2
#endif

// Shape of the kernel for element type T; kBig selects the large-unit mode.
template <typename T, bool kBig = false>
struct PipeShape {
    static constexpr int kRowBytes = kD * static_cast<int>(sizeof(T));  // 256 / 512
    static constexpr int kKPT = sizeof(T) == 2 ? 4 : 2;                 // keys per lane
    static constexpr int kTile = 32 * kKPT;                             // rows per tile
    // A slice is one TMA box: a column band of the tile, 32 bytes wide
    // (small units, whose rings must leave room for the gather) or 64
    // bytes wide (large units), with the TMA swizzle of the same span.
    static constexpr int kSliceBytes = kBig ? 64 : 32;
    static constexpr int kSliceChunks = kSliceBytes / 16;               // 16-byte chunks
    static constexpr int kSlices = kRowBytes / kSliceBytes;
    static constexpr int kSliceElems = kSliceBytes / static_cast<int>(sizeof(T));
    static constexpr int kSlotBytes = kTile * kSliceBytes;              // 4 KB / 8 KB (bf16)
    static constexpr int kQ = kBig ? 2 : TRI_PIPE_RING_SLOTS;           // ring slots per math warp
    static constexpr int kPfAhead = TRI_PIPE_PF_AHEAD;                  // L2 prefetch, warp tiles
    // Six math warps and two engines (or seven and one): 256 threads, so
    // that a thread may hold up to 255 registers (the register file is split
    // over the four SM sub-partitions, two warps each).
    static constexpr int kEngWarps = TRI_PIPE_ENGINE_WARPS;
    static constexpr int kMathWarps = 8 - kEngWarps;
    static constexpr int kMath = 32 * kMathWarps;
    static constexpr int kThreads = 256;
    // Gather pieces: kGRows consecutive destination rows of K and of V in
    // one buffer (K at 0, V at kGHalf).
    static constexpr int kGHalf = 8192;
    static constexpr int kGSlotBytes = 2 * kGHalf;
    static constexpr int kGRows = kGHalf / kRowBytes;  // 32 / 16 destination rows
    // Gather buffers: as many as shared memory leaves room for (runtime,
    // kMinGSlots..kMaxGSlots, shared by the engine warps); all but kGGap of
    // an engine warp's buffers may be loading.
    static constexpr int kMinGSlots = kEngWarps == 1 ? 3 : 2 * kEngWarps;
    static constexpr int kMaxGSlots = 12;
    static constexpr int kGGap = 1;
    static constexpr int kHand = 2;                // index buffers (units handed to the engine)
    static_assert(kGRows <= 32, "one lane per destination row of a gather piece");
    static_assert(kMinGSlots >= (kGGap + 1) * kEngWarps, "gather ring too shallow");
    static_assert(kEngWarps <= 2, "run-start scratch for two engine warps");
};

constexpr int kPipeCand = 1024;   // threshold-bin candidates listed in shared memory
// Large units merge their chunks' moment partials in the idle rings, after
// the histogram and the candidate list.
constexpr int kPartOff = 16384;

// Tiles per work item of a large unit: a multiple of the math warps' count.
constexpr int kChunkTiles = 6 * PipeShape<float>::kMathWarps;

// "Full" barriers per math warp, enough for either mode's ring.
template <typename T>
__host__ __device__ constexpr int pipe_full_bars() {
    return PipeShape<T, false>::kQ > 2 * PipeShape<T, true>::kQ ? PipeShape<T, false>::kQ
                                                                  : 2 * PipeShape<T, true>::kQ;
}

struct PipeLayout {
    size_t ring, gbuf, w, fin, hist, cand, kidx, smask, bars, red, misc, total;
};

// Shared-memory layout (dynamic part, from a 1024-byte aligned base).  The
// z-bin histogram, the candidate list and (small units) the final scores of
// a unit are only live between the end of its scoring and its hand-off to
// the engine, when the math warps' rings are idle: they alias the rings.
// Index buffers hold int32 for large units, uint16 for small ones (cap <=
// 65536); each index buffer has one run-start mask per gather piece.
template <typename T>
__host__ __device__ inline PipeLayout pipe_layout(int G, int64_t cap, int64_t B, bool big,
                                                  int gslots) {
    using SB = PipeShape<T, true>;
    using SS = PipeShape<T, false>;
    PipeLayout L;
    const int64_t m = B < cap ? B : cap;
    size_t o = 0;
    L.ring = o;
    L.hist = o;
    L.cand = o + kZBins * 4;
    L.fin = L.cand + kPipeCand * 8;
    o += static_cast<size_t>(SS::kMathWarps) *
         (big ? SB::kQ * SB::kSlotBytes : SS::kQ * SS::kSlotBytes);
    L.gbuf = o;
    o += static_cast<size_t>(gslots) * SS::kGSlotBytes;
    L.w = o;
    o += static_cast<size_t>(G) * kWHead * 4;
    L.kidx = o;
    o += SS::kHand * ((static_cast<size_t>(m) * (big ? 4 : 2) + 15) & ~size_t(15));
    L.smask = o;
    o += SS::kHand * ((static_cast<size_t>((m + SS::kGRows - 1) / SS::kGRows) * 8 + 15) & ~size_t(15));
    L.bars = o;
    o += (SS::kMathWarps * pipe_full_bars<T>() + SS::kMaxGSlots + 2 * SS::kHand) * 8;
    L.red = o;
    o += static_cast<size_t>(SS::kMathWarps) * kMaxG * 2 * 8;
    L.misc = o;
    o += 1024;
    // alignment slack of the dynamic base; the fold's static shared memory
    L.total = o + 1024 + sizeof(FoldShared);
    return L;
}

// Whether a unit's final scores (with the histogram and candidate list) fit
// the idle rings of the small-unit mode, and its indices uint16.
template <typename T>
__host__ __device__ inline bool pipe_small_unit(int64_t cap) {
    using S = PipeShape<T, false>;
    const size_t ring = static_cast<size_t>(S::kMathWarps) * S::kQ * S::kSlotBytes;
    return cap <= 65536 &&
           kZBins * 4 + kPipeCand * 8 + static_cast<size_t>((cap + 31) & ~int64_t(31)) * 4 <= ring;
}

// Small shared state of the math warps (in the misc area).
struct PipeMisc {
    SelState st;            // 16 bytes
    float2 mom[kMaxG];      // mu, 1/sigma per head
    uint32_t wcnt[PipeShape<float>::kMathWarps][2];
    uint32_t wadd[PipeShape<float>::kMathWarps][2];
    uint32_t zb0;
    int32_t ncand;
    int32_t abort;          // the engine gave up a wait
    int32_t stop;           // the math warps stop (written before, read after a math barrier)
    int32_t last;           // large units: this CTA completed the unit
    int64_t item;           // large units: current work item
    int64_t hdr_u[PipeShape<float>::kHand];  // unit of each index buffer (-1: end)
    int32_t hdr_m[PipeShape<float>::kHand];
    uint32_t gdst_rows[PipeShape<float>::kMaxGSlots];  // engine: rows of each gather buffer
    int64_t gdst[PipeShape<float>::kMaxGSlots];        // engine: destination byte offset
    int32_t runst[2][64];                              // engine: start row of each run
    uint64_t gseq[PipeShape<float>::kMaxGSlots];       // engine: (unit << 32) | piece of each buffer
    uint64_t landed[2];                                // in place: 1 + last piece each engine saw land
};
static_assert(sizeof(PipeMisc) <= 1024, "misc state exceeds its budget");

__device__ __forceinline__ void math_sync() { named_sync(1, PipeShape<float>::kMath); }

// A bounded wait whose outcome every lane of the warp shares (a lane whose
// own wait gave up makes the whole warp give up), so that control flow
// around later warp and group barriers never diverges.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, uint32_t* flag) {
    return __all_sync(0xffffffffu, mbar_wait(bar, parity, flag));
}

// Bulk store shared -> global with an L2 cache policy.
__device__ __forceinline__ void bulk_store_hint(void* gdst, const void* smem_src, uint32_t bytes,
                                                uint64_t policy) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group.L2::cache_hint [%0], [%1], %2, %3;" ::
                     "l"(reinterpret_cast<uint64_t>(gdst)),
                 "r"(smem_u32(smem_src)), "r"(bytes), "l"(policy)
                 : "memory");
}

// Score KPT keys (rows lane + 32 k of the tile) on the chunks of one slice
// of SB bytes (32 or 64), swizzled by TMA with the same span: 16-byte chunk
// cc of row r sits at r * SB + ((cc ^ sw(r)) << 4) with sw(r) = (r >> 2) & 1
// (32-byte swizzle) or (r >> 1) & 3 (64-byte swizzle); with r = lane + 32 k
// the term is the same for every k.  c0: first 16-byte chunk of the slice
// within the row.  The arithmetic is that of score_core.cuh.
template <typename T, int G, int KPT, int SB>
__device__ __forceinline__ void score_slice(const uint8_t* slot, int c0, const float* w, int lane,
                                            float2 (&acc)[KPT][G]) {
    constexpr int kCh = SB / 16;
    const int sw = SB == 64 ? ((lane >> 1) & 3) : ((lane >> 2) & 1);
    if constexpr (sizeof(T) == 2) {
#pragma unroll
        for (int cc = 0; cc < kCh; ++cc) {
            const int c = c0 + cc;
            float2 xy[KPT][4];
            float2 nn[KPT][2];
#pragma unroll
            for (int k = 0; k < KPT; ++k) {
                const uint4 v = *reinterpret_cast<const uint4*>(slot + (lane + 32 * k) * SB +
                                                                ((cc ^ sw) << 4));
                band_pairs_bf16(v, xy[k], nn[k]);
            }
#pragma unroll
            for (int h = 0; h < G; ++h) {
                const float4* rec = reinterpret_cast<const float4*>(w + h * kWHead + c * kWChunk);
                const float4 a = rec[0], b = rec[1], cw = rec[2];
#pragma unroll
                for (int k = 0; k < KPT; ++k) {
                    float2 t = acc[k][h];
                    t = __ffma2_rn(xy[k][0], make_float2(a.x, a.y), t);
                    t = __ffma2_rn(xy[k][1], make_float2(a.z, a.w), t);
                    t = __ffma2_rn(xy[k][2], make_float2(b.x, b.y), t);
                    t = __ffma2_rn(xy[k][3], make_float2(b.z, b.w), t);
                    t = __ffma2_rn(nn[k][0], make_float2(cw.x, cw.y), t);
                    t = __ffma2_rn(nn[k][1], make_float2(cw.z, cw.w), t);
                    acc[k][h] = t;
                }
            }
        }
    } else {
        // float32 rows: a 16-byte chunk holds 2 bands.
#pragma unroll
        for (int cc = 0; cc < kCh; ++cc) {
            const int c = c0 + cc;
            float2 xy[KPT][2];
            float2 nn[KPT];
#pragma unroll
            for (int k = 0; k < KPT; ++k) {
                const float4 v = *reinterpret_cast<const float4*>(slot + (lane + 32 * k) * SB +
                                                                  ((cc ^ sw) << 4));
                band_pair_f32(v, xy[k], nn[k]);
            }
            const int half = c & 1;
#pragma unroll
            for (int h = 0; h < G; ++h) {
                const float* rec = w + h * kWHead + (c >> 1) * kWChunk;
                const float4 a = *reinterpret_cast<const float4*>(rec + 4 * half);
                const float2 cw = *reinterpret_cast<const float2*>(rec + 8 + 2 * half);
#pragma unroll
                for (int k = 0; k < KPT; ++k) {
                    float2 t = acc[k][h];
                    t = __ffma2_rn(xy[k][0], make_float2(a.x, a.y), t);
                    t = __ffma2_rn(xy[k][1], make_float2(a.z, a.w), t);
                    t = __ffma2_rn(nn[k], cw, t);
                    acc[k][h] = t;
                }
            }
        }
    }
}

// Final-score storage: shared memory (small units) or global memory through
// L2 (large units; written by this CTA, read back with .cg loads).  Rows are
// padded to a multiple of 32 keys, so every aligned group of 4 keys can be
// moved as one 16-byte access (keys at or past n hold garbage, never read as
// valid).
struct FinShared {
    float* p;
    __device__ __forceinline__ float4 get4(int j) const {
        return *reinterpret_cast<const float4*>(p + j);
    }
    __device__ __forceinline__ void put4(int j, float4 v) const {
        *reinterpret_cast<float4*>(p + j) = v;
    }
};
struct FinGlobal {
    float* p;
    __device__ __forceinline__ float4 get4(int j) const {
        return __ldcg(reinterpret_cast<const float4*>(p + j));
    }
    __device__ __forceinline__ void put4(int j, float4 v) const {
        __stcg(reinterpret_cast<float4*>(p + j), v);
    }
};

__device__ __forceinline__ float f4at(const float4& v, int i) {
    return i == 0 ? v.x : (i == 1 ? v.y : (i == 2 ? v.z : v.w));
}

// Round a key count up to the padded row length of the score scratch.
__host__ __device__ __forceinline__ int64_t pipe_pad(int64_t n) { return (n + 31) & ~int64_t(31); }

// Rank the listed threshold-bin candidates (at most kPipeCand): the B-th
// key's full 32-bit key T into ms->st.prefix and the number of its ties that
// are kept into ms->st.k.  Directly (one candidate per thread) when they are
// few, else by a three-digit radix of their keys.  Every math thread calls it.
__device__ __forceinline__ void rank_listed(int nc, uint32_t* hist, const int2* cand, PipeMisc* ms) {
    using S = PipeShape<float>;
    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    if (nc <= S::kMath) {
        const uint32_t k0 = ms->st.k;
        math_sync();  // k0 read before st changes
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
            ms->st.prefix = mk;
            ms->st.k = k0 - above;  // ties of the threshold key that are kept
        }
        math_sync();
        return;
    }
    for (int p = 0; p < 3; ++p) {
        const int nb = 1 << pass_bits(p);
        for (int b = tid; b < nb; b += S::kMath) hist[b] = 0;
        math_sync();
        const uint32_t prefix = ms->st.prefix;
        const int shift = pass_shift(p);
        const int hi_shift = shift + pass_bits(p);
        for (int i = tid; i < nc; i += S::kMath) {
            const uint32_t key = static_cast<uint32_t>(cand[i].x);
            if (p == 0 || (key >> hi_shift) == prefix) atomicAdd(&hist[(key >> shift) & (nb - 1)], 1u);
        }
        math_sync();
        if (warp == 0) {
            uint32_t bin, above;
            warp_find_bin(hist, nb, ms->st.k, bin, above);
            if (lane == 0) {
                ms->st.prefix = (prefix << pass_bits(p)) | bin;
                ms->st.k -= above;
                ms->st.gt += above;
            }
        }
        math_sync();
    }
}

// The z-bin b0 holding the B-th key, and the selection state that follows
// from it (warp 0), from a unit's z-bin histogram.
__device__ __forceinline__ void threshold_bin(const uint32_t* hist, int64_t B, PipeMisc* ms) {
    const int lane = threadIdx.x & 31;
    uint32_t bin, above;
    warp_find_bin(hist, kZBins, static_cast<uint32_t>(B), bin, above);
    if (lane == 0) {
        ms->zb0 = bin;
        ms->ncand = 0;
        ms->st.prefix = 0;
        ms->st.k = static_cast<uint32_t>(B) - above;  // to take from bin b0
        ms->st.gt = above;
        ms->st.keep_all = 0;
    }
}

// Ordered write of one 128-key block of final scores v (lane l holds keys
// 4l .. 4l + 3 of the block, the first at index jb): every key above T and
// the ties of T while fewer than kt have been taken; pos / ties run on.
template <typename Idx>
__device__ __forceinline__ void write_block(const float4& v, int jb, int valid_to, uint32_t Tk,
                                            uint32_t kt, int m, uint32_t& pos, uint32_t& ties,
                                            Idx* kidx) {
    const int lane = threadIdx.x & 31;
    const uint32_t lt = (1u << lane) - 1u;
    uint32_t gtm = 0, eqm = 0;  // 4-bit masks of this lane's keys
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint32_t key = ordered_key(f4at(v, i));
        const bool valid = jb + i < valid_to;
        gtm |= (valid && key > Tk) ? (1u << i) : 0u;
        eqm |= (valid && key == Tk) ? (1u << i) : 0u;
    }
    // Keys are ordered lane-major: ties before this lane's keys.
    uint32_t eq_before = 0, eq_total = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint32_t bal = __ballot_sync(0xffffffffu, (eqm >> i) & 1u);
        eq_before += __popc(bal & lt);
        eq_total += __popc(bal);
    }
    uint32_t keepm = gtm;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint32_t my_tie = ties + eq_before + __popc(eqm & ((1u << i) - 1u));
        if (((eqm >> i) & 1u) && my_tie < kt) keepm |= 1u << i;
    }
    uint32_t keep_before = 0, keep_total = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint32_t bal = __ballot_sync(0xffffffffu, (keepm >> i) & 1u);
        keep_before += __popc(bal & lt);
        keep_total += __popc(bal);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        if ((keepm >> i) & 1u) {
            const uint32_t r = pos + keep_before + __popc(keepm & ((1u << i) - 1u));
            if (r < static_cast<uint32_t>(m)) kidx[r] = static_cast<Idx>(jb + i);
        }
    }
    pos += keep_total;
    ties += eq_total;
}

// Selection of one unit by the math threads, from its final scores (padded
// row, 16-byte groups) and their z-bin histogram.
//   1. the z-bin b0 of the B-th key (a descending scan of the histogram);
//   2. one pass: each math warp walks a contiguous segment of whole 128-key
//      blocks, counts its keys above b0 and lists the keys inside b0 (the
//      candidates, at most kPipeCand);
//   3. the candidates are ranked directly (one per thread) or by a three-digit
//      radix of their full keys; if they did not fit the list, by the same
//      radix in place over every key of b0, with a counting pass;
//   4. one ordered pass writes the kept indices: every key above the
//      threshold key T and the first (B - above) keys equal to T.
// Loads keep 4 groups of 4 keys in flight per lane.
template <typename Fin, typename Idx>
__device__ __forceinline__ void select_unit(const Fin fin, int n, int64_t B, int m, uint32_t* hist,
                                         int2* cand, PipeMisc* ms, Idx* kidx) {
    using S = PipeShape<float>;
    // 128-key blocks whose loads are in flight at once.
    constexpr int kLook = 4;
    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    if (warp == 0) threshold_bin(hist, B, ms);
    if (tid < S::kMathWarps * 2) ms->wadd[tid >> 1][tid & 1] = 0u;
    math_sync();
    const uint32_t b0 = ms->zb0;
    const int nblk = (n + 127) >> 7;
    const int bpw = (nblk + S::kMathWarps - 1) / S::kMathWarps;  // blocks per warp segment
    const int blk0 = warp * bpw;
    const int blk1 = min(blk0 + bpw, nblk);
    // ---- pass: keys above b0 per segment, candidates ----
    {
        uint32_t above_bin = 0;
        for (int bb = blk0; bb < blk1; bb += kLook) {
            float4 v[kLook];
#pragma unroll
            for (int q = 0; q < kLook; ++q)
                if (bb + q < blk1) v[q] = fin.get4(((bb + q) << 7) + 4 * lane);
#pragma unroll
            for (int q = 0; q < kLook; ++q) {
                if (bb + q >= blk1) break;
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int j = ((bb + q) << 7) + 4 * lane + i;
                    const float f = f4at(v[q], i);
                    if (j < n) {
                        const uint32_t zb = zbin(f);
                        above_bin += zb > b0;
                        if (zb == b0) {
                            const int r = atomicAdd(&ms->ncand, 1);
                            if (r < kPipeCand) cand[r] = make_int2(static_cast<int>(ordered_key(f)), j);
                        }
                    }
                }
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) above_bin += __shfl_xor_sync(0xffffffffu, above_bin, o);
        if (lane == 0) ms->wcnt[warp][0] = above_bin;
    }
    math_sync();
    const int nc = ms->ncand;
    const bool listed = nc <= kPipeCand;
    if (listed) {
        rank_listed(nc, hist, cand, ms);
    } else {
        // Too many keys share b0 to list: the same radix in place over them.
        for (int p = 0; p < 3; ++p) {
            const int nb = 1 << pass_bits(p);
            for (int b = tid; b < nb; b += S::kMath) hist[b] = 0;
            math_sync();
            const uint32_t prefix = ms->st.prefix;
            const int shift = pass_shift(p);
            const int hi_shift = shift + pass_bits(p);
            for (int g = tid; 4 * g < n; g += S::kMath) {
                const float4 v = fin.get4(4 * g);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float f = f4at(v, i);
                    const uint32_t key = ordered_key(f);
                    if (4 * g + i < n && zbin(f) == b0 && (p == 0 || (key >> hi_shift) == prefix))
                        atomicAdd(&hist[(key >> shift) & (nb - 1)], 1u);
                }
            }
            math_sync();
            if (warp == 0) {
                uint32_t bin, above;
                warp_find_bin(hist, nb, ms->st.k, bin, above);
                if (lane == 0) {
                    ms->st.prefix = (prefix << pass_bits(p)) | bin;
                    ms->st.k -= above;
                    ms->st.gt += above;
                }
            }
            math_sync();
        }
    }
    const uint32_t Tk = ms->st.prefix, kt = ms->st.k;
    // ---- kept keys above T and ties of T per segment ----
    if (listed) {
        // From the list: a segment's keys above T are its keys above b0 and
        // its candidates above T; its ties are its candidates equal to T.
        const int seg_keys = bpw << 7;
        for (int i = tid; i < nc; i += S::kMath) {
            const int2 e = cand[i];
            const uint32_t ek = static_cast<uint32_t>(e.x);
            const int sgi = e.y / seg_keys;
            if (ek > Tk) atomicAdd(&ms->wadd[sgi][0], 1u);
            if (ek == Tk) atomicAdd(&ms->wadd[sgi][1], 1u);
        }
    } else {
        uint32_t gt = 0, eq = 0;
        for (int bb = blk0; bb < blk1; bb += kLook) {
            float4 v[kLook];
#pragma unroll
            for (int q = 0; q < kLook; ++q)
                if (bb + q < blk1) v[q] = fin.get4(((bb + q) << 7) + 4 * lane);
#pragma unroll
            for (int q = 0; q < kLook; ++q) {
                if (bb + q >= blk1) break;
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int j = ((bb + q) << 7) + 4 * lane + i;
                    const uint32_t key = ordered_key(f4at(v[q], i));
                    gt += j < n && key > Tk;
                    eq += j < n && key == Tk;
                }
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            gt += __shfl_xor_sync(0xffffffffu, gt, o);
            eq += __shfl_xor_sync(0xffffffffu, eq, o);
        }
        if (lane == 0) {
            ms->wcnt[warp][0] = 0u;
            ms->wadd[warp][0] = gt;
            ms->wadd[warp][1] = eq;
        }
    }
    math_sync();
    // ---- ordered write of the kept indices ----
    uint32_t pos = 0, ties = 0;
    for (int v = 0; v < warp; ++v) {
        const uint32_t gtv = ms->wcnt[v][0] + ms->wadd[v][0];
        const uint32_t eqv = ms->wadd[v][1];
        const uint32_t take = ties < kt ? min(eqv, kt - ties) : 0u;
        pos += gtv + take;
        ties += eqv;
    }
    for (int bb = blk0; bb < blk1; bb += kLook) {
        float4 v[kLook];
#pragma unroll
        for (int q = 0; q < kLook; ++q)
            if (bb + q < blk1) v[q] = fin.get4(((bb + q) << 7) + 4 * lane);
#pragma unroll
        for (int q = 0; q < kLook; ++q) {
            if (bb + q >= blk1) break;
            write_block(v[q], ((bb + q) << 7) + 4 * lane, n, Tk, kt, m, pos, ties, kidx);
        }
    }
}

// z-scores of the unit's keys from the per-head scores in global memory
// (padded rows of stride ldr), their maximum over the group into fin (and
// into final_out, when given), the z-bin histogram into hist (zeroed by the
// caller), NaN flagged.  Groups of 4 keys move as 16-byte accesses.
template <int G, typename Fin>
__device__ __forceinline__ void zmax_unit(const float* raw, int64_t ldr, int n, const PipeMisc* ms,
                                       const Fin fin, float* final_out, uint32_t* hist,
                                       int64_t n_sink, int64_t n_recent, uint32_t* flag) {
    using S = PipeShape<float>;
    const int tid = threadIdx.x;
    float mu[G], inv[G];
#pragma unroll
    for (int h = 0; h < G; ++h) {
        mu[h] = ms->mom[h].x;
        inv[h] = ms->mom[h].y;
    }
    bool nonfinite = false;
    // Groups of 4 keys in flight per thread: 16-byte loads of every head.
    constexpr int kU = G <= 4 ? 2 : 1;
    const int n4 = (n + 3) >> 2;
    for (int g0 = tid; g0 < n4; g0 += S::kMath * kU) {
        float4 sv[kU][G];
#pragma unroll
        for (int q = 0; q < kU; ++q) {
            const int g = g0 + q * S::kMath;
#pragma unroll
            for (int h = 0; h < G; ++h)
                if (g < n4) sv[q][h] = __ldcg(reinterpret_cast<const float4*>(raw + h * ldr) + g);
        }
#pragma unroll
        for (int q = 0; q < kU; ++q) {
            const int g = g0 + q * S::kMath;
            if (g >= n4) break;
            float best[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
#pragma unroll
                for (int h = 0; h < G; ++h) {
                    const float z = (f4at(sv[q][h], i) - mu[h]) * inv[h];
                    best[i] = (h == 0) ? z : fmaxf(best[i], z);
                }
                if (best[i] != best[i] && 4 * g + i < n) nonfinite = true;
                // Protected sink / recent keys rank above every score.
                if (4 * g + i < n_sink || 4 * g + i >= n - n_recent) best[i] = INFINITY;
            }
            fin.put4(4 * g, make_float4(best[0], best[1], best[2], best[3]));
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                if (4 * g + i < n) {
                    atomicAdd(&hist[zbin(best[i])], 1u);
                    if (final_out) final_out[4 * g + i] = best[i];
                }
            }
        }
    }
    if (nonfinite) raise_flag(flag, TRI_FLAG_NONFINITE);
}

// (mu, 1/sigma) from float64 sums over n keys; NaN propagates.
__device__ __forceinline__ float2 moments_from_sums(double s1, double s2, int n) {
    if (n <= 0) return make_float2(0.f, 0.f);
    const double mu = s1 / n;
    double var = s2 / n - mu * mu;
    if (var < 0.0) var = 0.0;
    const double sd = sqrt(var);
    float inv = sd > 0.0 ? static_cast<float>(1.0 / sd) : 0.f;
    if (!(sd == sd)) inv = __int_as_float(0x7fc00000);
    return make_float2(static_cast<float>(mu), inv);
}

__device__ __forceinline__ void pipe_trace(const PipeArgs& a, int64_t u, int p, int slot) {
    if (a.trace && (threadIdx.x & 31) == 0)
        a.trace[(u * kTracePoints + p) * kTraceWarps + slot] = globaltimer_ns();
}

// ---------------------------------------------------------------------------
// The gather engine (kEngWarps warps).
//
// Pieces: destination rows [kGRows q, kGRows (q + 1)) of a unit (32 bf16 or
// 16 float32 rows), of K and of V together in one 16 KB buffer; engine warp
// e takes pieces e, e + kEngWarps, ... of every unit, through its own share
// of the buffers.  The math warps have marked the rows of each piece that
// start a run of consecutive source rows (the piece's run-start mask).  Loading a piece: lane o takes bulk load o, the K (o even) or V (o
// odd) rows of run o / 2, so one instruction issues up to 32 loads, all
// completing on the buffer's barrier (a bulk-copy instruction costs its warp
// a few hundred cycles whatever its size, its lanes little more).
// Up to (buffers - kGGap) pieces load while older ones are stored, K by lane
// 0 and V by lane 1 of one instruction, so loads, stores and the next unit's
// loads overlap.
// ---------------------------------------------------------------------------
template <typename T, typename Idx>
__device__ void pipe_engine(const PipeArgs& a, int eng, uint8_t* gbuf, int gs, const Idx* kidx_base,
                            size_t kidx_stride, const uint64_t* smask_base, size_t smask_stride,
                            uint64_t* gfull, uint64_t* kready, uint64_t* kfree, PipeMisc* ms) {
    using S = PipeShape<T>;
    const int lane = threadIdx.x & 31;
    const uint64_t pol = policy_evict_first();
    const char* ks = static_cast<const char*>(a.k_src);
    const char* vs = static_cast<const char*>(a.v_src);
    char* kd = static_cast<char*>(a.k_dst);
    char* vd = static_cast<char*>(a.v_dst);
    const bool has_v = a.v_src != nullptr;
    const uint32_t ahead = static_cast<uint32_t>(gs - S::kGGap);  // pieces loading at once
    uint32_t issued = 0, stored = 0, hs = 0;
    bool have = false, done = false, failed = false;
    int64_t u = 0;
    int m = 0, P = 0, q = 0;
    const Idx* kx = nullptr;
    const uint64_t* smask = nullptr;

    // Store the oldest loaded piece.  Returns false if its wait gave up.
    auto store_one = [&]() -> bool {
        const int sl = stored % gs;
        if (!warp_wait(&gfull[sl], (stored / gs) & 1, a.flag)) return false;
        if (S::kEngWarps > 1 && a.inplace) {
            // In place, a piece is stored only after the piece before it
            // (the other engine's) has landed, so that every earlier piece's
            // source rows are read before this piece's rows are written.
            const uint64_t seq = ms->gseq[eng * gs + sl];
            bool ok = true;
            if (lane == 0) {
                volatile uint64_t* mine = &ms->landed[eng];
                *mine = seq + 1u;
                __threadfence_block();
                const volatile uint64_t* other = &ms->landed[1 - eng];
                if ((seq & 0xffffffffu) != 0u && *other < seq) {
                    const uint64_t t0 = globaltimer_ns();
                    while (*other < seq) {
                        if (globaltimer_ns() - t0 > kWaitLimitNs) {
                            raise_flag(a.flag, TRI_FLAG_TIMEOUT);
                            ok = false;
                            break;
                        }
                        __nanosleep(32);
                    }
                }
                __threadfence_block();
            }
            if (!__shfl_sync(0xffffffffu, ok, 0)) return false;
        }
        if (lane < (has_v ? 2 : 1)) {
            const int g = eng * gs + sl;
            const int64_t off = ms->gdst[g];
            const uint32_t bytes = ms->gdst_rows[g] * S::kRowBytes;
            bulk_store_hint((lane ? vd : kd) + off, gbuf + sl * S::kGSlotBytes + lane * S::kGHalf, bytes,
                            pol);
            bulk_commit();
        }
        __syncwarp();
        ++stored;
        return true;
    };

    while (true) {
        if (!have && !done) {
            const int slot = hs % S::kHand;
            const uint32_t par = (hs / S::kHand) & 1;
            // Drain loaded pieces while the next unit is not ready (a phase
            // seen complete by any lane is complete for all).
            if (stored < issued && !__any_sync(0xffffffffu, mbar_try_wait(&kready[slot], par))) {
                if (!store_one()) {
                    failed = true;
                    break;
                }
                continue;
            }
            if (!warp_wait(&kready[slot], par, a.flag)) {
                failed = true;
                break;
            }
            u = ms->hdr_u[slot];
            if (u < 0) {
                done = true;
                continue;
            }
            m = ms->hdr_m[slot];
            kx = kidx_base + slot * kidx_stride;
            smask = smask_base + slot * smask_stride;
            P = (m + S::kGRows - 1) / S::kGRows;
            // Warp e takes pieces e, e + kEngWarps, ... (in place, each
            // store also waits for the other engine's previous piece).
            q = eng;
            if (eng == 0) pipe_trace(a, u, 4, 0);
            if (q >= P) {
                __syncwarp();
                if (lane == 0) mbar_arrive(&kfree[slot]);
                ++hs;
            } else {
                have = true;
            }
            continue;
        }
        if (have && issued - stored < ahead) {
            const int sl = issued % gs;
            // The store that last read this buffer (piece issued - gs) must
            // be done reading it: stored >= issued - ahead + 1, so at least
            // gs - ahead = kGGap stores were committed after it, and it is
            // complete once no more than the kGGap newest are pending.
            if (issued >= static_cast<uint32_t>(gs) && lane < (has_v ? 2 : 1))
                bulk_wait_read<S::kGGap>();  // lanes 0 and 1 each track their own stores
            __syncwarp();
            const int r0 = q * S::kGRows;
            const int rows = min(S::kGRows, m - r0);
            // Only the piece's own rows, and its first row always starts a
            // run: the runs then partition the piece exactly, whatever the mask.
            const uint64_t row_mask = rows >= 64 ? ~0ull : ((1ull << rows) - 1ull);
            const uint64_t starts = (smask[q] & row_mask) | 1ull;
            const int n_runs = __popcll(starts);
            int32_t* rs = ms->runst[eng];
#pragma unroll
            for (int hb = 0; hb < 2; ++hb) {
                const int bit = lane + 32 * hb;
                if ((starts >> bit) & 1ull) rs[__popcll(starts & ((1ull << bit) - 1ull))] = bit;
            }
            uint64_t* landed = &gfull[sl];
            if (lane == 0) {
                mbar_arrive_expect_tx(landed, static_cast<uint32_t>(rows * S::kRowBytes * (has_v ? 2 : 1)));
                ms->gdst[eng * gs + sl] = (u * a.cap_dst + r0) * S::kRowBytes;
                ms->gdst_rows[eng * gs + sl] = static_cast<uint32_t>(rows);
                ms->gseq[eng * gs + sl] = (static_cast<uint64_t>(hs) << 32) | static_cast<uint32_t>(q);
            }
            __syncwarp();
            uint8_t* buf = gbuf + sl * S::kGSlotBytes;
            const int n_ops = n_runs * (has_v ? 2 : 1);
            for (int o = lane; o - lane < n_ops; o += 32) {
                if (o < n_ops) {
                    const int r = has_v ? (o >> 1) : o;
                    const int t = has_v ? (o & 1) : 0;
                    const int l0 = rs[r];
                    const int l1 = r + 1 < n_runs ? rs[r + 1] : rows;
                    const int32_t j = static_cast<int32_t>(kx[r0 + l0]);
                    // A run that would leave the source cache (cannot happen)
                    // lands copies of row 0 instead, so that the barrier completes.
                    const bool ok = j >= 0 && j + (l1 - l0) <= a.cap;
                    if (!ok) raise_flag(a.flag, TRI_FLAG_INDEX_RANGE);
                    const char* src = (t ? vs : ks) + (u * a.cap + (ok ? j : 0)) * S::kRowBytes;
                    uint8_t* dst = buf + t * S::kGHalf + l0 * S::kRowBytes;
                    if (ok) {
                        bulk_load_hint(dst, src, static_cast<uint32_t>((l1 - l0) * S::kRowBytes), landed, pol);
                    } else {
                        for (int l = 0; l < l1 - l0; ++l)
                            bulk_load_hint(dst + l * S::kRowBytes, src, S::kRowBytes, landed, pol);
                    }
                }
            }
            __syncwarp();  // the run starts are read before the next piece rewrites them
            ++issued;
            q += S::kEngWarps;
            if (q >= P) {
                // Every load of this warp's pieces of the unit is issued.
                __syncwarp();
                if (eng == 0) pipe_trace(a, u, 5, 0);
                if (lane == 0) mbar_arrive(&kfree[hs % S::kHand]);
                ++hs;
                have = false;
            }
            continue;
        }
        if (stored < issued) {
            if (!store_one()) {
                failed = true;
                break;
            }
            continue;
        }
        if (done) break;
    }
    if (failed) ms->abort = 1;
    if (lane < 2) bulk_wait_all();
    if (failed) {
        // Loads still in flight into the buffers: give them time to land.
        const uint64_t t0 = globaltimer_ns();
        while (globaltimer_ns() - t0 < 200000) __nanosleep(1000);
    }
    __syncwarp();
}

__device__ __forceinline__ bool pipe_aborted(const PipeMisc* ms) {
    return *reinterpret_cast<const volatile int32_t*>(&ms->abort) != 0;
}

// ---------------------------------------------------------------------------
// The kernel.
// ---------------------------------------------------------------------------
template <typename T, int G, bool kBig>
__global__ void __launch_bounds__(PipeShape<T, kBig>::kThreads, 1)
prune_pipe_kernel(const __grid_constant__ CUtensorMap kmap, PipeArgs a) {
    using S = PipeShape<T, kBig>;
    using Idx = typename std::conditional<kBig, int32_t, uint16_t>::type;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const PipeLayout L = pipe_layout<T>(G, a.cap, a.B, kBig, a.gslots);
    uint8_t* ring = base + L.ring;
    uint8_t* gbuf = base + L.gbuf;
    float* w = reinterpret_cast<float*>(base + L.w);
    float* fin_s = reinterpret_cast<float*>(base + L.fin);       // aliases the rings
    uint32_t* hist = reinterpret_cast<uint32_t*>(base + L.hist);  // aliases the rings
    int2* cand = reinterpret_cast<int2*>(base + L.cand);          // aliases the rings
    Idx* kidx = reinterpret_cast<Idx*>(base + L.kidx);
    uint64_t* smask = reinterpret_cast<uint64_t*>(base + L.smask);
    const int64_t m_max = a.B < a.cap ? a.B : a.cap;
    const size_t kidx_stride =
        ((static_cast<size_t>(m_max) * sizeof(Idx) + 15) & ~size_t(15)) / sizeof(Idx);
    const size_t smask_stride =
        ((static_cast<size_t>((m_max + S::kGRows - 1) / S::kGRows) * 8 + 15) & ~size_t(15)) / 8;
    uint64_t* full = reinterpret_cast<uint64_t*>(base + L.bars);  // [warp][kQ]
    uint64_t* gfull = full + S::kMathWarps * pipe_full_bars<T>();  // [gslots]
    uint64_t* kready = gfull + S::kMaxGSlots;                       // [kHand]
    uint64_t* kfree = kready + S::kHand;                            // [kHand]
    double* red = reinterpret_cast<double*>(base + L.red);         // [warp][kMaxG][2]
    PipeMisc* ms = reinterpret_cast<PipeMisc*>(base + L.misc);
    __shared__ FoldShared fs;

    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int gs = a.gslots / S::kEngWarps;  // gather buffers per engine warp
    if (tid == 0) {
        for (int i = 0; i < S::kMathWarps * S::kQ; ++i) mbar_init(&full[i], 1);
        for (int i = 0; i < a.gslots; ++i) mbar_init(&gfull[i], 1);
        for (int i = 0; i < S::kHand; ++i) {
            mbar_init(&kready[i], 1);
            mbar_init(&kfree[i], S::kEngWarps);
        }
        fence_barrier_init();
        prefetch_tensormap(&kmap);
        ms->abort = 0;
        ms->stop = 0;
        ms->landed[0] = ms->landed[1] = 0ull;
        ms->item = -1;
    }
    __syncthreads();  // barriers and state initialised before anyone uses them

    if (warp >= S::kMathWarps) {
        const int e = warp - S::kMathWarps;
        pipe_engine<T, Idx>(a, e, gbuf + static_cast<size_t>(e) * gs * S::kGSlotBytes, gs, kidx,
                            kidx_stride, smask, smask_stride, gfull + e * gs, kready, kfree, ms);
        return;
    }

    // ----------------------------- math warps -----------------------------
    const int64_t B = a.B;
    // Keys of small units are read again by the gather (keep them in L2);
    // of large units only a few are, so their tiles are loaded as last use,
    // but fetched into L2 ahead of that with normal priority.
    const uint64_t kpol = kBig ? policy_evict_first() : policy_evict_last();
    const uint64_t pfpol = kBig ? policy_evict_normal() : policy_evict_last();
    uint8_t* my_ring = ring + static_cast<size_t>(warp) * S::kQ * S::kSlotBytes;
    uint64_t* my_full = full + warp * S::kQ;
    uint32_t sq = 0;  // slices this warp has consumed (ring position)
    uint32_t hs = 0;  // units handed to the engine
    const char* kbytes = static_cast<const char*>(a.k_src);

    // Issue slice i of this warp's tiles of unit u (tile t0 + warp +
    // kMathWarps (i / kSlices), column slice i % kSlices) into its ring slot.
    auto issue = [&](int64_t u, int t0, int i) {
        const uint32_t qn = sq + static_cast<uint32_t>(i);
        const int slot = qn % S::kQ;
        const int tile = t0 + warp + S::kMathWarps * (i / S::kSlices);
        const int slice = i % S::kSlices;
        uint64_t* bar = &my_full[slot];
        mbar_arrive_expect_tx(bar, S::kSlotBytes);
        tma_load_2d_hint(my_ring + slot * S::kSlotBytes, &kmap, bar, slice * S::kSliceElems,
                         static_cast<int32_t>(u * a.cap + static_cast<int64_t>(tile) * S::kTile),
                         kpol);
    };
    // Ask L2 for tile `tile` of unit u (rows inside the unit's buffer only).
    auto prefetch_tile = [&](int64_t u, int tile, int t_end) {
        if (tile >= t_end) return;
        const int rows = min(S::kTile, static_cast<int>(a.cap) - tile * S::kTile);
        if (rows <= 0) return;
        prefetch_l2_bulk(kbytes + (u * a.cap + static_cast<int64_t>(tile) * S::kTile) * S::kRowBytes,
                         static_cast<uint32_t>(rows * S::kRowBytes), pfpol);
    };
    auto warp_slices = [&](int t0, int t1) {
        const int nt = t1 - t0;
        const int nt_w = warp < nt ? (nt - 1 - warp) / S::kMathWarps + 1 : 0;
        return nt_w * S::kSlices;
    };
    // First kQ slices of this warp's tiles of [t0, t1) of unit u.  The rings
    // may hold the histogram, candidates and final scores of the previous
    // unit, written through the generic proxy: fence before TMA overwrites.
    auto first_loads = [&](int64_t u, int t0, int t1) {
        const int total = warp_slices(t0, t1);
        if (lane == 0) {
            fence_proxy_async();
            for (int i = 0; i < S::kQ && i < total; ++i) issue(u, t0, i);
            for (int k = 0; k <= S::kPfAhead; ++k) prefetch_tile(u, t0 + warp + k * S::kMathWarps, t1);
        }
    };

    // Score this warp's tiles of [t0, t1) of unit u (n valid keys): per-head
    // scores to raw (row stride ldr), float64 moments into red[warp].  A
    // wait that gives up sets ms->stop (read after the caller's barrier).
    auto score_range = [&](int64_t u, int n, int t0, int t1, float* raw, int64_t ldr) {
        const int total = warp_slices(t0, t1);
        double m1[G], m2[G];
#pragma unroll
        for (int h = 0; h < G; ++h) m1[h] = m2[h] = 0.0;
        float2 acc[S::kKPT][G];
        for (int i = 0; i < total; ++i) {
            const uint32_t qn = sq + static_cast<uint32_t>(i);
            const int slot = qn % S::kQ;
            const int slice = i % S::kSlices;
            const int tile = t0 + warp + S::kMathWarps * (i / S::kSlices);
            if (slice == 0) {
                score_acc_zero<G, S::kKPT>(acc);
                if (lane == 0) prefetch_tile(u, tile + (S::kPfAhead + 1) * S::kMathWarps, t1);
            }
            if (!warp_wait(&my_full[slot], (qn / S::kQ) & 1, a.flag)) {
                if (lane == 0) ms->stop = 1;
                break;
            }
            score_slice<T, G, S::kKPT, S::kSliceBytes>(my_ring + slot * S::kSlotBytes,
                                                       slice * S::kSliceChunks, w, lane, acc);
            __syncwarp();
            if (lane == 0 && i + S::kQ < total) {
                fence_proxy_async();
                issue(u, t0, i + S::kQ);
            }
            if (slice == S::kSlices - 1) {
#pragma unroll
                for (int k = 0; k < S::kKPT; ++k) {
                    const int j = tile * S::kTile + lane + 32 * k;
                    if (j < n) {
#pragma unroll
                        for (int h = 0; h < G; ++h) {
                            const float sc = acc[k][h].x + acc[k][h].y;
                            __stcg(raw + h * ldr + j, sc);
                            const double d = sc;
                            m1[h] += d;
                            m2[h] = fma(d, d, m2[h]);
                        }
                    }
                }
            }
        }
        sq += static_cast<uint32_t>(total);
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
    };

    // Hand unit u (m kept rows) to the engine: `fill` writes the kept
    // indices into the next index buffer once the engine is done with it,
    // the run-start mask of every gather piece follows, the engine is told,
    // and then the kept / n_kept outputs and the kept rows' positions are
    // written by the math warps while the engine gathers K and V.
    auto handoff = [&](int64_t u, int m, auto&& fill) -> bool {
        const int slot = hs % S::kHand;
        // One thread waits for the engine to release the index buffer; the
        // outcome reaches every math thread through the barrier.
        if (tid == 0 && hs >= static_cast<uint32_t>(S::kHand) &&
            !mbar_wait(&kfree[slot], ((hs / S::kHand) - 1) & 1, a.flag))
            ms->stop = 1;
        math_sync();
        if (ms->stop) return false;
        Idx* kx = kidx + slot * kidx_stride;
        uint64_t* sm = smask + slot * smask_stride;
        fill(kx);
        math_sync();
        const int P = (m + S::kGRows - 1) / S::kGRows;
        for (int q = warp; q < P; q += S::kMathWarps) {
            // Rows q kGRows + lane (and + 32): a row starts a run unless its
            // source row follows that of the row before it in the piece.
            const int ra = q * S::kGRows + lane;
            const bool va = lane < S::kGRows && ra < m;
            const int32_t ja = va ? static_cast<int32_t>(kx[ra]) : 0;
            const int32_t pa = __shfl_up_sync(0xffffffffu, ja, 1);
            uint64_t st = __ballot_sync(0xffffffffu, va && (lane == 0 || ja != pa + 1));
            if (S::kGRows > 32) {
                const int rb = ra + 32;
                const bool vb = rb < m;
                const int32_t jb = vb ? static_cast<int32_t>(kx[rb]) : 0;
                int32_t pb = __shfl_up_sync(0xffffffffu, jb, 1);
                const int32_t last_a = __shfl_sync(0xffffffffu, ja, 31);
                if (lane == 0) pb = last_a;
                st |= static_cast<uint64_t>(__ballot_sync(0xffffffffu, vb && jb != pb + 1)) << 32;
            }
            if (lane == 0) sm[q] = st;
        }
        math_sync();
        if (tid == 0) {
            ms->hdr_u[slot] = u;
            ms->hdr_m[slot] = m;
            mbar_arrive(&kready[slot]);
            a.n_kept[u] = m;
        }
        if (a.kept) {
            for (int r = tid; r < B; r += S::kMath)
                a.kept[u * B + r] = r < m ? static_cast<int32_t>(kx[r]) : -1;
        }
        if (a.pos_src) {
            // Rounds of kU * kMath rows.  In place, a round's stores may land
            // on rows the same round reads (never on rows a later round
            // reads: sources are at or after their destination), so the
            // round's loads are performed before the barrier, its stores
            // after it.
            constexpr int kU = 8;
            for (int b0 = 0; b0 < m; b0 += S::kMath * kU) {
                int32_t pv[kU];
#pragma unroll
                for (int qq = 0; qq < kU; ++qq) {
                    const int r = b0 + tid + qq * S::kMath;
                    pv[qq] = r < m ? a.pos_src[u * a.cap + kx[r]] : 0;
                }
                if (a.inplace) math_sync();
#pragma unroll
                for (int qq = 0; qq < kU; ++qq) {
                    const int r = b0 + tid + qq * S::kMath;
                    if (r < m) a.pos_dst[u * a.cap_dst + r] = pv[qq];
                }
            }
        }
        ++hs;
        return true;
    };
    auto send_end = [&]() {
        const int slot = hs % S::kHand;
        if (tid == 0) {
            if (hs >= static_cast<uint32_t>(S::kHand))
                mbar_wait(&kfree[slot], ((hs / S::kHand) - 1) & 1, a.flag);
            ms->hdr_u[slot] = -1;
            mbar_arrive(&kready[slot]);
        }
        ++hs;
    };
    // Moments of the unit from the math warps' partials (fixed order).
    auto warp_sums = [&](double& s1, double& s2) {
        s1 = 0.0;
        s2 = 0.0;
#pragma unroll
        for (int v = 0; v < S::kMathWarps; ++v) {
            s1 += red[(v * kMaxG + tid) * 2];
            s2 += red[(v * kMaxG + tid) * 2 + 1];
        }
    };
    bool failed = false;

    if constexpr (!kBig) {
        const int64_t capP = pipe_pad(a.cap);  // padded row of the score scratch
        float* raw = a.raw + static_cast<int64_t>(blockIdx.x) * G * capP;
        for (int64_t u = blockIdx.x; u < a.n_units; u += gridDim.x) {
            if (tid == 0 && pipe_aborted(ms)) ms->stop = 1;
            math_sync();
            if (ms->stop) {
                failed = true;
                break;
            }
            const int n = clamp_nvalid(a.n_valid, u, a.cap, tid == 0 ? a.flag : nullptr);
            const int64_t Bu = unit_budget(a.ub, u, B);
            const int m = static_cast<int>(n < Bu ? n : Bu);
            pipe_trace(a, u, 0, warp);
            if (n > Bu && Bu > 0) {
                const int n_tiles = (n + S::kTile - 1) / S::kTile;
                first_loads(u, 0, n_tiles);
                fold_unit_sync<G>(fs, a.fc, w, a.stats, a.p_cur, u, a.n_layers, a.n_kvheads, 1,
                                  S::kMath);
                score_range(u, n, 0, n_tiles, raw, capP);
                pipe_trace(a, u, 1, warp);
                math_sync();
                if (ms->stop) {
                    failed = true;
                    break;
                }
                if (tid < G) {
                    double s1, s2;
                    warp_sums(s1, s2);
                    ms->mom[tid] = moments_from_sums(s1, s2, n);
                }
                for (int b = tid; b < kZBins; b += S::kMath) hist[b] = 0;
                math_sync();
                zmax_unit<G>(raw, capP, n, ms, FinShared{fin_s},
                             a.final_out ? a.final_out + u * a.cap : nullptr, hist, a.n_sink,
                             a.n_recent, a.flag);
                math_sync();
                pipe_trace(a, u, 2, warp);
                // This warp's first tile of the next unit into L2.
                const int64_t un = u + gridDim.x;
                if (lane == 0 && un < a.n_units) {
                    const int nn = clamp_nvalid(a.n_valid, un, a.cap, nullptr);
                    if (nn > unit_budget(a.ub, un, B))
                        prefetch_tile(un, warp, (nn + S::kTile - 1) / S::kTile);
                }
                const bool ok = handoff(u, m, [&](Idx* kx) {
                    select_unit(FinShared{fin_s}, n, Bu, m, hist, cand, ms, kx);
                });
                if (!ok) {
                    failed = true;
                    break;
                }
            } else {
                const bool ok = handoff(u, m, [&](Idx* kx) {
                    for (int r = tid; r < m; r += S::kMath) kx[r] = static_cast<Idx>(r);
                });
                if (!ok) {
                    failed = true;
                    break;
                }
            }
            pipe_trace(a, u, 3, warp);
        }
    } else {
        // Large units: work items (unit, chunk of kChunkTiles tiles) from an
        // atomic queue; thread 0 fetches the next item while this one runs,
        // and asks L2 for the next item's first tiles and weights.
        const int64_t capP = pipe_pad(a.cap);  // padded row of the score scratch
        const int64_t ck = static_cast<int64_t>(kChunkTiles) * S::kTile;
        const int64_t cpu = (a.cap + ck - 1) / ck;  // chunks per unit
        const int64_t n_items = a.n_units * cpu;
        uint32_t next = 0;
        if (tid == 0) next = atomicAdd(a.queue, 1u);
        while (true) {
            if (tid == 0) {
                ms->item = next;
                if (next < n_items) next = atomicAdd(a.queue, 1u);
                if (pipe_aborted(ms)) ms->stop = 1;
            }
            math_sync();
            const int64_t item = ms->item;
            if (ms->stop) {
                failed = true;
                break;
            }
            if (item >= n_items) break;
            const int64_t u = item / cpu;
            const int c = static_cast<int>(item % cpu);
            const int n = clamp_nvalid(a.n_valid, u, a.cap, (tid == 0 && c == 0) ? a.flag : nullptr);
            const int64_t Bu = unit_budget(a.ub, u, B);
            const int m = static_cast<int>(n < Bu ? n : Bu);
            if (n <= Bu || Bu == 0) {
                if (c == 0) {
                    const bool ok = handoff(u, m, [&](Idx* kx) {
                        for (int r = tid; r < m; r += S::kMath) kx[r] = r;
                    });
                    if (!ok) {
                        failed = true;
                        break;
                    }
                }
                math_sync();
                continue;
            }
            const int n_tiles = (n + S::kTile - 1) / S::kTile;
            const int chunks = (n_tiles + kChunkTiles - 1) / kChunkTiles;
            if (c >= chunks) {
                math_sync();
                continue;
            }
            const int t0 = c * kChunkTiles;
            const int t1 = min(t0 + kChunkTiles, n_tiles);
            first_loads(u, t0, t1);
            {
                const float4* src = reinterpret_cast<const float4*>(a.wts + u * G * kWHead);
                float4* dst = reinterpret_cast<float4*>(w);
                for (int e = tid; e < G * kWHead / 4; e += S::kMath) dst[e] = __ldg(src + e);
            }
            if (tid == 0 && next < n_items) {
                // The next item's first tiles and weights into L2.
                const int64_t un = next / cpu;
                const int cn = static_cast<int>(next % cpu);
                const int nn = clamp_nvalid(a.n_valid, un, a.cap, nullptr);
                const int ntn = (nn + S::kTile - 1) / S::kTile;
                if (nn > unit_budget(a.ub, un, B) && cn * kChunkTiles < ntn) {
                    for (int t = 0; t < S::kMathWarps; ++t)
                        prefetch_tile(un, cn * kChunkTiles + t, min(cn * kChunkTiles + kChunkTiles, ntn));
                    prefetch_l2_bulk(a.wts + un * G * kWHead, G * kWHead * 4, pfpol);
                }
            }
            math_sync();
            float* raw = a.raw + u * G * capP;
            score_range(u, n, t0, t1, raw, capP);
            math_sync();
            if (ms->stop) {
                failed = true;
                break;
            }
            if (tid < G) {
                double s1, s2;
                warp_sums(s1, s2);
                double* part = a.partial + (u * cpu + c) * G * 2;
                __stcg(part + 2 * tid, s1);
                __stcg(part + 2 * tid + 1, s2);
            }
            math_sync();
            if (tid == 0) {
                __threadfence();
                const uint32_t prev = atomicAdd(&a.counters[u], 1u);
                ms->last = prev == static_cast<uint32_t>(chunks - 1);
            }
            math_sync();
            if (!ms->last) continue;
            __threadfence();
            // This CTA completed unit u: moments in chunk order, final
            // scores, selection, hand-off.  The chunks' partials are loaded
            // at once (into the idle rings) and summed in chunk order.
            {
                double* pp = reinterpret_cast<double*>(ring + kPartOff);
                const double* part = a.partial + u * cpu * G * 2;
                for (int e = tid; e < chunks * G * 2; e += S::kMath) pp[e] = __ldcg(part + e);
                math_sync();
                if (tid < G) {
                    double s1 = 0.0, s2 = 0.0;
                    for (int cc = 0; cc < chunks; ++cc) {
                        s1 += pp[(cc * G + tid) * 2];
                        s2 += pp[(cc * G + tid) * 2 + 1];
                    }
                    ms->mom[tid] = moments_from_sums(s1, s2, n);
                }
            }
            if (tid == 0) a.counters[u] = 0u;
            for (int b = tid; b < kZBins; b += S::kMath) hist[b] = 0;
            math_sync();
            float* fin_g = a.fin_scratch + static_cast<int64_t>(blockIdx.x) * capP;
            float* fo = a.final_out ? a.final_out + u * a.cap : nullptr;
            zmax_unit<G>(raw, capP, n, ms, FinGlobal{fin_g}, fo, hist, a.n_sink, a.n_recent,
                         a.flag);
            math_sync();
            const bool ok = handoff(u, m, [&](Idx* kx) {
                select_unit(FinGlobal{fin_g}, n, Bu, m, hist, cand, ms, kx);
            });
            if (!ok) {
                failed = true;
                break;
            }
        }
    }
    if (failed) ms->abort = 1;
    math_sync();
    send_end();
    if (failed) {
        // Loads still in flight into the ring: give them time to land.
        const uint64_t t0 = globaltimer_ns();
        while (globaltimer_ns() - t0 < 200000) __nanosleep(1000);
    }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
size_t pipe_smem_bytes(tri_dtype dt, int G, int64_t cap, int64_t B, bool big, int gslots) {
    return dt == TRI_BF16 ? pipe_layout<__nv_bfloat16>(G, cap, B, big, gslots).total
                          : pipe_layout<float>(G, cap, B, big, gslots).total;
}

int pipe_min_gslots() { return PipeShape<float>::kMinGSlots; }
int pipe_max_gslots() { return PipeShape<float>::kMaxGSlots; }
int pipe_engine_warps() { return PipeShape<float>::kEngWarps; }

int pipe_tile_keys(tri_dtype dt) {
    return dt == TRI_BF16 ? PipeShape<__nv_bfloat16>::kTile : PipeShape<float>::kTile;
}

int pipe_chunk_keys(tri_dtype dt) { return pipe_tile_keys(dt) * kChunkTiles; }

bool pipe_small_fits(tri_dtype dt, int64_t cap) {
    return dt == TRI_BF16 ? pipe_small_unit<__nv_bfloat16>(cap) : pipe_small_unit<float>(cap);
}

bool pipe_big_fits(int64_t cap) {
    // The chunks' moment partials of one unit fit the rings after the
    // histogram and candidates.
    using S = PipeShape<float, true>;
    const int64_t chunks = (cap + kChunkTiles * S::kTile - 1) / (kChunkTiles * S::kTile);
    return kPartOff + chunks * kMaxG * 16 <= static_cast<int64_t>(S::kMathWarps) * S::kQ * S::kSlotBytes;
}

int pipe_slice_bytes(bool big) { return big ? PipeShape<float, true>::kSliceBytes
                                            : PipeShape<float, false>::kSliceBytes; }

template <typename T, int G, bool kBig>
static cudaError_t launch_pipe_t(const CUtensorMap& map, const PipeArgs& a, int n_ctas,
                                 cudaStream_t s) {
    // Dynamic part only; the fold's static shared memory is in the total.
    const size_t smem = pipe_layout<T>(G, a.cap, a.B, kBig, a.gslots).total - sizeof(FoldShared);
    auto kern = prune_pipe_kernel<T, G, kBig>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    kern<<<n_ctas, PipeShape<T, kBig>::kThreads, smem, s>>>(map, a);
    note_launch(s);
    return cudaGetLastError();
}

template <typename T, bool kBig>
static cudaError_t launch_pipe_g(int G, const CUtensorMap& map, const PipeArgs& a, int n_ctas,
                                 cudaStream_t s) {
    switch (G) {
        case 1: return launch_pipe_t<T, 1, kBig>(map, a, n_ctas, s);
        case 2: return launch_pipe_t<T, 2, kBig>(map, a, n_ctas, s);
        case 3: return launch_pipe_t<T, 3, kBig>(map, a, n_ctas, s);
        case 4: return launch_pipe_t<T, 4, kBig>(map, a, n_ctas, s);
        case 5: return launch_pipe_t<T, 5, kBig>(map, a, n_ctas, s);
        case 6: return launch_pipe_t<T, 6, kBig>(map, a, n_ctas, s);
        case 7: return launch_pipe_t<T, 7, kBig>(map, a, n_ctas, s);
        case 8: return launch_pipe_t<T, 8, kBig>(map, a, n_ctas, s);
    }
    return cudaErrorInvalidValue;
}

cudaError_t launch_pipe(tri_dtype dt, int G, bool big, const CUtensorMap& map, const PipeArgs& a,
                        int n_ctas, cudaStream_t s) {
    if (dt == TRI_BF16)
        return big ? launch_pipe_g<__nv_bfloat16, true>(G, map, a, n_ctas, s)
                   : launch_pipe_g<__nv_bfloat16, false>(G, map, a, n_ctas, s);
    return big ? launch_pipe_g<float, true>(G, map, a, n_ctas, s)
               : launch_pipe_g<float, false>(G, map, a, n_ctas, s);
}

}  // namespace tri
