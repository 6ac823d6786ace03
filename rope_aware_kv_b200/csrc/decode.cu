// decode.cu -- attention of the next token over the compacted cache.
//
// For each unit (sequence, layer, KV head) and each of its G query heads h:
//   o_h = sum_{j < n} a_j v_j,  a_j = exp(s_j - m) / sum_{j' < n} exp(s_j' - m),
//   s_j = scale * (q_h . k_j),  m = max_j s_j,
// the softmax renormalised over the kept rows (jaedaily.cn tutorial,
// KV-compression objective: the output over the kept subset S uses the
// weights renormalised over S).  This is the consumer of what the prune step
// keeps; K and V rows are read once each, so the kernel is bound by HBM.
//
// One CTA per SM (per unit, or per chunk of a unit's keys when units are
// fewer than SMs), 256 threads.  Tiles of 32 KB of keys and 32 KB of values
// (128 bf16 / 64 float32 rows) are staged in shared memory by bulk copies
// (one for the keys, one for the values, completing on the stage's
// mbarrier), three tiles in flight, so HBM streams while the CTA computes:
//   scores  2 (bf16) or 4 (float32) threads per key, each 8 of its 16-byte
//           chunks in an order rotated by thread (conflict-free shared
//           loads), dims paired into packed FFMA2 products against the
//           queries (pre-scaled by scale * log2 e), partial sums combined by
//           shuffles;
//   softmax one warp per head: the tile's maximum, the running maximum and
//           sum, the accumulators' rescale factor (an online softmax);
//   values  thread t owns dims 2 (t % 64) and 2 (t % 64) + 1 of the keys of
//           block t / 64 (a quarter of the tile): 4-byte shared loads, the
//           weights of 4 keys in one 16-byte load, packed FFMA2 per key and
//           head; the 4 blocks are summed through shared memory at the end.
// A unit split over several CTAs writes per-chunk (maximum, sum,
// unnormalised output) that decode_combine_kernel merges in chunk order.
#include "tri_internal.cuh"
#include "tri_launch.h"

namespace tri {

constexpr int kDecThreads = 256;

struct DecodeArgs {
    const void* q;       // [U][G][128]
    const void* k;       // [U][cap][128]
    const void* v;
    int64_t cap;
    const int32_t* n_valid;
    float scale;
    int64_t chunk;       // keys per CTA (a multiple of the tile)
    int splits;          // CTAs per unit
    float* out;          // [U][G][128]
    float* part;         // [U][splits][G][2 + 128] when splits > 1
    uint32_t* flag;
};

// Shape of the staged tiles: 32 KB of keys and 32 KB of values per tile (128
// bf16 or 64 float32 rows), three tiles in flight.
template <typename T>
struct DecShape {
    static constexpr int kRowBytes = kD * static_cast<int>(sizeof(T));
    static constexpr int kTileBytes = 32768;
    static constexpr int kTile = kTileBytes / kRowBytes;          // keys per tile
    static constexpr int kStages = 3;
    static constexpr int kTpk = kDecThreads / kTile;               // threads per key (2 / 4)
    static constexpr int kChunks = kRowBytes / 16 / kTpk;          // 16-byte chunks per thread
    static constexpr int kBlk = kTile / 4;                         // keys per value block
    static constexpr size_t kSmem = static_cast<size_t>(kStages) * 2 * kTileBytes + 1024;
    static_assert(kChunks == 8, "chunk swizzle assumes 8 chunks per thread");
};

template <typename T, int G>
__global__ void __launch_bounds__(kDecThreads, 1)
decode_attn_kernel(const DecodeArgs a) {
    using S = DecShape<T>;
    extern __shared__ uint8_t dsm_raw[];
    uint8_t* stage0 = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(dsm_raw) + 1023) & ~uintptr_t(1023));
    __shared__ float4 qs[G][kD / 4];                 // scale * log2(e) * q
    __shared__ __align__(16) float sc[G][S::kTile];  // tile scores, then weights
    __shared__ float mrow[G], lrow[G], alpha[G];
    __shared__ float2 red[4][G][64];                 // key-block partials of the outputs
    __shared__ uint64_t full[S::kStages];
    __shared__ int abort_s;
    const int t = threadIdx.x;
    const int64_t u = blockIdx.y;
    const int c = blockIdx.x;
    const int n = clamp_nvalid(a.n_valid, u, a.cap, c == 0 && t == 0 ? a.flag : nullptr);
    const int64_t j0 = static_cast<int64_t>(c) * a.chunk;
    const int64_t j1 = min(j0 + a.chunk, static_cast<int64_t>(n));
    const int ntiles = j1 > j0 ? static_cast<int>((j1 - j0 + S::kTile - 1) / S::kTile) : 0;
    constexpr float kLog2e = 1.4426950408889634f;
    const T* qu = static_cast<const T*>(a.q) + u * G * kD;
    const char* ku = static_cast<const char*>(a.k) + u * a.cap * S::kRowBytes;
    const char* vu = static_cast<const char*>(a.v) + u * a.cap * S::kRowBytes;
    const uint64_t pol = policy_evict_first();
    // Tile i of this CTA into stage i % kStages: K rows, then V rows, one
    // bulk copy each, both completing on the stage's barrier.
    auto issue = [&](int i) {
        const int64_t b = j0 + static_cast<int64_t>(i) * S::kTile;
        const uint32_t rows = static_cast<uint32_t>(min(static_cast<int64_t>(S::kTile), j1 - b));
        const uint32_t bytes = rows * S::kRowBytes;
        uint8_t* st = stage0 + static_cast<size_t>(i % S::kStages) * 2 * S::kTileBytes;
        uint64_t* bar = &full[i % S::kStages];
        mbar_arrive_expect_tx(bar, 2 * bytes);
        bulk_load_hint(st, ku + b * S::kRowBytes, bytes, bar, pol);
        bulk_load_hint(st + S::kTileBytes, vu + b * S::kRowBytes, bytes, bar, pol);
    };
    if (t == 0) {
        for (int i = 0; i < S::kStages; ++i) mbar_init(&full[i], 1);
        fence_barrier_init();
        abort_s = 0;
        for (int i = 0; i < S::kStages && i < ntiles; ++i) issue(i);
    }
    for (int e = t; e < G * kD; e += kDecThreads)
        reinterpret_cast<float*>(qs)[e] = to_float(qu[e]) * a.scale * kLog2e;
    if (t < G) {
        mrow[t] = -INFINITY;
        lrow[t] = 0.f;
    }
    const int dp = t & 63;   // dims 2 dp, 2 dp + 1 in the value phase
    const int kb = t >> 6;   // value block: keys [kb * kBlk, (kb + 1) * kBlk) of a tile
    const int kk = t / S::kTpk;         // key of the score phase
    const int part = t % S::kTpk;       // its part of the row (kChunks chunks)
    const int sw = t & 7;               // chunk order: conflict-free 16-byte loads
    float2 acc[G];
#pragma unroll
    for (int h = 0; h < G; ++h) acc[h] = make_float2(0.f, 0.f);
    __syncthreads();
    for (int i = 0; i < ntiles; ++i) {
        const int64_t b = j0 + static_cast<int64_t>(i) * S::kTile;
        const int nt = static_cast<int>(min(static_cast<int64_t>(S::kTile), j1 - b));
        const uint8_t* kt = stage0 + static_cast<size_t>(i % S::kStages) * 2 * S::kTileBytes;
        const uint8_t* vt = kt + S::kTileBytes;
        const bool ok = mbar_wait(&full[i % S::kStages], (i / S::kStages) & 1, a.flag);
        if (__syncthreads_or(!ok)) {
            if (t == 0) abort_s = 1;
            break;
        }
        // ---- scores (log2 domain): S::kTpk threads per key ----
        {
            float2 a2[G];
#pragma unroll
            for (int h = 0; h < G; ++h) a2[h] = make_float2(0.f, 0.f);
            const uint8_t* row = kt + kk * S::kRowBytes;
#pragma unroll
            for (int cc = 0; cc < S::kChunks; ++cc) {
                const int ch = part * S::kChunks + (cc ^ sw);
                const uint4 w = *reinterpret_cast<const uint4*>(row + ch * 16);
                if constexpr (sizeof(T) == 2) {
                    const float2 k2[4] = {make_float2(bf16_lo(w.x), bf16_hi(w.x)),
                                          make_float2(bf16_lo(w.y), bf16_hi(w.y)),
                                          make_float2(bf16_lo(w.z), bf16_hi(w.z)),
                                          make_float2(bf16_lo(w.w), bf16_hi(w.w))};
#pragma unroll
                    for (int h = 0; h < G; ++h) {
                        const float4 qa = qs[h][2 * ch], qb = qs[h][2 * ch + 1];
                        a2[h] = __ffma2_rn(k2[0], make_float2(qa.x, qa.y), a2[h]);
                        a2[h] = __ffma2_rn(k2[1], make_float2(qa.z, qa.w), a2[h]);
                        a2[h] = __ffma2_rn(k2[2], make_float2(qb.x, qb.y), a2[h]);
                        a2[h] = __ffma2_rn(k2[3], make_float2(qb.z, qb.w), a2[h]);
                    }
                } else {
                    const float4 x = make_float4(__uint_as_float(w.x), __uint_as_float(w.y),
                                                 __uint_as_float(w.z), __uint_as_float(w.w));
#pragma unroll
                    for (int h = 0; h < G; ++h) {
                        const float4 qv = qs[h][ch];
                        a2[h] = __ffma2_rn(make_float2(x.x, x.y), make_float2(qv.x, qv.y), a2[h]);
                        a2[h] = __ffma2_rn(make_float2(x.z, x.w), make_float2(qv.z, qv.w), a2[h]);
                    }
                }
            }
#pragma unroll
            for (int h = 0; h < G; ++h) {
                float sv = a2[h].x + a2[h].y;
#pragma unroll
                for (int o = 1; o < S::kTpk; o <<= 1) sv += __shfl_xor_sync(0xffffffffu, sv, o);
                if (part == 0 && kk < nt) sc[h][kk] = sv;
            }
        }
        __syncthreads();
        // ---- tile maximum per head (warp h), new running maximum ----
        const int warp = t >> 5, lane = t & 31;
        for (int h = warp; h < G; h += kDecThreads / 32) {
            float mx = -INFINITY;
            for (int k = lane; k < nt; k += 32) mx = fmaxf(mx, sc[h][k]);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
            const float m_old = mrow[h];
            const float m_new = fmaxf(m_old, mx);
            float sum = 0.f;
            for (int k = lane; k < nt; k += 32) {
                const float p = exp2f(sc[h][k] - m_new);
                sc[h][k] = p;
                sum += p;
            }
            for (int k = nt + lane; k < ((nt + 3) & ~3); k += 32) sc[h][k] = 0.f;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
            if (lane == 0) {
                const float al = exp2f(m_old - m_new);  // 0 when m_old is -inf
                alpha[h] = al;
                lrow[h] = lrow[h] * al + sum;
                mrow[h] = m_new;
            }
        }
        __syncthreads();
        // ---- weighted values of this thread's key block, from shared memory ----
#pragma unroll
        for (int h = 0; h < G; ++h) {
            const float al = alpha[h];
            acc[h].x *= al;
            acc[h].y *= al;
        }
        const int k0 = kb * S::kBlk;
        const int k1 = min(k0 + S::kBlk, nt);
        for (int k = k0; k < k1; k += 4) {
            float2 vv[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const uint8_t* vr = vt + (k + q) * S::kRowBytes;
                if (k + q >= k1) {
                    vv[q] = make_float2(0.f, 0.f);
                } else if constexpr (sizeof(T) == 2) {
                    const uint32_t wv = *reinterpret_cast<const uint32_t*>(vr + dp * 4);
                    vv[q] = make_float2(bf16_lo(wv), bf16_hi(wv));
                } else {
                    vv[q] = *reinterpret_cast<const float2*>(vr + dp * 8);
                }
            }
#pragma unroll
            for (int h = 0; h < G; ++h) {
                const float4 p = *reinterpret_cast<const float4*>(&sc[h][k]);
                acc[h] = __ffma2_rn(make_float2(p.x, p.x), vv[0], acc[h]);
                acc[h] = __ffma2_rn(make_float2(p.y, p.y), vv[1], acc[h]);
                acc[h] = __ffma2_rn(make_float2(p.z, p.z), vv[2], acc[h]);
                acc[h] = __ffma2_rn(make_float2(p.w, p.w), vv[3], acc[h]);
            }
        }
        __syncthreads();  // the stage and sc are free again
        if (t == 0 && i + S::kStages < ntiles) {
            fence_proxy_async();  // generic reads of the stage before the copy overwrites it
            issue(i + S::kStages);
        }
    }
    __syncthreads();
    if (abort_s) {
        // Copies still in flight into the stages: give them time to land.
        if (t == 0) {
            const uint64_t t0 = globaltimer_ns();
            while (globaltimer_ns() - t0 < 200000) __nanosleep(1000);
        }
        __syncthreads();
        return;
    }
    // ---- the 4 key blocks in a fixed order ----
#pragma unroll
    for (int h = 0; h < G; ++h) red[kb][h][dp] = acc[h];
    __syncthreads();
    for (int e = t; e < G * 64; e += kDecThreads) {
        const int h = e / 64, d2 = e % 64;
        float2 o = red[0][h][d2];
#pragma unroll
        for (int l = 1; l < 4; ++l) {
            o.x += red[l][h][d2].x;
            o.y += red[l][h][d2].y;
        }
        if (a.splits == 1) {
            const float l = lrow[h];
            const float inv = l > 0.f ? 1.f / l : 0.f;
            reinterpret_cast<float2*>(a.out + (u * G + h) * kD)[d2] = make_float2(o.x * inv, o.y * inv);
        } else {
            float* p = a.part + ((u * a.splits + c) * G + h) * (2 + kD);
            reinterpret_cast<float2*>(p + 2)[d2] = o;
            if (d2 == 0) {
                p[0] = mrow[h];
                p[1] = lrow[h];
            }
        }
    }
}

// Merge the chunks of each (unit, head) in chunk order: o = sum_c 2^(m_c - M)
// acc_c / sum_c 2^(m_c - M) l_c.  grid U * G, 128 threads (one per dim).
__global__ void __launch_bounds__(kD)
decode_combine_kernel(const float* __restrict__ part, int splits, int G, float* __restrict__ out) {
    const int64_t uh = blockIdx.x;
    const int64_t u = uh / G, h = uh % G;
    const int d = threadIdx.x;
    float M = -INFINITY;
    for (int c = 0; c < splits; ++c) M = fmaxf(M, part[((u * splits + c) * G + h) * (2 + kD)]);
    float num = 0.f, den = 0.f;
    for (int c = 0; c < splits; ++c) {
        const float* p = part + ((u * splits + c) * G + h) * (2 + kD);
        const float w = p[1] > 0.f ? exp2f(p[0] - M) : 0.f;
        num = fmaf(w, p[2 + d], num);
        den = fmaf(w, p[1], den);
    }
    out[uh * kD + d] = den > 0.f ? num / den : 0.f;
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
int decode_splits(int64_t n_units, int64_t cap, int n_sm) {
    // One CTA per SM (the staged tiles fill its shared memory): split units
    // over several CTAs only when there are fewer units than SMs.
    const int64_t tiles = (cap + DecShape<__nv_bfloat16>::kTile - 1) / DecShape<__nv_bfloat16>::kTile;
    int64_t s = (static_cast<int64_t>(n_sm) + n_units - 1) / n_units;
    if (s > tiles) s = tiles;
    if (s < 1) s = 1;
    if (s > 1024) s = 1024;
    return static_cast<int>(s);
}

size_t decode_part_bytes(int64_t n_units, int G, int64_t cap, int n_sm) {
    const int s = decode_splits(n_units, cap, n_sm);
    return s > 1 ? static_cast<size_t>(n_units * s * G) * (2 + kD) * sizeof(float) : 0;
}

template <typename T>
static cudaError_t launch_decode_t(int G, const DecodeArgs& a, int64_t n_units, cudaStream_t s) {
    dim3 grid(static_cast<unsigned>(a.splits), static_cast<unsigned>(n_units));
    const size_t smem = DecShape<T>::kSmem;
    switch (G) {
#define TRI_DCASE(g)                                                                        \
    case g: {                                                                               \
        cudaError_t e = cudaFuncSetAttribute(decode_attn_kernel<T, g>,                      \
                                             cudaFuncAttributeMaxDynamicSharedMemorySize,   \
                                             static_cast<int>(smem));                       \
        if (e != cudaSuccess) return e;                                                     \
        decode_attn_kernel<T, g><<<grid, kDecThreads, smem, s>>>(a);                        \
        break;                                                                              \
    }
        TRI_DCASE(1) TRI_DCASE(2) TRI_DCASE(3) TRI_DCASE(4)
        TRI_DCASE(5) TRI_DCASE(6) TRI_DCASE(7) TRI_DCASE(8)
#undef TRI_DCASE
        default: return cudaErrorInvalidValue;
    }
    note_launch(s);
    return cudaGetLastError();
}

cudaError_t launch_decode(tri_dtype dt, int G, const void* q, const void* k, const void* v,
                          int64_t n_units, int64_t cap, const int32_t* n_valid, float scale,
                          float* out, float* part, uint32_t* flag, int n_sm, cudaStream_t s) {
    DecodeArgs a;
    a.q = q;
    a.k = k;
    a.v = v;
    a.cap = cap;
    a.n_valid = n_valid;
    a.scale = scale;
    a.splits = decode_splits(n_units, cap, n_sm);
    const int64_t tile = dt == TRI_BF16 ? DecShape<__nv_bfloat16>::kTile : DecShape<float>::kTile;
    const int64_t tiles = (cap + tile - 1) / tile;
    a.chunk = ((tiles + a.splits - 1) / a.splits) * tile;
    a.out = out;
    a.part = part;
    a.flag = flag;
    cudaError_t e = dt == TRI_BF16 ? launch_decode_t<__nv_bfloat16>(G, a, n_units, s)
                                   : launch_decode_t<float>(G, a, n_units, s);
    if (e != cudaSuccess || a.splits == 1) return e;
    decode_combine_kernel<<<static_cast<unsigned>(n_units * G), kD, 0, s>>>(part, a.splits, G, out);
    note_launch(s);
    return cudaGetLastError();
}

}  // namespace tri
