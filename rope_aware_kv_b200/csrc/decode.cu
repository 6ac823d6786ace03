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
// Split-K over the keys when units are few: CTA (c, u) handles the keys
// [c * chunk, (c + 1) * chunk) of unit u in tiles of 256 keys with an online
// softmax (running maximum and sum per head, accumulators rescaled when the
// maximum grows), then either writes o_h (one chunk per unit) or its
// (maximum, sum, unnormalised accumulator) for a combine kernel that merges
// the chunks in order.
//   scores  thread t scores key t of the tile for every head (its 256-byte
//           row through 16-byte loads, the G queries from shared memory);
//   values  thread t owns dims 2 (t % 64) and 2 (t % 64) + 1 for the keys
//           t / 64, t / 64 + 4, ... of the tile (4-byte coalesced loads of V),
//           the 4 key lanes summed through shared memory at the end.
#include "tri_internal.cuh"
#include "tri_launch.h"

namespace tri {

constexpr int kDecThreads = 256;
constexpr int kDecTile = 256;  // keys per tile (one per thread in the score phase)

struct DecodeArgs {
    const void* q;       // [U][G][128]
    const void* k;       // [U][cap][128]
    const void* v;
    int64_t cap;
    const int32_t* n_valid;
    float scale;
    int64_t chunk;       // keys per CTA (a multiple of kDecTile)
    int splits;          // CTAs per unit
    float* out;          // [U][G][128]
    float* part;         // [U][splits][G][2 + 128] when splits > 1
    uint32_t* flag;
};

template <typename T>
__device__ __forceinline__ float2 load_pair(const T* row, int i) {
    if constexpr (sizeof(T) == 2) {
        const uint32_t w = __ldg(reinterpret_cast<const uint32_t*>(row) + i);
        return make_float2(bf16_lo(w), bf16_hi(w));
    } else {
        return __ldg(reinterpret_cast<const float2*>(row) + i);
    }
}

template <typename T, int G>
__global__ void __launch_bounds__(kDecThreads)
decode_attn_kernel(const DecodeArgs a) {
    __shared__ float4 qs[G][kD / 4];          // scale * log2(e) * q
    __shared__ float sc[G][kDecTile];         // tile scores, then weights
    __shared__ float mrow[G], lrow[G], alpha[G];
    __shared__ float2 red[4][G][64];          // key-lane partials of the outputs
    const int t = threadIdx.x;
    const int64_t u = blockIdx.y;
    const int c = blockIdx.x;
    const int n = clamp_nvalid(a.n_valid, u, a.cap, c == 0 && t == 0 ? a.flag : nullptr);
    const int64_t j0 = static_cast<int64_t>(c) * a.chunk;
    const int64_t j1 = min(j0 + a.chunk, static_cast<int64_t>(n));
    constexpr float kLog2e = 1.4426950408889634f;
    const T* qu = static_cast<const T*>(a.q) + u * G * kD;
    for (int e = t; e < G * kD; e += kDecThreads) {
        const float x = to_float(qu[e]) * a.scale * kLog2e;
        reinterpret_cast<float*>(qs)[e] = x;
    }
    if (t < G) {
        mrow[t] = -INFINITY;
        lrow[t] = 0.f;
    }
    const int dp = t & 63;   // dims 2 dp, 2 dp + 1
    const int kl = t >> 6;   // key lane 0..3
    float2 acc[G];
#pragma unroll
    for (int h = 0; h < G; ++h) acc[h] = make_float2(0.f, 0.f);
    __syncthreads();
    const T* ku = static_cast<const T*>(a.k) + u * a.cap * kD;
    const T* vu = static_cast<const T*>(a.v) + u * a.cap * kD;
    constexpr int64_t kRowBytes = kD * sizeof(T);
    if (t == 0 && j1 > j0) {
        // The first tile's values into L2 while its keys are scored.
        const int64_t r = min(static_cast<int64_t>(kDecTile), j1 - j0);
        prefetch_l2_bulk(vu + j0 * kD, static_cast<uint32_t>(r * kRowBytes), policy_evict_first());
    }
    for (int64_t b = j0; b < j1; b += kDecTile) {
        const int nt = static_cast<int>(min(static_cast<int64_t>(kDecTile), j1 - b));
        if (t == 0 && b + kDecTile < j1) {
            // The next tile's keys and values into L2 while this one is used.
            const int64_t r = min(static_cast<int64_t>(kDecTile), j1 - b - kDecTile);
            const uint64_t pol = policy_evict_first();
            prefetch_l2_bulk(ku + (b + kDecTile) * kD, static_cast<uint32_t>(r * kRowBytes), pol);
            prefetch_l2_bulk(vu + (b + kDecTile) * kD, static_cast<uint32_t>(r * kRowBytes), pol);
        }
        // ---- scores (log2 domain) of key b + t for every head ----
        if (t < nt) {
            const T* row = ku + (b + t) * kD;
            float s[G];
#pragma unroll
            for (int h = 0; h < G; ++h) s[h] = 0.f;
            if constexpr (sizeof(T) == 2) {
                // 16 x 16-byte loads: 8 bf16 components each.
#pragma unroll 4
                for (int i = 0; i < kD / 8; ++i) {
                    const uint4 w = __ldg(reinterpret_cast<const uint4*>(row) + i);
                    const float4 xa = make_float4(bf16_lo(w.x), bf16_hi(w.x), bf16_lo(w.y), bf16_hi(w.y));
                    const float4 xb = make_float4(bf16_lo(w.z), bf16_hi(w.z), bf16_lo(w.w), bf16_hi(w.w));
#pragma unroll
                    for (int h = 0; h < G; ++h) {
                        const float4 qa = qs[h][2 * i], qb = qs[h][2 * i + 1];
                        float r = s[h];
                        r = fmaf(qa.x, xa.x, r);
                        r = fmaf(qa.y, xa.y, r);
                        r = fmaf(qa.z, xa.z, r);
                        r = fmaf(qa.w, xa.w, r);
                        r = fmaf(qb.x, xb.x, r);
                        r = fmaf(qb.y, xb.y, r);
                        r = fmaf(qb.z, xb.z, r);
                        r = fmaf(qb.w, xb.w, r);
                        s[h] = r;
                    }
                }
            } else {
#pragma unroll 4
                for (int i = 0; i < kD / 4; ++i) {
                    const float4 x = __ldg(reinterpret_cast<const float4*>(row) + i);
#pragma unroll
                    for (int h = 0; h < G; ++h) {
                        const float4 qv = qs[h][i];
                        float r = s[h];
                        r = fmaf(qv.x, x.x, r);
                        r = fmaf(qv.y, x.y, r);
                        r = fmaf(qv.z, x.z, r);
                        r = fmaf(qv.w, x.w, r);
                        s[h] = r;
                    }
                }
            }
#pragma unroll
            for (int h = 0; h < G; ++h) sc[h][t] = s[h];
        }
        __syncthreads();
        // ---- tile maximum per head (warp h), new running maximum ----
        const int warp = t >> 5, lane = t & 31;
        for (int h = warp; h < G; h += kDecThreads / 32) {
            float mx = -INFINITY;
            for (int i = lane; i < nt; i += 32) mx = fmaxf(mx, sc[h][i]);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
            const float m_old = mrow[h];
            const float m_new = fmaxf(m_old, mx);
            float sum = 0.f;
            for (int i = lane; i < nt; i += 32) {
                const float p = exp2f(sc[h][i] - m_new);
                sc[h][i] = p;
                sum += p;
            }
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
        // ---- accumulate the weighted values ----
#pragma unroll
        for (int h = 0; h < G; ++h) {
            const float al = alpha[h];
            acc[h].x *= al;
            acc[h].y *= al;
        }
        for (int i = kl; i < nt; i += 4) {
            const float2 vv = load_pair(vu + (b + i) * kD, dp);
#pragma unroll
            for (int h = 0; h < G; ++h) {
                const float p = sc[h][i];
                acc[h].x = fmaf(p, vv.x, acc[h].x);
                acc[h].y = fmaf(p, vv.y, acc[h].y);
            }
        }
        __syncthreads();  // sc is rewritten by the next tile
    }
    // ---- the 4 key lanes in a fixed order ----
#pragma unroll
    for (int h = 0; h < G; ++h) red[kl][h][dp] = acc[h];
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
    const int64_t tiles = (cap + kDecTile - 1) / kDecTile;
    int64_t s = (2LL * n_sm + n_units - 1) / n_units;
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
    switch (G) {
#define TRI_DCASE(g) \
    case g: decode_attn_kernel<T, g><<<grid, kDecThreads, 0, s>>>(a); break;
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
    const int64_t tiles = (cap + kDecTile - 1) / kDecTile;
    a.chunk = ((tiles + a.splits - 1) / a.splits) * kDecTile;
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
