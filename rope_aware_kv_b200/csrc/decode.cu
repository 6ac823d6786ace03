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
//   scores  thread t scores keys t and t + 256 of a 512-key tile for every
//           head (their rows through 16-byte loads, the G queries from
//           shared memory), dims paired into packed FFMA2 products;
//   values  thread t owns dims 2 (t % 64) and 2 (t % 64) + 1 of the keys of
//           block t / 64 (128 consecutive keys of the tile): 4-byte loads,
//           coalesced over the 64 threads of a block, the weights of 4 keys
//           in one 16-byte shared load, packed FFMA2 per key and head; the 4
//           blocks are summed through shared memory at the end.
#include "tri_internal.cuh"
#include "tri_launch.h"

namespace tri {

constexpr int kDecThreads = 256;
constexpr int kDecTile = 512;  // keys per tile (two per thread in the score phase)

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

// Score of two keys (rows r0, r1) for every head, packed: the key's dims
// (2j, 2j + 1) as one float2 against the query's, accumulated with FFMA2
// into (even-dim, odd-dim) partial sums.
template <typename T, int G>
__device__ __forceinline__ void score_two(const T* r0, const T* r1, bool has1,
                                          const float4 (&qs)[G][kD / 4], float (&s0)[G],
                                          float (&s1)[G]) {
    float2 a0[G], a1[G];
#pragma unroll
    for (int h = 0; h < G; ++h) a0[h] = a1[h] = make_float2(0.f, 0.f);
    if constexpr (sizeof(T) == 2) {
#pragma unroll 2
        for (int i = 0; i < kD / 8; ++i) {  // 16-byte chunk i: dims 8i .. 8i + 7
            const uint4 w0 = __ldg(reinterpret_cast<const uint4*>(r0) + i);
            const uint4 w1 = has1 ? __ldg(reinterpret_cast<const uint4*>(r1) + i) : w0;
            const float2 k0[4] = {make_float2(bf16_lo(w0.x), bf16_hi(w0.x)),
                                  make_float2(bf16_lo(w0.y), bf16_hi(w0.y)),
                                  make_float2(bf16_lo(w0.z), bf16_hi(w0.z)),
                                  make_float2(bf16_lo(w0.w), bf16_hi(w0.w))};
            const float2 k1[4] = {make_float2(bf16_lo(w1.x), bf16_hi(w1.x)),
                                  make_float2(bf16_lo(w1.y), bf16_hi(w1.y)),
                                  make_float2(bf16_lo(w1.z), bf16_hi(w1.z)),
                                  make_float2(bf16_lo(w1.w), bf16_hi(w1.w))};
#pragma unroll
            for (int h = 0; h < G; ++h) {
                const float4 qa = qs[h][2 * i], qb = qs[h][2 * i + 1];
                const float2 q[4] = {make_float2(qa.x, qa.y), make_float2(qa.z, qa.w),
                                     make_float2(qb.x, qb.y), make_float2(qb.z, qb.w)};
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    a0[h] = __ffma2_rn(k0[j], q[j], a0[h]);
                    a1[h] = __ffma2_rn(k1[j], q[j], a1[h]);
                }
            }
        }
    } else {
#pragma unroll 2
        for (int i = 0; i < kD / 4; ++i) {  // dims 4i .. 4i + 3
            const float4 x0 = __ldg(reinterpret_cast<const float4*>(r0) + i);
            const float4 x1 = has1 ? __ldg(reinterpret_cast<const float4*>(r1) + i) : x0;
#pragma unroll
            for (int h = 0; h < G; ++h) {
                const float4 qv = qs[h][i];
                a0[h] = __ffma2_rn(make_float2(x0.x, x0.y), make_float2(qv.x, qv.y), a0[h]);
                a0[h] = __ffma2_rn(make_float2(x0.z, x0.w), make_float2(qv.z, qv.w), a0[h]);
                a1[h] = __ffma2_rn(make_float2(x1.x, x1.y), make_float2(qv.x, qv.y), a1[h]);
                a1[h] = __ffma2_rn(make_float2(x1.z, x1.w), make_float2(qv.z, qv.w), a1[h]);
            }
        }
    }
#pragma unroll
    for (int h = 0; h < G; ++h) {
        s0[h] = a0[h].x + a0[h].y;
        s1[h] = a1[h].x + a1[h].y;
    }
}

template <typename T, int G>
__global__ void __launch_bounds__(kDecThreads, 3)
decode_attn_kernel(const DecodeArgs a) {
    __shared__ float4 qs[G][kD / 4];          // scale * log2(e) * q
    __shared__ __align__(16) float sc[G][kDecTile];  // tile scores, then weights
    __shared__ float mrow[G], lrow[G], alpha[G];
    __shared__ float2 red[4][G][64];          // key-block partials of the outputs
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
    const int kb = t >> 6;   // key block 0..3: keys [kb * kBlk, (kb + 1) * kBlk) of a tile
    constexpr int kBlk = kDecTile / 4;
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
        // ---- scores (log2 domain) of keys b + t and b + t + 256 ----
        if (t < nt) {
            const bool has1 = t + kDecThreads < nt;
            float s0[G], s1[G];
            score_two<T, G>(ku + (b + t) * kD, ku + (b + t + (has1 ? kDecThreads : 0)) * kD, has1,
                            qs, s0, s1);
#pragma unroll
            for (int h = 0; h < G; ++h) {
                sc[h][t] = s0[h];
                if (has1) sc[h][t + kDecThreads] = s1[h];
            }
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
            // Weights past the tile's keys are zero (the value phase reads
            // whole groups of 4).
            for (int i = nt + lane; i < ((nt + 3) & ~3); i += 32) sc[h][i] = 0.f;
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
        // ---- accumulate the weighted values: this thread's key block ----
#pragma unroll
        for (int h = 0; h < G; ++h) {
            const float al = alpha[h];
            acc[h].x *= al;
            acc[h].y *= al;
        }
        const int i0 = kb * kBlk;
        const int i1 = min(i0 + kBlk, nt);
        for (int i = i0; i < i1; i += 4) {
            float2 vv[4];
#pragma unroll
            for (int q = 0; q < 4; ++q)
                vv[q] = i + q < i1 ? load_pair(vu + (b + i + q) * kD, dp) : make_float2(0.f, 0.f);
#pragma unroll
            for (int h = 0; h < G; ++h) {
                const float4 p = *reinterpret_cast<const float4*>(&sc[h][i]);
                acc[h] = __ffma2_rn(make_float2(p.x, p.x), vv[0], acc[h]);
                acc[h] = __ffma2_rn(make_float2(p.y, p.y), vv[1], acc[h]);
                acc[h] = __ffma2_rn(make_float2(p.z, p.z), vv[2], acc[h]);
                acc[h] = __ffma2_rn(make_float2(p.w, p.w), vv[3], acc[h]);
            }
        }
        __syncthreads();  // sc is rewritten by the next tile
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
