// score_core.cuh -- per-key score arithmetic on a shared-memory key tile.
//
// For key k' (post-RoPE) and query head h the folded score is
//   s_h = sum_f (ReA_hf * x_f + ImA_hf * y_f) + sum_f c_hf * |k'_f|
// with k'_f = x_f + i y_f the interleaved pair (x_2f, x_2f+1), A_hf the
// offset-averaged rotated query centre and c_hf = (1 - R_hf) E|q_hf| (see
// score.cu).  Products are formed with packed float32x2 FMAs on band pairs:
// (x_i, x_i+1) against (ReA_i, ReA_i+1), (y_i, y_i+1) against (ImA_i,
// ImA_i+1), and the pair's norms against (c_i, c_i+1); the squared norms of a
// pair are one packed multiply and one packed FMA of the same registers.
#pragma once

#include "tri_internal.cuh"

// Unroll factor of the 16-chunk loop: full unrolling lets the compiler hoist
// shared-memory loads, partial unrolling keeps the instruction footprint small.
#ifndef TRI_SCORE_UNROLL
#define TRI_SCORE_UNROLL 4
#endif

namespace tri {

constexpr int kScoreUnroll = TRI_SCORE_UNROLL;

// One 16-byte chunk of a bf16 row (bands i..i+3, words (x_i, y_i) with x in
// the low half) as register pairs xy = {(x_i, x_i+1), (y_i, y_i+1),
// (x_i+2, x_i+3), (y_i+2, y_i+3)} and the band norms nn = {(|k_i|, |k_i+1|),
// (|k_i+2|, |k_i+3|)}.
__device__ __forceinline__ void band_pairs_bf16(const uint4 v, float2 (&xy)[4], float2 (&nn)[2]) {
    xy[0] = make_float2(bf16_lo(v.x), bf16_lo(v.y));
    xy[1] = make_float2(bf16_hi(v.x), bf16_hi(v.y));
    xy[2] = make_float2(bf16_lo(v.z), bf16_lo(v.w));
    xy[3] = make_float2(bf16_hi(v.z), bf16_hi(v.w));
    const float2 q01 = __ffma2_rn(xy[1], xy[1], __fmul2_rn(xy[0], xy[0]));
    const float2 q23 = __ffma2_rn(xy[3], xy[3], __fmul2_rn(xy[2], xy[2]));
    nn[0] = make_float2(sqrt_approx(q01.x), sqrt_approx(q01.y));
    nn[1] = make_float2(sqrt_approx(q23.x), sqrt_approx(q23.y));
}

// The same for a 16-byte chunk of a float32 row (bands i, i+1: x_i, y_i,
// x_i+1, y_i+1): xy = {(x_i, x_i+1), (y_i, y_i+1)}, nn = (|k_i|, |k_i+1|).
__device__ __forceinline__ void band_pair_f32(const float4 v, float2 (&xy)[2], float2& nn) {
    xy[0] = make_float2(v.x, v.z);
    xy[1] = make_float2(v.y, v.w);
    const float2 q = __ffma2_rn(xy[1], xy[1], __fmul2_rn(xy[0], xy[0]));
    nn = make_float2(sqrt_approx(q.x), sqrt_approx(q.y));
}

// Chunks (16 bytes: 4 bf16 bands or 2 float32 bands) per key row.
template <typename T>
__host__ __device__ constexpr int row_chunks() { return sizeof(T) == 2 ? kChunks : 2 * kChunks; }

// Accumulate chunks [c0, c1) of KPT keys into acc.  The keys live in
// swizzled shared memory as 128-byte TMA boxes: chunk c of row r is at
// boxes + ((c >> 3) - (c0 >> 3)) * kBoxBytes + r * 128 + (((c & 7) ^ (r & 7)) << 4)
// (TMA 128-byte swizzle: 8 consecutive threads reading the same logical
// chunk of 8 consecutive rows hit 8 different bank groups), so `boxes` may
// hold the whole tile (c0 = 0) or only the boxes from c0 on.  Rows
// first_row + kRowStride * k (k < KPT); w points at the weight record of the
// first of the G heads scored here.  Scoring a tile in parts accumulates in
// the same order as scoring it whole.
template <typename T, int G, int KPT, int kBoxBytes, int kRowStride>
__device__ __forceinline__ void score_rows_acc(const uint8_t* boxes, int c0, int c1, const float* w,
                                               int first_row, float2 (&acc)[KPT][G]) {
    const int box0 = c0 >> 3;
    if constexpr (sizeof(T) == 2) {
#pragma unroll kScoreUnroll
        for (int c = c0; c < c1; ++c) {
            float2 xy[KPT][4];
            float2 nn[KPT][2];
#pragma unroll
            for (int k = 0; k < KPT; ++k) {
                const int r = first_row + kRowStride * k;
                const uint4 v = *reinterpret_cast<const uint4*>(
                    boxes + ((c >> 3) - box0) * kBoxBytes + r * 128 + (((c & 7) ^ (r & 7)) << 4));
                band_pairs_bf16(v, xy[k], nn[k]);
            }
#pragma unroll
            for (int h = 0; h < G; ++h) {
                const float4* rec = reinterpret_cast<const float4*>(w + h * kWHead + c * kWChunk);
                const float4 a = rec[0], b = rec[1], cc = rec[2];
#pragma unroll
                for (int k = 0; k < KPT; ++k) {
                    float2 t = acc[k][h];
                    t = __ffma2_rn(xy[k][0], make_float2(a.x, a.y), t);
                    t = __ffma2_rn(xy[k][1], make_float2(a.z, a.w), t);
                    t = __ffma2_rn(xy[k][2], make_float2(b.x, b.y), t);
                    t = __ffma2_rn(xy[k][3], make_float2(b.z, b.w), t);
                    t = __ffma2_rn(nn[k][0], make_float2(cc.x, cc.y), t);
                    t = __ffma2_rn(nn[k][1], make_float2(cc.z, cc.w), t);
                    acc[k][h] = t;
                }
            }
        }
    } else {
        // float32 rows: 32 chunks of 4 floats (2 bands each).
#pragma unroll 4
        for (int c = c0; c < c1; ++c) {
            float2 xy[KPT][2];
            float2 nn[KPT];
#pragma unroll
            for (int k = 0; k < KPT; ++k) {
                const int r = first_row + kRowStride * k;
                const float4 v = *reinterpret_cast<const float4*>(
                    boxes + ((c >> 3) - box0) * kBoxBytes + r * 128 + (((c & 7) ^ (r & 7)) << 4));
                band_pair_f32(v, xy[k], nn[k]);
            }
            const int half = c & 1;
#pragma unroll
            for (int h = 0; h < G; ++h) {
                const float* rec = w + h * kWHead + (c >> 1) * kWChunk;
                const float4 a = *reinterpret_cast<const float4*>(rec + 4 * half);
                const float2 cc = *reinterpret_cast<const float2*>(rec + 8 + 2 * half);
#pragma unroll
                for (int k = 0; k < KPT; ++k) {
                    float2 t = acc[k][h];
                    t = __ffma2_rn(xy[k][0], make_float2(a.x, a.y), t);
                    t = __ffma2_rn(xy[k][1], make_float2(a.z, a.w), t);
                    t = __ffma2_rn(nn[k], cc, t);
                    acc[k][h] = t;
                }
            }
        }
    }
}

template <int G, int KPT>
__device__ __forceinline__ void score_acc_zero(float2 (&acc)[KPT][G]) {
#pragma unroll
    for (int k = 0; k < KPT; ++k)
#pragma unroll
        for (int h = 0; h < G; ++h) acc[k][h] = make_float2(0.f, 0.f);
}

template <int G, int KPT>
__device__ __forceinline__ void score_acc_final(const float2 (&acc)[KPT][G], float (&s)[KPT][G]) {
#pragma unroll
    for (int k = 0; k < KPT; ++k)
#pragma unroll
        for (int h = 0; h < G; ++h) s[k][h] = acc[k][h].x + acc[k][h].y;
}

// Score KPT keys of a whole tile (all chunks) into s.
template <typename T, int G, int KPT, int kBoxBytes, int kRowStride>
__device__ __forceinline__ void score_rows(const uint8_t* tile, const float* w, int first_row,
                                           float (&s)[KPT][G]) {
    float2 acc[KPT][G];
    score_acc_zero<G, KPT>(acc);
    score_rows_acc<T, G, KPT, kBoxBytes, kRowStride>(tile, 0, row_chunks<T>(), w, first_row, acc);
    score_acc_final<G, KPT>(acc, s);
}

}  // namespace tri
