// calibrate.cu -- per-head, per-band query statistics from pre-RoPE queries.
//
// For query head h and RoPE band f (pair (x_2f, x_2f+1)):
//   E[q_f] = mean over tokens of x_2f + i x_2f+1,  E[|q_f|] = mean of the
//   pair's norm,  R_f = |E[q_f]| / E[|q_f|]  (R_f = 1 where E[|q_f|] = 0).
// (TriAttention talk announcement, qingkeai.online: S_norm equation and the
// R_f definition; shibing624 paper reading, offline calibration on ~10K
// tokens; hyper.ai summary of arXiv 2604.04921, Method section.)
//
// Two launches: a column reduction over token chunks writing float64 partial
// sums, then a fixed-order merge per head.  No atomics on floating point, so
// the result is bitwise reproducible.
#include "tri_internal.cuh"
#include "tri_launch.h"
#include "calibrate_dp.h"

namespace tri {

constexpr int kCalThreads = 256;   // 4 rows x 64 bands per step
constexpr int kCalChunk = 1024;    // tokens per CTA

// Options of the extended calibration: post-RoPE queries are rotated back
// by -w_f p (p the token's position, qpos[t]) before they are averaged, which
// gives their pre-RoPE bands (shibing624 paper reading, Q/K concentration
// section: the centres live in the pre-RoPE space); `half` takes band f from
// components (x_f, x_{f+64}).  Keys calibrated the same way give the K centres.
struct CalibOpts {
    const int32_t* qpos = nullptr;  // [n_tok] positions of post-RoPE rows, or null
    int half = 0;
    double theta = 10000.0;
};

template <typename T>
__global__ void __launch_bounds__(kCalThreads)
calib_partial_kernel(const T* __restrict__ q, int64_t n_tok, int n_chunks,
                     double* __restrict__ part, CalibOpts opt) {
    const int f = threadIdx.x & 63;
    const int r = threadIdx.x >> 6;
    const int64_t h = blockIdx.y;
    const int64_t t0 = static_cast<int64_t>(blockIdx.x) * kCalChunk;
    const int64_t t1 = min(t0 + kCalChunk, n_tok);
    const double w = opt.qpos ? pow(opt.theta, -2.0 * static_cast<double>(f) / kD) : 0.0;
    double sx = 0.0, sy = 0.0, sn = 0.0;
    for (int64_t t = t0 + r; t < t1; t += 4) {
        const T* row = q + (h * n_tok + t) * kD;
        float x, y;
        if (opt.half) {
            x = to_float(row[f]);
            y = to_float(row[f + 64]);
        } else if constexpr (sizeof(T) == 2) {
            const uint32_t wd = reinterpret_cast<const uint32_t*>(row)[f];
            x = bf16_lo(wd);
            y = bf16_hi(wd);
        } else {
            const float2 v = reinterpret_cast<const float2*>(row)[f];
            x = v.x;
            y = v.y;
        }
        double dx = x, dy = y;
        if (opt.qpos) {
            double sa, ca;
            sincos(w * static_cast<double>(opt.qpos[t]), &sa, &ca);
            const double rx = ca * dx + sa * dy;
            dy = -sa * dx + ca * dy;
            dx = rx;
        }
        sx += dx;
        sy += dy;
        sn += sqrt(dx * dx + dy * dy);
    }
    __shared__ double red[4][64][3];
    red[r][f][0] = sx;
    red[r][f][1] = sy;
    red[r][f][2] = sn;
    __syncthreads();
    if (r == 0) {
        double a = 0.0, b = 0.0, c = 0.0;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            a += red[i][f][0];
            b += red[i][f][1];
            c += red[i][f][2];
        }
        double* o = part + ((h * n_chunks + blockIdx.x) * 64 + f) * 3;
        o[0] = a;
        o[1] = b;
        o[2] = c;
    }
}

__global__ void __launch_bounds__(64)
calib_merge_kernel(const double* __restrict__ part, int n_chunks, int64_t n_tok,
                   float* __restrict__ stats) {
    const int f = threadIdx.x;
    const int64_t h = blockIdx.x;
    double a = 0.0, b = 0.0, c = 0.0;
    for (int i = 0; i < n_chunks; ++i) {
        const double* o = part + ((h * n_chunks + i) * 64 + f) * 3;
        a += o[0];
        b += o[1];
        c += o[2];
    }
    const double inv = 1.0 / static_cast<double>(n_tok);
    const double mre = a * inv, mim = b * inv, mn = c * inv;
    const double R = (mn > 0.0) ? sqrt(mre * mre + mim * mim) / mn : 1.0;
    float* s = stats + (h * 64 + f) * 4;
    s[0] = static_cast<float>(mre);
    s[1] = static_cast<float>(mim);
    s[2] = static_cast<float>(mn);
    s[3] = static_cast<float>(R);
}

// Data-parallel calibration: the chunk partials of a shard summed in chunk
// order into float64 totals, and statistics formed from (all-reduced) totals.
__global__ void __launch_bounds__(64)
calib_sum_kernel(const double* __restrict__ part, int n_chunks, double* __restrict__ sums) {
    const int f = threadIdx.x;
    const int64_t h = blockIdx.x;
    double a = 0.0, b = 0.0, c = 0.0;
    for (int i = 0; i < n_chunks; ++i) {
        const double* o = part + ((h * n_chunks + i) * 64 + f) * 3;
        a += o[0];
        b += o[1];
        c += o[2];
    }
    double* o = sums + (h * 64 + f) * 3;
    o[0] = a;
    o[1] = b;
    o[2] = c;
}

__global__ void __launch_bounds__(64)
calib_finish_kernel(const double* __restrict__ sums, int64_t n_tok, float* __restrict__ stats) {
    const int f = threadIdx.x;
    const int64_t h = blockIdx.x;
    const double* o = sums + (h * 64 + f) * 3;
    const double inv = 1.0 / static_cast<double>(n_tok);
    const double mre = o[0] * inv, mim = o[1] * inv, mn = o[2] * inv;
    const double R = (mn > 0.0) ? sqrt(mre * mre + mim * mim) / mn : 1.0;
    float* s = stats + (h * 64 + f) * 4;
    s[0] = static_cast<float>(mre);
    s[1] = static_cast<float>(mim);
    s[2] = static_cast<float>(mn);
    s[3] = static_cast<float>(R);
}

cudaError_t launch_calibrate_sums(const void* q, tri_dtype dt, int64_t n_heads, int64_t n_tok,
                                  double* sums, void* ws, cudaStream_t s) {
    const int n_chunks = static_cast<int>((n_tok + kCalChunk - 1) / kCalChunk);
    double* part = reinterpret_cast<double*>(static_cast<char*>(ws) + kWsHeader);
    dim3 grid(n_chunks, static_cast<unsigned>(n_heads));
    if (dt == TRI_BF16) {
        calib_partial_kernel<__nv_bfloat16><<<grid, kCalThreads, 0, s>>>(
            static_cast<const __nv_bfloat16*>(q), n_tok, n_chunks, part, CalibOpts());
    } else {
        calib_partial_kernel<float><<<grid, kCalThreads, 0, s>>>(static_cast<const float*>(q),
                                                                  n_tok, n_chunks, part,
                                                                  CalibOpts());
    }
    note_launch(s);
    calib_sum_kernel<<<static_cast<unsigned>(n_heads), 64, 0, s>>>(part, n_chunks, sums);
    note_launch(s);
    return cudaGetLastError();
}

cudaError_t launch_calibrate_finish(const double* sums, int64_t n_heads, int64_t n_tok,
                                    float* stats, cudaStream_t s) {
    calib_finish_kernel<<<static_cast<unsigned>(n_heads), 64, 0, s>>>(sums, n_tok, stats);
    note_launch(s);
    return cudaGetLastError();
}

size_t calibrate_ws_bytes(int64_t n_heads, int64_t n_tok) {
    const int64_t n_chunks = (n_tok + kCalChunk - 1) / kCalChunk;
    return kWsHeader + static_cast<size_t>(n_heads * n_chunks * 64 * 3) * sizeof(double);
}

cudaError_t launch_calibrate(const void* q, tri_dtype dt, int64_t n_heads, int64_t n_tok,
                             float* stats, void* ws, cudaStream_t s, const int32_t* qpos,
                             int half, double theta) {
    const int n_chunks = static_cast<int>((n_tok + kCalChunk - 1) / kCalChunk);
    double* part = reinterpret_cast<double*>(static_cast<char*>(ws) + kWsHeader);
    dim3 grid(n_chunks, static_cast<unsigned>(n_heads));
    CalibOpts opt;
    opt.qpos = qpos;
    opt.half = half;
    opt.theta = theta;
    if (dt == TRI_BF16) {
        calib_partial_kernel<__nv_bfloat16><<<grid, kCalThreads, 0, s>>>(
            static_cast<const __nv_bfloat16*>(q), n_tok, n_chunks, part, opt);
        note_launch(s);
    } else {
        calib_partial_kernel<float><<<grid, kCalThreads, 0, s>>>(static_cast<const float*>(q),
                                                                  n_tok, n_chunks, part, opt);
        note_launch(s);
    }
    calib_merge_kernel<<<static_cast<unsigned>(n_heads), 64, 0, s>>>(part, n_chunks, n_tok, stats);
    note_launch(s);
    return cudaGetLastError();
}

}  // namespace tri
