// logit.cu -- the attention logit as a function of distance: reconstructed
// from the Q/K centres, measured on post-RoPE sequences, and their Pearson
// correlation (the check behind the centre approximation).
//
// Talk page: the RoPE logit general form
//   logit = sum_f |q_f| |k_f| cos(w_f Delta + phi_f),  phi_f = arg q_f - arg k_f,
// and with q_f ~ E[q_f], k_f ~ E[k_f] (the centres) a trigonometric series
// in the distance Delta alone; shibing624 paper reading, Fig. 1(D): the
// series against the measured logits, per head, by Pearson correlation.
//   reconstruct  recon[h][i] = sum_f |E q_f| |E k_f| cos(w_f deltas[i] + phi_f)
//                (query head h, its KV head h / G; float64, one block per head)
//   curve        curve[h][i] = mean over t in [deltas[i], n_tok) of
//                q[h][t] . k[h / G][t - deltas[i]] (token t at position t;
//                float32 dot products summed in float64, one block per
//                (delta, head))
//   pearson      r[row] of two [rows][n] float arrays (two passes, float64)
#include "tri_internal.cuh"
#include "tri_launch.h"

namespace tri {

__global__ void __launch_bounds__(256)
logit_reconstruct_kernel(const float* __restrict__ qs, const float* __restrict__ ks, int G,
                         double theta, const int64_t* __restrict__ deltas, int64_t n_delta,
                         float* __restrict__ recon) {
    __shared__ double amp[kF], phi[kF], om[kF];
    const int64_t h = blockIdx.x;
    if (threadIdx.x < kF) {
        const int f = threadIdx.x;
        const float* q = qs + (h * kF + f) * 4;
        const float* k = ks + ((h / G) * kF + f) * 4;
        const double qr = q[0], qi = q[1], kr = k[0], ki = k[1];
        amp[f] = sqrt(qr * qr + qi * qi) * sqrt(kr * kr + ki * ki);
        phi[f] = atan2(qi, qr) - atan2(ki, kr);
        om[f] = pow(theta, -2.0 * static_cast<double>(f) / kD);
    }
    __syncthreads();
    for (int64_t i = threadIdx.x; i < n_delta; i += blockDim.x) {
        const double dl = static_cast<double>(deltas[i]);
        double s = 0.0;
        for (int f = 0; f < kF; ++f) s += amp[f] * cos(om[f] * dl + phi[f]);
        recon[h * n_delta + i] = static_cast<float>(s);
    }
}

__device__ __forceinline__ double block_sum_d(double v, double* red) {
    red[threadIdx.x] = v;
    __syncthreads();
    for (int w = blockDim.x / 2; w > 0; w >>= 1) {
        if (threadIdx.x < w) red[threadIdx.x] += red[threadIdx.x + w];
        __syncthreads();
    }
    const double r = red[0];
    __syncthreads();
    return r;
}

template <typename T>
__global__ void __launch_bounds__(256)
logit_curve_kernel(const T* __restrict__ q, const T* __restrict__ k, int G, int64_t n_tok,
                   const int64_t* __restrict__ deltas, int64_t n_delta, float* __restrict__ curve) {
    __shared__ double red[256];
    const int64_t i = blockIdx.x, h = blockIdx.y;
    const int64_t D = deltas[i];
    const int64_t t0 = D > 0 ? D : 0;
    const int64_t t1 = D < 0 ? n_tok + D : n_tok;
    const T* qh = q + h * n_tok * kD;
    const T* kh = k + (h / G) * n_tok * kD;
    double sum = 0.0;
    for (int64_t t = t0 + threadIdx.x; t < t1; t += blockDim.x) {
        const T* qr = qh + t * kD;
        const T* kr = kh + (t - D) * kD;
        float dot = 0.f;
        for (int e = 0; e < kD; ++e) dot = fmaf(to_float(qr[e]), to_float(kr[e]), dot);
        sum += dot;
    }
    sum = block_sum_d(sum, red);
    if (threadIdx.x == 0) {
        const int64_t cnt = t1 > t0 ? t1 - t0 : 0;
        curve[h * n_delta + i] = cnt > 0 ? static_cast<float>(sum / static_cast<double>(cnt)) : 0.f;
    }
}

__global__ void __launch_bounds__(256)
pearson_kernel(const float* __restrict__ a, const float* __restrict__ b, int64_t n,
               float* __restrict__ r) {
    __shared__ double red[256];
    const float* x = a + blockIdx.x * n;
    const float* y = b + blockIdx.x * n;
    double sx = 0.0, sy = 0.0;
    for (int64_t i = threadIdx.x; i < n; i += blockDim.x) {
        sx += x[i];
        sy += y[i];
    }
    const double mx = block_sum_d(sx, red) / static_cast<double>(n > 0 ? n : 1);
    const double my = block_sum_d(sy, red) / static_cast<double>(n > 0 ? n : 1);
    double sxy = 0.0, sxx = 0.0, syy = 0.0;
    for (int64_t i = threadIdx.x; i < n; i += blockDim.x) {
        const double dx = x[i] - mx, dy = y[i] - my;
        sxy += dx * dy;
        sxx += dx * dx;
        syy += dy * dy;
    }
    sxy = block_sum_d(sxy, red);
    sxx = block_sum_d(sxx, red);
    syy = block_sum_d(syy, red);
    if (threadIdx.x == 0)
        r[blockIdx.x] = (sxx > 0.0 && syy > 0.0) ? static_cast<float>(sxy / sqrt(sxx * syy)) : 0.f;
}

cudaError_t launch_logit_reconstruct(const float* qs, const float* ks, int64_t n_qheads, int G,
                                     double theta, const int64_t* deltas, int64_t n_delta,
                                     float* recon, cudaStream_t s) {
    logit_reconstruct_kernel<<<static_cast<unsigned>(n_qheads), 256, 0, s>>>(qs, ks, G, theta,
                                                                             deltas, n_delta, recon);
    note_launch(s);
    return cudaGetLastError();
}

cudaError_t launch_logit_curve(tri_dtype dt, const void* q, const void* k, int64_t n_qheads, int G,
                               int64_t n_tok, const int64_t* deltas, int64_t n_delta, float* curve,
                               cudaStream_t s) {
    dim3 grid(static_cast<unsigned>(n_delta), static_cast<unsigned>(n_qheads));
    if (dt == TRI_BF16)
        logit_curve_kernel<__nv_bfloat16><<<grid, 256, 0, s>>>(
            static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k), G, n_tok,
            deltas, n_delta, curve);
    else
        logit_curve_kernel<float><<<grid, 256, 0, s>>>(static_cast<const float*>(q),
                                                       static_cast<const float*>(k), G, n_tok,
                                                       deltas, n_delta, curve);
    note_launch(s);
    return cudaGetLastError();
}

cudaError_t launch_pearson(const float* a, const float* b, int64_t n_rows, int64_t n, float* r,
                           cudaStream_t s) {
    pearson_kernel<<<static_cast<unsigned>(n_rows), 256, 0, s>>>(a, b, n, r);
    note_launch(s);
    return cudaGetLastError();
}

}  // namespace tri
