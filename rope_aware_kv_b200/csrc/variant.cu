// variant.cu -- the method variants that change the per-key arithmetic, and
// per-layer budgets.
//
// TRI_VAR_MAX_OFFSET: the score of a key for a query head is the maximum over
// the future offsets delta of S_trig(delta) + S_norm, not their mean
// (shibing624 paper reading, future-offset paragraph: the maximum is the
// key's score).  The offset average no longer folds into one weight vector,
// so each offset keeps its own rotated centre
//   A_{f,delta} = E[q_f] e^{i w_f (p_cur + delta)}
// and a key costs one 128-wide dot product per offset and head.
// TRI_VAR_HALF_SPLIT: band f pairs components (x_f, x_{f+64}) (the
// rotate-half RoPE layout) instead of (x_2f, x_2f+1).
//
// Both run on the split path: variant_score_kernel scores one key per
// thread with the key's 64 bands staged in shared memory (and, for the
// maximum, each head's per-offset centres), moments_kernel forms each head's mean and
// 1/sigma (two passes in float64, fixed order), and the z-max / selection /
// gather kernels follow unchanged.  These are correctness paths for the
// variants, not tuned like the main score kernel.
#include "tri_internal.cuh"
#include "tri_launch.h"

namespace tri {

// One thread per key of one unit (blockIdx.y); 128 keys per block.  wts:
// the fold_kernel records (chunk-major, 12 floats per 4 bands: the folded A
// pairs, then the norm weights c).  With max_off, each head's per-offset
// centres A_{f,delta} = E[q_f] e^{i w_f (p_cur + delta)} are formed by the
// block in shared memory (float64, rounded once), zero under
// TRI_VAR_NO_TRIG; otherwise the folded A of wts (the mean over the offsets).
constexpr int kVarThreads = 128;

struct VariantArgs {
    int64_t cap;
    const int32_t* n_valid;
    const float* wts;          // fold records [U*G][kWHead]
    const float* stats;        // [L][Hkv*G][64][4]
    const int64_t* p_cur;      // [n_seq]
    int64_t n_layers, n_kvheads;
    double theta;
    FoldOffsets off;
    int max_off;               // maximum over the offsets (else their mean)
    int half;                  // half-split band pairing
    int variant;
    float* raw;                // [U][G][cap]
    uint32_t* flag;
    PageMap pm;                // paged key pool, or contiguous
};

template <typename T, int G>
__global__ void __launch_bounds__(kVarThreads)
variant_score_kernel(const T* __restrict__ keys, const VariantArgs a) {
    extern __shared__ float2 kb[];  // [kF][kVarThreads] bands, [kF][kVarThreads] norms, A
    float* nb = reinterpret_cast<float*>(kb + kF * kVarThreads);
    float2* aw = reinterpret_cast<float2*>(nb + kF * kVarThreads);  // [n_off][kF]
    const int64_t u = blockIdx.y;
    const int n =
        clamp_nvalid(a.n_valid, u, a.cap, blockIdx.x == 0 && threadIdx.x == 0 ? a.flag : nullptr);
    const int t = threadIdx.x;
    const int j = blockIdx.x * kVarThreads + t;
    if (blockIdx.x * kVarThreads >= n) return;  // uniform over the block
    const int64_t pr = j < n ? phys_row(a.pm, u, a.cap, j) : -1;
    if (j < n && pr < 0) raise_flag(a.flag, TRI_FLAG_INDEX_RANGE);
    const bool valid = pr >= 0;
    if (valid) {
        const T* row = keys + pr * kD;
        for (int f = 0; f < kF; ++f) {
            const float x = to_float(row[a.half ? f : 2 * f]);
            const float y = to_float(row[a.half ? f + kF : 2 * f + 1]);
            kb[f * kVarThreads + t] = make_float2(x, y);
            nb[f * kVarThreads + t] = sqrtf(fmaf(x, x, y * y));
        }
    }
    const int64_t kvh = u % a.n_kvheads;
    const int64_t layer = (u / a.n_kvheads) % a.n_layers;
    const int64_t seq = u / (a.n_kvheads * a.n_layers);
    const bool trig = (a.variant & TRI_VAR_NO_TRIG) == 0;
#pragma unroll 1
    for (int h = 0; h < G; ++h) {
        const float* rec = a.wts + (u * G + h) * kWHead;
        if (a.max_off) {
            __syncthreads();  // the previous head's centres are no longer read
            const float* st = a.stats + ((layer * a.n_kvheads + kvh) * G + h) * kF * 4;
            for (int e = t; e < a.off.n * kF; e += kVarThreads) {
                const int o = e / kF, f = e % kF;
                const double w =
                    pow(a.theta, -2.0 * static_cast<double>(f) / static_cast<double>(kD));
                double sn, cs;
                sincos(w * static_cast<double>(a.p_cur[seq] + a.off.v[o]), &sn, &cs);
                const double mre = st[f * 4], mim = st[f * 4 + 1];
                aw[e] = trig ? make_float2(static_cast<float>(mre * cs - mim * sn),
                                           static_cast<float>(mre * sn + mim * cs))
                             : make_float2(0.f, 0.f);
            }
            __syncthreads();
        }
        if (!valid) continue;
        float s_norm = 0.f;
        for (int f = 0; f < kF; ++f)
            s_norm = fmaf(__ldg(rec + wrec_c(f)), nb[f * kVarThreads + t],
                          s_norm);
        float s;
        if (a.max_off) {
            float best = -INFINITY;
#pragma unroll 1
            for (int o = 0; o < a.off.n; ++o) {
                float tr = 0.f;
                for (int f = 0; f < kF; ++f) {
                    const float2 c = aw[o * kF + f];
                    const float2 k = kb[f * kVarThreads + t];
                    tr = fmaf(c.x, k.x, fmaf(c.y, k.y, tr));
                }
                best = fmaxf(best, tr + s_norm);
            }
            s = best;
        } else {
            float tr = 0.f;
            for (int f = 0; f < kF; ++f) {
                const float2 k = kb[f * kVarThreads + t];
                tr = fmaf(__ldg(rec + wrec_re(f)), k.x, fmaf(__ldg(rec + wrec_im(f)), k.y, tr));
            }
            s = tr + s_norm;
        }
        a.raw[(u * G + h) * a.cap + j] = s;
    }
}

// Mean and 1/sigma (population) of each (unit, head) over the unit's valid
// keys, in float64: a fixed-order block reduction, two passes.  grid U * G.
__global__ void __launch_bounds__(256)
moments_kernel(const float* __restrict__ raw, int64_t cap, const int32_t* __restrict__ n_valid,
               int G, float2* __restrict__ mom) {
    __shared__ double red[256];
    const int64_t uh = blockIdx.x;
    const int64_t u = uh / G;
    const int n = clamp_nvalid(n_valid, u, cap, nullptr);
    const float* s = raw + uh * cap;
    auto block_sum = [&](double v) -> double {
        red[threadIdx.x] = v;
        __syncthreads();
        for (int w = 128; w > 0; w >>= 1) {
            if (threadIdx.x < w) red[threadIdx.x] += red[threadIdx.x + w];
            __syncthreads();
        }
        const double r = red[0];
        __syncthreads();
        return r;
    };
    double a = 0.0;
    for (int j = threadIdx.x; j < n; j += 256) a += s[j];
    const double mu = n > 0 ? block_sum(a) / n : 0.0;
    double b = 0.0;
    for (int j = threadIdx.x; j < n; j += 256) {
        const double d = s[j] - mu;
        b = fma(d, d, b);
    }
    const double var = n > 0 ? block_sum(b) / n : 0.0;
    if (threadIdx.x == 0) {
        const double sd = sqrt(var);
        float inv = sd > 0.0 ? static_cast<float>(1.0 / sd) : 0.f;
        if (!(sd == sd)) inv = __int_as_float(0x7fc00000);
        mom[uh] = make_float2(static_cast<float>(mu), inv);
    }
}

// ub[u] = layer_budget[layer of u]: per-layer budgets to per-unit budgets.
__global__ void unit_budget_kernel(const int32_t* __restrict__ layer_budget, int64_t n_units,
                                   int64_t n_layers, int64_t n_kvheads, int32_t* __restrict__ ub) {
    for (int64_t u = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; u < n_units;
         u += static_cast<int64_t>(gridDim.x) * blockDim.x)
        ub[u] = layer_budget[(u / n_kvheads) % n_layers];
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
size_t variant_score_smem() {
    return static_cast<size_t>(kF) * kVarThreads * (8 + 4) + static_cast<size_t>(TRI_MAX_OFFSETS) * kF * 8;
}

template <typename T>
static cudaError_t launch_vscore_t(int G, const void* keys, int64_t n_units,
                                   const VariantArgs& a, cudaStream_t s) {
    const size_t smem = variant_score_smem();
    dim3 grid(static_cast<unsigned>((a.cap + kVarThreads - 1) / kVarThreads),
              static_cast<unsigned>(n_units));
    const T* k = static_cast<const T*>(keys);
    switch (G) {
#define TRI_VCASE(g)                                                                      \
    case g: {                                                                             \
        cudaError_t e = cudaFuncSetAttribute(variant_score_kernel<T, g>,                  \
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, \
                                             static_cast<int>(smem));                     \
        if (e != cudaSuccess) return e;                                                   \
        variant_score_kernel<T, g><<<grid, kVarThreads, smem, s>>>(k, a);                 \
        break;                                                                            \
    }
        TRI_VCASE(1) TRI_VCASE(2) TRI_VCASE(3) TRI_VCASE(4)
        TRI_VCASE(5) TRI_VCASE(6) TRI_VCASE(7) TRI_VCASE(8)
#undef TRI_VCASE
        default: return cudaErrorInvalidValue;
    }
    note_launch(s);
    return cudaGetLastError();
}

cudaError_t launch_variant_score(tri_dtype dt, int G, const void* keys, int64_t n_units,
                                 int64_t cap, const int32_t* n_valid, const float* wts,
                                 const float* stats, const int64_t* p_cur, int64_t n_layers,
                                 int64_t n_kvheads, double theta, const FoldOffsets& off,
                                 int variant, float* raw, uint32_t* flag, cudaStream_t s,
                                 const PageMap& pm) {
    VariantArgs a;
    a.pm = pm;
    a.cap = cap;
    a.n_valid = n_valid;
    a.wts = wts;
    a.stats = stats;
    a.p_cur = p_cur;
    a.n_layers = n_layers;
    a.n_kvheads = n_kvheads;
    a.theta = theta;
    a.off = off;
    a.max_off = (variant & TRI_VAR_MAX_OFFSET) ? 1 : 0;
    a.half = (variant & TRI_VAR_HALF_SPLIT) ? 1 : 0;
    a.variant = variant;
    a.raw = raw;
    a.flag = flag;
    if (dt == TRI_BF16) return launch_vscore_t<__nv_bfloat16>(G, keys, n_units, a, s);
    return launch_vscore_t<float>(G, keys, n_units, a, s);
}

cudaError_t launch_moments(const float* raw, int64_t n_units, int64_t cap, const int32_t* n_valid,
                           int G, float2* mom, cudaStream_t s) {
    moments_kernel<<<static_cast<unsigned>(n_units * G), 256, 0, s>>>(raw, cap, n_valid, G, mom);
    note_launch(s);
    return cudaGetLastError();
}

cudaError_t launch_unit_budget(const int32_t* layer_budget, int64_t n_units, int64_t n_layers,
                               int64_t n_kvheads, int32_t* ub, cudaStream_t s) {
    const int64_t blocks = (n_units + 255) / 256;
    unit_budget_kernel<<<static_cast<unsigned>(blocks < 1024 ? blocks : 1024), 256, 0, s>>>(
        layer_budget, n_units, n_layers, n_kvheads, ub);
    note_launch(s);
    return cudaGetLastError();
}

}  // namespace tri
