// fold_core.cuh -- the per-head fold computed inside the prune kernels.
//
// A_f = E[q_f] e^{i w_f p_cur} C_f with C_f = (1/|D|) sum_delta e^{i w_f delta}
// and c_f = (1 - R_f) E|q_f| (talk page: S_trig, S_norm and the
// offset-averaged S~; the key position cancels, see score.cu); the ablations
// TRI_VAR_NO_TRIG (A_f = 0) and TRI_VAR_NO_R (c_f = E|q_f|) change only
// these weights.  The
// config-only factors w_f and C_f arrive as a kernel parameter (FoldConst);
// each unit needs 64 phases e^{i w_f p_cur} and G x 64 complex products, all
// in float64, rounded once to the float32 weight records the score loop reads
// (16 chunks x 12 floats per head: 4 bands' (Re A, Im A) pairs, then their c).
#pragma once

#include "tri_internal.cuh"
#include "tri_launch.h"

namespace tri {

struct FoldShared {
    double ef[64][2];
};
static_assert(sizeof(FoldShared) <= kFoldStaticBytes, "fold factors exceed their budget");

// Weight records of the G query heads of unit u into w (shared memory),
// computed by the first nthreads threads of the CTA: with bar_id 0 they are
// all of its threads (two __syncthreads inside), otherwise the named barrier
// bar_id synchronises exactly those threads.
template <int G>
__device__ __forceinline__ void fold_unit_sync(FoldShared& fs, const FoldConst& fc, float* w,
                                               const float* stats, const int64_t* p_cur,
                                               int64_t u, int64_t n_layers, int64_t n_kvheads,
                                               int bar_id, int nthreads) {
    const int t = threadIdx.x;
    const int64_t kvh = u % n_kvheads;
    const int64_t layer = (u / n_kvheads) % n_layers;
    const int64_t seq = u / (n_kvheads * n_layers);
    auto sync = [&]() {
        if (bar_id == 0)
            __syncthreads();
        else
            named_sync(bar_id, nthreads);
    };
    if (t < kF) {
        double ps, pc;
        sincos(fc.omega[t] * static_cast<double>(p_cur[seq]), &ps, &pc);
        fs.ef[t][0] = pc;
        fs.ef[t][1] = ps;
    }
    sync();
    const float* st_base = stats + ((layer * n_kvheads + kvh) * G) * kF * 4;
    for (int e = t; e < G * kF; e += nthreads) {
        const int h = e / kF, f = e % kF;
        const float4 st = *reinterpret_cast<const float4*>(st_base + (h * kF + f) * 4);
        const double mre = st.x, mim = st.y;
        const double tre = mre * fs.ef[f][0] - mim * fs.ef[f][1];
        const double tim = mre * fs.ef[f][1] + mim * fs.ef[f][0];
        const bool trig = (fc.variant & TRI_VAR_NO_TRIG) == 0;
        const double are = trig ? tre * fc.cf[f][0] - tim * fc.cf[f][1] : 0.0;
        const double aim = trig ? tre * fc.cf[f][1] + tim * fc.cf[f][0] : 0.0;
        const double rw = (fc.variant & TRI_VAR_NO_R) ? 1.0 : 1.0 - static_cast<double>(st.w);
        const double cw = rw * static_cast<double>(st.z);
        float* rec = w + h * kWHead;
        rec[wrec_re(f)] = static_cast<float>(are);
        rec[wrec_im(f)] = static_cast<float>(aim);
        rec[wrec_c(f)] = static_cast<float>(cw);
    }
    sync();
}

// Every thread of the CTA computes the fold (two __syncthreads inside).
template <int G>
__device__ __forceinline__ void fold_unit(FoldShared& fs, const FoldConst& fc, float* w,
                                          const float* stats, const int64_t* p_cur, int64_t u,
                                          int64_t n_layers, int64_t n_kvheads) {
    fold_unit_sync<G>(fs, fc, w, stats, p_cur, u, n_layers, n_kvheads, 0,
                      static_cast<int>(blockDim.x));
}

}  // namespace tri
