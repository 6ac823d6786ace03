// select.cu -- top-B selection and order-preserving compaction of indices.
//
// Keep the B keys with the highest final score, in ascending index order
// (talk page: keep only the top-B; jaedaily.cn tutorial, eviction step:
// top-k then sort to keep the temporal order).  Ranking: score descending,
// NaN lowest, -0.0 == +0.0, equal scores by ascending index.
//
// Method: MSB-first radix select on the order-preserving 32-bit key of each
// score, three digit passes of 11, 11 and 10 bits.  Each pass builds a
// histogram of the keys that match the digits fixed so far (shared-memory
// counts, one global atomic per non-empty bin); the digit holding the B-th
// largest key is found by a descending warp scan that every CTA of the next
// launch repeats redundantly (no extra launch, no global state to carry).
// After the last pass the threshold key T, the count of keys above it and the
// number of ties to keep are known exactly; the compaction then walks each
// unit in index order with warp ballots, taking every key above T and the
// first ties by index.
#include "tri_internal.cuh"
#include "tri_launch.h"
#include "select_core.cuh"

namespace tri {

// State after `passes` digit passes; executed by one warp, result in *out.
__device__ void compute_state(const uint32_t* hists, int64_t n_units, int64_t u, int n, int64_t B,
                              int passes, SelState* out) {
    SelState st;
    st.prefix = 0;
    st.k = static_cast<uint32_t>(B);
    st.gt = 0;
    st.keep_all = (n <= B) ? 1 : 0;
    if (!st.keep_all) {
        for (int p = 0; p < passes; ++p) {
            const uint32_t* h = hists + (static_cast<int64_t>(p) * n_units + u) * kHistBins0;
            uint32_t bin, above;
            warp_find_bin(h, 1 << pass_bits(p), st.k, bin, above);
            st.gt += above;
            st.k -= above;
            st.prefix = (st.prefix << pass_bits(p)) | bin;
        }
    }
    if ((threadIdx.x & 31) == 0) *out = st;
}

// Histogram of digit `pass` of the keys matching the prefix of earlier passes.
__global__ void __launch_bounds__(256)
radix_pass_kernel(const float* __restrict__ fin, int64_t n_units, int64_t cap,
                  const int32_t* __restrict__ n_valid, int64_t B, uint32_t* __restrict__ hists,
                  int pass, uint32_t* flag) {
    __shared__ uint32_t hist[kHistBins0];
    __shared__ SelState st;
    const int64_t u = blockIdx.y;
    const int n = clamp_nvalid(n_valid, u, cap, nullptr);
    if (threadIdx.x < 32) compute_state(hists, n_units, u, n, B, pass, &st);
    const int nb = 1 << pass_bits(pass);
    for (int b = threadIdx.x; b < nb; b += blockDim.x) hist[b] = 0;
    __syncthreads();
    if (st.keep_all) return;
    const int shift = pass_shift(pass);
    const int hi_shift = shift + pass_bits(pass);
    const uint32_t mask = static_cast<uint32_t>(nb - 1);
    const int j0 = blockIdx.x * kZChunk;
    const int j1 = min(j0 + kZChunk, n);
    bool nonfinite = false;
    for (int j = j0 + threadIdx.x; j < j1; j += blockDim.x) {
        const float x = fin[u * cap + j];
        if (pass == 0 && x != x) nonfinite = true;
        const uint32_t key = ordered_key(x);
        const bool match = (hi_shift >= 32) ? true : ((key >> hi_shift) == st.prefix);
        if (match) atomicAdd(&hist[(key >> shift) & mask], 1u);
    }
    if (nonfinite) raise_flag(flag, TRI_FLAG_NONFINITE);
    __syncthreads();
    uint32_t* g = hists + (static_cast<int64_t>(pass) * n_units + u) * kHistBins0;
    for (int b = threadIdx.x; b < nb; b += blockDim.x)
        if (hist[b]) atomicAdd(&g[b], hist[b]);
}

// Per chunk of kZChunk keys: count of keys above T and equal to T.
__global__ void __launch_bounds__(256)
select_count_kernel(const float* __restrict__ fin, int64_t n_units, int64_t cap,
                    const int32_t* __restrict__ n_valid, int64_t B,
                    const uint32_t* __restrict__ hists, uint2* __restrict__ counts) {
    __shared__ SelState st;
    __shared__ uint32_t red[8][2];
    const int64_t u = blockIdx.y;
    const int n = clamp_nvalid(n_valid, u, cap, nullptr);
    if (threadIdx.x < 32) compute_state(hists, n_units, u, n, B, 3, &st);
    __syncthreads();
    const int j0 = blockIdx.x * kZChunk;
    const int j1 = min(j0 + kZChunk, n);
    uint32_t gt = 0, eq = 0;
    if (!st.keep_all) {
        for (int j = j0 + threadIdx.x; j < j1; j += blockDim.x) {
            const uint32_t key = ordered_key(fin[u * cap + j]);
            gt += key > st.prefix;
            eq += key == st.prefix;
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        gt += __shfl_xor_sync(0xffffffffu, gt, o);
        eq += __shfl_xor_sync(0xffffffffu, eq, o);
    }
    if ((threadIdx.x & 31) == 0) {
        red[threadIdx.x >> 5][0] = gt;
        red[threadIdx.x >> 5][1] = eq;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        uint32_t a = 0, b = 0;
        for (int w = 0; w < 8; ++w) {
            a += red[w][0];
            b += red[w][1];
        }
        counts[u * gridDim.x + blockIdx.x] = make_uint2(a, b);
    }
}

// Ordered compaction of kept indices.  Warp w of the CTA walks keys
// j0 + 256 w + 32 i + lane, i = 0..7, in index order; ballots give each kept
// key its rank.
__global__ void __launch_bounds__(256)
select_compact_kernel(const float* __restrict__ fin, int64_t n_units, int64_t cap,
                      const int32_t* __restrict__ n_valid, int64_t B,
                      const uint32_t* __restrict__ hists, const uint2* __restrict__ counts,
                      int32_t* __restrict__ kept, int32_t* __restrict__ n_kept) {
    __shared__ SelState st;
    __shared__ uint32_t wgt[8], weq[8];
    __shared__ uint32_t base_kept, base_ties;
    const int64_t u = blockIdx.y;
    const int n = clamp_nvalid(n_valid, u, cap, nullptr);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x < 32) compute_state(hists, n_units, u, n, B, 3, &st);
    if (threadIdx.x == 32) {
        // Kept keys and ties in the chunks before this one.
        uint32_t k = 0, t = 0;
        const uint2* c = counts + u * gridDim.x;
        for (unsigned i = 0; i < blockIdx.x; ++i) {
            k += c[i].x;
            t += c[i].y;
        }
        base_kept = k;
        base_ties = t;
    }
    __syncthreads();
    const int64_t m = (n < B) ? n : B;
    int32_t* out = kept + u * B;
    const int j0 = blockIdx.x * kZChunk + warp * 256;
    if (st.keep_all) {
        for (int i = 0; i < 8; ++i) {
            const int j = j0 + 32 * i + lane;
            if (j < n) out[j] = j;
        }
    } else {
        // Pass 1: this warp's counts.
        uint32_t key[8];
        uint32_t gt = 0, eq = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int j = j0 + 32 * i + lane;
            key[i] = (j < n) ? ordered_key(fin[u * cap + j]) : 0u;
            const bool valid = j < n;
            gt += __popc(__ballot_sync(0xffffffffu, valid && key[i] > st.prefix));
            eq += __popc(__ballot_sync(0xffffffffu, valid && key[i] == st.prefix));
        }
        if (lane == 0) {
            wgt[warp] = gt;
            weq[warp] = eq;
        }
        __syncthreads();
        // Ties before this warp (global order) and kept keys before this warp.
        uint32_t ties = base_ties, pos = 0;
        for (int w = 0; w < warp; ++w) ties += weq[w];
        // Kept before this chunk: strict-above counts plus ties taken.
        {
            // counts[].x are strict counts; ties taken before the chunk:
            const uint32_t taken_before = min(base_ties, st.k);
            pos = base_kept + taken_before;
            uint32_t t = base_ties;
            for (int w = 0; w < warp; ++w) {
                const uint32_t take = (t < st.k) ? min(weq[w], st.k - t) : 0u;
                pos += wgt[w] + take;
                t += weq[w];
            }
        }
        const uint32_t lt = (1u << lane) - 1u;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int j = j0 + 32 * i + lane;
            const bool valid = j < n;
            const bool is_eq = valid && key[i] == st.prefix;
            const uint32_t beq = __ballot_sync(0xffffffffu, is_eq);
            const uint32_t my_tie = ties + __popc(beq & lt);
            const bool keep = valid && (key[i] > st.prefix || (is_eq && my_tie < st.k));
            const uint32_t bk = __ballot_sync(0xffffffffu, keep);
            if (keep) {
                const uint32_t r = pos + __popc(bk & lt);
                if (r < static_cast<uint32_t>(B)) out[r] = j;
            }
            pos += __popc(bk);
            ties += __popc(beq);
        }
    }
    if (blockIdx.x == 0) {
        if (threadIdx.x == 0) n_kept[u] = static_cast<int32_t>(m);
        for (int64_t r = m + threadIdx.x; r < B; r += blockDim.x) out[r] = -1;
    }
}

cudaError_t launch_radix_pass(const float* fin, int64_t n_units, int64_t cap,
                              const int32_t* n_valid, int64_t B, uint32_t* hists, int pass,
                              uint32_t* flag, cudaStream_t s) {
    dim3 grid(static_cast<unsigned>((cap + kZChunk - 1) / kZChunk), static_cast<unsigned>(n_units));
    radix_pass_kernel<<<grid, 256, 0, s>>>(fin, n_units, cap, n_valid, B, hists, pass, flag);
    note_launch(s);
    return cudaGetLastError();
}

cudaError_t launch_select_finish(const float* fin, int64_t n_units, int64_t cap,
                                 const int32_t* n_valid, int64_t B, const uint32_t* hists,
                                 uint2* counts, int32_t* kept, int32_t* n_kept, cudaStream_t s) {
    dim3 grid(static_cast<unsigned>((cap + kZChunk - 1) / kZChunk), static_cast<unsigned>(n_units));
    select_count_kernel<<<grid, 256, 0, s>>>(fin, n_units, cap, n_valid, B, hists, counts);
    note_launch(s);
    select_compact_kernel<<<grid, 256, 0, s>>>(fin, n_units, cap, n_valid, B, hists, counts, kept,
                                               n_kept);
    note_launch(s);
    return cudaGetLastError();
}

}  // namespace tri
