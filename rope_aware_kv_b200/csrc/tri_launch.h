// tri_launch.h -- host-side launch interfaces between the libtri translation
// units (not part of the public C ABI, which is include/tri.h).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/tri.h"

namespace tri {

constexpr int kZChunk = 2048;      // keys per CTA in the z-max / radix / compaction kernels
constexpr int kHistBins0 = 2048;   // bins of the first (and largest) radix digit
constexpr int kShift0 = 21;        // the first digit is key bits 31..21

struct FoldOffsets {
    int n;
    int64_t v[TRI_MAX_OFFSETS];
};

// Config-only fold factors (RoPE frequencies w_f and the offset-averaged
// phasor C_f = (1/|D|) sum_delta e^{i w_f delta}), formed once per call by the
// host code of the library in float64 and passed as a kernel parameter.
struct FoldConst {
    double omega[64];
    double cf[64][2];
    int variant;  // TRI_VAR_* bits (the fold applies NO_TRIG and NO_R)
};

// Static shared memory of the fused and cooperative kernels (the fold's
// per-unit phases), counted in their shared-memory budgets.
constexpr size_t kFoldStaticBytes = 4096;

// Paged cache layout: logical row j of unit u lives in physical page
// table[u * per_unit + j / rows] of a pool of n_pages pages of `rows` rows.
// With no table the layout is contiguous: unit u's rows start at u * cap.
struct PageMap {
    const int32_t* table = nullptr;
    int64_t rows = 0;
    int64_t per_unit = 0;
    int64_t n_pages = 0;
};

// Physical row of logical row j of unit u, or -1 when its page index is
// outside the pool.
__device__ __forceinline__ int64_t phys_row(const PageMap& pm, int64_t u, int64_t cap, int64_t j) {
    if (!pm.table) return u * cap + j;
    const int64_t pg = pm.table[u * pm.per_unit + j / pm.rows];
    if (pg < 0 || pg >= pm.n_pages) return -1;
    return pg * pm.rows + j % pm.rows;
}

struct ScoreArgs {
    const void* keys;            // [U][cap][128] (for L2 prefetch; loads go through the map)
    int64_t n_units;
    int64_t cap;
    int64_t tpu;                 // tiles per unit
    const int32_t* n_valid;
    const float* wts;            // fold output, [U*G][192]
    float* raw;                  // [U][G][cap]
    double* partial;             // [U][tpu][G][2]
    uint32_t* counters;          // [U], zero on entry
    float2* mom;                 // [U][G] (mu, 1/sigma)
    uint32_t* flag;
    PageMap pm;                  // paged key pool (table null: contiguous [U][cap])
};

struct FusedArgs {
    int64_t n_units;
    int stages;                  // TMA ring depth, 4..6
    // fold inputs (the kernel forms the per-head weights itself)
    const float* stats;          // [L][Hkv*G][64][4]
    const int64_t* p_cur;        // [n_seq]
    int64_t n_layers;
    int64_t n_kvheads;
    FoldConst fc;
    int64_t cap;
    int64_t cap_dst;
    int64_t B;
    const int32_t* n_valid;
    const void* k_src;
    const void* v_src;
    const int32_t* pos_src;
    void* k_dst;
    void* v_dst;
    int32_t* pos_dst;
    int32_t* kept;               // [U][B] or null
    int32_t* n_kept;             // [U]
    float* final_out;            // [U][cap] final scores, or null
    float* scratch;              // [grid][G][cap] per-CTA score scratch
    uint64_t* trace;             // [U][kTracePoints] phase timestamps, or null
    uint32_t* flag;
};

// The pipelined kernel (pipe.cu).
struct PipeArgs {
    int64_t n_units;
    int gslots;                  // gather buffers (shared memory permitting)
    int64_t cap;
    int64_t cap_dst;
    int64_t B;
    const int32_t* n_valid;
    // fold inputs of the small-unit mode (the kernel forms the weights itself)
    const float* stats;          // [L][Hkv*G][64][4]
    const int64_t* p_cur;        // [n_seq]
    int64_t n_layers;
    int64_t n_kvheads;
    FoldConst fc;
    const float* wts;            // large-unit mode: fold output [U*G][192]
    const void* k_src;
    const void* v_src;
    const int32_t* pos_src;
    void* k_dst;
    void* v_dst;
    int32_t* pos_dst;
    int inplace;                 // destinations are the sources (cap_dst == cap)
    int64_t n_sink;              // protected first keys of every unit
    int64_t n_recent;            // protected last keys of every unit
    const int32_t* ub;           // [U] per-unit budgets (<= B) or null
    int32_t* kept;               // [U][B] or null
    int32_t* n_kept;             // [U]
    float* final_out;            // [U][cap] or null
    float* raw;                  // small: [grid][G][cap]; large: [U][G][cap]
    float* fin_scratch;          // large: [grid][cap] (when final_out is null)
    double* partial;             // large: [U][chunks][G][2]
    uint32_t* counters;          // large: [U], zero on entry
    uint32_t* queue;             // large: work-item counter, zero on entry
    uint64_t* trace;             // [U][kTracePoints][kTraceWarps] or null (small mode)
    uint32_t* flag;
};

constexpr int kTracePoints = 8;  // phase points per unit (fused) or CTA (coop)
constexpr int kTraceWarps = 8;   // one slot per warp

// Threshold-bin candidates one unit of the cooperative path can exchange
// (8 bytes each; staged in the CTA's TMA ring of at least 2 x 32 KB).
constexpr int kCandMax = 8192;
// Most CTAs the cooperative path splits one unit over (a multiple of 32).
constexpr int kMaxCtasPerUnit = 160;

struct CoopArgs {
    int64_t n_units;
    const float* stats;          // fold inputs, as in FusedArgs
    const int64_t* p_cur;
    int64_t n_layers;
    int64_t n_kvheads;
    FoldConst fc;
    int64_t cap;
    int64_t cap_dst;
    int64_t B;
    int64_t keys_max;            // most keys one CTA takes
    int stages;                  // TMA ring depth
    int ctas_per_unit;           // C
    uint64_t barrier_wait_ns;    // bound of each unit-barrier wait
    const int32_t* n_valid;
    const void* k_src;
    const void* v_src;
    const int32_t* pos_src;
    void* k_dst;
    void* v_dst;
    int32_t* pos_dst;
    int32_t* kept;               // [U][B] or null
    int32_t* n_kept;             // [U]
    float* final_out;            // [U][cap] final scores, or null
    float* scratch;              // [grid][G][keys_max]
    double* partial;             // [U][C][G][2]
    uint32_t* hists;             // [U][2048] z-bin histograms, zero on entry
    uint32_t* hists_key;         // [3][U][2048] full-key digits (zeroed in the kernel)
    uint2* counts;               // [U][C]
    uint32_t* bar;               // [U], zero on entry
    uint32_t* cand_count;        // [U], zero on entry
    int2* cand;                  // [U][kCandMax] (ordered key, key index)
    uint64_t* trace;             // [grid][kTracePoints][kTraceWarps] or null
    uint32_t* flag;
};


// api.cu: byte offsets of the selection's scratch from `start` (the flag
// word comes first): three radix histograms per unit, then per-chunk
// counts.  Shared by tri_select_topB and its static-scratch variant.
struct SelectWs {
    size_t hists, counts, total;
};
SelectWs select_ws(size_t start, int64_t n_units, int64_t cap);

// api.cu: every exported call that launches kernels starts a fresh launch
// count for tri_last_launch_count.
void begin_launches();

// api.cu: the caller's phase-trace buffer for the next launches (or null).
uint64_t* phase_trace_buffer(int64_t n_units);

// api.cu: call after every kernel launch (counts launches and records the
// caller's timing event for that launch, if any).
void note_launch(cudaStream_t s);

// calibrate.cu
size_t calibrate_ws_bytes(int64_t n_heads, int64_t n_tok);
// qpos (nullable): positions of post-RoPE rows, rotated back first; half:
// half-split band pairing.
cudaError_t launch_calibrate(const void* q, tri_dtype dt, int64_t n_heads, int64_t n_tok,
                             float* stats, void* ws, cudaStream_t s,
                             const int32_t* qpos = nullptr, int half = 0, double theta = 10000.0);

// score.cu
int score_tile_keys(tri_dtype dt);
cudaError_t launch_fold(const float* stats, const int64_t* p_cur, int64_t n_seq, int64_t n_layers,
                        int64_t n_qheads, double theta, const FoldOffsets& off, int variant,
                        float* wts, cudaStream_t s);
cudaError_t launch_score(tri_dtype dt, int G, const CUtensorMap& map, const ScoreArgs& a,
                         int n_sm, cudaStream_t s);
// hist0 (nullable): per-unit histogram of the final scores, of their z-bins
// (zbins != 0) or of their first radix digit.
// Keys j < n_sink or j >= n_valid - n_recent get the final score +inf
// (protected: kept before every other key).
cudaError_t launch_zmax(int G, const float* raw, int64_t n_units, int64_t cap,
                        const int32_t* n_valid, const float2* mom, float* fin, uint32_t* hist0,
                        int zbins, int64_t n_sink, int64_t n_recent, uint32_t* flag,
                        cudaStream_t s);

// variant.cu: the max-over-offsets and half-split variants of the score,
// two-pass moments, per-layer budgets to per-unit budgets.
size_t variant_score_smem();
cudaError_t launch_variant_score(tri_dtype dt, int G, const void* keys, int64_t n_units,
                                 int64_t cap, const int32_t* n_valid, const float* wts,
                                 const float* stats, const int64_t* p_cur, int64_t n_layers,
                                 int64_t n_kvheads, double theta, const FoldOffsets& off,
                                 int variant, float* raw, uint32_t* flag, cudaStream_t s,
                                 const PageMap& pm = PageMap());
cudaError_t launch_moments(const float* raw, int64_t n_units, int64_t cap, const int32_t* n_valid,
                           int G, float2* mom, cudaStream_t s);
cudaError_t launch_unit_budget(const int32_t* layer_budget, int64_t n_units, int64_t n_layers,
                               int64_t n_kvheads, int32_t* ub, cudaStream_t s);

// decode.cu: attention of one query token per head over the cache rows.
int decode_splits(int64_t n_units, int64_t cap, int n_sm);
size_t decode_part_bytes(int64_t n_units, int G, int64_t cap, int n_sm);
cudaError_t launch_decode(tri_dtype dt, int G, const void* q, const void* k, const void* v,
                          int64_t n_units, int64_t cap, const int32_t* n_valid, float scale,
                          float* out, float* part, uint32_t* flag, int n_sm, cudaStream_t s);

// logit.cu: logit(Delta) from the centres, measured, and their correlation.
cudaError_t launch_logit_reconstruct(const float* qs, const float* ks, int64_t n_qheads, int G,
                                     double theta, const int64_t* deltas, int64_t n_delta,
                                     float* recon, cudaStream_t s);
cudaError_t launch_logit_curve(tri_dtype dt, const void* q, const void* k, int64_t n_qheads, int G,
                               int64_t n_tok, const int64_t* deltas, int64_t n_delta, float* curve,
                               cudaStream_t s);
cudaError_t launch_pearson(const float* a, const float* b, int64_t n_rows, int64_t n, float* r,
                           cudaStream_t s);

// zselect.cu: top-B by z-bins on the split path (zhist from launch_zmax with
// zbins; counts [U][chunks] and cand [U][kCandMax] scratch, cand_count [U]
// zero on entry, state [U] of zsel_state_bytes()).
size_t zsel_state_bytes();
// ub (nullable): per-unit budgets [U] (clamped to [0, B]); B is the row
// stride of kept.
cudaError_t launch_zselect(const float* fin, int64_t n_units, int64_t cap, const int32_t* n_valid,
                           int64_t B, const int32_t* ub, const uint32_t* zhist, uint2* counts,
                           int2* cand, uint32_t* cand_count, void* state, int32_t* kept,
                           int32_t* n_kept, cudaStream_t s);

// select.cu
cudaError_t launch_radix_pass(const float* fin, int64_t n_units, int64_t cap,
                              const int32_t* n_valid, int64_t B, uint32_t* hists, int pass,
                              uint32_t* flag, cudaStream_t s);
cudaError_t launch_select_finish(const float* fin, int64_t n_units, int64_t cap,
                                 const int32_t* n_valid, int64_t B, const uint32_t* hists,
                                 uint2* counts, int32_t* kept, int32_t* n_kept, cudaStream_t s);

// compact.cu
cudaError_t launch_gather(tri_dtype dt, const void* k_src, const void* v_src,
                          const int32_t* pos_src, int64_t n_units, int64_t cap_src,
                          const int32_t* kept, const int32_t* n_kept, int64_t B, void* k_dst,
                          void* v_dst, int32_t* pos_dst, int64_t cap_dst, uint32_t* flag,
                          int n_blocks, cudaStream_t s);
// pm: paged K/V pool (positions stay [U][cap]); default contiguous.
cudaError_t launch_compact_inplace(tri_dtype dt, void* k, void* v, int32_t* pos, int64_t n_units,
                                   int64_t cap, const int32_t* kept, const int32_t* n_kept,
                                   int64_t B, uint32_t* flag, int n_blocks, cudaStream_t s,
                                   const PageMap& pm = PageMap());
cudaError_t launch_append(tri_dtype dt, void* k_cache, void* v_cache, int32_t* pos_cache,
                          int64_t n_seq, int64_t n_units, int64_t cap, int32_t* n_valid,
                          int64_t* p_cur, const void* k_new, const void* v_new,
                          const int32_t* pos_new, int64_t n_new, uint32_t* flag, cudaStream_t s);

// coop.cu
size_t coop_smem_bytes(tri_dtype dt, int G, int64_t keys_max, int stages);
int coop_tile_keys(tri_dtype dt);
int coop_max_stages();
cudaError_t launch_coop(tri_dtype dt, int G, const CUtensorMap& map, const CoopArgs& a,
                        int n_ctas, cudaStream_t s);

// fused.cu
size_t fused_smem_bytes(tri_dtype dt, int G, int64_t cap, int64_t B, int stages);
int fused_max_stages();
size_t fused_smem_limit();
int fused_tile_keys(tri_dtype dt);
cudaError_t launch_fused(tri_dtype dt, int G, const CUtensorMap& map, const FusedArgs& a,
                         int n_ctas, cudaStream_t s);

// pipe.cu
size_t pipe_smem_bytes(tri_dtype dt, int G, int64_t cap, int64_t B, bool big, int gslots);
int pipe_min_gslots();
int pipe_max_gslots();
bool pipe_small_fits(tri_dtype dt, int64_t cap);
bool pipe_big_fits(int64_t cap);
int pipe_slice_bytes(bool big);
int pipe_engine_warps();
int pipe_tile_keys(tri_dtype dt);
int pipe_chunk_keys(tri_dtype dt);
cudaError_t launch_pipe(tri_dtype dt, int G, bool big, const CUtensorMap& map, const PipeArgs& a,
                        int n_ctas, cudaStream_t s);

}  // namespace tri
