/*
 * tri.h -- C ABI of libtri, a B200 (sm_100a) implementation of the KV-cache
 * pruning hot path of TriAttention ("TriAttention: Efficient Long Reasoning
 * with Trigonometric KV Compression", arXiv 2604.04921).
 *
 * The method, as the pages state it:
 *   - RoPE rotates each pair (x_2f, x_2f+1) of a d-wide head vector by the
 *     angle w_f p, w_f = theta^(-2f/d), theta = 10000
 *     (TriAttention talk announcement, qingkeai.online: RoPE rotation equation;
 *     hyper.ai summary of arXiv 2604.04921, Method section).
 *   - Offline calibration collects, per query head and band f, the centre
 *     E[q_f], the mean norm E[|q_f|] and R_f = |E[q_f]| / E[|q_f|] from
 *     pre-RoPE queries (talk page: S_norm equation and the R_f definition;
 *     shibing624 paper reading, "complete scoring framework", step 1).
 *   - Each cached key k is scored with
 *         S_trig(k, Delta) = sum_f |E[q_f]| |k_f| cos(w_f Delta + phi_f)
 *         S_norm(k)        = sum_f (1 - R_f) E[|q_f|] |k_f|
 *     averaged over the future offsets D = {1, 2, 4, ..., 2^16}
 *     (talk page: S_trig, S_norm and the offset-averaged score S~).
 *   - Scores are z-normalised per query head and combined by max over each
 *     GQA group (hyper.ai summary, Method section, "normalise then aggregate").
 *   - The top-B keys are kept in their original temporal order and K/V are
 *     gathered into a compacted cache (jaedaily.cn KV-compression tutorial,
 *     eviction step: top-k, then sort to keep the temporal order).
 *   - Scoring and pruning fire once every 128 generated tokens (hyper.ai
 *     summary, Method section).
 *
 * How the library computes S~ (exact algebra, no approximation): with
 * phi_f = arg E[q_f] - arg k_f, the trigonometric term of band f equals
 * Re(E[q_f] conj(k_f) e^{i w_f Delta}).  The pre-RoPE key is
 * k_f = k'_f e^{-i w_f p_k} and Delta = p_cur + delta - p_k, so the key's own
 * position cancels and the average over D is Re(A_f conj(k'_f)) with
 * A_f = E[q_f] e^{i w_f p_cur} C_f and C_f = (1/|D|) sum_delta e^{i w_f delta}.
 * The per-head fold A_f is computed in float64 on the device; the per-key work
 * is one 128-wide dot product plus 64 band norms per query head, in float32.
 *
 * Conventions shared by every call
 * --------------------------------
 * Pointers are DEVICE pointers unless a comment says "host".  The caller
 * allocates every buffer, including the workspace ("ws"); the library
 * allocates, frees and retains nothing and keeps no state between calls,
 * except three per-host-thread profiling settings (tri_set_timing_events,
 * tri_set_phase_trace, tri_last_launch_count) and the cached device address
 * of tri_select_topB_static's static scratch.
 * Calls are asynchronous on the given CUDA stream ("stream" is a
 * cudaStream_t passed as void*; NULL is the legacy default stream) and are
 * safe to capture in a CUDA graph.  Two calls that share a workspace must not
 * overlap on the GPU.
 *
 * Layouts:
 *   unit u = (seq * n_layers + layer) * n_kvheads + kvh: one KV head's cache.
 *   K, V:   [U][cap][head_dim] row-major, element type dt, 16-byte aligned.
 *   pos:    [U][cap] int32 token positions of the cached rows.
 *   n_valid:[U] int32 number of valid rows of each unit (NULL: every unit
 *           holds cap rows).  Rows >= n_valid are ignored.
 *   p_cur:  [n_seq] int64 current position of each sequence (the position of
 *           the next query).  Future queries sit at p_cur + delta.
 *   stats:  [n_layers][n_kvheads * G][head_dim/2][4] float32 calibration
 *           (Re E[q_f], Im E[q_f], E[|q_f|], R_f); query head kvh*G + g
 *           belongs to KV head kvh (contiguous GQA groups).
 *
 * Selection semantics: keys are ranked by final score descending; NaN ranks
 * below every number; -0.0 equals +0.0; equal scores rank by ascending index.
 * The kept set is the first min(B, n_valid) keys of that ranking, written in
 * ascending index order.
 *
 * Errors: arguments are validated on the host before anything is launched
 * (TRI_ERR_INVALID_ARG, TRI_ERR_UNSUPPORTED, TRI_ERR_WORKSPACE); a failed
 * launch returns TRI_ERR_CUDA.  Conditions only the device can see (n_valid
 * outside [0, cap], a kept index outside the source cache, a non-finite final
 * score) set bits in a flag word at the start of the workspace, which each
 * call clears when it starts; tri_check_device_error reads it.
 */
#ifndef TRI_H_
#define TRI_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum tri_status {
    TRI_OK = 0,
    TRI_ERR_INVALID_ARG = 1, /* null / misaligned pointer, bad size or shape */
    TRI_ERR_UNSUPPORTED = 2, /* valid but not implemented (head_dim, G, dtype) */
    TRI_ERR_WORKSPACE = 3,   /* ws is NULL or smaller than the *_workspace_bytes query */
    TRI_ERR_CUDA = 4,        /* a CUDA runtime call or kernel launch failed */
    TRI_ERR_DEVICE = 5,      /* tri_check_device_error found a device-side flag */
    TRI_ERR_SCRATCH_LIMIT = 6 /* the request needs more than the static scratch holds */
} tri_status;

typedef enum tri_dtype {
    TRI_F32 = 0, /* IEEE float32 */
    TRI_BF16 = 1 /* bfloat16 */
} tri_dtype;

/* Device flag bits (tri_check_device_error). */
#define TRI_FLAG_NVALID_RANGE 0x1u /* some n_valid[u] outside [0, cap]; clamped */
#define TRI_FLAG_INDEX_RANGE 0x2u  /* a kept index outside [0, cap_src) or n_kept > B; row skipped */
#define TRI_FLAG_NONFINITE 0x4u    /* a final score was NaN (ranked last) */
#define TRI_FLAG_TIMEOUT 0x8u      /* a bounded wait inside a kernel gave up */

#define TRI_MAX_OFFSETS 64
#define TRI_MAX_GROUP 8

/* Method parameters.  tri_config_default fills the pages' values. */
/* Kernel path of tri_prune. */
#define TRI_PATH_AUTO 0  /* coop for fewer units than SMs, else pipe, else split */
#define TRI_PATH_FUSED 1 /* one CTA per unit (TRI_ERR_UNSUPPORTED if it does not fit) */
#define TRI_PATH_SPLIT 2 /* separate score / z-max / select / gather kernels */
#define TRI_PATH_COOP 3  /* each unit split over several CTAs of one kernel (few large units) */
#define TRI_PATH_PIPE 4  /* persistent kernel, gather of one unit overlapping the next's score */

/* Method variants (tri_config.variant bits; 0 is the method as the pages'
 * main text states it).  Ablations of the shibing624 paper reading's
 * ablation section and alternatives the pages name:
 *   TRI_VAR_NO_TRIG     S_trig left out: the score is S_norm alone;
 *   TRI_VAR_NO_R        the norm weight E[|q_f|] without the (1 - R_f) factor;
 *   TRI_VAR_MAX_OFFSET  the maximum over the offsets D of S_trig + S_norm
 *                       instead of their mean (future-offset paragraph: the
 *                       maximum is the key's score);
 *   TRI_VAR_HALF_SPLIT  band f pairs components (x_f, x_{f+d/2}), the
 *                       rotate-half RoPE layout, for keys and (tri_calibrate_ex)
 *                       queries, instead of (x_2f, x_2f+1).
 * NO_TRIG and NO_R change only the folded weights and run on every path;
 * MAX_OFFSET and HALF_SPLIT run on the split path (TRI_PATH_AUTO takes it;
 * another forced path returns TRI_ERR_UNSUPPORTED). */
#define TRI_VAR_NO_TRIG 0x1
#define TRI_VAR_NO_R 0x2
#define TRI_VAR_MAX_OFFSET 0x4
#define TRI_VAR_HALF_SPLIT 0x8
#define TRI_VAR_ALL 0xf

typedef struct tri_config {
    int head_dim;                      /* d; 128 is supported */
    double theta;                      /* RoPE base, 10000 */
    int n_offsets;                     /* |D|, 1..TRI_MAX_OFFSETS */
    int64_t offsets[TRI_MAX_OFFSETS];  /* future offsets delta >= 0 */
    int path;                          /* TRI_PATH_* (tri_prune only) */
    int variant;                       /* TRI_VAR_* bits, 0 by default */
    /* Protected keys (jaedaily.cn tutorial, streaming section: the most
     * recent tokens are kept from eviction): keys j < n_sink and
     * j >= n_valid - n_recent of every unit get the final score +inf, so
     * they rank before every other key (ties by index: the lowest-indexed
     * protected keys when they alone exceed the budget).  Both 0 by default. */
    int64_t n_sink;
    int64_t n_recent;
    /* Per-layer budgets (same tutorial, budget paragraph: pyramid-shaped
     * budgets per layer): device array [n_layers], entry l the budget of
     * every unit of layer l, clamped to [0, B]; B remains the row stride of
     * kept_idx and the bound of cap_dst.  NULL: B everywhere (tri_prune only). */
    const int32_t* layer_budget;
    /* Bound, in nanoseconds, of each wait at the unit-wide barriers of the
     * cooperative path (TRI_PATH_COOP); 0: 2 s.  A wait that runs out sets
     * TRI_FLAG_TIMEOUT and its CTA skips the rest of the unit (no copy is in
     * flight into its shared memory at any unit barrier), so the call's
     * outputs for that unit are incomplete; the next call starts clean.  Only
     * for testing the timeout path: production calls leave it 0. */
    int64_t barrier_wait_ns;
} tri_config;

/* Fill cfg (host) with head_dim, theta = 10000, D = {2^0, ..., 2^16}
 * (talk page, offset-averaged score S~), TRI_PATH_AUTO and no variant,
 * protection or per-layer budget.
 * Protection and per-layer budgets run on the pipelined and split paths
 * (TRI_PATH_AUTO picks one; TRI_PATH_FUSED or TRI_PATH_COOP returns
 * TRI_ERR_UNSUPPORTED). */
void tri_config_default(tri_config* cfg, int head_dim);

/* Human-readable name of a status code (static string). */
const char* tri_status_str(tri_status s);

/* Library version string (static). */
const char* tri_version(void);

/* ---------------------------------------------------------------------- */
/* Calibration (offline, once per model)                                   */
/* ---------------------------------------------------------------------- */

/* Workspace bytes tri_calibrate needs for n_heads heads of n_tok tokens. */
size_t tri_calibrate_workspace_bytes(int64_t n_heads, int64_t n_tok, int head_dim);

/*
 * Per-head, per-band query statistics from pre-RoPE queries
 * (talk page: R_f = |E[q_f]| / E[|q_f|]; paper reading, offline calibration
 * on about 10K tokens; hyper.ai summary, R = |E[q]| / E[|q|]).
 *   q_pre:  [n_heads][n_tok][head_dim] pre-RoPE queries (dt); n_heads is the
 *           flattened [n_layers][n_qheads].
 *   stats:  out, [n_heads][head_dim/2][4] float32:
 *           Re E[q_f], Im E[q_f], E[|q_f|], R_f (R_f = 1 where E[|q_f|] = 0).
 * Sums are taken in float64 in a fixed order (bitwise deterministic).
 * Errors: n_heads < 1, n_tok < 1, head_dim != 128 or a null pointer ->
 * INVALID_ARG / UNSUPPORTED; ws too small -> TRI_ERR_WORKSPACE.
 */
tri_status tri_calibrate(const void* q_pre, tri_dtype dt, int64_t n_heads, int64_t n_tok,
                         int head_dim, float* stats, void* ws, size_t ws_bytes, void* stream);

/*
 * Calibration with the config's options: head_dim, theta and the band
 * pairing (TRI_VAR_HALF_SPLIT in cfg->variant) from cfg.  q_pos (nullable,
 * device [n_tok] int32): q holds post-RoPE rows, token t at position
 * q_pos[t] in every head; each band is rotated back by -w_f q_pos[t] (the
 * inverse of the talk page's RoPE matrix) before it is averaged, so the
 * statistics are those of the pre-RoPE queries (shibing624 paper reading,
 * Q/K concentration section: the centres live in the pre-RoPE space).  The
 * same call on keys gives the K centres.  Layouts, results and workspace as
 * tri_calibrate.
 */
tri_status tri_calibrate_ex(const tri_config* cfg, const void* q, tri_dtype dt, int64_t n_heads,
                            int64_t n_tok, int head_dim, const int32_t* q_pos, float* stats,
                            void* ws, size_t ws_bytes, void* stream);

/*
 * Calibration split for data-parallel shards of the calibration tokens: each
 * shard reduces its tokens to float64 sums, the shards' sums are added (an
 * all-reduce over the ranks), and the statistics are formed from the totals.
 * Not in the pages (they calibrate offline on one batch); the statistics
 * equal tri_calibrate's on all tokens up to float64 rounding of the sum order.
 *   tri_calibrate_sums: q_pre as in tri_calibrate; sums: out,
 *     [n_heads][head_dim/2][3] float64 = (sum Re q_f, sum Im q_f, sum |q_f|)
 *     over the shard's n_tok tokens; workspace as tri_calibrate's.
 *   tri_calibrate_finish: sums: [n_heads][head_dim/2][3] float64 totals;
 *     n_tok_total: tokens summed (>= 1); stats: out, as tri_calibrate's.
 * Errors as tri_calibrate.
 */
tri_status tri_calibrate_sums(const void* q_pre, tri_dtype dt, int64_t n_heads, int64_t n_tok,
                              int head_dim, double* sums, void* ws, size_t ws_bytes,
                              void* stream);
tri_status tri_calibrate_finish(const double* sums, int64_t n_heads, int64_t n_tok_total,
                                int head_dim, float* stats, void* stream);

/* ---------------------------------------------------------------------- */
/* Score                                                                   */
/* ---------------------------------------------------------------------- */

size_t tri_score_workspace_bytes(int64_t n_seq, int64_t n_layers, int64_t n_kvheads, int G,
                                 int64_t cap, int head_dim);

/*
 * Offset-averaged score S~ of every valid key for each query head of its
 * group, then the GQA "normalise then aggregate" final score (talk page:
 * S_trig, S_norm, S~; hyper.ai summary, Method section).
 *   cfg:    host pointer; theta, offsets, head_dim.
 *   k_post: [U][cap][head_dim] post-RoPE keys (dt), 16-byte aligned.
 *   G:      query heads per KV head, 1..TRI_MAX_GROUP.
 *   raw:    out (nullable), [U][G][cap] float32 per-head S~.
 *   final:  out, [U][cap] float32: max over the group of (S~ - mu_h) / sigma_h,
 *           with mu_h, sigma_h the mean and population standard deviation of
 *           head h's S~ over the unit's n_valid keys (z = 0 where sigma_h = 0).
 * Entries at rows >= n_valid are not written.  Keys' positions are not needed:
 * the fold cancels them exactly (see the header comment).
 */
tri_status tri_score(const tri_config* cfg, const void* k_post, tri_dtype dt, int64_t n_seq,
                     int64_t n_layers, int64_t n_kvheads, int G, int64_t cap,
                     const int32_t* n_valid, const int64_t* p_cur, const float* stats, float* raw,
                     float* final_score, void* ws, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------- */
/* Top-B selection                                                         */
/* ---------------------------------------------------------------------- */

size_t tri_select_workspace_bytes(int64_t n_units, int64_t cap, int64_t B);

/*
 * Keep the top-B keys of each unit by final score, in ascending index order
 * (talk page: keep only the top-B; tutorial eviction step: top-k then sort).
 * MSB-first radix select on order-preserving 32-bit keys; ties at the B-th
 * score go to the lowest indices, so the result is unique and deterministic.
 *   final:    [U][cap] float32 scores.
 *   B:        budget >= 1.
 *   kept_idx: out, [U][B] int32, ascending; slots >= n_kept[u] are set to -1.
 *   n_kept:   out, [U] int32 = min(B, n_valid[u]).
 */
tri_status tri_select_topB(const float* final_score, int64_t n_units, int64_t cap,
                           const int32_t* n_valid, int64_t B, int32_t* kept_idx, int32_t* n_kept,
                           void* ws, size_t ws_bytes, void* stream);

/*
 * tri_select_topB without a workspace, for callers that cannot allocate
 * device memory (a serving engine whose memory manager owns all device memory
 * and hands a plugin only its inputs and outputs; a latency-critical path
 * where cudaMalloc, which may synchronise the device or fail, is forbidden).
 * The pages have no counterpart: this is an integration variant of the
 * selection above and returns exactly its results.
 *
 * The scratch (radix histograms and per-chunk counts) lives in a statically
 * allocated device array of tri_select_static_scratch_bytes() bytes (1 MiB)
 * that every GPU which loads the library reserves until the process exits.
 * Arguments, layouts and results are those of tri_select_topB.  A request
 * whose scratch would not fit (3 * 8 KiB per unit plus 8 bytes per 2048 keys
 * per unit, plus 256 bytes) returns TRI_ERR_SCRATCH_LIMIT before anything is
 * launched; e.g. 40 units of up to 131072 keys fit.  Nothing is allocated:
 * no cudaMalloc, cudaFree or allocating library call.
 *
 * Each call made outside stream capture looks up the array's device address
 * with the device current (cudaGetSymbolAddress) and remembers it for calls
 * made while a stream is being captured, so the first call on a device (and
 * the first after a cudaDeviceReset) must come before any stream capture on
 * it; a captured call with no earlier uncaptured call returns TRI_ERR_CUDA.  Every call shares the one array
 * and clears what must start at zero itself, so calls whose executions overlap
 * on the GPU (different streams, or different host threads) race and must be
 * serialised by the caller.  Device-side flags are not reported.
 */
tri_status tri_select_topB_static(const float* final_score, int64_t n_units, int64_t cap,
                                  const int32_t* n_valid, int64_t B, int32_t* kept_idx,
                                  int32_t* n_kept, void* stream);

/* Size in bytes of the static scratch array of tri_select_topB_static. */
size_t tri_select_static_scratch_bytes(void);

/* ---------------------------------------------------------------------- */
/* Order-preserving compaction                                             */
/* ---------------------------------------------------------------------- */

size_t tri_compact_workspace_bytes(void);

/*
 * Gather the kept rows: for r < n_kept[u],
 *   k_dst[u][r] = k_src[u][kept_idx[u][r]], v_dst likewise, pos_dst likewise
 * (bit copies; tutorial eviction step: keys[idx], values[idx]).
 *   k_src, v_src: [U][cap_src][head_dim] (dt); v_src/v_dst may both be NULL.
 *   pos_src/pos_dst: [U][cap_src] / [U][cap_dst] int32; may both be NULL.
 *   kept_idx: [U][B]; n_kept: [U].
 *   k_dst, v_dst: [U][cap_dst][head_dim], cap_dst >= min(B, cap_src); must not
 *   overlap the sources.
 * Rows r >= n_kept[u] of the destination are left untouched.
 */
tri_status tri_compact(const void* k_src, const void* v_src, const int32_t* pos_src, tri_dtype dt,
                       int64_t n_units, int64_t cap_src, int head_dim, const int32_t* kept_idx,
                       const int32_t* n_kept, int64_t B, void* k_dst, void* v_dst,
                       int32_t* pos_dst, int64_t cap_dst, void* ws, size_t ws_bytes, void* stream);

/*
 * In-place order-preserving compaction of one cache buffer: for r < n_kept[u],
 *   k[u][r] = k[u][kept_idx[u][r]] (as it was on entry), v and pos likewise
 * (tutorial eviction step, keys[idx] / values[idx] kept in temporal order,
 * without a second cache buffer).  kept_idx rows must satisfy
 * kept_idx[u][r] >= r, which every ascending list of distinct indices does
 * (the lists tri_select_topB writes); a row whose index breaks this or lies
 * outside [0, cap) is left unwritten and sets TRI_FLAG_INDEX_RANGE.  Rows
 * that already hold their kept row (the prefix before the first dropped row)
 * are not moved; rows r >= n_kept[u] keep their old contents.
 *   k, v: [U][cap][head_dim] (dt), v nullable; pos: [U][cap] int32, nullable.
 *   The three buffers must not overlap one another.
 *   ws: tri_compact_workspace_bytes() bytes (the device flag word).
 */
tri_status tri_compact_inplace(void* k, void* v, int32_t* pos, tri_dtype dt, int64_t n_units,
                               int64_t cap, int head_dim, const int32_t* kept_idx,
                               const int32_t* n_kept, int64_t B, void* ws, size_t ws_bytes,
                               void* stream);

/* ---------------------------------------------------------------------- */
/* One whole prune step (score + select + compact)                         */
/* ---------------------------------------------------------------------- */

size_t tri_prune_workspace_bytes(int64_t n_seq, int64_t n_layers, int64_t n_kvheads, int G,
                                 int64_t cap, int64_t B, int head_dim);

/*
 * One prune step over every unit of a batch: score, z-normalise and max,
 * select the top-B, gather K, V and positions into the destination cache.
 * Units whose n_valid <= B are copied whole.  With fewer units than SMs, one
 * kernel splits each unit over several CTAs (TRI_PATH_COOP); otherwise one
 * persistent kernel scores, selects and gathers, the gather of each unit
 * overlapping the scoring of the next (TRI_PATH_PIPE; a unit too large for
 * one CTA is scored in chunks by many CTAs and selected by the CTA that
 * completes it); the separate kernels of tri_score / tri_select_topB /
 * tri_compact (TRI_PATH_SPLIT) and the earlier whole-unit fused kernel
 * (TRI_PATH_FUSED) can be forced through cfg->path.  Arguments as in the
 * calls above; kept_idx (nullable, [U][B]) receives the kept indices;
 * n_kept ([U], required) receives min(B, n_valid[u]), the destination's
 * n_valid for the next step; final_score (nullable, [U][cap_src] float32)
 * receives the final scores of tri_score for every unit with n_valid > B
 * (rows of units that are copied whole may be left unwritten).
 */
tri_status tri_prune(const tri_config* cfg, const void* k_src, const void* v_src,
                     const int32_t* pos_src, tri_dtype dt, int64_t n_seq, int64_t n_layers,
                     int64_t n_kvheads, int G, int64_t cap_src, const int32_t* n_valid,
                     const int64_t* p_cur, const float* stats, int64_t B, void* k_dst,
                     void* v_dst, int32_t* pos_dst, int64_t cap_dst, int32_t* kept_idx,
                     int32_t* n_kept, float* final_score, void* ws, size_t ws_bytes,
                     void* stream);

/*
 * The same prune step with the cache compacted in place: the kept rows of
 * unit u end up in rows 0 .. n_kept[u]-1 of k, v and pos themselves, in
 * temporal order, so one cache buffer serves every step (no ping-pong
 * destination).  Arguments as in tri_prune with k_dst = k_src = k (likewise v,
 * pos) and cap_dst = cap_src = cap; k, v and pos must not overlap one
 * another, and n_kept must not be n_valid (a caller that wants the new count
 * in place alternates two count arrays).  Served by the pipelined kernel
 * (its gather stores each piece of destination rows only after every earlier
 * piece's source rows have been read) or by the split kernels ending in the
 * in-place compaction of tri_compact_inplace; cfg->path TRI_PATH_FUSED or
 * TRI_PATH_COOP returns TRI_ERR_UNSUPPORTED.  Workspace:
 * tri_prune_workspace_bytes.
 */
tri_status tri_prune_inplace(const tri_config* cfg, void* k, void* v, int32_t* pos,
                             tri_dtype dt, int64_t n_seq, int64_t n_layers, int64_t n_kvheads,
                             int G, int64_t cap, const int32_t* n_valid, const int64_t* p_cur,
                             const float* stats, int64_t B, int32_t* kept_idx, int32_t* n_kept,
                             float* final_score, void* ws, size_t ws_bytes, void* stream);

/*
 * The in-place prune step on a paged cache (the page-table layout of paged
 * KV caches): the K and V rows of all units live in one pool of n_pages
 * pages of page_rows rows each, [n_pages][page_rows][head_dim] (dt); logical
 * row j of unit u is row j % page_rows of page
 * page_table[u * pages_per_unit + j / page_rows] (device int32).  Logical
 * rows are what every other argument means (n_valid, kept_idx, final_score
 * and the positions pos, which stay [U][cap] int32, nullable): after the
 * call rows 0 .. n_kept[u]-1 of unit u hold its kept rows in temporal order,
 * so the pages past ceil(n_kept[u] / page_rows) hold nothing the unit needs.
 * page_rows is a multiple of 128 (whole score tiles per page) and
 * pages_per_unit * page_rows >= cap; a page index outside [0, n_pages) sets
 * TRI_FLAG_INDEX_RANGE, its keys score as zeros and its rows are not moved.
 * Runs the split kernels (score tiles located through the table, in-place
 * compaction through it); cfg->path other than TRI_PATH_AUTO and
 * TRI_PATH_SPLIT returns TRI_ERR_UNSUPPORTED.  Workspace:
 * tri_prune_workspace_bytes.
 */
tri_status tri_prune_paged_inplace(const tri_config* cfg, void* k_pool, void* v_pool, int32_t* pos,
                                   tri_dtype dt, int64_t n_seq, int64_t n_layers,
                                   int64_t n_kvheads, int G, int64_t cap, const int32_t* n_valid,
                                   const int64_t* p_cur, const float* stats, int64_t B,
                                   const int32_t* page_table, int64_t page_rows,
                                   int64_t pages_per_unit, int64_t n_pages, int32_t* kept_idx,
                                   int32_t* n_kept, float* final_score, void* ws, size_t ws_bytes,
                                   void* stream);

/* The kernel path (TRI_PATH_PIPE, TRI_PATH_COOP, TRI_PATH_FUSED or TRI_PATH_SPLIT) that
 * tri_prune (inplace = 0) or tri_prune_inplace (inplace = 1) takes for these
 * shapes on the current device when cfg->path is `path`; -1 when `path`
 * cannot serve them or the shapes are invalid. */
int tri_prune_path(int64_t n_seq, int64_t n_layers, int64_t n_kvheads, int G, int64_t cap,
                   int64_t B, tri_dtype dt, int path, int inplace);

/* ---------------------------------------------------------------------- */
/* logit(Delta) from the centres, measured, and their correlation          */
/* ---------------------------------------------------------------------- */

/*
 * The attention logit as a trigonometric series in the distance Delta, from
 * the Q and K centres (talk page: RoPE logit general form and the centre
 * approximation q_f ~ E[q_f], k_f ~ E[k_f]):
 *   recon[h][i] = sum_f |E q_f| |E k_f| cos(w_f deltas[i] + arg E q_f - arg E k_f)
 * with w_f = theta^(-2f/d) (cfg->theta).  q_stats: [n_qheads][64][4] and
 * k_stats: [n_qheads / G][64][4] as tri_calibrate / tri_calibrate_ex write
 * them (keys calibrated like queries give the K centres); query head h uses
 * KV head h / G.  deltas: device int64 [n_delta]; recon: [n_qheads][n_delta]
 * float32 (float64 inside).  No workspace.
 */
tri_status tri_logit_reconstruct(const tri_config* cfg, const float* q_stats,
                                 const float* k_stats, int64_t n_qheads, int G,
                                 const int64_t* deltas, int64_t n_delta, float* recon,
                                 void* stream);

/*
 * The measured counterpart on one sequence of post-RoPE rows, token t at
 * position t:  curve[h][i] = mean over t of q[h][t] . k[h / G][t - deltas[i]]
 * over the pairs inside [0, n_tok) (0 when there is none).  q_post:
 * [n_qheads][n_tok][head_dim], k_post: [n_qheads / G][n_tok][head_dim] (dt);
 * deltas: device int64 [n_delta]; curve: [n_qheads][n_delta] float32.
 */
tri_status tri_logit_curve(const void* q_post, const void* k_post, tri_dtype dt, int64_t n_qheads,
                           int G, int64_t n_tok, int head_dim, const int64_t* deltas,
                           int64_t n_delta, float* curve, void* stream);

/* Pearson correlation of each row of a and b ([n_rows][n] float32) into
 * r[n_rows] (shibing624 paper reading, Fig. 1(D): reconstruction against the
 * measured logits per head); 0 for a constant row. */
tri_status tri_pearson(const float* a, const float* b, int64_t n_rows, int64_t n, float* r,
                       void* stream);

/* ---------------------------------------------------------------------- */
/* Decode attention over the compacted cache                               */
/* ---------------------------------------------------------------------- */

size_t tri_decode_workspace_bytes(int64_t n_units, int G, int64_t cap);

/*
 * Attention of the next token over each unit's kept rows, the softmax
 * renormalised over them (jaedaily.cn tutorial, KV-compression objective:
 * the output over the kept subset S is sum_{j in S} a_j v_j with
 * a_j = exp(s_j) / sum_{j' in S} exp(s_j')):
 *   out[u][h] = sum_{j < n} a_j v[u][j],  s_j = scale * (q[u][h] . k[u][j]),
 *   n = n_valid[u] (NULL: cap); a unit with n = 0 gives zeros.
 *   q: [U][G][head_dim] (dt), the post-RoPE queries of the current token, the
 *      G query heads of unit u's KV head (unit order as tri_prune).
 *   k, v: [U][cap][head_dim] (dt), e.g. tri_prune's destination cache.
 *   scale > 0 (1/sqrt(head_dim) for the usual attention).
 *   out: [U][G][head_dim] float32.
 *   ws: tri_decode_workspace_bytes(U, G, cap) bytes (per-chunk partials when
 *   a unit's keys are split over several CTAs).
 * Float32 accumulation with an online (running-maximum) softmax.
 */
tri_status tri_decode_attention(const void* q, const void* k, const void* v, tri_dtype dt,
                                int64_t n_units, int G, int64_t cap, int head_dim,
                                const int32_t* n_valid, float scale, float* out, void* ws,
                                size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------- */
/* Streaming helper: append generated tokens                               */
/* ---------------------------------------------------------------------- */

/*
 * Append n_new rows per unit to a cache: rows n_valid[u] .. n_valid[u]+n_new-1
 * of unit u receive k_new[u][i], v_new[u][i], pos_new[u][i]; n_valid[u] grows by
 * n_new; p_cur[seq] is set to 1 + the largest position in pos_new of the
 * sequence's units.  Used by the windowed driver that prunes every 128
 * generated tokens (hyper.ai summary, Method section).  A unit whose rows
 * would exceed cap is left unchanged and sets TRI_FLAG_NVALID_RANGE.
 *   k_new, v_new: [U][n_new][head_dim] (dt); pos_new: [U][n_new] int32.
 *   n_valid: in/out [U]; p_cur: out [n_seq] (nullable).
 */
tri_status tri_append(void* k_cache, void* v_cache, int32_t* pos_cache, tri_dtype dt,
                      int64_t n_seq, int64_t n_units, int64_t cap, int head_dim,
                      int32_t* n_valid, int64_t* p_cur, const void* k_new, const void* v_new,
                      const int32_t* pos_new, int64_t n_new, void* ws, size_t ws_bytes,
                      void* stream);

/* ---------------------------------------------------------------------- */
/* Launch accounting (profiling)                                           */
/* ---------------------------------------------------------------------- */

/*
 * Per-kernel timing for the calling host thread.  events (host array of
 * cudaEvent_t handles passed as void*, caller-owned, must stay valid while
 * set) receives one cudaEventRecord on the call's stream right after each
 * kernel the next calls launch: event i after launch i of each call.  Pass
 * (NULL, 0) to stop.  Works under stream capture (the records become graph
 * nodes).  Returns TRI_ERR_INVALID_ARG for n_events < 0 or a NULL array with
 * n_events > 0.
 */
tri_status tri_set_timing_events(void* const* events, int n_events);

/* Number of kernels the most recent tri_* call on this host thread launched
 * (memsets are not counted). */
int tri_last_launch_count(void);

/*
 * Phase tracing for the calling host thread.  When device_buf (device
 * memory, caller-owned, at least n_units * 512 bytes) is set, the fused
 * kernel of tri_prune writes %globaltimer nanoseconds into
 * device_buf[(u * 8 + p) * 8 + w] (uint64): lane 0 of warp w records phase
 * point p of unit u just before the barrier that ends the phase, so a phase
 * ends at the largest w entry.  p = 0: start of the unit; 1: scored;
 * 2: z-max done; 3: selected; 4: gathered.  The cooperative kernel (a few
 * units, each split over several CTAs) indexes by CTA instead of unit and
 * needs grid * 512 bytes: points 0 start, 1 scored, 2 after the first unit
 * barrier, 3 z-max done, 4 after the second barrier, 5 threshold known (past
 * the third barrier), 6 compaction done, 7 gather done.  Pass (NULL, 0) to
 * stop.
 */
tri_status tri_set_phase_trace(void* device_buf, size_t bytes);

/* ---------------------------------------------------------------------- */
/* Device-side error flag                                                  */
/* ---------------------------------------------------------------------- */

/*
 * Synchronise the stream and read the flag word of ws (written by the last
 * call that used ws).  *flags_out (host, nullable) receives the TRI_FLAG_*
 * bits.  Returns TRI_OK when no bit is set, TRI_ERR_DEVICE otherwise, or
 * TRI_ERR_CUDA if the synchronisation fails.
 */
tri_status tri_check_device_error(const void* ws, void* stream, uint32_t* flags_out);

#ifdef __cplusplus
}
#endif

#endif /* TRI_H_ */
