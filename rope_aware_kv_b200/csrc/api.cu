// api.cu -- the libtri C ABI (include/tri.h): host-side argument checks,
// workspace layout, TMA descriptors and kernel dispatch.
//
// Nothing here computes any part of the method; every step runs in the
// kernels of calibrate.cu, score.cu, select.cu, compact.cu and fused.cu.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstring>
#include <mutex>

#include "tri_internal.cuh"
#include "tri_launch.h"
#include "calibrate_dp.h"

using namespace tri;

// Launch accounting for callers that time each kernel (tri_set_timing_events).
namespace {
thread_local cudaEvent_t* t_events = nullptr;
thread_local int t_n_events = 0;
thread_local int t_launches = 0;
}  // namespace

namespace {
thread_local uint64_t* t_trace = nullptr;
thread_local size_t t_trace_bytes = 0;
}  // namespace

uint64_t* tri::phase_trace_buffer(int64_t n_units) {
    if (!t_trace || t_trace_bytes < static_cast<size_t>(n_units) * kTracePoints * kTraceWarps * 8)
        return nullptr;
    return t_trace;
}

void tri::begin_launches() { t_launches = 0; }

SelectWs tri::select_ws(size_t start, int64_t U, int64_t cap) {
    SelectWs w;
    size_t off = start;
    auto take = [&](size_t bytes) {
        const size_t o = off;
        off = (off + bytes + 255) & ~size_t(255);
        return o;
    };
    w.hists = take(static_cast<size_t>(3 * U) * kHistBins0 * 4);
    const int64_t chunks = (cap + kZChunk - 1) / kZChunk;
    w.counts = take(static_cast<size_t>(U * chunks) * 8);
    w.total = off;
    return w;
}

void tri::note_launch(cudaStream_t s) {
    if (t_events && t_launches < t_n_events) {
        // Under stream capture a plain record only marks a dependency; an
        // external record becomes an event-record node that can be timed.
        cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
        cudaStreamIsCapturing(s, &cs);
        if (cs == cudaStreamCaptureStatusActive)
            cudaEventRecordWithFlags(t_events[t_launches], s, cudaEventRecordExternal);
        else
            cudaEventRecord(t_events[t_launches], s);
    }
    ++t_launches;
}

namespace {

constexpr size_t kAlign = 256;

size_t align_up(size_t x) { return (x + kAlign - 1) & ~(kAlign - 1); }

// Workspace carving: returns offsets of consecutive, 256-byte aligned regions.
bool overlaps(const void* a, size_t an, const void* b, size_t bn) {
    const char* pa = static_cast<const char*>(a);
    const char* pb = static_cast<const char*>(b);
    return pa < pb + bn && pb < pa + an;
}

// Whether any destination (K, V, positions; null ones skipped) overlaps any
// source: the gather reads the sources while it writes the destinations.
bool gather_buffers_overlap(const void* k_src, const void* v_src, const void* pos_src,
                            const void* k_dst, const void* v_dst, const void* pos_dst,
                            int64_t n_units, int64_t cap_src, int64_t cap_dst, size_t esz) {
    const size_t sb = static_cast<size_t>(n_units * cap_src) * kD * esz;
    const size_t db = static_cast<size_t>(n_units * cap_dst) * kD * esz;
    const size_t spb = static_cast<size_t>(n_units * cap_src) * 4;
    const size_t dpb = static_cast<size_t>(n_units * cap_dst) * 4;
    const void* src[3] = {k_src, v_src, pos_src};
    const size_t sn[3] = {sb, sb, spb};
    const void* dst[3] = {k_dst, v_dst, pos_dst};
    const size_t dn[3] = {db, db, dpb};
    for (int i = 0; i < 3; ++i)
        for (int j = 0; j < 3; ++j)
            if (src[i] && dst[j] && overlaps(src[i], sn[i], dst[j], dn[j])) return true;
    return false;
}

// The three in-place buffers (K, V, positions; V and positions nullable)
// must be disjoint.
bool inplace_buffers_overlap(const void* k, const void* v, const void* pos, int64_t n_units,
                             int64_t cap, size_t esz) {
    const size_t kb = static_cast<size_t>(n_units * cap) * kD * esz;
    const size_t pb = static_cast<size_t>(n_units * cap) * 4;
    return (v && overlaps(k, kb, v, kb)) || (pos && overlaps(k, kb, pos, pb)) ||
           (v && pos && overlaps(v, kb, pos, pb));
}

struct Carve {
    size_t off = kWsHeader;
    size_t take(size_t bytes) {
        const size_t o = off;
        off = align_up(off + bytes);
        return o;
    }
};

struct DeviceInfo {
    int sm_count = 0;
};

DeviceInfo device_info() {
    static std::mutex mu;
    static DeviceInfo cache[64];
    int dev = 0;
    cudaGetDevice(&dev);
    std::lock_guard<std::mutex> lock(mu);
    DeviceInfo& d = cache[dev & 63];
    if (!d.sm_count) cudaDeviceGetAttribute(&d.sm_count, cudaDevAttrMultiProcessorCount, dev);
    return d;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static std::once_flag once;
    static EncodeTiledFn fn = nullptr;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// 2-D view of a key cache [rows][128] for TMA: boxes of box_bytes (128, 64
// or 32) bytes x box_rows rows, swizzled with the same span.
tri_status make_key_map(CUtensorMap* map, const void* k, tri_dtype dt, int64_t rows,
                        int box_rows, int box_bytes = 128) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return TRI_ERR_CUDA;
    const int esz = dt == TRI_BF16 ? 2 : 4;
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(kD), static_cast<cuuint64_t>(rows)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(kD * esz)};
    const cuuint32_t box[2] = {static_cast<cuuint32_t>(box_bytes / esz),
                               static_cast<cuuint32_t>(box_rows)};
    const cuuint32_t estr[2] = {1, 1};
    const CUresult r = fn(map,
                          dt == TRI_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                         : CU_TENSOR_MAP_DATA_TYPE_FLOAT32,
                          2, const_cast<void*>(k), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE,
                          box_bytes == 32   ? CU_TENSOR_MAP_SWIZZLE_32B
                          : box_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                                            : CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? TRI_OK : TRI_ERR_CUDA;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }
bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3) == 0; }
bool dtype_ok(tri_dtype dt) { return dt == TRI_BF16 || dt == TRI_F32; }

tri_status cuda_status(cudaError_t e) { return e == cudaSuccess ? TRI_OK : TRI_ERR_CUDA; }

#define TRI_TRY(expr)                              \
    do {                                           \
        const tri_status _st = (expr);             \
        if (_st != TRI_OK) return _st;             \
    } while (0)

#define TRI_CUDA(expr)                             \
    do {                                           \
        if ((expr) != cudaSuccess) return TRI_ERR_CUDA; \
    } while (0)

tri_status check_cfg(const tri_config* cfg, FoldOffsets* off) {
    if (!cfg) return TRI_ERR_INVALID_ARG;
    if (cfg->head_dim != kD) return TRI_ERR_UNSUPPORTED;
    if (!(cfg->theta > 1.0) || cfg->n_offsets < 1 || cfg->n_offsets > TRI_MAX_OFFSETS)
        return TRI_ERR_INVALID_ARG;
    if (cfg->path < TRI_PATH_AUTO || cfg->path > TRI_PATH_PIPE) return TRI_ERR_INVALID_ARG;
    if ((cfg->variant & ~TRI_VAR_ALL) != 0 || cfg->n_sink < 0 || cfg->n_recent < 0 ||
        cfg->barrier_wait_ns < 0)
        return TRI_ERR_INVALID_ARG;
    if (cfg->layer_budget && !aligned4(cfg->layer_budget)) return TRI_ERR_INVALID_ARG;
    off->n = cfg->n_offsets;
    for (int i = 0; i < cfg->n_offsets; ++i) {
        if (cfg->offsets[i] < 0) return TRI_ERR_INVALID_ARG;
        off->v[i] = cfg->offsets[i];
    }
    return TRI_OK;
}

// w_f = theta^(-2f/d) and C_f = (1/|D|) sum_delta e^{i w_f delta} in float64
// (talk page: RoPE frequencies and the offset-averaged score S~).  These
// depend on the configuration only.
FoldConst fold_const(const tri_config* cfg) {
    FoldConst fc;
    for (int f = 0; f < kF; ++f) {
        const double w = std::pow(cfg->theta, -2.0 * f / static_cast<double>(kD));
        double cre = 0.0, cim = 0.0;
        for (int i = 0; i < cfg->n_offsets; ++i) {
            const double a = w * static_cast<double>(cfg->offsets[i]);
            cre += std::cos(a);
            cim += std::sin(a);
        }
        fc.omega[f] = w;
        fc.cf[f][0] = cre / cfg->n_offsets;
        fc.cf[f][1] = cim / cfg->n_offsets;
    }
    fc.variant = cfg->variant;
    return fc;
}

// Shape limits shared by score / prune: grid dimensions and 32-bit TMA row
// coordinates.
tri_status check_units(int64_t n_seq, int64_t n_layers, int64_t n_kvheads, int G, int64_t cap) {
    if (n_seq < 1 || n_layers < 1 || n_kvheads < 1 || cap < 1) return TRI_ERR_INVALID_ARG;
    if (G < 1 || G > kMaxG) return TRI_ERR_UNSUPPORTED;
    const int64_t U = n_seq * n_layers * n_kvheads;
    if (U > 65535 || U * cap >= (int64_t(1) << 31) || cap > (int64_t(1) << 30))
        return TRI_ERR_UNSUPPORTED;
    return TRI_OK;
}

// ---- score workspace ----
struct ScoreWs {
    size_t wts, raw, partial, counters, mom, total;
    int64_t tpu;
};

ScoreWs score_ws(int64_t n_seq, int64_t n_layers, int64_t n_kvheads, int G, int64_t cap,
                 tri_dtype dt, bool own_raw) {
    ScoreWs w;
    const int64_t U = n_seq * n_layers * n_kvheads;
    const int tile = score_tile_keys(dt);
    w.tpu = (cap + tile - 1) / tile;
    Carve c;
    w.wts = c.take(static_cast<size_t>(U * G) * kWHead * 4);
    w.raw = own_raw ? c.take(static_cast<size_t>(U * G * cap) * 4) : 0;
    w.partial = c.take(static_cast<size_t>(U * w.tpu * G * 2) * 8);
    w.counters = c.take(static_cast<size_t>(U) * 4);
    w.mom = c.take(static_cast<size_t>(U * G) * 8);
    w.total = c.off;
    return w;
}


// ---- prune workspace ----
struct CoopPlan {
    bool ok = false;
    int ctas_per_unit = 0, stages = 0;
    int64_t keys_max = 0;
};

struct PipePlan {
    bool ok = false;
    bool big = false;   // large-unit mode (chunks, last-arriver selection)
    int gslots = 0;     // gather buffers
    int64_t grid = 0;
    int64_t cpu = 0;    // chunks per unit (large mode)
};

struct PruneWs {
    bool fused = false;
    bool coop = false;
    bool pipe = false;
    CoopPlan cp;
    PipePlan pp;
    size_t queue = 0, counters = 0, wts = 0, raw = 0, fin_scratch = 0;
    size_t zcand = 0, zcount = 0, zstate = 0;  // split path: z-bin selection
    size_t ub = 0;                             // per-unit budgets (per-layer budgets given)
    ScoreWs sc;
    size_t fin = 0, kept = 0;
    SelectWs sel;
    size_t partial = 0, hists = 0, counts = 0, bar = 0, zero_end = 0, hists_key = 0, cand = 0,
           cand_count = 0;
    size_t total = 0;
};

// Deepest TMA ring (4..6 stages of 32 KB) the fused kernel fits in shared
// memory, or 0 when even 4 stages do not fit.
int fused_stages(tri_dtype dt, int G, int64_t cap, int64_t B) {
    for (int st = fused_max_stages(); st >= 4; --st)
        if (fused_smem_bytes(dt, G, cap, B, st) <= fused_smem_limit()) return st;
    return 0;
}

bool use_fused(tri_dtype dt, int G, int64_t cap, int64_t B, int path) {
    const int st = fused_stages(dt, G, cap, B);
    return path == TRI_PATH_FUSED ? st >= 4 : st >= 5;
}

int64_t sm_count_or_default() {
    const int64_t sms = device_info().sm_count;
    return sms > 0 ? sms : 148;
}

// CTAs of the persistent fused kernel: one per SM (its shared memory allows
// no more), never more than the units.
int64_t fused_ctas(int64_t U) {
    const int64_t sms = sm_count_or_default();
    return U < sms ? U : sms;
}

// Cooperative plan: C = floor(SMs / U) CTAs per unit (at most one per key
// tile), each with the deepest TMA ring its keys leave room for.
CoopPlan coop_plan(tri_dtype dt, int G, int64_t U, int64_t cap) {
    CoopPlan p;
    const int64_t sms = sm_count_or_default();
    const int64_t tile = coop_tile_keys(dt);
    const int64_t tiles = (cap + tile - 1) / tile;
    int64_t C = sms / U;
    if (C > tiles) C = tiles;
    if (C > kMaxCtasPerUnit) C = kMaxCtasPerUnit;
    if (C < 2) return p;
    p.keys_max = ((tiles + C - 1) / C) * tile;
    for (int st = coop_max_stages(); st >= 2; --st) {
        if (coop_smem_bytes(dt, G, p.keys_max, st) <= fused_smem_limit()) {
            p.stages = st;
            break;
        }
    }
    if (!p.stages) return p;
    p.ctas_per_unit = static_cast<int>(C);
    p.ok = true;
    return p;
}

// Pipelined kernel: the small-unit mode when a unit's final scores fit its
// idle rings (uint16 indices), else the large-unit mode; either needs its
// shared-memory layout to fit one CTA.
PipePlan pipe_plan(tri_dtype dt, int G, int64_t U, int64_t cap, int64_t B) {
    PipePlan p;
    const int64_t sms = sm_count_or_default();
    const bool small = pipe_small_fits(dt, cap);
    if (!small && !pipe_big_fits(cap)) return p;
    const int e = pipe_engine_warps();
    for (int g = pipe_max_gslots() / e * e; g >= pipe_min_gslots(); g -= e) {
        if (pipe_smem_bytes(dt, G, cap, B, !small, g) <= fused_smem_limit()) {
            p.gslots = g;
            break;
        }
    }
    if (!p.gslots) return p;
    p.ok = true;
    p.big = !small;
    if (small) {
        p.grid = U < sms ? U : sms;
    } else {
        const int64_t ck = pipe_chunk_keys(dt);
        p.cpu = (cap + ck - 1) / ck;
        const int64_t items = U * p.cpu;
        p.grid = items < sms ? items : sms;
    }
    return p;
}

// Rows of a page of a paged pool: whole score tiles (128 bf16 / 64 float32
// keys) per page.
constexpr int64_t kPageRowQuantum = 128;

// Which kernel paths can serve a call: 0 every path; 1 the pipelined and
// split paths (protected keys, per-layer budgets, in-place compaction); 2
// the split path alone (the max-over-offsets and half-split scores).
enum { kAnyPath = 0, kPipeOrSplit = 1, kSplitOnly = 2 };

int path_restriction(const tri_config* cfg, bool inplace) {
    if (cfg->variant & (TRI_VAR_MAX_OFFSET | TRI_VAR_HALF_SPLIT)) return kSplitOnly;
    if (cfg->n_sink > 0 || cfg->n_recent > 0 || cfg->layer_budget || inplace) return kPipeOrSplit;
    return kAnyPath;
}

// In place (destination = source) only the pipelined kernel (one engine
// warp then stores the pieces in order) and the split path (in-place
// compaction kernel) serve.
PruneWs prune_ws(int64_t n_seq, int64_t n_layers, int64_t n_kvheads, int G, int64_t cap,
                 int64_t B, tri_dtype dt, bool own_kept, int path, bool inplace = false,
                 int restrict_to = kAnyPath) {
    PruneWs w;
    const int64_t U = n_seq * n_layers * n_kvheads;
    const int64_t sms = sm_count_or_default();
    if (inplace && restrict_to < kPipeOrSplit) restrict_to = kPipeOrSplit;
    if (restrict_to >= kPipeOrSplit && (path == TRI_PATH_FUSED || path == TRI_PATH_COOP)) return w;
    if (restrict_to >= kSplitOnly && path == TRI_PATH_PIPE) return w;
    if ((path == TRI_PATH_PIPE || path == TRI_PATH_AUTO) && restrict_to < kSplitOnly) {
        const PipePlan pp = pipe_plan(dt, G, U, cap, B);
        const CoopPlan cp0 = path == TRI_PATH_AUTO && restrict_to == kAnyPath
                                 ? coop_plan(dt, G, U, cap)
                                 : CoopPlan();
        // AUTO takes the pipelined kernel for units that fit one CTA (whole
        // units per CTA); units scored in chunks run faster on the split
        // kernels.
        const bool take = pp.ok && (path == TRI_PATH_PIPE || (!pp.big && !(cp0.ok && U < sms)));
        if (take) {
            w.pipe = true;
            w.pp = pp;
            Carve c;
            w.queue = c.take(4);
            w.counters = c.take(static_cast<size_t>(U) * 4);
            w.zero_end = c.off;
            w.ub = c.take(static_cast<size_t>(U) * 4);
            // Score rows are padded to a multiple of 32 keys (16-byte groups).
            const int64_t capP = (cap + 31) & ~int64_t(31);
            if (pp.big) {
                w.wts = c.take(static_cast<size_t>(U * G) * kWHead * 4);
                w.raw = c.take(static_cast<size_t>(U * G * capP) * 4);
                w.partial = c.take(static_cast<size_t>(U * pp.cpu * G * 2) * 8);
                w.fin_scratch = c.take(static_cast<size_t>(pp.grid * capP) * 4);
            } else {
                w.raw = c.take(static_cast<size_t>(pp.grid * G * capP) * 4);
            }
            w.kept = own_kept ? c.take(static_cast<size_t>(U * B) * 4) : 0;
            w.total = c.off;
            return w;
        }
        if (path == TRI_PATH_PIPE) return w;  // not possible: tri_prune reports it
    }
    const bool fused_ok = restrict_to == kAnyPath && path != TRI_PATH_SPLIT &&
                          path != TRI_PATH_COOP && use_fused(dt, G, cap, B, path);
    const CoopPlan cp = restrict_to == kAnyPath && (path == TRI_PATH_AUTO || path == TRI_PATH_COOP)
                            ? coop_plan(dt, G, U, cap)
                            : CoopPlan();
    const bool want_coop =
        path == TRI_PATH_COOP || (path == TRI_PATH_AUTO && cp.ok && (U < sms || !fused_ok));
    if (want_coop && cp.ok) {
        w.coop = true;
        w.cp = cp;
        const int64_t grid = U * cp.ctas_per_unit;
        Carve c;
        w.hists = c.take(static_cast<size_t>(U) * kHistBins0 * 4);
        w.bar = c.take(static_cast<size_t>(U) * 4);
        w.cand_count = c.take(static_cast<size_t>(U) * 4);
        w.zero_end = c.off;
        w.hists_key = c.take(static_cast<size_t>(3 * U) * kHistBins0 * 4);
        w.cand = c.take(static_cast<size_t>(U) * kCandMax * 8);
        w.sc.wts = c.take(256);
        w.sc.raw = c.take(static_cast<size_t>(grid * G * cp.keys_max) * 4);
        w.partial = c.take(static_cast<size_t>(grid * G * 2) * 8);
        w.counts = c.take(static_cast<size_t>(grid) * 8);
        w.kept = own_kept ? c.take(static_cast<size_t>(U * B) * 4) : 0;
        w.total = c.off;
        return w;
    }
    if (path == TRI_PATH_COOP) return w;  // not possible: tri_prune reports it
    w.fused = fused_ok;
    if (w.fused) {
        Carve c;
        w.sc.wts = c.take(256);
        w.sc.raw = c.take(static_cast<size_t>(fused_ctas(U) * G * cap) * 4);
        w.kept = own_kept ? c.take(static_cast<size_t>(U * B) * 4) : 0;
        w.fin = 0;
        w.total = c.off;
        return w;
    }
    w.sc = score_ws(n_seq, n_layers, n_kvheads, G, cap, dt, true);
    Carve c;
    c.off = w.sc.total;
    w.fin = c.take(static_cast<size_t>(U * cap) * 4);
    w.kept = own_kept ? c.take(static_cast<size_t>(U * B) * 4) : 0;
    w.sel = select_ws(c.off, U, cap);
    c.off = w.sel.total;
    w.zcand = c.take(static_cast<size_t>(U) * kCandMax * 8);
    w.zcount = c.take(static_cast<size_t>(U) * 4);
    w.zstate = c.take(static_cast<size_t>(U) * zsel_state_bytes());
    w.ub = c.take(static_cast<size_t>(U) * 4);
    w.total = c.off;
    return w;
}

// Per-head raw scores and their moments (mean, 1/sigma): the TMA score
// kernel, or for the max-over-offsets / half-split variants the variant
// score kernel followed by the moments kernel.
cudaError_t score_any(const tri_config* cfg, const FoldOffsets& off, tri_dtype dt, int G,
                      const CUtensorMap& map, const ScoreArgs& a, const float* stats,
                      const int64_t* p_cur, int64_t n_layers, int64_t n_kvheads, int n_sm,
                      cudaStream_t s) {
    if (cfg->variant & (TRI_VAR_MAX_OFFSET | TRI_VAR_HALF_SPLIT)) {
        cudaError_t e = launch_variant_score(dt, G, a.keys, a.n_units, a.cap, a.n_valid, a.wts,
                                             stats, p_cur, n_layers, n_kvheads, cfg->theta, off,
                                             cfg->variant, a.raw, a.flag, s, a.pm);
        if (e != cudaSuccess) return e;
        return launch_moments(a.raw, a.n_units, a.cap, a.n_valid, G, a.mom, s);
    }
    return launch_score(dt, G, map, a, n_sm, s);
}

// Every exported call that launches kernels starts a fresh launch count.
struct LaunchScope {
    LaunchScope() { begin_launches(); }
};

char* ws_at(void* ws, size_t off) { return static_cast<char*>(ws) + off; }
uint32_t* ws_flag(void* ws) { return reinterpret_cast<uint32_t*>(ws); }

}  // namespace

// ===========================================================================
// Exported C ABI
// ===========================================================================
extern "C" {

void tri_config_default(tri_config* cfg, int head_dim) {
    if (!cfg) return;
    std::memset(cfg, 0, sizeof(*cfg));
    cfg->head_dim = head_dim;
    cfg->theta = 10000.0;
    cfg->n_offsets = 17;
    for (int i = 0; i < 17; ++i) cfg->offsets[i] = int64_t(1) << i;
}

const char* tri_status_str(tri_status s) {
    switch (s) {
        case TRI_OK: return "ok";
        case TRI_ERR_INVALID_ARG: return "invalid argument";
        case TRI_ERR_UNSUPPORTED: return "unsupported shape or type";
        case TRI_ERR_WORKSPACE: return "workspace missing or too small";
        case TRI_ERR_CUDA: return "CUDA error";
        case TRI_ERR_DEVICE: return "device-side flag set";
        case TRI_ERR_SCRATCH_LIMIT: return "request exceeds the static scratch";
    }
    return "unknown status";
}

const char* tri_version(void) { return "libtri 0.1 sm_100a"; }

size_t tri_calibrate_workspace_bytes(int64_t n_heads, int64_t n_tok, int head_dim) {
    (void)head_dim;
    if (n_heads < 1 || n_tok < 1) return kWsHeader;
    return calibrate_ws_bytes(n_heads, n_tok);
}

tri_status tri_calibrate(const void* q_pre, tri_dtype dt, int64_t n_heads, int64_t n_tok,
                         int head_dim, float* stats, void* ws, size_t ws_bytes, void* stream) {
    LaunchScope scope_;
    if (!q_pre || !stats || n_heads < 1 || n_tok < 1) return TRI_ERR_INVALID_ARG;
    if (!dtype_ok(dt)) return TRI_ERR_UNSUPPORTED;
    if (head_dim != kD) return TRI_ERR_UNSUPPORTED;
    if (n_heads > 65535) return TRI_ERR_UNSUPPORTED;
    if (!aligned16(q_pre) || !aligned4(stats)) return TRI_ERR_INVALID_ARG;
    if (!ws || ws_bytes < calibrate_ws_bytes(n_heads, n_tok) || !aligned16(ws))
        return TRI_ERR_WORKSPACE;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    TRI_CUDA(cudaMemsetAsync(ws, 0, kWsHeader, s));
    return cuda_status(launch_calibrate(q_pre, dt, n_heads, n_tok, stats, ws, s));
}

tri_status tri_calibrate_ex(const tri_config* cfg, const void* q, tri_dtype dt, int64_t n_heads,
                            int64_t n_tok, int head_dim, const int32_t* q_pos, float* stats,
                            void* ws, size_t ws_bytes, void* stream) {
    LaunchScope scope_;
    FoldOffsets off;
    TRI_TRY(check_cfg(cfg, &off));
    if (!q || !stats || n_heads < 1 || n_tok < 1) return TRI_ERR_INVALID_ARG;
    if (!dtype_ok(dt)) return TRI_ERR_UNSUPPORTED;
    if (head_dim != kD) return TRI_ERR_UNSUPPORTED;
    if (n_heads > 65535) return TRI_ERR_UNSUPPORTED;
    if (!aligned16(q) || !aligned4(stats) || (q_pos && !aligned4(q_pos))) return TRI_ERR_INVALID_ARG;
    if (!ws || ws_bytes < calibrate_ws_bytes(n_heads, n_tok) || !aligned16(ws))
        return TRI_ERR_WORKSPACE;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    TRI_CUDA(cudaMemsetAsync(ws, 0, kWsHeader, s));
    return cuda_status(launch_calibrate(q, dt, n_heads, n_tok, stats, ws, s, q_pos,
                                        (cfg->variant & TRI_VAR_HALF_SPLIT) ? 1 : 0, cfg->theta));
}

tri_status tri_calibrate_sums(const void* q_pre, tri_dtype dt, int64_t n_heads, int64_t n_tok,
                              int head_dim, double* sums, void* ws, size_t ws_bytes,
                              void* stream) {
    LaunchScope scope_;
    if (!q_pre || !sums || n_heads < 1 || n_tok < 1) return TRI_ERR_INVALID_ARG;
    if (!dtype_ok(dt)) return TRI_ERR_UNSUPPORTED;
    if (head_dim != kD) return TRI_ERR_UNSUPPORTED;
    if (n_heads > 65535) return TRI_ERR_UNSUPPORTED;
    if (!aligned16(q_pre) || (reinterpret_cast<uintptr_t>(sums) & 7)) return TRI_ERR_INVALID_ARG;
    if (!ws || ws_bytes < calibrate_ws_bytes(n_heads, n_tok) || !aligned16(ws))
        return TRI_ERR_WORKSPACE;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    TRI_CUDA(cudaMemsetAsync(ws, 0, kWsHeader, s));
    return cuda_status(launch_calibrate_sums(q_pre, dt, n_heads, n_tok, sums, ws, s));
}

tri_status tri_calibrate_finish(const double* sums, int64_t n_heads, int64_t n_tok_total,
                                int head_dim, float* stats, void* stream) {
    LaunchScope scope_;
    if (!sums || !stats || n_heads < 1 || n_tok_total < 1) return TRI_ERR_INVALID_ARG;
    if (head_dim != kD) return TRI_ERR_UNSUPPORTED;
    if (n_heads > 65535) return TRI_ERR_UNSUPPORTED;
    if ((reinterpret_cast<uintptr_t>(sums) & 7) || !aligned4(stats)) return TRI_ERR_INVALID_ARG;
    return cuda_status(launch_calibrate_finish(sums, n_heads, n_tok_total, stats,
                                               static_cast<cudaStream_t>(stream)));
}

size_t tri_score_workspace_bytes(int64_t n_seq, int64_t n_layers, int64_t n_kvheads, int G,
                                 int64_t cap, int head_dim) {
    (void)head_dim;
    if (check_units(n_seq, n_layers, n_kvheads, G, cap) != TRI_OK) return kWsHeader;
    // Large enough whether or not the caller supplies `raw` (bf16 tiles are
    // the smaller unit, so the bf16 layout bounds both types).
    const size_t a = score_ws(n_seq, n_layers, n_kvheads, G, cap, TRI_BF16, true).total;
    const size_t b = score_ws(n_seq, n_layers, n_kvheads, G, cap, TRI_F32, true).total;
    return a > b ? a : b;
}

tri_status tri_score(const tri_config* cfg, const void* k_post, tri_dtype dt, int64_t n_seq,
                     int64_t n_layers, int64_t n_kvheads, int G, int64_t cap,
                     const int32_t* n_valid, const int64_t* p_cur, const float* stats, float* raw,
                     float* final_score, void* ws, size_t ws_bytes, void* stream) {
    LaunchScope scope_;
    FoldOffsets off;
    TRI_TRY(check_cfg(cfg, &off));
    if (!dtype_ok(dt)) return TRI_ERR_UNSUPPORTED;
    TRI_TRY(check_units(n_seq, n_layers, n_kvheads, G, cap));
    if (!k_post || !p_cur || !stats || !final_score) return TRI_ERR_INVALID_ARG;
    if (!aligned16(k_post) || !aligned4(final_score) || (raw && !aligned4(raw)) ||
        (n_valid && !aligned4(n_valid)) || !aligned4(stats))
        return TRI_ERR_INVALID_ARG;
    const ScoreWs w = score_ws(n_seq, n_layers, n_kvheads, G, cap, dt, raw == nullptr);
    if (!ws || !aligned16(ws) || ws_bytes < w.total) return TRI_ERR_WORKSPACE;
    const int64_t U = n_seq * n_layers * n_kvheads;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    CUtensorMap map;
    TRI_TRY(make_key_map(&map, k_post, dt, U * cap, score_tile_keys(dt)));
    TRI_CUDA(cudaMemsetAsync(ws, 0, kWsHeader, s));
    TRI_CUDA(cudaMemsetAsync(ws_at(ws, w.counters), 0, static_cast<size_t>(U) * 4, s));
    float* wts = reinterpret_cast<float*>(ws_at(ws, w.wts));
    TRI_CUDA(launch_fold(stats, p_cur, n_seq, n_layers, n_kvheads * G, cfg->theta, off,
                         cfg->variant, wts, s));
    ScoreArgs a;
    a.keys = k_post;
    a.n_units = U;
    a.cap = cap;
    a.tpu = w.tpu;
    a.n_valid = n_valid;
    a.wts = wts;
    a.raw = raw ? raw : reinterpret_cast<float*>(ws_at(ws, w.raw));
    a.partial = reinterpret_cast<double*>(ws_at(ws, w.partial));
    a.counters = reinterpret_cast<uint32_t*>(ws_at(ws, w.counters));
    a.mom = reinterpret_cast<float2*>(ws_at(ws, w.mom));
    a.flag = ws_flag(ws);
    TRI_CUDA(score_any(cfg, off, dt, G, map, a, stats, p_cur, n_layers, n_kvheads,
                       device_info().sm_count, s));
    TRI_CUDA(launch_zmax(G, a.raw, U, cap, n_valid, a.mom, final_score, nullptr, 0, cfg->n_sink,
                         cfg->n_recent, a.flag, s));
    return TRI_OK;
}

size_t tri_select_workspace_bytes(int64_t n_units, int64_t cap, int64_t B) {
    (void)B;
    if (n_units < 1 || cap < 1) return kWsHeader;
    return select_ws(kWsHeader, n_units, cap).total;
}

tri_status tri_select_topB(const float* final_score, int64_t n_units, int64_t cap,
                           const int32_t* n_valid, int64_t B, int32_t* kept_idx, int32_t* n_kept,
                           void* ws, size_t ws_bytes, void* stream) {
    LaunchScope scope_;
    if (!final_score || !kept_idx || !n_kept || n_units < 1 || cap < 1 || B < 1)
        return TRI_ERR_INVALID_ARG;
    if (B > INT32_MAX || n_units > 65535 || cap > (int64_t(1) << 30)) return TRI_ERR_UNSUPPORTED;
    if (!aligned4(final_score) || !aligned4(kept_idx) || !aligned4(n_kept) ||
        (n_valid && !aligned4(n_valid)))
        return TRI_ERR_INVALID_ARG;
    const SelectWs w = select_ws(kWsHeader, n_units, cap);
    if (!ws || !aligned16(ws) || ws_bytes < w.total) return TRI_ERR_WORKSPACE;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint32_t* hists = reinterpret_cast<uint32_t*>(ws_at(ws, w.hists));
    TRI_CUDA(cudaMemsetAsync(ws, 0, w.counts, s));  // header + histograms
    for (int p = 0; p < 3; ++p)
        TRI_CUDA(launch_radix_pass(final_score, n_units, cap, n_valid, B, hists, p, ws_flag(ws), s));
    TRI_CUDA(launch_select_finish(final_score, n_units, cap, n_valid, B, hists,
                                  reinterpret_cast<uint2*>(ws_at(ws, w.counts)), kept_idx, n_kept,
                                  s));
    return TRI_OK;
}

size_t tri_compact_workspace_bytes(void) { return kWsHeader; }

tri_status tri_compact(const void* k_src, const void* v_src, const int32_t* pos_src, tri_dtype dt,
                       int64_t n_units, int64_t cap_src, int head_dim, const int32_t* kept_idx,
                       const int32_t* n_kept, int64_t B, void* k_dst, void* v_dst,
                       int32_t* pos_dst, int64_t cap_dst, void* ws, size_t ws_bytes,
                       void* stream) {
    LaunchScope scope_;
    if (!k_src || !k_dst || !kept_idx || !n_kept || n_units < 1 || cap_src < 1 || B < 1)
        return TRI_ERR_INVALID_ARG;
    if (!dtype_ok(dt) || head_dim != kD) return TRI_ERR_UNSUPPORTED;
    if ((v_src == nullptr) != (v_dst == nullptr) || (pos_src == nullptr) != (pos_dst == nullptr))
        return TRI_ERR_INVALID_ARG;
    if (cap_dst < (B < cap_src ? B : cap_src)) return TRI_ERR_INVALID_ARG;
    if (!aligned16(k_src) || !aligned16(k_dst) || (v_src && (!aligned16(v_src) || !aligned16(v_dst))))
        return TRI_ERR_INVALID_ARG;
    const size_t esz = dt == TRI_BF16 ? 2 : 4;
    if (gather_buffers_overlap(k_src, v_src, pos_src, k_dst, v_dst, pos_dst, n_units, cap_src,
                               cap_dst, esz))
        return TRI_ERR_INVALID_ARG;
    if (!ws || ws_bytes < kWsHeader || !aligned16(ws)) return TRI_ERR_WORKSPACE;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    TRI_CUDA(cudaMemsetAsync(ws, 0, kWsHeader, s));
    return cuda_status(launch_gather(dt, k_src, v_src, pos_src, n_units, cap_src, kept_idx, n_kept,
                                     B, k_dst, v_dst, pos_dst, cap_dst, ws_flag(ws),
                                     device_info().sm_count * 8, s));
}

tri_status tri_compact_inplace(void* k, void* v, int32_t* pos, tri_dtype dt, int64_t n_units,
                               int64_t cap, int head_dim, const int32_t* kept_idx,
                               const int32_t* n_kept, int64_t B, void* ws, size_t ws_bytes,
                               void* stream) {
    LaunchScope scope_;
    if (!k || !kept_idx || !n_kept || n_units < 1 || cap < 1 || B < 1) return TRI_ERR_INVALID_ARG;
    if (!dtype_ok(dt) || head_dim != kD) return TRI_ERR_UNSUPPORTED;
    if (!aligned16(k) || (v && !aligned16(v)) || (pos && !aligned4(pos)) || !aligned4(kept_idx) ||
        !aligned4(n_kept))
        return TRI_ERR_INVALID_ARG;
    const size_t esz = dt == TRI_BF16 ? 2 : 4;
    if (inplace_buffers_overlap(k, v, pos, n_units, cap, esz)) return TRI_ERR_INVALID_ARG;
    if (!ws || ws_bytes < kWsHeader || !aligned16(ws)) return TRI_ERR_WORKSPACE;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    TRI_CUDA(cudaMemsetAsync(ws, 0, kWsHeader, s));
    return cuda_status(launch_compact_inplace(dt, k, v, pos, n_units, cap, kept_idx, n_kept, B,
                                              ws_flag(ws), device_info().sm_count * 8, s));
}

size_t tri_prune_workspace_bytes(int64_t n_seq, int64_t n_layers, int64_t n_kvheads, int G,
                                 int64_t cap, int64_t B, int head_dim) {
    (void)head_dim;
    if (check_units(n_seq, n_layers, n_kvheads, G, cap) != TRI_OK || B < 1) return kWsHeader;
    size_t best = 0;
    for (tri_dtype dt : {TRI_BF16, TRI_F32}) {
        for (int path : {TRI_PATH_AUTO, TRI_PATH_FUSED, TRI_PATH_SPLIT, TRI_PATH_COOP,
                         TRI_PATH_PIPE}) {
            const size_t t = prune_ws(n_seq, n_layers, n_kvheads, G, cap, B, dt, true, path).total;
            if (t > best) best = t;
        }
    }
    return best;
}

int tri_prune_path(int64_t n_seq, int64_t n_layers, int64_t n_kvheads, int G, int64_t cap,
                   int64_t B, tri_dtype dt, int path, int inplace) {
    if (check_units(n_seq, n_layers, n_kvheads, G, cap) != TRI_OK || B < 1 || !dtype_ok(dt))
        return -1;
    const PruneWs w = prune_ws(n_seq, n_layers, n_kvheads, G, cap, B, dt, false, path, inplace != 0);
    if (w.pipe) return TRI_PATH_PIPE;
    if (w.coop) return TRI_PATH_COOP;
    if (w.fused) return TRI_PATH_FUSED;
    if (path == TRI_PATH_FUSED || path == TRI_PATH_COOP || path == TRI_PATH_PIPE) return -1;
    return TRI_PATH_SPLIT;
}

// tri_prune and tri_prune_inplace (k_dst == k_src, v_dst == v_src,
// pos_dst == pos_src, cap_dst == cap_src).
static tri_status prune_impl(const tri_config* cfg, const void* k_src, const void* v_src,
                             const int32_t* pos_src, tri_dtype dt, int64_t n_seq,
                             int64_t n_layers, int64_t n_kvheads, int G, int64_t cap_src,
                             const int32_t* n_valid, const int64_t* p_cur, const float* stats,
                             int64_t B, void* k_dst, void* v_dst, int32_t* pos_dst,
                             int64_t cap_dst, int32_t* kept_idx, int32_t* n_kept,
                             float* final_score, void* ws, size_t ws_bytes, void* stream,
                             bool inplace, const PageMap* paged = nullptr) {
    LaunchScope scope_;
    FoldOffsets off;
    TRI_TRY(check_cfg(cfg, &off));
    if (!dtype_ok(dt)) return TRI_ERR_UNSUPPORTED;
    TRI_TRY(check_units(n_seq, n_layers, n_kvheads, G, cap_src));
    if (!k_src || !k_dst || !p_cur || !stats || !n_kept || B < 1) return TRI_ERR_INVALID_ARG;
    if (B > INT32_MAX) return TRI_ERR_UNSUPPORTED;
    if ((v_src == nullptr) != (v_dst == nullptr) || (pos_src == nullptr) != (pos_dst == nullptr))
        return TRI_ERR_INVALID_ARG;
    if (cap_dst < (B < cap_src ? B : cap_src)) return TRI_ERR_INVALID_ARG;
    if (!aligned16(k_src) || !aligned16(k_dst) ||
        (v_src && (!aligned16(v_src) || !aligned16(v_dst))) || !aligned16(stats) ||
        !aligned4(n_kept) || (kept_idx && !aligned4(kept_idx)) || (n_valid && !aligned4(n_valid)) ||
        (final_score && !aligned4(final_score)))
        return TRI_ERR_INVALID_ARG;
    const int64_t U = n_seq * n_layers * n_kvheads;
    const size_t esz = dt == TRI_BF16 ? 2 : 4;
    if (paged) {
        const size_t pool = static_cast<size_t>(paged->n_pages * paged->rows) * kD * esz;
        const size_t pb = static_cast<size_t>(U * cap_src) * 4;
        if ((v_src && overlaps(k_src, pool, v_src, pool)) || (pos_src && overlaps(k_src, pool, pos_src, pb)) ||
            (v_src && pos_src && overlaps(v_src, pool, pos_src, pb)) ||
            (n_valid && static_cast<const void*>(n_valid) == static_cast<const void*>(n_kept)))
            return TRI_ERR_INVALID_ARG;
    } else if (inplace) {
        if (inplace_buffers_overlap(k_src, v_src, pos_src, U, cap_src, esz) ||
            (n_valid && static_cast<const void*>(n_valid) == static_cast<const void*>(n_kept)))
            return TRI_ERR_INVALID_ARG;
    } else if (gather_buffers_overlap(k_src, v_src, pos_src, k_dst, v_dst, pos_dst, U, cap_src,
                                      cap_dst, esz)) {
        return TRI_ERR_INVALID_ARG;
    }
    const int restrict_to = paged ? kSplitOnly : path_restriction(cfg, inplace);
    const PruneWs w = prune_ws(n_seq, n_layers, n_kvheads, G, cap_src, B, dt, kept_idx == nullptr,
                               cfg->path, inplace, restrict_to);
    if (cfg->path == TRI_PATH_FUSED && !w.fused) return TRI_ERR_UNSUPPORTED;
    if (cfg->path == TRI_PATH_COOP && !w.coop) return TRI_ERR_UNSUPPORTED;
    if (cfg->path == TRI_PATH_PIPE && !w.pipe) return TRI_ERR_UNSUPPORTED;
    if (restrict_to >= kPipeOrSplit && (cfg->path == TRI_PATH_FUSED || cfg->path == TRI_PATH_COOP))
        return TRI_ERR_UNSUPPORTED;
    if (restrict_to >= kSplitOnly && cfg->path == TRI_PATH_PIPE) return TRI_ERR_UNSUPPORTED;
    if (!ws || !aligned16(ws) || ws_bytes < w.total) return TRI_ERR_WORKSPACE;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    float* wts = reinterpret_cast<float*>(ws_at(ws, w.sc.wts));
    int32_t* kept = kept_idx ? kept_idx : reinterpret_cast<int32_t*>(ws_at(ws, w.kept));
    uint32_t* flag = ws_flag(ws);
    int32_t* ub = cfg->layer_budget ? reinterpret_cast<int32_t*>(ws_at(ws, w.ub)) : nullptr;
    if (ub)
        TRI_CUDA(launch_unit_budget(cfg->layer_budget, U, n_layers, n_kvheads, ub, s));

    if (w.pipe) {
        CUtensorMap map;
        TRI_TRY(make_key_map(&map, k_src, dt, U * cap_src, pipe_tile_keys(dt),
                             pipe_slice_bytes(w.pp.big)));
        // One memset: the flag word, the work-item queue and the unit counters.
        TRI_CUDA(cudaMemsetAsync(ws, 0, w.zero_end, s));
        PipeArgs a;
        a.n_units = U;
        a.gslots = w.pp.gslots;
        a.cap = cap_src;
        a.cap_dst = cap_dst;
        a.B = B;
        a.n_valid = n_valid;
        a.stats = stats;
        a.p_cur = p_cur;
        a.n_layers = n_layers;
        a.n_kvheads = n_kvheads;
        a.fc = fold_const(cfg);
        a.wts = nullptr;
        a.k_src = k_src;
        a.v_src = v_src;
        a.pos_src = pos_src;
        a.k_dst = k_dst;
        a.v_dst = v_dst;
        a.pos_dst = pos_dst;
        a.inplace = inplace ? 1 : 0;
        a.n_sink = cfg->n_sink;
        a.n_recent = cfg->n_recent;
        a.ub = ub;
        a.kept = kept_idx;
        a.n_kept = n_kept;
        a.final_out = final_score;
        a.raw = reinterpret_cast<float*>(ws_at(ws, w.raw));
        a.fin_scratch = w.pp.big ? reinterpret_cast<float*>(ws_at(ws, w.fin_scratch)) : nullptr;
        a.partial = w.pp.big ? reinterpret_cast<double*>(ws_at(ws, w.partial)) : nullptr;
        a.counters = reinterpret_cast<uint32_t*>(ws_at(ws, w.counters));
        a.queue = reinterpret_cast<uint32_t*>(ws_at(ws, w.queue));
        a.trace = w.pp.big ? nullptr : phase_trace_buffer(U);
        a.flag = flag;
        if (w.pp.big) {
            float* pw = reinterpret_cast<float*>(ws_at(ws, w.wts));
            TRI_CUDA(launch_fold(stats, p_cur, n_seq, n_layers, n_kvheads * G, cfg->theta, off, cfg->variant, pw,
                                 s));
            a.wts = pw;
        }
        return cuda_status(launch_pipe(dt, G, w.pp.big, map, a, static_cast<int>(w.pp.grid), s));
    }

    if (w.coop) {
        CUtensorMap map;
        TRI_TRY(make_key_map(&map, k_src, dt, U * cap_src, coop_tile_keys(dt)));
        // One memset: the flag word, the unit histograms and barrier counters.
        TRI_CUDA(cudaMemsetAsync(ws, 0, w.zero_end, s));
        CoopArgs a;
        a.n_units = U;
        a.stats = stats;
        a.p_cur = p_cur;
        a.n_layers = n_layers;
        a.n_kvheads = n_kvheads;
        a.fc = fold_const(cfg);
        a.cap = cap_src;
        a.cap_dst = cap_dst;
        a.B = B;
        a.keys_max = w.cp.keys_max;
        a.stages = w.cp.stages;
        a.ctas_per_unit = w.cp.ctas_per_unit;
        a.barrier_wait_ns = cfg->barrier_wait_ns > 0 ? static_cast<uint64_t>(cfg->barrier_wait_ns)
                                                     : kWaitLimitNs;
        a.n_valid = n_valid;
        a.k_src = k_src;
        a.v_src = v_src;
        a.pos_src = pos_src;
        a.k_dst = k_dst;
        a.v_dst = v_dst;
        a.pos_dst = pos_dst;
        a.kept = kept_idx;
        a.n_kept = n_kept;
        a.final_out = final_score;
        a.scratch = reinterpret_cast<float*>(ws_at(ws, w.sc.raw));
        a.partial = reinterpret_cast<double*>(ws_at(ws, w.partial));
        a.hists = reinterpret_cast<uint32_t*>(ws_at(ws, w.hists));
        a.hists_key = reinterpret_cast<uint32_t*>(ws_at(ws, w.hists_key));
        a.counts = reinterpret_cast<uint2*>(ws_at(ws, w.counts));
        a.bar = reinterpret_cast<uint32_t*>(ws_at(ws, w.bar));
        a.cand_count = reinterpret_cast<uint32_t*>(ws_at(ws, w.cand_count));
        a.cand = reinterpret_cast<int2*>(ws_at(ws, w.cand));
        a.trace = phase_trace_buffer(U * w.cp.ctas_per_unit);
        a.flag = flag;
        return cuda_status(
            launch_coop(dt, G, map, a, static_cast<int>(U * w.cp.ctas_per_unit), s));
    }

    if (w.fused) {
        CUtensorMap map;
        TRI_TRY(make_key_map(&map, k_src, dt, U * cap_src, fused_tile_keys(dt)));
        TRI_CUDA(cudaMemsetAsync(ws, 0, kWsHeader, s));
        FusedArgs a;
        a.stats = stats;
        a.p_cur = p_cur;
        a.n_layers = n_layers;
        a.n_kvheads = n_kvheads;
        a.fc = fold_const(cfg);
        a.n_units = U;
        a.stages = fused_stages(dt, G, cap_src, B);
        a.cap = cap_src;
        a.cap_dst = cap_dst;
        a.B = B;
        a.n_valid = n_valid;
        a.k_src = k_src;
        a.v_src = v_src;
        a.pos_src = pos_src;
        a.k_dst = k_dst;
        a.v_dst = v_dst;
        a.pos_dst = pos_dst;
        a.kept = kept_idx;
        a.n_kept = n_kept;
        a.final_out = final_score;
        a.scratch = reinterpret_cast<float*>(ws_at(ws, w.sc.raw));
        a.trace = phase_trace_buffer(U);
        a.flag = flag;
        return cuda_status(launch_fused(dt, G, map, a, static_cast<int>(fused_ctas(U)), s));
    }

    CUtensorMap map;
    TRI_TRY(make_key_map(&map, k_src, dt, paged ? paged->n_pages * paged->rows : U * cap_src,
                         score_tile_keys(dt)));
    // Zero the flag word, the moment counters and the radix histograms.
    TRI_CUDA(cudaMemsetAsync(ws, 0, kWsHeader, s));
    TRI_CUDA(cudaMemsetAsync(ws_at(ws, w.sc.counters), 0, static_cast<size_t>(U) * 4, s));
    TRI_CUDA(cudaMemsetAsync(ws_at(ws, w.sel.hists), 0, w.sel.counts - w.sel.hists, s));
    TRI_CUDA(cudaMemsetAsync(ws_at(ws, w.zcount), 0, static_cast<size_t>(U) * 4, s));
    TRI_CUDA(launch_fold(stats, p_cur, n_seq, n_layers, n_kvheads * G, cfg->theta, off,
                         cfg->variant, wts, s));
    ScoreArgs a;
    a.keys = k_src;
    a.n_units = U;
    a.cap = cap_src;
    a.tpu = w.sc.tpu;
    a.n_valid = n_valid;
    a.wts = wts;
    a.raw = reinterpret_cast<float*>(ws_at(ws, w.sc.raw));
    a.partial = reinterpret_cast<double*>(ws_at(ws, w.sc.partial));
    a.counters = reinterpret_cast<uint32_t*>(ws_at(ws, w.sc.counters));
    a.mom = reinterpret_cast<float2*>(ws_at(ws, w.sc.mom));
    a.flag = flag;
    if (paged) a.pm = *paged;
    const int n_sm = device_info().sm_count;
    TRI_CUDA(score_any(cfg, off, dt, G, map, a, stats, p_cur, n_layers, n_kvheads, n_sm, s));
    float* fin = final_score ? final_score : reinterpret_cast<float*>(ws_at(ws, w.fin));
    uint32_t* hists = reinterpret_cast<uint32_t*>(ws_at(ws, w.sel.hists));
    TRI_CUDA(launch_zmax(G, a.raw, U, cap_src, n_valid, a.mom, fin, hists, 1, cfg->n_sink,
                         cfg->n_recent, flag, s));
    TRI_CUDA(launch_zselect(fin, U, cap_src, n_valid, B, ub, hists,
                            reinterpret_cast<uint2*>(ws_at(ws, w.sel.counts)),
                            reinterpret_cast<int2*>(ws_at(ws, w.zcand)),
                            reinterpret_cast<uint32_t*>(ws_at(ws, w.zcount)), ws_at(ws, w.zstate), kept,
                            n_kept, s));
    if (inplace)
        return cuda_status(launch_compact_inplace(dt, k_dst, v_dst, pos_dst, U, cap_src, kept,
                                                  n_kept, B, flag, n_sm * 8, s,
                                                  paged ? *paged : PageMap()));
    return cuda_status(launch_gather(dt, k_src, v_src, pos_src, U, cap_src, kept, n_kept, B, k_dst,
                                     v_dst, pos_dst, cap_dst, flag, n_sm * 8, s));
}

tri_status tri_prune(const tri_config* cfg, const void* k_src, const void* v_src,
                     const int32_t* pos_src, tri_dtype dt, int64_t n_seq, int64_t n_layers,
                     int64_t n_kvheads, int G, int64_t cap_src, const int32_t* n_valid,
                     const int64_t* p_cur, const float* stats, int64_t B, void* k_dst,
                     void* v_dst, int32_t* pos_dst, int64_t cap_dst, int32_t* kept_idx,
                     int32_t* n_kept, float* final_score, void* ws, size_t ws_bytes,
                     void* stream) {
    return prune_impl(cfg, k_src, v_src, pos_src, dt, n_seq, n_layers, n_kvheads, G, cap_src,
                      n_valid, p_cur, stats, B, k_dst, v_dst, pos_dst, cap_dst, kept_idx, n_kept,
                      final_score, ws, ws_bytes, stream, false);
}

tri_status tri_prune_paged_inplace(const tri_config* cfg, void* k_pool, void* v_pool, int32_t* pos,
                                   tri_dtype dt, int64_t n_seq, int64_t n_layers,
                                   int64_t n_kvheads, int G, int64_t cap, const int32_t* n_valid,
                                   const int64_t* p_cur, const float* stats, int64_t B,
                                   const int32_t* page_table, int64_t page_rows,
                                   int64_t pages_per_unit, int64_t n_pages, int32_t* kept_idx,
                                   int32_t* n_kept, float* final_score, void* ws, size_t ws_bytes,
                                   void* stream) {
    if (!page_table || !aligned4(page_table) || page_rows < 1 || page_rows % kPageRowQuantum != 0 ||
        n_pages < 1 || pages_per_unit < 1 || cap < 1 || pages_per_unit * page_rows < cap ||
        n_pages * page_rows > INT32_MAX)
        return TRI_ERR_INVALID_ARG;
    PageMap pm;
    pm.table = page_table;
    pm.rows = page_rows;
    pm.per_unit = pages_per_unit;
    pm.n_pages = n_pages;
    return prune_impl(cfg, k_pool, v_pool, pos, dt, n_seq, n_layers, n_kvheads, G, cap, n_valid,
                      p_cur, stats, B, k_pool, v_pool, pos, cap, kept_idx, n_kept, final_score, ws,
                      ws_bytes, stream, true, &pm);
}

tri_status tri_prune_inplace(const tri_config* cfg, void* k, void* v, int32_t* pos,
                             tri_dtype dt, int64_t n_seq, int64_t n_layers, int64_t n_kvheads,
                             int G, int64_t cap, const int32_t* n_valid, const int64_t* p_cur,
                             const float* stats, int64_t B, int32_t* kept_idx, int32_t* n_kept,
                             float* final_score, void* ws, size_t ws_bytes, void* stream) {
    return prune_impl(cfg, k, v, pos, dt, n_seq, n_layers, n_kvheads, G, cap, n_valid, p_cur,
                      stats, B, k, v, pos, cap, kept_idx, n_kept, final_score, ws, ws_bytes,
                      stream, true);
}

tri_status tri_logit_reconstruct(const tri_config* cfg, const float* q_stats,
                                 const float* k_stats, int64_t n_qheads, int G,
                                 const int64_t* deltas, int64_t n_delta, float* recon,
                                 void* stream) {
    LaunchScope scope_;
    FoldOffsets off;
    TRI_TRY(check_cfg(cfg, &off));
    if (!q_stats || !k_stats || !deltas || !recon || n_qheads < 1 || G < 1 || n_delta < 1 ||
        n_qheads % G != 0)
        return TRI_ERR_INVALID_ARG;
    if (n_qheads > 65535) return TRI_ERR_UNSUPPORTED;
    if (!aligned4(q_stats) || !aligned4(k_stats) || !aligned4(recon) ||
        (reinterpret_cast<uintptr_t>(deltas) & 7))
        return TRI_ERR_INVALID_ARG;
    return cuda_status(launch_logit_reconstruct(q_stats, k_stats, n_qheads, G, cfg->theta, deltas,
                                                n_delta, recon,
                                                static_cast<cudaStream_t>(stream)));
}

tri_status tri_logit_curve(const void* q_post, const void* k_post, tri_dtype dt, int64_t n_qheads,
                           int G, int64_t n_tok, int head_dim, const int64_t* deltas,
                           int64_t n_delta, float* curve, void* stream) {
    LaunchScope scope_;
    if (!q_post || !k_post || !deltas || !curve || n_qheads < 1 || G < 1 || n_tok < 1 ||
        n_delta < 1 || n_qheads % G != 0)
        return TRI_ERR_INVALID_ARG;
    if (!dtype_ok(dt) || head_dim != kD) return TRI_ERR_UNSUPPORTED;
    if (n_qheads > 65535 || n_delta > INT32_MAX) return TRI_ERR_UNSUPPORTED;
    if (!aligned4(q_post) || !aligned4(k_post) || !aligned4(curve) ||
        (reinterpret_cast<uintptr_t>(deltas) & 7))
        return TRI_ERR_INVALID_ARG;
    return cuda_status(launch_logit_curve(dt, q_post, k_post, n_qheads, G, n_tok, deltas, n_delta,
                                          curve, static_cast<cudaStream_t>(stream)));
}

tri_status tri_pearson(const float* a, const float* b, int64_t n_rows, int64_t n, float* r,
                       void* stream) {
    LaunchScope scope_;
    if (!a || !b || !r || n_rows < 1 || n < 1) return TRI_ERR_INVALID_ARG;
    if (n_rows > INT32_MAX) return TRI_ERR_UNSUPPORTED;
    if (!aligned4(a) || !aligned4(b) || !aligned4(r)) return TRI_ERR_INVALID_ARG;
    return cuda_status(launch_pearson(a, b, n_rows, n, r, static_cast<cudaStream_t>(stream)));
}

size_t tri_decode_workspace_bytes(int64_t n_units, int G, int64_t cap) {
    if (n_units < 1 || cap < 1 || G < 1 || G > TRI_MAX_GROUP) return kWsHeader;
    return kWsHeader + decode_part_bytes(n_units, G, cap, static_cast<int>(sm_count_or_default()));
}

tri_status tri_decode_attention(const void* q, const void* k, const void* v, tri_dtype dt,
                                int64_t n_units, int G, int64_t cap, int head_dim,
                                const int32_t* n_valid, float scale, float* out, void* ws,
                                size_t ws_bytes, void* stream) {
    LaunchScope scope_;
    if (!q || !k || !v || !out || n_units < 1 || cap < 1 || !(scale > 0.f))
        return TRI_ERR_INVALID_ARG;
    if (!dtype_ok(dt) || head_dim != kD || G < 1 || G > TRI_MAX_GROUP) return TRI_ERR_UNSUPPORTED;
    if (n_units > 65535) return TRI_ERR_UNSUPPORTED;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) ||
        (n_valid && !aligned4(n_valid)))
        return TRI_ERR_INVALID_ARG;
    const int n_sm = static_cast<int>(sm_count_or_default());
    if (!ws || !aligned16(ws) || ws_bytes < kWsHeader + decode_part_bytes(n_units, G, cap, n_sm))
        return TRI_ERR_WORKSPACE;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    TRI_CUDA(cudaMemsetAsync(ws, 0, kWsHeader, s));
    return cuda_status(launch_decode(dt, G, q, k, v, n_units, cap, n_valid, scale, out,
                                     reinterpret_cast<float*>(ws_at(ws, kWsHeader)), ws_flag(ws),
                                     n_sm, s));
}

tri_status tri_append(void* k_cache, void* v_cache, int32_t* pos_cache, tri_dtype dt,
                      int64_t n_seq, int64_t n_units, int64_t cap, int head_dim,
                      int32_t* n_valid, int64_t* p_cur, const void* k_new, const void* v_new,
                      const int32_t* pos_new, int64_t n_new, void* ws, size_t ws_bytes,
                      void* stream) {
    LaunchScope scope_;
    if (!k_cache || !n_valid || n_seq < 1 || n_units < 1 || cap < 1 || n_new < 0)
        return TRI_ERR_INVALID_ARG;
    if (n_new > 0 && !k_new) return TRI_ERR_INVALID_ARG;  // nothing is read when n_new == 0
    if (!dtype_ok(dt) || head_dim != kD) return TRI_ERR_UNSUPPORTED;
    if (n_units % n_seq != 0 || n_units > 65535) return TRI_ERR_INVALID_ARG;
    if (n_new > 0 && ((v_cache == nullptr) != (v_new == nullptr) ||
                      (pos_cache == nullptr) != (pos_new == nullptr)))
        return TRI_ERR_INVALID_ARG;
    if (p_cur && !pos_new) return TRI_ERR_INVALID_ARG;
    if (!aligned16(k_cache) || !aligned16(k_new) ||
        (v_cache && (!aligned16(v_cache) || !aligned16(v_new))))
        return TRI_ERR_INVALID_ARG;
    if (!ws || ws_bytes < kWsHeader || !aligned16(ws)) return TRI_ERR_WORKSPACE;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    TRI_CUDA(cudaMemsetAsync(ws, 0, kWsHeader, s));
    if (n_new == 0) return TRI_OK;
    return cuda_status(launch_append(dt, k_cache, v_cache, pos_cache, n_seq, n_units, cap, n_valid,
                                     p_cur, k_new, v_new, pos_new, n_new, ws_flag(ws), s));
}

tri_status tri_set_timing_events(void* const* events, int n_events) {
    if (n_events < 0 || (n_events > 0 && !events)) return TRI_ERR_INVALID_ARG;
    t_events = n_events ? reinterpret_cast<cudaEvent_t*>(const_cast<void**>(events)) : nullptr;
    t_n_events = n_events;
    return TRI_OK;
}

int tri_last_launch_count(void) { return t_launches; }

tri_status tri_set_phase_trace(void* device_buf, size_t bytes) {
    if (bytes && !device_buf) return TRI_ERR_INVALID_ARG;
    t_trace = static_cast<uint64_t*>(device_buf);
    t_trace_bytes = device_buf ? bytes : 0;
    return TRI_OK;
}

tri_status tri_check_device_error(const void* ws, void* stream, uint32_t* flags_out) {
    if (!ws) return TRI_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint32_t f = 0;
    if (cudaMemcpyAsync(&f, ws, sizeof(f), cudaMemcpyDeviceToHost, s) != cudaSuccess)
        return TRI_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return TRI_ERR_CUDA;
    if (flags_out) *flags_out = f;
    return f ? TRI_ERR_DEVICE : TRI_OK;
}

}  // extern "C"
