/*
 * tri_oracle.c -- plain float64 CPU oracle for TriAttention KV-cache pruning.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the correctness reference that the
 * CUDA path is compared against.  Only the tests, the smoke check and the CPU
 * baseline leg of the benchmark may load it; the library (libtri) never links,
 * calls or imports it, and the two share no code, header, table or constant.
 *
 * It computes the method the way the pages state it, step by step, in double
 * precision, with no folding, blocking or reordering beyond the definitions:
 *
 *   calibrate  per-band query centre E[q_f], mean norm E[|q_f|] and
 *              concentration R_f = |E[q_f]| / E[|q_f|]
 *              (TriAttention talk announcement, qingkeai.online, "S_norm"
 *              equation and the R_f definition beside it; hyper.ai summary of
 *              arXiv 2604.04921, Method section, R = |E[q]| / E[|q|]).
 *   score      each post-RoPE key is de-rotated by its own position (inverse of
 *              the talk page's RoPE rotation matrix), its band amplitude and
 *              phase are taken, and for every future offset delta in D the
 *              trigonometric score
 *                  S_trig(k, Delta) = sum_f |E[q_f]| |k_f| cos(w_f Delta + phi_f),
 *                  phi_f = arg E[q_f] - arg k_f,   Delta = p_cur - p_k + delta
 *              plus the norm score
 *                  S_norm(k) = sum_f (1 - R_f) E[|q_f|] |k_f|
 *              is evaluated explicitly and averaged over D
 *              (talk page: RoPE logit general form, S_trig, S_norm and the
 *              offset-averaged score S~ with D = {1, 2, 4, ..., 2^16}).
 *   normalise  per query head a z-score over the unit's keys, then the maximum
 *              over the heads of the GQA group (hyper.ai summary, Method
 *              section: "normalise then aggregate" for grouped-query attention).
 *   select     the top-B keys by (score descending, index ascending), returned
 *              in ascending index order (jaedaily.cn KV-compression tutorial,
 *              eviction step: top-k then sort to keep temporal order; talk
 *              page: keep only the top-B).
 *   gather     bit-exact copy of the kept K, V and position rows.
 *
 * Readings where the pages are silent (each also listed in the design notes):
 *   - average (not max) over the offsets, as the talk page's S~ equation says;
 *   - phi_f uses the pre-RoPE key phase (the key de-rotated by its position);
 *   - bands pair interleaved components (x_2f, x_2f+1), f = 0..d/2-1;
 *   - population standard deviation; sigma == 0 gives z = 0;
 *   - the head maximum ignores NaN (fmax semantics) and is NaN only when every
 *     head is NaN; NaN scores rank below every number; -0.0 equals +0.0;
 *   - ties at the B-th score go to the lowest index;
 *   - R_f = 1 when E[|q_f|] = 0 (the norm weight (1-R_f)E|q_f| is 0 anyway).
 *
 * Method variants (each off by default; the pages name them as ablations or
 * alternatives, the readings are listed in the design notes):
 *   ORA_VAR_NO_TRIG     S_trig left out, the score is S_norm alone (shibing624
 *                       paper reading, ablation section: without S_trig);
 *   ORA_VAR_NO_R        the norm weight without the concentration factor,
 *                       E[|q_f|] instead of (1 - R_f) E[|q_f|] (same section:
 *                       without the R weighting);
 *   ORA_VAR_MAX_OFFSET  the maximum over the offsets of S_trig + S_norm
 *                       instead of their mean (same page, future-offset
 *                       paragraph: the maximum is the key's score);
 *   ORA_VAR_HALF_SPLIT  band f pairs components (x_f, x_{f+d/2}) instead of
 *                       (x_2f, x_2f+1) (the rotate-half RoPE layout);
 *   protection          the n_sink first and n_recent last keys of a unit are
 *                       always kept (jaedaily.cn tutorial, streaming section:
 *                       the most recent tokens are protected from eviction);
 *   layer budgets       a budget per layer instead of one B (same tutorial,
 *                       budget paragraph: pyramid-shaped budgets per layer).
 *
 * Element types: 0 = float32, 1 = bfloat16 (upper half of a float32).  Both
 * decode exactly to double.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORA_F32 0
#define ORA_BF16 1

#define ORA_VAR_NO_TRIG 1
#define ORA_VAR_NO_R 2
#define ORA_VAR_MAX_OFFSET 4
#define ORA_VAR_HALF_SPLIT 8

#define ORA_OK 0
#define ORA_EINVAL 1
#define ORA_ENOMEM 2

static double ora_decode(const void* base, int dtype, int64_t i) {
    if (dtype == ORA_F32) {
        return (double)((const float*)base)[i];
    }
    uint32_t bits = (uint32_t)((const uint16_t*)base)[i] << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

/* Components (x, y) of band f of the d-vector starting at element `row`:
 * interleaved (x_2f, x_2f+1) as the talk page's RoPE matrix pairs them, or
 * half-split (x_f, x_{f+d/2}) for the rotate-half layout. */
static void ora_band(const void* base, int dtype, int64_t row, int f, int d, int half,
                     double* x, double* y) {
    if (half) {
        *x = ora_decode(base, dtype, row + f);
        *y = ora_decode(base, dtype, row + f + d / 2);
    } else {
        *x = ora_decode(base, dtype, row + 2 * f);
        *y = ora_decode(base, dtype, row + 2 * f + 1);
    }
}

/* RoPE angular frequency of band f: w_f = theta^(-2f/d) (talk page, RoPE
 * rotation; hyper.ai summary, Method section). */
static double ora_omega(double theta, int f, int d) {
    return pow(theta, -2.0 * (double)f / (double)d);
}

int oracle_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void oracle_set_threads(int n) {
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

/*
 * Calibration.  q: queries [n_heads][n_tok][d]; stats out:
 * [n_heads][d/2][4] = (Re E[q_f], Im E[q_f], E[|q_f|], R_f).
 * Pre-RoPE queries are averaged as they are.  Post-RoPE queries (qpos
 * non-NULL: the position of each token, [n_tok], shared by the heads) are
 * first rotated back by -w_f p, the inverse of the talk page's RoPE matrix,
 * which gives the pre-RoPE band (shibing624 paper reading, Q/K concentration
 * section: the centres live in the pre-RoPE space).  `half` selects the
 * half-split band pairing.  The same statistics of keys are the K centres.
 */
int oracle_calibrate_ex(const void* q, int dtype, int64_t n_heads, int64_t n_tok, int d,
                        const int32_t* qpos, double theta, int half, double* stats) {
    if (!q || !stats || n_heads < 0 || n_tok <= 0 || d <= 0 || (d & 1)) return ORA_EINVAL;
    const int F = d / 2;
    int64_t h;
#pragma omp parallel for schedule(dynamic)
    for (h = 0; h < n_heads; ++h) {
        for (int f = 0; f < F; ++f) {
            const double w = ora_omega(theta, f, d);
            double sx = 0.0, sy = 0.0, sn = 0.0;
            for (int64_t n = 0; n < n_tok; ++n) {
                const int64_t row = (h * n_tok + n) * (int64_t)d;
                double x, y;
                ora_band(q, dtype, row, f, d, half, &x, &y);
                if (qpos) {
                    const double a = w * (double)qpos[n];
                    const double c = cos(a), sn_ = sin(a);
                    const double xr = c * x + sn_ * y;
                    const double yr = -sn_ * x + c * y;
                    x = xr;
                    y = yr;
                }
                sx += x;
                sy += y;
                sn += hypot(x, y);
            }
            const double mre = sx / (double)n_tok;
            const double mim = sy / (double)n_tok;
            const double mn = sn / (double)n_tok;
            const double R = (mn > 0.0) ? hypot(mre, mim) / mn : 1.0;
            double* o = stats + ((int64_t)h * F + f) * 4;
            o[0] = mre;
            o[1] = mim;
            o[2] = mn;
            o[3] = R;
        }
    }
    return ORA_OK;
}

/* Calibration of pre-RoPE queries with interleaved bands. */
int oracle_calibrate(const void* q, int dtype, int64_t n_heads, int64_t n_tok, int d,
                     double* stats) {
    return oracle_calibrate_ex(q, dtype, n_heads, n_tok, d, NULL, 10000.0, 0, stats);
}

/*
 * Score one unit (one KV head's cache) for the G query heads of its group,
 * in the pages' unfolded form.
 *   k:       post-RoPE keys [n][d]
 *   pos:     position of each key [n]
 *   stats:   calibration of the G query heads [G][d/2][4]
 *   offsets: the future offsets D [n_off]
 *   raw out: per-head offset-averaged score S~ [G][n]
 */
static void ora_score_unit(const void* k, int dtype, int64_t n, int d, const int32_t* pos,
                           int64_t p_cur, const double* stats, int G, double theta,
                           const int64_t* offsets, int n_off, int variant, double* raw,
                           double* kmag, double* karg, const double* omega) {
    const int F = d / 2;
    const int half = (variant & ORA_VAR_HALF_SPLIT) != 0;
    const int use_trig = (variant & ORA_VAR_NO_TRIG) == 0;
    const int use_r = (variant & ORA_VAR_NO_R) == 0;
    const int use_max = (variant & ORA_VAR_MAX_OFFSET) != 0;
    double qmag[512], qarg[512], qnw[512];
    (void)theta;
    for (int64_t j = 0; j < n; ++j) {
        const double pj = (double)pos[j];
        /* De-rotate: k_f = R(-w_f p_j) k'_f, the inverse of the RoPE matrix. */
        for (int f = 0; f < F; ++f) {
            double xr, yr;
            ora_band(k, dtype, j * d, f, d, half, &xr, &yr);
            const double a = omega[f] * pj;
            const double c = cos(a), s = sin(a);
            const double x = c * xr + s * yr;
            const double y = -s * xr + c * yr;
            kmag[f] = hypot(x, y);
            karg[f] = atan2(y, x);
        }
        for (int h = 0; h < G; ++h) {
            const double* st = stats + (int64_t)h * F * 4;
            /* Per band of this head: |E[q_f]|, arg E[q_f] and the norm weight
             * (1 - R_f) E[|q_f|]; none of them depends on the offset. */
            for (int f = 0; f < F; ++f) {
                qmag[f] = hypot(st[f * 4 + 0], st[f * 4 + 1]);
                qarg[f] = atan2(st[f * 4 + 1], st[f * 4 + 0]);
                qnw[f] = (use_r ? 1.0 - st[f * 4 + 3] : 1.0) * st[f * 4 + 2];
            }
            double total = 0.0, best = -INFINITY;
            for (int o = 0; o < n_off; ++o) {
                const double Delta = (double)(p_cur - (int64_t)pos[j] + offsets[o]);
                double s_trig = 0.0, s_norm = 0.0;
                for (int f = 0; f < F; ++f) {
                    const double phi = qarg[f] - karg[f];
                    if (use_trig) s_trig += qmag[f] * kmag[f] * cos(omega[f] * Delta + phi);
                    s_norm += qnw[f] * kmag[f];
                }
                total += s_trig + s_norm;
                if (s_trig + s_norm > best) best = s_trig + s_norm;
            }
            raw[(int64_t)h * n + j] = use_max ? best : total / (double)n_off;
        }
    }
}

/* z-score per head over the n keys, then the maximum over the heads. */
static void ora_znorm_max(const double* raw, int G, int64_t n, double* z, double* fin,
                          double* mu_out, double* sd_out) {
    for (int h = 0; h < G; ++h) {
        const double* s = raw + (int64_t)h * n;
        double sum = 0.0;
        for (int64_t j = 0; j < n; ++j) sum += s[j];
        const double mu = (n > 0) ? sum / (double)n : 0.0;
        double ss = 0.0;
        for (int64_t j = 0; j < n; ++j) ss += (s[j] - mu) * (s[j] - mu);
        const double sd = (n > 0) ? sqrt(ss / (double)n) : 0.0;
        for (int64_t j = 0; j < n; ++j) {
            z[(int64_t)h * n + j] = (sd > 0.0) ? (s[j] - mu) / sd : (sd == 0.0 ? 0.0 : NAN);
        }
        if (mu_out) mu_out[h] = mu;
        if (sd_out) sd_out[h] = sd;
    }
    for (int64_t j = 0; j < n; ++j) {
        double m = z[j];
        for (int h = 1; h < G; ++h) m = fmax(m, z[(int64_t)h * n + j]);
        fin[j] = m;
    }
}

typedef struct {
    double v;
    int32_t idx;
    int nan;
} ora_item;

/* Order: larger score first; NaN after every number; equal scores (and -0 vs
 * +0, which compare equal) by ascending index. */
static int ora_cmp_rank(const void* pa, const void* pb) {
    const ora_item* a = (const ora_item*)pa;
    const ora_item* b = (const ora_item*)pb;
    if (a->nan != b->nan) return a->nan ? 1 : -1;
    if (!a->nan) {
        if (a->v > b->v) return -1;
        if (a->v < b->v) return 1;
    }
    return (a->idx < b->idx) ? -1 : (a->idx > b->idx);
}

static int ora_cmp_i32(const void* pa, const void* pb) {
    const int32_t a = *(const int32_t*)pa, b = *(const int32_t*)pb;
    return (a > b) - (a < b);
}

/*
 * Top-B selection on one unit's final scores.  kept out: min(B, n) indices in
 * ascending order.  threshold out (optional): the B-th score in rank order
 * (NaN when n == 0).  Returns the number kept, or -1 on allocation failure.
 */
int64_t oracle_select(const double* fin, int64_t n, int64_t B, int32_t* kept, double* threshold) {
    if (n < 0 || B < 0) return -1;
    const int64_t m = (B < n) ? B : n;
    if (threshold) *threshold = NAN;
    if (n == 0) return 0;
    ora_item* it = (ora_item*)malloc((size_t)n * sizeof(ora_item));
    if (!it) return -1;
    for (int64_t j = 0; j < n; ++j) {
        it[j].v = fin[j];
        it[j].idx = (int32_t)j;
        it[j].nan = isnan(fin[j]) ? 1 : 0;
    }
    qsort(it, (size_t)n, sizeof(ora_item), ora_cmp_rank);
    for (int64_t r = 0; r < m; ++r) kept[r] = it[r].idx;
    if (threshold && m > 0) *threshold = it[m - 1].v;
    free(it);
    qsort(kept, (size_t)m, sizeof(int32_t), ora_cmp_i32);
    return m;
}

/*
 * Top-B selection with protected keys: every key j < n_sink or
 * j >= n - n_recent is kept, the lowest indices of them when they alone are
 * more than B; the places left go to the other keys in the order of
 * oracle_select.  threshold out (optional): the score of the last unprotected
 * key kept, NaN when none is.  Returns the number kept, or -1.
 */
int64_t oracle_select_protected(const double* fin, int64_t n, int64_t B, int64_t n_sink,
                                int64_t n_recent, int32_t* kept, double* threshold) {
    if (n < 0 || B < 0 || n_sink < 0 || n_recent < 0) return -1;
    const int64_t m = (B < n) ? B : n;
    if (threshold) *threshold = NAN;
    if (n == 0) return 0;
    int64_t p = 0;
    for (int64_t j = 0; j < n && p < m; ++j)
        if (j < n_sink || j >= n - n_recent) kept[p++] = (int32_t)j;
    if (p == m) return m;
    ora_item* it = (ora_item*)malloc((size_t)n * sizeof(ora_item));
    if (!it) return -1;
    int64_t c = 0;
    for (int64_t j = 0; j < n; ++j) {
        if (j < n_sink || j >= n - n_recent) continue;
        it[c].v = fin[j];
        it[c].idx = (int32_t)j;
        it[c].nan = isnan(fin[j]) ? 1 : 0;
        ++c;
    }
    qsort(it, (size_t)c, sizeof(ora_item), ora_cmp_rank);
    const int64_t rest = m - p;
    for (int64_t r = 0; r < rest; ++r) kept[p + r] = it[r].idx;
    if (threshold && rest > 0) *threshold = it[rest - 1].v;
    free(it);
    qsort(kept, (size_t)m, sizeof(int32_t), ora_cmp_i32);
    return m;
}

/*
 * Whole prune step over a batch of units, one unit at a time per thread.
 * Unit u = (seq * n_layers + layer) * n_kvheads + kvh; its query heads are
 * kvh*G .. kvh*G+G-1 of that layer.
 *   k, v:       [U][cap][d] post-RoPE keys and values (dtype)
 *   pos:        [U][cap] int32 key positions
 *   n_valid:    [U] number of valid keys in each unit (NULL: cap)
 *   p_cur:      [n_seq] current position of each sequence
 *   stats:      [n_layers][n_kvheads*G][d/2][4] calibration (double)
 *   offsets:    D, n_off entries
 *   raw:        [U][G][cap] per-head S~ (optional, NULL to skip)
 *   fin:        [U][cap] final score (optional)
 *   kept:       [U][B] kept indices, ascending (optional)
 *   n_kept:     [U] (optional)
 *   thr:        [U] B-th score (optional)
 *   k_dst, v_dst, pos_dst: [U][cap_dst][d] gathered rows (optional)
 *   unit_list:  subset of units to process (NULL: all), n_list entries
 *   variant:    ORA_VAR_* bits (0: the method as the pages' main text states it)
 *   n_sink, n_recent: protected first / last keys of each unit (0: none)
 *   layer_budget: [n_layers] budget of each layer's units, at most B (NULL: B)
 */
int oracle_prune(const void* k, const void* v, const int32_t* pos, int dtype, int64_t n_seq,
                 int64_t n_layers, int64_t n_kvheads, int G, int64_t cap, int d,
                 const int32_t* n_valid, const int64_t* p_cur, const double* stats, double theta,
                 const int64_t* offsets, int n_off, int64_t B, double* raw, double* fin,
                 int32_t* kept, int64_t* n_kept, double* thr, void* k_dst, void* v_dst,
                 int32_t* pos_dst, int64_t cap_dst, const int64_t* unit_list, int64_t n_list,
                 int variant, int64_t n_sink, int64_t n_recent, const int64_t* layer_budget) {
    if (!k || !pos || !p_cur || !stats || !offsets || n_off <= 0 || G <= 0 || cap < 0 || d <= 0 ||
        d > 1024 || (d & 1) || B < 0 || n_sink < 0 || n_recent < 0)
        return ORA_EINVAL;
    if ((k_dst || v_dst || pos_dst) && cap_dst < ((B < cap) ? B : cap)) return ORA_EINVAL;
    if (layer_budget)
        for (int64_t l = 0; l < n_layers; ++l)
            if (layer_budget[l] < 0 || layer_budget[l] > B) return ORA_EINVAL;
    const int F = d / 2;
    const int64_t U = n_seq * n_layers * n_kvheads;
    const int64_t count = unit_list ? n_list : U;
    const size_t esize = (dtype == ORA_F32) ? 4 : 2;
    double* omega = (double*)malloc((size_t)F * sizeof(double));
    if (!omega) return ORA_ENOMEM;
    for (int f = 0; f < F; ++f) omega[f] = ora_omega(theta, f, d);
    int err = ORA_OK;
    int64_t i;
#pragma omp parallel for schedule(dynamic)
    for (i = 0; i < count; ++i) {
        const int64_t u = unit_list ? unit_list[i] : i;
        if (u < 0 || u >= U) {
#pragma omp atomic write
            err = ORA_EINVAL;
            continue;
        }
        const int64_t seq = u / (n_layers * n_kvheads);
        const int64_t layer = (u / n_kvheads) % n_layers;
        const int64_t kvh = u % n_kvheads;
        const int64_t n = n_valid ? n_valid[u] : cap;
        double* r = (double*)malloc(((size_t)G * (size_t)(n > 0 ? n : 1)) * sizeof(double));
        double* z = (double*)malloc(((size_t)G * (size_t)(n > 0 ? n : 1)) * sizeof(double));
        double* fn = (double*)malloc((size_t)(n > 0 ? n : 1) * sizeof(double));
        int32_t* kp = (int32_t*)malloc((size_t)(B > 0 ? B : 1) * sizeof(int32_t));
        double* kmag = (double*)malloc((size_t)F * sizeof(double));
        double* karg = (double*)malloc((size_t)F * sizeof(double));
        if (n < 0 || n > cap) {
#pragma omp atomic write
            err = ORA_EINVAL;
        } else if (!r || !z || !fn || !kp || !kmag || !karg) {
#pragma omp atomic write
            err = ORA_ENOMEM;
        } else {
            const double* st = stats + ((layer * n_kvheads + kvh) * (int64_t)G) * F * 4;
            const void* ku = (const char*)k + (size_t)(u * cap * d) * esize;
            ora_score_unit(ku, dtype, n, d, pos + u * cap, p_cur[seq], st, G, theta, offsets,
                           n_off, variant, r, kmag, karg, omega);
            ora_znorm_max(r, G, n, z, fn, NULL, NULL);
            double t;
            const int64_t Bu = layer_budget ? layer_budget[layer] : B;
            const int64_t m = (n_sink > 0 || n_recent > 0)
                                  ? oracle_select_protected(fn, n, Bu, n_sink, n_recent, kp, &t)
                                  : oracle_select(fn, n, Bu, kp, &t);
            if (raw)
                for (int h = 0; h < G; ++h)
                    memcpy(raw + (u * G + h) * cap, r + (int64_t)h * n, (size_t)n * sizeof(double));
            if (fin) memcpy(fin + u * cap, fn, (size_t)n * sizeof(double));
            if (kept) memcpy(kept + u * B, kp, (size_t)m * sizeof(int32_t));
            if (n_kept) n_kept[u] = m;
            if (thr) thr[u] = t;
            for (int64_t rr = 0; rr < m; ++rr) {
                const int64_t src = u * cap + kp[rr];
                const int64_t dst = u * cap_dst + rr;
                if (k_dst)
                    memcpy((char*)k_dst + (size_t)(dst * d) * esize,
                           (const char*)k + (size_t)(src * d) * esize, (size_t)d * esize);
                if (v_dst && v)
                    memcpy((char*)v_dst + (size_t)(dst * d) * esize,
                           (const char*)v + (size_t)(src * d) * esize, (size_t)d * esize);
                if (pos_dst) pos_dst[dst] = pos[src];
            }
        }
        free(r);
        free(z);
        free(fn);
        free(kp);
        free(kmag);
        free(karg);
    }
    free(omega);
    return err;
}

/* Score only (per-head S~) for one unit; exposed for the pins. */
int oracle_score(const void* k, int dtype, int64_t n, int d, const int32_t* pos, int64_t p_cur,
                 const double* stats, int G, double theta, const int64_t* offsets, int n_off,
                 int variant, double* raw) {
    if (!k || !pos || !stats || !offsets || !raw || n < 0 || G <= 0 || d <= 0 || d > 1024 ||
        (d & 1) || n_off <= 0)
        return ORA_EINVAL;
    const int F = d / 2;
    double* omega = (double*)malloc((size_t)F * sizeof(double));
    double* kmag = (double*)malloc((size_t)F * sizeof(double));
    double* karg = (double*)malloc((size_t)F * sizeof(double));
    if (!omega || !kmag || !karg) {
        free(omega);
        free(kmag);
        free(karg);
        return ORA_ENOMEM;
    }
    for (int f = 0; f < F; ++f) omega[f] = ora_omega(theta, f, d);
    ora_score_unit(k, dtype, n, d, pos, p_cur, stats, G, theta, offsets, n_off, variant, raw,
                   kmag, karg, omega);
    free(omega);
    free(kmag);
    free(karg);
    return ORA_OK;
}

/* z-score per head then max over heads, for one unit; exposed for the pins. */
int oracle_znorm_max(const double* raw, int G, int64_t n, double* z, double* fin, double* mu,
                     double* sd) {
    if (!raw || !z || !fin || G <= 0 || n < 0) return ORA_EINVAL;
    ora_znorm_max(raw, G, n, z, fin, mu, sd);
    return ORA_OK;
}

/*
 * Decode attention of one new query token over a (compacted) cache, one unit
 * at a time (jaedaily.cn tutorial, KV-compression objective: the output over
 * the kept subset S is sum_{j in S} a_j v_j with the softmax weights
 * a_j = exp(q.k_j / sqrt(d)) / sum_{j' in S} exp(q.k_j' / sqrt(d)),
 * renormalised over S).  scale multiplies the dot products (1/sqrt(d) for
 * the usual attention; any positive value).
 *   q:   [U][G][d] post-RoPE query of the current token for the G query heads
 *        of each unit (float32 or bf16 codes, like k and v)
 *   k,v: [U][cap][d] cache rows; the first n_valid[u] are attended
 *   out: [U][G][d] double
 * A unit with no valid key gives zeros.  The maximum score is subtracted
 * before exponentiating (the value is the same in exact arithmetic).
 */
int oracle_decode_attention(const void* q, const void* k, const void* v, int dtype,
                            int64_t n_units, int G, int64_t cap, int d, const int32_t* n_valid,
                            double scale, double* out) {
    if (!q || !k || !v || !out || n_units < 0 || G <= 0 || cap < 0 || d <= 0) return ORA_EINVAL;
    int64_t u;
    int err = ORA_OK;
#pragma omp parallel for schedule(dynamic)
    for (u = 0; u < n_units; ++u) {
        const int64_t n = n_valid ? n_valid[u] : cap;
        if (n < 0 || n > cap) {
#pragma omp atomic write
            err = ORA_EINVAL;
            continue;
        }
        double* sc = (double*)malloc((size_t)(n > 0 ? n : 1) * sizeof(double));
        if (!sc) {
#pragma omp atomic write
            err = ORA_ENOMEM;
            continue;
        }
        for (int h = 0; h < G; ++h) {
            const int64_t qrow = (u * G + h) * (int64_t)d;
            double* o = out + (u * G + h) * (int64_t)d;
            for (int e = 0; e < d; ++e) o[e] = 0.0;
            if (n == 0) continue;
            double mx = -INFINITY;
            for (int64_t j = 0; j < n; ++j) {
                const int64_t krow = (u * cap + j) * (int64_t)d;
                double dot = 0.0;
                for (int e = 0; e < d; ++e)
                    dot += ora_decode(q, dtype, qrow + e) * ora_decode(k, dtype, krow + e);
                sc[j] = scale * dot;
                if (sc[j] > mx) mx = sc[j];
            }
            double den = 0.0;
            for (int64_t j = 0; j < n; ++j) {
                const double w = exp(sc[j] - mx);
                den += w;
                const int64_t vrow = (u * cap + j) * (int64_t)d;
                for (int e = 0; e < d; ++e) o[e] += w * ora_decode(v, dtype, vrow + e);
            }
            for (int e = 0; e < d; ++e) o[e] /= den;
        }
        free(sc);
    }
    return err;
}

/*
 * The attention logit as a function of the distance Delta, reconstructed from
 * the Q and K centres (talk page: the RoPE logit general form
 * logit = sum_f |q_f| |k_f| cos(w_f Delta + phi_f), phi_f = arg q_f - arg k_f,
 * and the centre approximation q_f ~ E[q_f], k_f ~ E[k_f] that turns it into
 * a trigonometric series in Delta; shibing624 paper reading, Fig. 1(D)):
 *   recon[h][i] = sum_f |E q_f| |E k_f| cos(w_f deltas[i] + arg E q_f - arg E k_f)
 * for query head h with statistics qstats[h] and its KV head's kstats[h / G]
 * ([..][d/2][4] as oracle_calibrate writes them).
 */
int oracle_logit_reconstruct(const double* qstats, const double* kstats, int64_t n_qheads, int G,
                             int d, double theta, const int64_t* deltas, int64_t n_delta,
                             double* recon) {
    if (!qstats || !kstats || !deltas || !recon || n_qheads < 0 || G <= 0 || d <= 0 || (d & 1))
        return ORA_EINVAL;
    const int F = d / 2;
    for (int64_t h = 0; h < n_qheads; ++h) {
        const double* qs = qstats + h * F * 4;
        const double* ks = kstats + (h / G) * F * 4;
        for (int64_t i = 0; i < n_delta; ++i) {
            double sum = 0.0;
            for (int f = 0; f < F; ++f) {
                const double amp = hypot(qs[f * 4], qs[f * 4 + 1]) * hypot(ks[f * 4], ks[f * 4 + 1]);
                const double phi = atan2(qs[f * 4 + 1], qs[f * 4]) - atan2(ks[f * 4 + 1], ks[f * 4]);
                sum += amp * cos(ora_omega(theta, f, d) * (double)deltas[i] + phi);
            }
            recon[h * n_delta + i] = sum;
        }
    }
    return ORA_OK;
}

/*
 * The measured counterpart: the mean post-RoPE attention logit over every
 * query/key pair of one sequence at distance Delta, token t at position t:
 *   curve[h][i] = mean over t in [Delta, n_tok) of q[h][t] . k[h / G][t - Delta]
 * (0 when no pair is that far apart).  q: [n_qheads][n_tok][d], k:
 * [n_qheads / G][n_tok][d], post-RoPE (dtype codes as elsewhere).
 */
int oracle_logit_curve(const void* q, const void* k, int dtype, int64_t n_qheads, int G,
                       int64_t n_tok, int d, const int64_t* deltas, int64_t n_delta,
                       double* curve) {
    if (!q || !k || !deltas || !curve || n_qheads < 0 || G <= 0 || n_tok < 0 || d <= 0)
        return ORA_EINVAL;
    int64_t h;
#pragma omp parallel for schedule(dynamic)
    for (h = 0; h < n_qheads; ++h) {
        const int64_t kh = h / G;
        for (int64_t i = 0; i < n_delta; ++i) {
            const int64_t D = deltas[i];
            double sum = 0.0;
            int64_t cnt = 0;
            for (int64_t t = (D > 0 ? D : 0); t < n_tok; ++t) {
                if (t - D >= n_tok) continue;
                double dot = 0.0;
                for (int e = 0; e < d; ++e)
                    dot += ora_decode(q, dtype, (h * n_tok + t) * (int64_t)d + e) *
                           ora_decode(k, dtype, (kh * n_tok + t - D) * (int64_t)d + e);
                sum += dot;
                ++cnt;
            }
            curve[h * n_delta + i] = cnt > 0 ? sum / (double)cnt : 0.0;
        }
    }
    return ORA_OK;
}

/* Pearson correlation of rows a[r][0..n) and b[r][0..n) (two-pass; 0 when a
 * row is constant). */
int oracle_pearson(const double* a, const double* b, int64_t n_rows, int64_t n, double* r) {
    if (!a || !b || !r || n_rows < 0 || n < 0) return ORA_EINVAL;
    for (int64_t row = 0; row < n_rows; ++row) {
        const double* x = a + row * n;
        const double* y = b + row * n;
        double mx = 0.0, my = 0.0;
        for (int64_t i = 0; i < n; ++i) {
            mx += x[i];
            my += y[i];
        }
        mx /= (double)(n > 0 ? n : 1);
        my /= (double)(n > 0 ? n : 1);
        double sxy = 0.0, sxx = 0.0, syy = 0.0;
        for (int64_t i = 0; i < n; ++i) {
            sxy += (x[i] - mx) * (y[i] - my);
            sxx += (x[i] - mx) * (x[i] - mx);
            syy += (y[i] - my) * (y[i] - my);
        }
        r[row] = (sxx > 0.0 && syy > 0.0) ? sxy / sqrt(sxx * syy) : 0.0;
    }
    return ORA_OK;
}
