/*
 * moe_oracle.c -- plain CPU fp64 oracle of the hard-routed sparse MoE layer
 * forward.
 *
 * TEST INFRASTRUCTURE. Only the tests, the smoke check and the benchmark's
 * CPU-baseline leg use this library. The product path never links it, and it
 * shares no code, header, table or helper with the CUDA library.
 *
 * It computes the plain definitions, one step at a time, in double precision:
 *
 *   1. router logits   L[t,e] = sum_i x[t,i] * W_r[i,e] + b[e]
 *      ("5.5 real sparse MoE kernels (Metal)", Scope -- in: "Top-K routing
 *      kernel: routing_logits -> (top_k_indices, top_k_weights)"; the router
 *      matmul is phase 1 of the "Mega Kernel Architecture" of
 *      MOE_OPTIMIZATION_COMPLETE.md)
 *   2. softmax over all experts, top-k selection, renormalised weights
 *      (same passages; phases 2-3 of the mega kernel)
 *   3. stable sort of the routed slots by expert: order, inv_order =
 *      argsort(order), row_map = order // k, per-expert counts and the row and
 *      tile prefix tables (DS4Server issue #112, "Current upstream route",
 *      sort_rows; "Kernel contract", _schedule)
 *   4. gate|up projection with the GLU epilogue act(gate) * up, act = silu
 *      (SwiGLU) or the tanh form of GELU (GeGLU), over the
 *      sorted rows, reading token rows through row_map (issue #112,
 *      swiglu_rows; mlxcel PR #275, "What it does")
 *   5. down projection of the sorted rows (issue #112, switch_linear with
 *      sorted indices)
 *   6. score-weighted unsort back to token order
 *      out[t] = sum_j w[t,j] * down_j(...)  (mlxcel PR #275, "What it does";
 *      issue #112, _scatter_unsort)
 *
 * Weight element values: f32 and bf16 are read as stored; the 4-bit affine
 * format is dequantised as w = scale * q + bias with q in [0,15] taken from
 * bits [4j, 4j+3] of each 32-bit word (element j of the word, low nibble
 * first) and one bf16 scale and bias per group of 64 input elements
 * (mlx-lm PR #2044, "When it applies": affine 4-bit, group size 64; mlxcel
 * PR #275, "Multi-bit handling": affine dequant with a shift-unpack).
 *
 * Readings where the pages are silent (each also listed in the design notes):
 *   - ties in top-k go to the lowest expert index; -0.0 equals +0.0; a NaN
 *     logit ranks below every number (its parity is not pinned);
 *   - the selection is made on the logits rounded to fp32 (the precision the
 *     kernels decide in); weights are softmax restricted to the selected
 *     experts, which equals softmax over all experts renormalised over the
 *     selection;
 *   - the router bias is added to the logits before softmax and selection;
 *   - the sort is stable (ties by slot index r = t*k + j);
 *   - tile_off is the exclusive scan of ceil(count_e / BM).
 *
 * Threads: loops over independent tokens or experts are split across
 * nthreads POSIX threads; each output element is still computed by one
 * sequential sum in the order the definition gives.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

enum { ORC_F32 = 0, ORC_BF16 = 1, ORC_F16 = 2 }; /* activation / dense dtypes */
/* 4-bit affine with group 64 (ORC_W_Q4), 32 or 128 input elements per
 * scale and bias (the group sizes of DS4Server issue #112, "Kernel contract") */
enum { ORC_W_F32 = 0, ORC_W_BF16 = 1, ORC_W_Q4 = 2, ORC_W_Q4G32 = 3, ORC_W_Q4G128 = 4,
       ORC_W_Q8 = 5 /* 8-bit affine, group 64: byte j of a word is element j */ };

static int q4_group(int fmt) {
    return fmt == ORC_W_Q4 ? 64 : fmt == ORC_W_Q4G32 ? 32 : fmt == ORC_W_Q4G128 ? 128 : 0;
}

/* a bf16 value is the upper 16 bits of the fp32 with the same bits */
static double bf16_value(uint16_t h) {
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* an IEEE 754 binary16 value: sign, 5 exponent bits (bias 15), 10 fraction
 * bits; exponent 0 is subnormal (2^-14 * fraction / 1024), 31 is inf/NaN */
static double f16_value(uint16_t h) {
    const int sign = h >> 15, ex = (h >> 10) & 0x1F, fr = h & 0x3FF;
    double v;
    if (ex == 0) v = ldexp((double)fr, -24);
    else if (ex == 31) v = fr ? NAN : INFINITY;
    else v = ldexp((double)(1024 + fr), ex - 25);
    return sign ? -v : v;
}

static double act_value(const void* p, int dt, size_t i) {
    if (dt == ORC_F32) return (double)((const float*)p)[i];
    if (dt == ORC_F16) return f16_value(((const uint16_t*)p)[i]);
    return bf16_value(((const uint16_t*)p)[i]);
}

/* One expert weight matrix of shape [rows][cols] inside a stack of E. */
typedef struct {
    int fmt;                 /* ORC_W_* */
    const void* w;           /* f32/bf16: [E][rows][cols]; q4: u32 [E][rows][cols/8] */
    const uint16_t* s;       /* q4 only: bf16 [E][rows][cols/group] */
    const uint16_t* b;       /* q4 only: bf16 [E][rows][cols/group] */
    int rows, cols;
} orc_wmat;

/* Value of element (e, r, c) of a weight stack (dequantised for q4). */
static double weight_value(const orc_wmat* m, int e, int r, int c) {
    size_t row = (size_t)e * m->rows + r;
    if (m->fmt == ORC_W_F32) return (double)((const float*)m->w)[row * m->cols + c];
    if (m->fmt == ORC_W_BF16) return bf16_value(((const uint16_t*)m->w)[row * m->cols + c]);
    if (m->fmt == ORC_W_Q8) {
        uint32_t word8 = ((const uint32_t*)m->w)[row * (m->cols / 4) + c / 4];
        int q8 = (int)((word8 >> (8 * (c % 4))) & 0xFFu);
        size_t g8 = row * (m->cols / 64) + c / 64;
        return bf16_value(m->s[g8]) * (double)q8 + bf16_value(m->b[g8]);
    }
    uint32_t word = ((const uint32_t*)m->w)[row * (m->cols / 8) + c / 8];
    int q = (int)((word >> (4 * (c % 8))) & 0xFu);
    const int gs = q4_group(m->fmt);
    size_t g = row * (m->cols / gs) + c / gs;
    return bf16_value(m->s[g]) * (double)q + bf16_value(m->b[g]);
}

/* Whole row r of expert e, as doubles. */
static void weight_row(const orc_wmat* m, int e, int r, double* out) {
    for (int c = 0; c < m->cols; ++c) out[c] = weight_value(m, e, r, c);
}

/* ---------------------------------------------------------------- threads */

typedef void (*orc_range_fn)(void* ctx, int lo, int hi);
typedef struct { orc_range_fn fn; void* ctx; int lo, hi; } orc_job;

static void* orc_job_run(void* a) {
    orc_job* j = (orc_job*)a;
    j->fn(j->ctx, j->lo, j->hi);
    return NULL;
}

/* run fn over [0, n) split into nthreads contiguous ranges */
static void orc_parallel(orc_range_fn fn, void* ctx, int n, int nthreads) {
    if (nthreads < 1) nthreads = 1;
    if (nthreads > n) nthreads = n;
    if (nthreads <= 1) { if (n > 0) fn(ctx, 0, n); return; }
    pthread_t* th = (pthread_t*)malloc(sizeof(pthread_t) * nthreads);
    orc_job* jobs = (orc_job*)malloc(sizeof(orc_job) * nthreads);
    for (int i = 0; i < nthreads; ++i) {
        jobs[i].fn = fn; jobs[i].ctx = ctx;
        jobs[i].lo = (int)((long long)n * i / nthreads);
        jobs[i].hi = (int)((long long)n * (i + 1) / nthreads);
    }
    char* ok = (char*)calloc((size_t)nthreads, 1);
    for (int i = 0; i < nthreads; ++i)
        ok[i] = pthread_create(&th[i], NULL, orc_job_run, &jobs[i]) == 0;
    for (int i = 0; i < nthreads; ++i) {
        if (ok[i]) pthread_join(th[i], NULL);
        else orc_job_run(&jobs[i]);           /* thread not started: run here */
    }
    free(ok);
    free(th);
    free(jobs);
}

/* ---------------------------------------------------------------- 1. logits */

typedef struct {
    const void* x; int xdt; const void* wr; const float* bias;
    int d, E; double* L;
} logits_ctx;

static void logits_range(void* p, int lo, int hi) {
    logits_ctx* c = (logits_ctx*)p;
    for (int t = lo; t < hi; ++t)
        for (int e = 0; e < c->E; ++e) {
            double acc = 0.0;
            for (int i = 0; i < c->d; ++i)
                acc += act_value(c->x, c->xdt, (size_t)t * c->d + i) *
                       act_value(c->wr, c->xdt, (size_t)e * c->d + i);
            if (c->bias) acc += (double)c->bias[e];
            c->L[(size_t)t * c->E + e] = acc;
        }
}

/* L [T][E] = x [T][d] . W_r + bias ; the router weight is stored as
 * w_router [E][d] (row e is column e of W_r). */
int orc_router_logits(const void* x, int xdt, const void* w_router, const float* bias,
                      int T, int d, int E, double* L, int nthreads) {
    if (T < 0 || d <= 0 || E <= 0) return 1;
    logits_ctx c = {x, xdt, w_router, bias, d, E, L};
    orc_parallel(logits_range, &c, T, nthreads);
    return 0;
}

/* ---------------------------------------------------------------- 2. top-k */

/* Ranking order of two experts of one token: a ranks before b when its
 * logit is larger, or equal with the smaller index; NaN ranks last. */
static int ranks_before(double va, int a, double vb, int b) {
    int na = isnan(va), nb = isnan(vb);
    if (na || nb) {
        if (na && nb) return a < b;
        return nb;                      /* a number ranks before NaN */
    }
    if (va > vb) return 1;
    if (va < vb) return 0;
    return a < b;                       /* equal (incl. -0 == +0): lower index */
}

/* Select the k best experts per token, best first, and their weights
 * w[t,j] = exp(L_j - m) / sum_{j' selected} exp(L_j' - m), m = max_e L[t,e]. */
int orc_topk(const double* L, int T, int E, int k, int32_t* idx, double* w) {
    if (k < 1 || k > E) return 1;
    char* taken = (char*)malloc((size_t)E);
    for (int t = 0; t < T; ++t) {
        const double* row = L + (size_t)t * E;
        memset(taken, 0, (size_t)E);
        for (int j = 0; j < k; ++j) {
            int best = -1;
            for (int e = 0; e < E; ++e) {
                if (taken[e]) continue;
                if (best < 0 || ranks_before(row[e], e, row[best], best)) best = e;
            }
            taken[best] = 1;
            idx[(size_t)t * k + j] = best;
        }
        double m = -INFINITY;
        for (int e = 0; e < E; ++e) if (row[e] > m) m = row[e];
        double den = 0.0;
        for (int j = 0; j < k; ++j) den += exp(row[idx[(size_t)t * k + j]] - m);
        for (int j = 0; j < k; ++j)
            w[(size_t)t * k + j] = exp(row[idx[(size_t)t * k + j]] - m) / den;
    }
    free(taken);
    return 0;
}

/* The same weights by the other reading of the pages: p = softmax over all E
 * experts, then w_j = p_{idx_j} / sum_j' p_{idx_j'} for the given selection. */
int orc_topk_weights_full_softmax(const double* L, const int32_t* idx, int T, int E, int k,
                                  double* w) {
    double* p = (double*)malloc(sizeof(double) * (size_t)E);
    for (int t = 0; t < T; ++t) {
        const double* row = L + (size_t)t * E;
        double m = -INFINITY;
        for (int e = 0; e < E; ++e) if (row[e] > m) m = row[e];
        double z = 0.0;
        for (int e = 0; e < E; ++e) z += exp(row[e] - m);
        for (int e = 0; e < E; ++e) p[e] = exp(row[e] - m) / z;
        double s = 0.0;
        for (int j = 0; j < k; ++j) s += p[idx[(size_t)t * k + j]];
        for (int j = 0; j < k; ++j) w[(size_t)t * k + j] = p[idx[(size_t)t * k + j]] / s;
    }
    free(p);
    return 0;
}

/* ---------------------------------------------------------------- 3. sort */

/* Stable sort of routed slots r = t*k + j by expert id idx_flat[r]:
 * order lists, expert by expert, the slots of that expert in increasing r. */
int orc_sort_rows(const int32_t* idx, int T, int k, int E, int BM,
                  uint32_t* order, uint32_t* inv_order, uint32_t* row_map,
                  int32_t* counts, int32_t* row_off, int32_t* tile_off) {
    long long R = (long long)T * k;
    if (BM < 1 || E < 1) return 1;
    for (long long r = 0; r < R; ++r)
        if (idx[r] < 0 || idx[r] >= E) return 1;
    long long pos = 0;
    row_off[0] = 0;
    tile_off[0] = 0;
    for (int e = 0; e < E; ++e) {
        long long start = pos;
        for (long long r = 0; r < R; ++r)
            if (idx[r] == e) order[pos++] = (uint32_t)r;
        counts[e] = (int32_t)(pos - start);
        row_off[e + 1] = (int32_t)pos;
        tile_off[e + 1] = tile_off[e] + (counts[e] + BM - 1) / BM;
    }
    for (long long i = 0; i < R; ++i) {
        inv_order[order[i]] = (uint32_t)i;
        row_map[i] = order[i] / (uint32_t)k;
    }
    return 0;
}

/* ------------------------------------------------- 4. gate|up with SwiGLU */

typedef struct {
    const void* x; int xdt; const uint32_t* row_map; const int32_t* row_off;
    orc_wmat gu; int d, F; double* h; int act;
} swiglu_ctx;

/* The gate's activation of the GLU. act 0: silu(g) = g * sigmoid(g) =
 * g / (1 + exp(-g)) (SwiGLU). act 1: the tanh form of GELU (Hendrycks and
 * Gimpel), 0.5 g (1 + tanh(sqrt(2/pi) (g + 0.044715 g^3))) -- the
 * "tanh-GELU GLU" of mlx-lm PR #2044, "When it applies" (Gemma-4's GeGLU). */
static double glu_gate(double g, int act) {
    if (act == 1) {
        const double c = sqrt(2.0 / (4.0 * atan(1.0)));   /* sqrt(2 / pi) */
        return 0.5 * g * (1.0 + tanh(c * (g + 0.044715 * g * g * g)));
    }
    return g / (1.0 + exp(-g));
}

static void swiglu_range(void* p, int lo, int hi) {
    swiglu_ctx* c = (swiglu_ctx*)p;
    double* wg = (double*)malloc(sizeof(double) * c->d);
    double* wu = (double*)malloc(sizeof(double) * c->d);
    for (int e = lo; e < hi; ++e) {
        int r0 = c->row_off[e], r1 = c->row_off[e + 1];
        if (r0 == r1) continue;
        for (int f = 0; f < c->F; ++f) {
            weight_row(&c->gu, e, f, wg);              /* gate row f   */
            weight_row(&c->gu, e, c->F + f, wu);       /* up row F + f */
            for (int i = r0; i < r1; ++i) {
                size_t t = c->row_map[i];
                double g = 0.0, u = 0.0;
                for (int a = 0; a < c->d; ++a) {
                    double xv = act_value(c->x, c->xdt, t * c->d + a);
                    g += xv * wg[a];
                    u += xv * wu[a];
                }
                c->h[(size_t)i * c->F + f] = glu_gate(g, c->act) * u;
            }
        }
    }
    free(wg);
    free(wu);
}

/* h [R][F] for sorted rows; rows of expert e are [row_off[e], row_off[e+1]),
 * row i reads token row_map[i] of x. Weights w_gu [E][2F][d] (gate rows
 * 0..F-1, up rows F..2F-1). */
int orc_expert_swiglu(const void* x, int xdt, const uint32_t* row_map, const int32_t* row_off,
                      int E, int d, int F, int wfmt, const void* w_gu, const uint16_t* s_gu,
                      const uint16_t* b_gu, double* h, int act, int nthreads) {
    if (act != 0 && act != 1) return 1;
    swiglu_ctx c = {x, xdt, row_map, row_off, {wfmt, w_gu, s_gu, b_gu, 2 * F, d}, d, F, h, act};
    orc_parallel(swiglu_range, &c, E, nthreads);
    return 0;
}

/* Pre-activations of the same rows, for error bounds in the tests: g and u
 * as above, and the sums of absolute products |x| . |w_gate| and |x| . |w_up|
 * (each output [R][F]). */
typedef struct {
    const void* x; int xdt; const uint32_t* row_map; const int32_t* row_off;
    orc_wmat gu; int d, F; double *g, *u, *ga, *ua;
} gate_up_ctx;

static void gate_up_range(void* p, int lo, int hi) {
    gate_up_ctx* c = (gate_up_ctx*)p;
    double* wg = (double*)malloc(sizeof(double) * c->d);
    double* wu = (double*)malloc(sizeof(double) * c->d);
    for (int e = lo; e < hi; ++e) {
        int r0 = c->row_off[e], r1 = c->row_off[e + 1];
        if (r0 == r1) continue;
        for (int f = 0; f < c->F; ++f) {
            weight_row(&c->gu, e, f, wg);
            weight_row(&c->gu, e, c->F + f, wu);
            for (int i = r0; i < r1; ++i) {
                size_t t = c->row_map[i];
                double g = 0.0, u = 0.0, ga = 0.0, ua = 0.0;
                for (int a = 0; a < c->d; ++a) {
                    double xv = act_value(c->x, c->xdt, t * c->d + a);
                    g += xv * wg[a];
                    u += xv * wu[a];
                    ga += fabs(xv * wg[a]);
                    ua += fabs(xv * wu[a]);
                }
                size_t o = (size_t)i * c->F + f;
                c->g[o] = g; c->u[o] = u; c->ga[o] = ga; c->ua[o] = ua;
            }
        }
    }
    free(wg);
    free(wu);
}

int orc_expert_gate_up(const void* x, int xdt, const uint32_t* row_map, const int32_t* row_off,
                       int E, int d, int F, int wfmt, const void* w_gu, const uint16_t* s_gu,
                       const uint16_t* b_gu, double* g, double* u, double* ga, double* ua,
                       int nthreads) {
    gate_up_ctx c = {x, xdt, row_map, row_off, {wfmt, w_gu, s_gu, b_gu, 2 * F, d}, d, F,
                     g, u, ga, ua};
    orc_parallel(gate_up_range, &c, E, nthreads);
    return 0;
}

/* ---------------------------------------------------------------- 5. down */

typedef struct {
    const double* h; const int32_t* row_off; orc_wmat dn; int d, F; double* ys;
} down_ctx;

static void down_range(void* p, int lo, int hi) {
    down_ctx* c = (down_ctx*)p;
    double* wd = (double*)malloc(sizeof(double) * c->F);
    for (int e = lo; e < hi; ++e) {
        int r0 = c->row_off[e], r1 = c->row_off[e + 1];
        if (r0 == r1) continue;
        for (int o = 0; o < c->d; ++o) {
            weight_row(&c->dn, e, o, wd);
            for (int i = r0; i < r1; ++i) {
                double acc = 0.0;
                for (int f = 0; f < c->F; ++f) acc += c->h[(size_t)i * c->F + f] * wd[f];
                c->ys[(size_t)i * c->d + o] = acc;
            }
        }
    }
    free(wd);
}

/* ys [R][d] = h [R][F] . W_dn[e]^T for the rows of each expert e.
 * Weights w_dn [E][d][F]. */
int orc_expert_down(const double* h, const int32_t* row_off, int E, int d, int F, int wfmt,
                    const void* w_dn, const uint16_t* s_dn, const uint16_t* b_dn, double* ys,
                    int nthreads) {
    down_ctx c = {h, row_off, {wfmt, w_dn, s_dn, b_dn, d, F}, d, F, ys};
    orc_parallel(down_range, &c, E, nthreads);
    return 0;
}

/* Sums of absolute products |h[i]| . |w_dn[e][o]| (for error bounds). */
typedef struct {
    const double* h; const int32_t* row_off; orc_wmat dn; int d, F; double* out;
} down_abs_ctx;

static void down_abs_range(void* p, int lo, int hi) {
    down_abs_ctx* c = (down_abs_ctx*)p;
    double* wd = (double*)malloc(sizeof(double) * c->F);
    for (int e = lo; e < hi; ++e) {
        int r0 = c->row_off[e], r1 = c->row_off[e + 1];
        if (r0 == r1) continue;
        for (int o = 0; o < c->d; ++o) {
            weight_row(&c->dn, e, o, wd);
            for (int i = r0; i < r1; ++i) {
                double acc = 0.0;
                for (int f = 0; f < c->F; ++f) acc += fabs(c->h[(size_t)i * c->F + f] * wd[f]);
                c->out[(size_t)i * c->d + o] = acc;
            }
        }
    }
    free(wd);
}

int orc_expert_down_abs(const double* h, const int32_t* row_off, int E, int d, int F, int wfmt,
                        const void* w_dn, const uint16_t* s_dn, const uint16_t* b_dn, double* out,
                        int nthreads) {
    down_abs_ctx c = {h, row_off, {wfmt, w_dn, s_dn, b_dn, d, F}, d, F, out};
    orc_parallel(down_abs_range, &c, E, nthreads);
    return 0;
}

/* ------------------------------------------------------------- 6. combine */

/* y [T][d] : y[t,o] = sum_j w[t,j] * ys[inv_order[t*k+j], o], j = 0..k-1 */
int orc_combine(const double* ys, const uint32_t* inv_order, const double* w, int T, int k, int d,
                double* y) {
    for (int t = 0; t < T; ++t)
        for (int o = 0; o < d; ++o) {
            double acc = 0.0;
            for (int j = 0; j < k; ++j)
                acc += w[(size_t)t * k + j] * ys[(size_t)inv_order[(size_t)t * k + j] * d + o];
            y[(size_t)t * d + o] = acc;
        }
    return 0;
}

/* ------------------------------------------------------------- forward */

/* Whole layer. Logits are computed in fp64 and rounded to fp32 before the
 * selection and the weights (the library's logits are fp32); everything after
 * that stays in fp64 with no intermediate rounding.
 * Optional outputs (may be NULL): logits64 [T][E] (before rounding),
 * idx [T][k], w [T][k], h [R][F], ys [R][d]. */
int orc_forward(const void* x, int xdt, const void* w_router, const float* bias,
                int T, int d, int E, int k, int F, int BM,
                int wfmt, const void* w_gu, const uint16_t* s_gu, const uint16_t* b_gu,
                const void* w_dn, const uint16_t* s_dn, const uint16_t* b_dn,
                double* y, double* logits64, int32_t* idx_out, double* w_out,
                double* h_out, double* ys_out, int act, int nthreads) {
    if (k < 1 || k > E || T < 0) return 1;
    size_t R = (size_t)T * k;
    double* L = (double*)malloc(sizeof(double) * ((size_t)T * E + 1));
    int32_t* idx = (int32_t*)malloc(sizeof(int32_t) * (R + 1));
    double* w = (double*)malloc(sizeof(double) * (R + 1));
    uint32_t* order = (uint32_t*)malloc(sizeof(uint32_t) * (R + 1));
    uint32_t* inv = (uint32_t*)malloc(sizeof(uint32_t) * (R + 1));
    uint32_t* rmap = (uint32_t*)malloc(sizeof(uint32_t) * (R + 1));
    int32_t* counts = (int32_t*)malloc(sizeof(int32_t) * E);
    int32_t* roff = (int32_t*)malloc(sizeof(int32_t) * (E + 1));
    int32_t* toff = (int32_t*)malloc(sizeof(int32_t) * (E + 1));
    double* h = (double*)malloc(sizeof(double) * (R * F + 1));
    double* ys = (double*)malloc(sizeof(double) * (R * d + 1));
    int rc = orc_router_logits(x, xdt, w_router, bias, T, d, E, L, nthreads);
    if (rc == 0 && logits64) memcpy(logits64, L, sizeof(double) * (size_t)T * E);
    for (size_t i = 0; rc == 0 && i < (size_t)T * E; ++i) L[i] = (double)(float)L[i];
    if (rc == 0) rc = orc_topk(L, T, E, k, idx, w);
    if (rc == 0) rc = orc_sort_rows(idx, T, k, E, BM, order, inv, rmap, counts, roff, toff);
    if (rc == 0) rc = orc_expert_swiglu(x, xdt, rmap, roff, E, d, F, wfmt, w_gu, s_gu, b_gu, h, act, nthreads);
    if (rc == 0) rc = orc_expert_down(h, roff, E, d, F, wfmt, w_dn, s_dn, b_dn, ys, nthreads);
    if (rc == 0) rc = orc_combine(ys, inv, w, T, k, d, y);
    if (rc == 0) {
        if (idx_out) memcpy(idx_out, idx, sizeof(int32_t) * R);
        if (w_out) memcpy(w_out, w, sizeof(double) * R);
        if (h_out) memcpy(h_out, h, sizeof(double) * R * F);
        if (ys_out) memcpy(ys_out, ys, sizeof(double) * R * d);
    }
    free(L); free(idx); free(w); free(order); free(inv); free(rmap);
    free(counts); free(roff); free(toff); free(h); free(ys);
    return rc;
}

/* Dequantised value of one weight element, exported for the format pins. */
double orc_weight_value(int wfmt, const void* w, const uint16_t* s, const uint16_t* b,
                        int rows, int cols, int e, int r, int c) {
    orc_wmat m = {wfmt, w, s, b, rows, cols};
    return weight_value(&m, e, r, c);
}
