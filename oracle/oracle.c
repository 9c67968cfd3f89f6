/*
 * oracle.c -- plain, slow, fp64 CPU oracle of the routed Mixture-of-Experts FFN layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the benchmark's CPU
 * baseline load this file's library; the product path never does.  It shares no code,
 * header, table or helper with the CUDA library.
 *
 * What it computes (the layer described on the pages, written out as its definition):
 *
 *   router     logits[t][e] = sum_i x[t][i] * Wr[e][i]                       (fp64)
 *              softmax router ("Glacial", section "What works": exact Granite MoE
 *              forward; top-k on the logits, softmax renormalised over the k chosen);
 *              sigmoid router ("colibri" README, section "What's implemented":
 *              DeepSeek-V3-style sigmoid router, noaux_tc, routed_scaling_factor):
 *              key = sigmoid(logit) + bias (bias used for selection only),
 *              weight = scaling * sigmoid / sum of chosen sigmoids.
 *   selection  the k largest keys; equal keys go to the lower expert index; the
 *              output order is by rank (key descending, index ascending).
 *   experts    SwiGLU per expert: g = Wg x, u = Wu x, h = silu(g) * u, y = Wd h,
 *              the fused gate/up matrix holding the gate rows first and the up rows
 *              after them (open-1b-verify, "Tensor mapping": w_gate_up split at the
 *              row boundary; iliria, "What's implemented": gate+up fused).
 *   weights    packed int4 with one fp32 scale per output row, dequantised on use
 *              (colibri README, "What's implemented": int8 / packed int4 / packed int2,
 *              per-row scales, dequant-on-use), or bf16, or the int8 container (which
 *              holds the codes of any tier, one per byte), or packed int2.
 *   combine    out[t] = sum over chosen experts in ascending index of w * y, plus the
 *              shared expert with weight 1 (colibri README, "What's implemented":
 *              shared expert).
 *   union      batch-union: each chosen expert is applied to every token routed to it
 *              (colibri README, "What's implemented": batch-union MoE).  Evaluated
 *              per (token, row) with exactly the same summation order as the per-token
 *              path, so the two agree bit for bit.
 *
 * Quantiser (int4 tier): per row m = max|w| (fp32), s = m / 7 (fp32 IEEE division),
 * q = clamp(round-half-even(w / s), -8, 7); a zero row has s = 0 and q = 0; two nibbles
 * per byte, the even column in the low nibble.  Non-finite input is an error.
 *
 * Build: gcc -O2 -fopenmp -ffp-contract=off (never -ffast-math).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

enum { ORACLE_ROUTER_SOFTMAX = 0, ORACLE_ROUTER_SIGMOID = 1 };
enum { ORACLE_W_INT4 = 0, ORACLE_W_BF16 = 1, ORACLE_W_INT8 = 2, ORACLE_W_INT2 = 3 };
enum { ORACLE_MODE_PER_TOKEN = 0, ORACLE_MODE_UNION = 1, ORACLE_MODE_DENSE = 2 };
enum { ORACLE_OK = 0, ORACLE_ERR_RANGE = 1, ORACLE_ERR_MISSING_EXPERT = 2, ORACLE_ERR_ARG = 3,
       ORACLE_ERR_NOMEM = 4 };

typedef struct {
    int32_t d, f, n_experts, top_k, n_shared, f_shared, router, wkind;
    double scaling;
    const float *router_w;          /* [E][d] */
    const float *router_bias;       /* [E] or NULL */
    const void *const *gate_up;     /* [E] pointers to [2f][d/2] u8 | [2f][d] bf16 | [2f][d] s8 | [2f][d/4] u8 */
    const float *const *gate_up_scale;  /* [E] pointers to [2f] (int4 / int8) */
    const void *const *down;        /* [E] pointers to [d][f/2] u8 | [d][f] bf16 | [d][f] s8 */
    const float *const *down_scale;     /* [E] pointers to [d] */
    const void *shared_gate_up;
    const float *shared_gate_up_scale;
    const void *shared_down;
    const float *shared_down_scale;
    /* router variants (colibri README: "noaux_tc" and the "--topp" adaptive expert top-p knob);
     * n_group <= 1 and top_p outside (0, 1) leave the plain top-k router */
    int32_t n_group, topk_group;
    double top_p;
} oracle_layer;

/* ------------------------------------------------------------------------------------ */
/* scalar helpers                                                                          */
/* ------------------------------------------------------------------------------------ */

static double bf16_value(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float v;
    memcpy(&v, &u, sizeof v);
    return (double)v;
}

static int nibble_value(uint8_t byte, int high)
{
    int n = high ? (byte >> 4) : (byte & 0xF);
    return n >= 8 ? n - 16 : n;     /* two's-complement 4-bit value */
}

/* Code i (0..3) of a packed int2 byte: bits 2i .. 2i+1, a two's-complement 2-bit value. */
static int crumb_value(uint8_t byte, int i)
{
    int n = (byte >> (2 * i)) & 3;
    return n >= 2 ? n - 4 : n;
}

/* One weight of a [rows][cols] matrix in the layer's storage kind, dequantised, in fp64.
 * The product q * s is exact in fp64 (4-bit times 24-bit significands). */
static double weight_at(int wkind, const void *m, const float *scale, int64_t row, int64_t col,
                        int64_t cols)
{
    if (wkind == ORACLE_W_BF16)
        return bf16_value(((const uint16_t *)m)[row * cols + col]);
    if (wkind == ORACLE_W_INT8)
        return (double)((const int8_t *)m)[row * cols + col] * (double)scale[row];
    if (wkind == ORACLE_W_INT2) {
        uint8_t byte = ((const uint8_t *)m)[row * (cols / 4) + col / 4];
        return (double)crumb_value(byte, (int)(col & 3)) * (double)scale[row];
    }
    const uint8_t *p = (const uint8_t *)m;
    uint8_t byte = p[row * (cols / 2) + col / 2];
    return (double)nibble_value(byte, (int)(col & 1)) * (double)scale[row];
}

/* ------------------------------------------------------------------------------------ */
/* quantiser / packer                                                                       */
/* ------------------------------------------------------------------------------------ */

int oracle_quantize_int8(const float *w, int64_t rows, int64_t cols, int8_t *q, float *scales)
{
    if (rows < 0 || cols < 0) return ORACLE_ERR_ARG;
    int bad = 0;
    for (int64_t r = 0; r < rows; ++r) {
        const float *row = w + r * cols;
        float m = 0.0f;
        for (int64_t c = 0; c < cols; ++c) {
            if (!isfinite(row[c])) bad = 1;
            float a = fabsf(row[c]);
            if (a > m) m = a;
        }
        float s = m / 7.0f;
        scales[r] = s;
        for (int64_t c = 0; c < cols; ++c) {
            float v = 0.0f;
            if (s != 0.0f && isfinite(row[c])) v = rintf(row[c] / s);
            if (v > 7.0f) v = 7.0f;
            if (v < -8.0f) v = -8.0f;
            q[r * cols + c] = (int8_t)v;
        }
    }
    return bad ? ORACLE_ERR_RANGE : ORACLE_OK;
}

int oracle_pack_int4(const float *w, int64_t rows, int64_t cols, uint8_t *packed, float *scales)
{
    if (rows < 0 || cols < 0 || (cols & 1)) return ORACLE_ERR_ARG;
    int8_t *q = (int8_t *)malloc((size_t)(rows * cols > 0 ? rows * cols : 1));
    if (!q) return ORACLE_ERR_NOMEM;
    int rc = oracle_quantize_int8(w, rows, cols, q, scales);
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t j = 0; j < cols / 2; ++j) {
            uint8_t lo = (uint8_t)(q[r * cols + 2 * j] & 0xF);
            uint8_t hi = (uint8_t)(q[r * cols + 2 * j + 1] & 0xF);
            packed[r * (cols / 2) + j] = (uint8_t)(lo | (hi << 4));
        }
    free(q);
    return rc;
}

void oracle_unpack_int4(const uint8_t *packed, int64_t rows, int64_t cols, int8_t *q)
{
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t c = 0; c < cols; ++c)
            q[r * cols + c] = (int8_t)nibble_value(packed[r * (cols / 2) + c / 2], (int)(c & 1));
}

/*
 * The quantiser of the b-bit tier (b = 2, 4 or 8) into the int8 container, one code per byte
 * (colibri README, "What's implemented": int8 / packed int4 / packed int2 quantisation with
 * per-row scales).  The same symmetric rule as the int4 tier, with qmax = 2^(b-1) - 1:
 * per row m = max|w| (fp32), s = m / qmax (fp32 IEEE division), q = clamp(round-half-even(
 * fp32(w / s)), -qmax - 1, qmax); a zero row has s = 0 and q = 0.  Non-finite input is an
 * error (its codes are 0).
 */
int oracle_quantize_tier(const float *w, int64_t rows, int64_t cols, int32_t bits, int8_t *q, float *scales)
{
    if (rows < 0 || cols < 0 || (bits != 2 && bits != 4 && bits != 8)) return ORACLE_ERR_ARG;
    const float qmax = (float)((1 << (bits - 1)) - 1);
    const float qmin = -qmax - 1.0f;
    int bad = 0;
    for (int64_t r = 0; r < rows; ++r) {
        const float *row = w + r * cols;
        float m = 0.0f;
        for (int64_t c = 0; c < cols; ++c) {
            if (!isfinite(row[c])) bad = 1;
            float a = fabsf(row[c]);
            if (a > m) m = a;
        }
        float s = m / qmax;
        scales[r] = s;
        for (int64_t c = 0; c < cols; ++c) {
            float v = 0.0f;
            if (s != 0.0f && isfinite(row[c])) v = rintf(row[c] / s);
            if (v > qmax) v = qmax;
            if (v < qmin) v = qmin;
            q[r * cols + c] = (int8_t)v;
        }
    }
    return bad ? ORACLE_ERR_RANGE : ORACLE_OK;
}

/* Packed int2 container: the 2-bit tier's codes, four per byte, column 4j + i of a row in bits
 * 2i .. 2i+1 of byte j (the lowest column in the lowest bits, as the int4 container puts the
 * even column in the low nibble).  cols must be a multiple of 4. */
int oracle_pack_int2(const float *w, int64_t rows, int64_t cols, uint8_t *packed, float *scales)
{
    if (rows < 0 || cols < 0 || (cols & 3)) return ORACLE_ERR_ARG;
    int8_t *q = (int8_t *)malloc((size_t)(rows * cols > 0 ? rows * cols : 1));
    if (!q) return ORACLE_ERR_NOMEM;
    int rc = oracle_quantize_tier(w, rows, cols, 2, q, scales);
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t j = 0; j < cols / 4; ++j) {
            uint8_t b = 0;
            for (int i = 0; i < 4; ++i) b |= (uint8_t)((q[r * cols + 4 * j + i] & 3) << (2 * i));
            packed[r * (cols / 4) + j] = b;
        }
    free(q);
    return rc;
}

void oracle_unpack_int2(const uint8_t *packed, int64_t rows, int64_t cols, int8_t *q)
{
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t c = 0; c < cols; ++c)
            q[r * cols + c] = (int8_t)crumb_value(packed[r * (cols / 4) + c / 4], (int)(c & 3));
}

/* ------------------------------------------------------------------------------------ */
/* router                                                                                   */
/* ------------------------------------------------------------------------------------ */

/* Group-limited selection (the DeepSeek-V3 router, "noaux_tc", with n_group > 1): the experts
 * form n_group contiguous groups of E / n_group; a group's score is the sum of its two largest
 * keys (its only key for groups of one); the topk_group best groups (score descending, lower group
 * index first on equal scores) stay selectable, and the experts of every other group are marked
 * taken, i.e. excluded. */
static void limit_groups(const oracle_layer *L, const double *key, unsigned char *taken)
{
    const int E = L->n_experts, G = L->n_group;
    if (G <= 1) return;
    const int per = E / G;
    double score[64];
    unsigned char keep[64];
    for (int g = 0; g < G; ++g) {
        double b1 = -INFINITY, b2 = -INFINITY;
        for (int e = g * per; e < (g + 1) * per; ++e) {
            if (key[e] > b1) { b2 = b1; b1 = key[e]; }
            else if (key[e] > b2) b2 = key[e];
        }
        score[g] = per >= 2 ? b1 + b2 : b1;
        keep[g] = 0;
    }
    for (int r = 0; r < L->topk_group; ++r) {
        int best = -1;
        for (int g = 0; g < G; ++g)
            if (!keep[g] && (best < 0 || score[g] > score[best])) best = g;
        keep[best] = 1;
    }
    for (int e = 0; e < E; ++e)
        if (!keep[e / per]) taken[e] = 1;
}

/* Adaptive expert top-p: in rank order, the first m experts whose weights, as a share of the k
 * weights' total, add up to at least p (1 <= m <= k) are kept; the others are dropped (index -1,
 * weight 0) and the kept weights are scaled back up to the k weights' total. */
static void apply_top_p(double p, int k, int32_t *idx, double *w)
{
    if (!(p > 0.0 && p < 1.0)) return;
    double total = 0.0;
    for (int r = 0; r < k; ++r) total += w[r];
    double cum = 0.0;
    int m = k;
    for (int r = 0; r < k; ++r) {
        cum += w[r];
        if (cum / total >= p) { m = r + 1; break; }
    }
    double kept = 0.0;
    for (int r = 0; r < m; ++r) kept += w[r];
    for (int r = 0; r < k; ++r) {
        if (r < m) {
            w[r] = w[r] * (total / kept);
        } else {
            w[r] = 0.0;
            idx[r] = -1;
        }
    }
}

/* Routes one token.  key/logit scratch of length E.  Writes idx[k] (rank order), w[k]
 * (fp64), and the gap between the k-th and (k+1)-th largest key (+inf when k == E). */
static void route_token(const oracle_layer *L, const uint16_t *xt, double *logit, double *key,
                        unsigned char *taken, int32_t *idx, double *w, double *gap)
{
    const int E = L->n_experts, d = L->d, k = L->top_k;
    for (int e = 0; e < E; ++e) {
        double acc = 0.0;
        const float *wr = L->router_w + (int64_t)e * d;
        for (int i = 0; i < d; ++i) acc += bf16_value(xt[i]) * (double)wr[i];
        logit[e] = acc;
        if (L->router == ORACLE_ROUTER_SIGMOID) {
            double sig = 1.0 / (1.0 + exp(-acc));
            key[e] = sig + (L->router_bias ? (double)L->router_bias[e] : 0.0);
        } else {
            key[e] = acc;
        }
        taken[e] = 0;
    }
    limit_groups(L, key, taken);
    for (int r = 0; r < k; ++r) {
        int best = -1;
        for (int e = 0; e < E; ++e)
            if (!taken[e] && (best < 0 || key[e] > key[best])) best = e;
        taken[best] = 1;
        idx[r] = best;
    }
    double next = -INFINITY;
    for (int e = 0; e < E; ++e)
        if (!taken[e] && key[e] > next) next = key[e];
    *gap = (k < E) ? key[idx[k - 1]] - next : INFINITY;

    if (L->router == ORACLE_ROUTER_SIGMOID) {
        double sum = 0.0;
        for (int r = 0; r < k; ++r) sum += 1.0 / (1.0 + exp(-logit[idx[r]]));
        for (int r = 0; r < k; ++r) w[r] = L->scaling * (1.0 / (1.0 + exp(-logit[idx[r]]))) / sum;
    } else {
        double m = logit[idx[0]];
        for (int r = 1; r < k; ++r) if (logit[idx[r]] > m) m = logit[idx[r]];
        double sum = 0.0;
        for (int r = 0; r < k; ++r) sum += exp(logit[idx[r]] - m);
        for (int r = 0; r < k; ++r) w[r] = L->scaling * exp(logit[idx[r]] - m) / sum;
    }
    apply_top_p(L->top_p, k, idx, w);
}

int oracle_route(const oracle_layer *L, const uint16_t *x, int32_t T, int32_t *idx, double *w,
                 double *logits, double *gap)
{
    const int E = L->n_experts;
    if (L->top_k < 1 || L->top_k > E || T < 0) return ORACLE_ERR_ARG;
    if (L->n_group > 1 && (L->n_group > 64 || E % L->n_group || L->topk_group < 1 || L->topk_group > L->n_group ||
                           L->topk_group * (E / L->n_group) < L->top_k))
        return ORACLE_ERR_ARG;
    int rc = ORACLE_OK;
#pragma omp parallel
    {
        double *key = (double *)malloc(sizeof(double) * (size_t)E);
        double *lg = (double *)malloc(sizeof(double) * (size_t)E);
        unsigned char *taken = (unsigned char *)malloc((size_t)E);
        if (!key || !lg || !taken) {
#pragma omp atomic write
            rc = ORACLE_ERR_NOMEM;
        } else {
#pragma omp for schedule(static)
            for (int t = 0; t < T; ++t) {
                route_token(L, x + (int64_t)t * L->d, lg, key, taken, idx + (int64_t)t * L->top_k,
                            w + (int64_t)t * L->top_k, gap + t);
                if (logits) memcpy(logits + (int64_t)t * E, lg, sizeof(double) * (size_t)E);
            }
        }
        free(key); free(lg); free(taken);
    }
    return rc;
}

/* ------------------------------------------------------------------------------------ */
/* expert FFN                                                                               */
/* ------------------------------------------------------------------------------------ */

typedef struct {
    const void *gate_up; const float *gate_up_scale;
    const void *down; const float *down_scale;
    int f;
} expert_ref;

static int get_expert(const oracle_layer *L, int e, expert_ref *out)
{
    if (e == L->n_experts) {        /* the shared expert */
        out->gate_up = L->shared_gate_up; out->gate_up_scale = L->shared_gate_up_scale;
        out->down = L->shared_down; out->down_scale = L->shared_down_scale;
        out->f = L->f_shared;
    } else {
        out->gate_up = L->gate_up ? L->gate_up[e] : NULL;
        out->gate_up_scale = L->gate_up_scale ? L->gate_up_scale[e] : NULL;
        out->down = L->down ? L->down[e] : NULL;
        out->down_scale = L->down_scale ? L->down_scale[e] : NULL;
        out->f = L->f;
    }
    if (!out->gate_up || !out->down) return ORACLE_ERR_MISSING_EXPERT;
    if (L->wkind != ORACLE_W_BF16 && (!out->gate_up_scale || !out->down_scale))
        return ORACLE_ERR_MISSING_EXPERT;
    return ORACLE_OK;
}

/* SwiGLU of one expert on one token, in fp64.  Optional exports g, u, h ([f]); y is [d].
 * Rows are independent, so they are split across threads; each row's sum runs over the
 * columns in ascending order whatever the thread count. */
static void expert_apply(const oracle_layer *L, const expert_ref *ex, const double *x, double *g_out,
                         double *u_out, double *h, double *y)
{
    const int d = L->d, f = ex->f, wk = L->wkind;
#pragma omp parallel for schedule(static) if (f >= 64)
    for (int r = 0; r < f; ++r) {
        double g = 0.0, u = 0.0;
        for (int i = 0; i < d; ++i) g += weight_at(wk, ex->gate_up, ex->gate_up_scale, r, i, d) * x[i];
        for (int i = 0; i < d; ++i)
            u += weight_at(wk, ex->gate_up, ex->gate_up_scale, (int64_t)f + r, i, d) * x[i];
        if (g_out) g_out[r] = g;
        if (u_out) u_out[r] = u;
        h[r] = g / (1.0 + exp(-g)) * u;
    }
#pragma omp parallel for schedule(static) if (d >= 64)
    for (int j = 0; j < d; ++j) {
        double acc = 0.0;
        for (int r = 0; r < f; ++r) acc += weight_at(wk, ex->down, ex->down_scale, j, r, f) * h[r];
        y[j] = acc;
    }
}

int oracle_expert_ffn(const oracle_layer *L, int32_t e, const uint16_t *xt, double *g, double *u,
                      double *h, double *y)
{
    expert_ref ex;
    if (e < 0 || e > L->n_experts || (e == L->n_experts && L->n_shared < 1)) return ORACLE_ERR_ARG;
    int rc = get_expert(L, e, &ex);
    if (rc) return rc;
    double *x = (double *)malloc(sizeof(double) * (size_t)L->d);
    if (!x) return ORACLE_ERR_NOMEM;
    for (int i = 0; i < L->d; ++i) x[i] = bf16_value(xt[i]);
    expert_apply(L, &ex, x, g, u, h, y);
    free(x);
    return ORACLE_OK;
}

/* ------------------------------------------------------------------------------------ */
/* layer forward                                                                            */
/* ------------------------------------------------------------------------------------ */

/* Sort the k chosen experts of one token by ascending index (insertion sort), carrying
 * their weights along: the combine adds experts in that order. */
static void ascending(int k, const int32_t *idx, const double *w, int32_t *si, double *sw)
{
    for (int r = 0; r < k; ++r) { si[r] = idx[r]; sw[r] = w[r]; }
    for (int a = 1; a < k; ++a) {
        int32_t ki = si[a]; double kw = sw[a]; int b = a - 1;
        while (b >= 0 && si[b] > ki) { si[b + 1] = si[b]; sw[b + 1] = sw[b]; --b; }
        si[b + 1] = ki; sw[b + 1] = kw;
    }
}

static int max_f(const oracle_layer *L) { return L->f_shared > L->f ? L->f_shared : L->f; }

/*
 * out    [T][d] fp64
 * idx    [T][k] rank order, w [T][k] fp64, gap [T] (may be NULL)
 * mode   per-token | batch-union | dense (all E experts, zero gate for the unchosen)
 */
int oracle_forward(const oracle_layer *L, const uint16_t *x, int32_t T, int32_t mode, double *out,
                   int32_t *idx, double *w, double *gap)
{
    const int d = L->d, E = L->n_experts, k = L->top_k;
    const int S = L->n_shared > 0 ? 1 : 0;
    if (T < 0 || k < 1 || k > E || (L->wkind == ORACLE_W_INT4 && ((d & 1) || (L->f & 1))) ||
        (L->wkind == ORACLE_W_INT2 && ((d & 3) || (L->f & 3) || (S && (L->f_shared & 3)))))
        return ORACLE_ERR_ARG;
    double *gap_buf = gap ? gap : (double *)malloc(sizeof(double) * (size_t)(T > 0 ? T : 1));
    int rc = oracle_route(L, x, T, idx, w, NULL, gap_buf);
    if (!gap) free(gap_buf);
    if (rc) return rc;

    double *xd = (double *)malloc(sizeof(double) * (size_t)d);
    double *h = (double *)malloc(sizeof(double) * (size_t)max_f(L));
    double *y = (double *)malloc(sizeof(double) * (size_t)d);
    int32_t *si = (int32_t *)malloc(sizeof(int32_t) * (size_t)k);
    double *sw = (double *)malloc(sizeof(double) * (size_t)k);
    if (!xd || !h || !y || !si || !sw) { rc = ORACLE_ERR_NOMEM; goto done; }

    if (mode == ORACLE_MODE_PER_TOKEN || mode == ORACLE_MODE_DENSE) {
        double *gate = (double *)malloc(sizeof(double) * (size_t)E);
        if (!gate) { rc = ORACLE_ERR_NOMEM; goto done; }
        for (int t = 0; t < T && !rc; ++t) {
            double *o = out + (int64_t)t * d;
            for (int i = 0; i < d; ++i) { xd[i] = bf16_value(x[(int64_t)t * d + i]); o[i] = 0.0; }
            ascending(k, idx + (int64_t)t * k, w + (int64_t)t * k, si, sw);
            if (mode == ORACLE_MODE_PER_TOKEN) {
                for (int r = 0; r < k && !rc; ++r) {
                    expert_ref ex;
                    if (si[r] < 0) continue;          /* dropped by top-p */
                    if ((rc = get_expert(L, si[r], &ex))) break;
                    expert_apply(L, &ex, xd, NULL, NULL, h, y);
                    for (int j = 0; j < d; ++j) o[j] += sw[r] * y[j];
                }
            } else {
                for (int e = 0; e < E; ++e) gate[e] = 0.0;
                for (int r = 0; r < k; ++r)
                    if (si[r] >= 0) gate[si[r]] = sw[r];
                for (int e = 0; e < E && !rc; ++e) {
                    expert_ref ex;
                    if ((rc = get_expert(L, e, &ex))) break;
                    expert_apply(L, &ex, xd, NULL, NULL, h, y);
                    for (int j = 0; j < d; ++j) o[j] += gate[e] * y[j];
                }
            }
            if (!rc && S) {
                expert_ref ex;
                if ((rc = get_expert(L, E, &ex))) break;
                expert_apply(L, &ex, xd, NULL, NULL, h, y);
                for (int j = 0; j < d; ++j) o[j] += y[j];
            }
        }
        free(gate);
    } else if (mode == ORACLE_MODE_UNION) {
        /* y_all[t][slot][d]: slot r holds the r-th chosen expert in ascending index, slot k the
         * shared expert.  Each unique expert is visited once and applied to its whole bucket. */
        const int slots = k + S;
        double *y_all = (double *)malloc(sizeof(double) * (size_t)T * (size_t)slots * (size_t)d + 8);
        int32_t *sorted_idx = (int32_t *)malloc(sizeof(int32_t) * (size_t)T * (size_t)k + 4);
        double *sorted_w = (double *)malloc(sizeof(double) * (size_t)T * (size_t)k + 8);
        if (!y_all || !sorted_idx || !sorted_w) {
            free(y_all); free(sorted_idx); free(sorted_w); rc = ORACLE_ERR_NOMEM; goto done;
        }
        for (int t = 0; t < T; ++t)
            ascending(k, idx + (int64_t)t * k, w + (int64_t)t * k, sorted_idx + (int64_t)t * k,
                      sorted_w + (int64_t)t * k);
        for (int e = 0; e <= E && !rc; ++e) {
            if (e == E && !S) break;
            int used = 0;
            expert_ref ex;
            for (int t = 0; t < T && !rc; ++t) {
                int slot = -1;
                if (e == E) slot = k;
                else
                    for (int r = 0; r < k; ++r) if (sorted_idx[(int64_t)t * k + r] == e) slot = r;
                if (slot < 0) continue;
                if (!used) { if ((rc = get_expert(L, e, &ex))) break; used = 1; }
                for (int i = 0; i < d; ++i) xd[i] = bf16_value(x[(int64_t)t * d + i]);
                expert_apply(L, &ex, xd, NULL, NULL, h, y_all + ((int64_t)t * slots + slot) * d);
            }
        }
        for (int t = 0; t < T && !rc; ++t) {
            double *o = out + (int64_t)t * d;
            for (int j = 0; j < d; ++j) o[j] = 0.0;
            for (int r = 0; r < k; ++r) {
                if (sorted_idx[(int64_t)t * k + r] < 0) continue;     /* dropped by top-p */
                const double *ys = y_all + ((int64_t)t * slots + r) * d;
                for (int j = 0; j < d; ++j) o[j] += sorted_w[(int64_t)t * k + r] * ys[j];
            }
            if (S) {
                const double *ys = y_all + ((int64_t)t * slots + k) * d;
                for (int j = 0; j < d; ++j) o[j] += ys[j];
            }
        }
        free(y_all); free(sorted_idx); free(sorted_w);
    } else {
        rc = ORACLE_ERR_ARG;
    }
done:
    free(xd); free(h); free(y); free(si); free(sw);
    return rc;
}

int oracle_num_threads(void)
{
#ifdef _OPENMP
    extern int omp_get_max_threads(void);
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Threads of the following oracle calls (n >= 1): only the timing of the CPU baseline on one
 * core uses it.  The results do not depend on it: every parallel loop writes disjoint outputs
 * and each sum runs in its own fixed order inside one thread. */
void oracle_set_num_threads(int n)
{
#ifdef _OPENMP
    extern void omp_set_num_threads(int);
    if (n >= 1) omp_set_num_threads(n);
#else
    (void)n;
#endif
}
