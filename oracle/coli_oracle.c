/*
 * CPU oracle for one routed-expert MoE layer with int4 gs64 experts.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the package's smoke check and
 * the benchmark's CPU-baseline leg may load this library.  It shares no code,
 * header or table with the CUDA library; it is plain, slow and written so a
 * reader can check it against the definitions by eye.  Everything is computed
 * per token, in double precision.
 *
 * What it computes (sources are the pages about the Colibri engine):
 *   - routing: k of E routed experts per token ("zhichai.net/topic/178503686",
 *     MoE-sparsity section: 256 experts, 8 + 1 active per layer, the router
 *     picks 8 per token); softmax over the chosen k (a reading: the pages do
 *     not name the scoring function);
 *   - the shared expert: always on, weight 1.0 (same page, three-tier storage
 *     section: the "+1" shared expert active in every layer);
 *   - batch-union: the per-expert lists of (token, slot) pairs, so an expert is
 *     read once for all positions that need it ("yunpan.plus/t/30351-1-1",
 *     capability two, batch-union bullet);
 *   - int4 gs64 weights ("yunpan.plus/t/30351-1-1", capability four: gs64 vs
 *     per-row int4): W[n][k] = q[n][k] * s[n][k / 64], q a signed nibble;
 *   - the expert FFN (SwiGLU; a reading): y = W_d (silu(W_g x) * (W_u x)).
 *
 * Readings where the pages are silent (each listed in the design notes):
 *   - selection runs on the logits; order is logit descending, ties to the
 *     lower expert index; -0 == +0; NaN ranks below -inf;
 *   - w_j = exp(l_j - m) / sum_i exp(l_i - m) over the chosen set, m the top
 *     value; NaN counts as exp() = 0; if m = +inf the +inf entries share the
 *     weight equally; if m is -inf or NaN every slot gets 1/k;
 *   - nibble order: low nibble = even k, high nibble = odd k; codes are
 *     two's complement in [-8, 7], no zero point;
 *   - scales: bf16, row-major [rows][K/64];
 *   - gate/up are [I][H], down is [H][I], packed along the reduction dim.
 *
 * Parity pins: every function here is checked by the CPU test suite against
 * closed forms, brute force, hand-packed bytes and an independent numpy
 * restatement; none of those checks call back into this file's arithmetic.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
    const uint8_t *gate_q, *up_q, *down_q;   /* [I][H/2], [I][H/2], [H][I/2] */
    const uint16_t *gate_s, *up_s, *down_s;  /* bf16 bits [I][H/64], [I][H/64], [H][I/64];
                                                per-row: [I][1], [I][1], [H][1] */
    int32_t group;                           /* 64: gs64; 0: one scale per row */
} oracle_expert;

/* ---- scalar formats --------------------------------------------------- */

/* bf16 is the top half of an IEEE binary32. */
double oracle_bf16_to_double(uint16_t bits) {
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* Signed int4 code number `k` of a row packed two per byte (even k in the
 * low nibble). */
int oracle_int4_code(const uint8_t *row, int64_t k) {
    uint8_t byte = row[k / 2];
    int nib = (k % 2 == 0) ? (byte & 0x0F) : (byte >> 4);
    return nib >= 8 ? nib - 16 : nib;
}

/* Inverse of oracle_int4_code over a row of n codes (n even). */
void oracle_int4_pack(const int8_t *codes, int64_t n, uint8_t *row) {
    for (int64_t i = 0; i < n / 2; ++i) {
        uint8_t lo = (uint8_t)(codes[2 * i] & 0x0F);
        uint8_t hi = (uint8_t)(codes[2 * i + 1] & 0x0F);
        row[i] = (uint8_t)(lo | (hi << 4));
    }
}

/* Dequantised weight W[n][k] of a [rows][K] matrix in the legacy per-row
 * int4 format: the same codes, one bf16 scale per row, W[n][k] = q[n][k] *
 * s[n] ("ssnai.com/JustVugg_colibri.html", decision guide: the older per-row
 * int4 GLM-5.2 mirror; "yunpan.plus/t/30351-1-1", capability four: gs64
 * against per-row int4).  The pages do not print the layout; this reading
 * keeps everything of gs64 but the scale index. */
double oracle_weight_per_row(const uint8_t *q, const uint16_t *s, int64_t K, int64_t n,
                             int64_t k) {
    const uint8_t *row = q + n * (K / 2);
    return (double)oracle_int4_code(row, k) * oracle_bf16_to_double(s[n]);
}

/* W[n][k] of an expert matrix in the expert's format (gs64 or per-row). */
static double weight_of(const uint8_t *q, const uint16_t *s, int64_t K, int32_t group, int64_t n,
                        int64_t k);

/* Dequantised weight W[n][k] of a [rows][K] gs64 matrix. */
double oracle_weight(const uint8_t *q, const uint16_t *s, int64_t K, int64_t n, int64_t k) {
    const uint8_t *row = q + n * (K / 2);
    double scale = oracle_bf16_to_double(s[n * (K / 64) + k / 64]);
    return (double)oracle_int4_code(row, k) * scale;
}

static double weight_of(const uint8_t *q, const uint16_t *s, int64_t K, int32_t group, int64_t n,
                        int64_t k) {
    return group == 0 ? oracle_weight_per_row(q, s, K, n, k) : oracle_weight(q, s, K, n, k);
}

/* ---- routing ----------------------------------------------------------- */

/* 1 if (va, a) is ranked before (vb, b). */
static int ranks_before(float va, int a, float vb, int b) {
    int nan_a = isnan(va), nan_b = isnan(vb);
    if (nan_a != nan_b) return nan_b;          /* any number beats NaN */
    if (!nan_a) {
        if (va > vb) return 1;
        if (va < vb) return 0;
    }
    return a < b;                              /* equal (or both NaN): lower index */
}

/* Top-k of each logits row and the renormalised softmax weights.
 * idx [T][k], w [T][k].  Returns 0, or -1 on bad sizes. */
int oracle_route(int T, int E, int k, const float *logits, int32_t *idx, double *w) {
    if (T < 0 || E < 1 || k < 1 || k > E) return -1;
    unsigned char *taken = (unsigned char *)malloc((size_t)E);
    if (!taken) return -1;
    for (int t = 0; t < T; ++t) {
        const float *l = logits + (int64_t)t * E;
        memset(taken, 0, (size_t)E);
        /* k passes, each picking the best expert not yet taken */
        for (int j = 0; j < k; ++j) {
            int best = -1;
            for (int e = 0; e < E; ++e) {
                if (taken[e]) continue;
                if (best < 0 || ranks_before(l[e], e, l[best], best)) best = e;
            }
            taken[best] = 1;
            idx[(int64_t)t * k + j] = best;
        }
        int32_t *S = idx + (int64_t)t * k;
        double *wt = w + (int64_t)t * k;
        double m = (double)l[S[0]];
        if (isinf(m) && m > 0) {
            int n_inf = 0;
            for (int j = 0; j < k; ++j) n_inf += (isinf(l[S[j]]) && l[S[j]] > 0);
            for (int j = 0; j < k; ++j)
                wt[j] = (isinf(l[S[j]]) && l[S[j]] > 0) ? 1.0 / n_inf : 0.0;
        } else if (isnan(m) || (isinf(m) && m < 0)) {
            for (int j = 0; j < k; ++j) wt[j] = 1.0 / k;
        } else {
            double z = 0.0;
            for (int j = 0; j < k; ++j) {
                double v = (double)l[S[j]];
                wt[j] = isnan(v) ? 0.0 : exp(v - m);
                z += wt[j];
            }
            for (int j = 0; j < k; ++j) wt[j] /= z;
        }
    }
    free(taken);
    return 0;
}

/* Router logits in double: logits[t][e] = sum_h x[t][h] * Wr[e][h]. */
void oracle_router_logits(int T, int E, int H, const uint16_t *x_bf16, const float *Wr,
                          double *logits) {
    for (int t = 0; t < T; ++t)
        for (int e = 0; e < E; ++e) {
            double acc = 0.0;
            for (int h = 0; h < H; ++h)
                acc += oracle_bf16_to_double(x_bf16[(int64_t)t * H + h]) *
                       (double)Wr[(int64_t)e * H + h];
            logits[(int64_t)t * E + e] = acc;
        }
}

/* ---- batch-union --------------------------------------------------------- */

/* Bucket the T*k (token, slot) pairs by expert.  A pair is p = t*k + j.
 * counts[e]: pairs routed to e; offsets[e]: start of e's list (offsets[E] =
 * T*k); pairs[]: the lists, expert-major, ascending token; active[]: experts
 * with a non-empty list, ascending; *n_active: their number.
 * Returns 0, or -1 if an index lies outside [0, E). */
int oracle_union(int T, int E, int k, const int32_t *idx, int32_t *counts,
                 int32_t *offsets, int32_t *pairs, int32_t *active, int32_t *n_active) {
    int64_t P = (int64_t)T * k;
    for (int64_t p = 0; p < P; ++p)
        if (idx[p] < 0 || idx[p] >= E) return -1;
    int64_t pos = 0;
    int na = 0;
    for (int e = 0; e < E; ++e) {
        offsets[e] = (int32_t)pos;
        int32_t c = 0;
        for (int t = 0; t < T; ++t)
            for (int j = 0; j < k; ++j)
                if (idx[(int64_t)t * k + j] == e) {
                    pairs[pos++] = t * k + j;
                    ++c;
                }
        counts[e] = c;
        if (c > 0) active[na++] = e;
    }
    offsets[E] = (int32_t)pos;
    for (int e = na; e < E; ++e) active[e] = -1;
    *n_active = na;
    return 0;
}

/* ---- expert FFN ---------------------------------------------------------- */

static double silu(double z) { return z / (1.0 + exp(-z)); }

/* y[H] = FFN_e(x[H]) with SwiGLU, all in double.  `tmp` holds I doubles. */
static void expert_ffn(int H, int I, const oracle_expert *ex, const double *x, double *y,
                       double *tmp) {
    for (int n = 0; n < I; ++n) {
        double g = 0.0, u = 0.0;
        for (int k = 0; k < H; ++k) {
            g += weight_of(ex->gate_q, ex->gate_s, H, ex->group, n, k) * x[k];
            u += weight_of(ex->up_q, ex->up_s, H, ex->group, n, k) * x[k];
        }
        tmp[n] = silu(g) * u;
    }
    for (int m = 0; m < H; ++m) {
        double acc = 0.0;
        for (int n = 0; n < I; ++n)
            acc += weight_of(ex->down_q, ex->down_s, I, ex->group, m, n) * tmp[n];
        y[m] = acc;
    }
}

void oracle_expert_ffn(int H, int I, const oracle_expert *ex, const double *x, double *y) {
    double *tmp = (double *)malloc(sizeof(double) * (size_t)I);
    expert_ffn(H, I, ex, x, y, tmp);
    free(tmp);
}

/* ---- whole layer, per token -------------------------------------------- */

typedef struct {
    int H, I, E, k, n_shared;
    const oracle_expert *experts;   /* E routed, then n_shared shared */
    const uint16_t *x_bf16;         /* [T][H] */
    const int32_t *idx;             /* [T][k] chosen experts */
    const int32_t *sample;          /* tokens to evaluate */
    int n_sample;
    double *ybuf;                   /* [n_sample][k + n_shared][H] expert outputs */
    int next;                       /* work counter */
    pthread_mutex_t lock;
} layer_job;

/* One work item: expert output FFN_e(x_t) for one (sampled token, slot). */
static void layer_item(const layer_job *J, int item, double *x, double *tmp) {
    int H = J->H, I = J->I, per = J->k + J->n_shared;
    int si = item / per, j = item % per, t = J->sample[si];
    int e = j < J->k ? J->idx[(int64_t)t * J->k + j] : J->E + (j - J->k);
    for (int h = 0; h < H; ++h) x[h] = oracle_bf16_to_double(J->x_bf16[(int64_t)t * H + h]);
    expert_ffn(H, I, &J->experts[e], x, J->ybuf + (int64_t)item * H, tmp);
}

static void *layer_worker(void *arg) {
    layer_job *J = (layer_job *)arg;
    double *x = (double *)malloc(sizeof(double) * (size_t)J->H);
    double *tmp = (double *)malloc(sizeof(double) * (size_t)J->I);
    int n_items = J->n_sample * (J->k + J->n_shared);
    for (;;) {
        pthread_mutex_lock(&J->lock);
        int item = J->next++;
        pthread_mutex_unlock(&J->lock);
        if (item >= n_items) break;
        layer_item(J, item, x, tmp);
    }
    free(x);
    free(tmp);
    return NULL;
}

/* out[s][H] = sum_j w[t][j] FFN_{idx[t][j]}(x_t) + sum_shared FFN_sh(x_t)
 *             (+ residual[t]),  t = sample[s].
 * Routing is given (idx, w from oracle_route).  Each expert output is computed
 * by one thread and the sum is formed afterwards in a fixed order, so the
 * result does not depend on the thread count. */
int oracle_layer(int H, int I, int E, int k, int n_shared, const oracle_expert *experts,
                 int T, const uint16_t *x_bf16, const int32_t *idx, const double *w,
                 const double *residual, const int32_t *sample, int n_sample, double *out,
                 int n_threads) {
    if (H % 128 || I % 128 || k < 1 || k > E || n_shared < 0 || T < 0) return -1;
    for (int s = 0; s < n_sample; ++s)
        if (sample[s] < 0 || sample[s] >= T) return -1;
    for (int s = 0; s < n_sample; ++s)
        for (int j = 0; j < k; ++j) {
            int e = idx[(int64_t)sample[s] * k + j];
            if (e < 0 || e >= E) return -1;
        }
    int per = k + n_shared;
    layer_job J;
    J.H = H; J.I = I; J.E = E; J.k = k; J.n_shared = n_shared; J.experts = experts;
    J.x_bf16 = x_bf16; J.idx = idx; J.sample = sample; J.n_sample = n_sample; J.next = 0;
    J.ybuf = (double *)malloc(sizeof(double) * (size_t)n_sample * per * H + 8);
    if (!J.ybuf) return -1;
    pthread_mutex_init(&J.lock, NULL);
    if (n_threads < 1) n_threads = 1;
    if (n_threads > 256) n_threads = 256;
    pthread_t th[256];
    int started = 0;
    for (int i = 1; i < n_threads; ++i)
        if (pthread_create(&th[started], NULL, layer_worker, &J) == 0) ++started;
    layer_worker(&J);
    for (int i = 0; i < started; ++i) pthread_join(th[i], NULL);
    pthread_mutex_destroy(&J.lock);

    for (int s = 0; s < n_sample; ++s) {
        int t = sample[s];
        double *o = out + (int64_t)s * H;
        const double *ys = J.ybuf + (int64_t)s * per * H;
        for (int h = 0; h < H; ++h) {
            double acc = 0.0;
            for (int j = 0; j < k; ++j) acc += w[(int64_t)t * k + j] * ys[(int64_t)j * H + h];
            for (int sh = 0; sh < n_shared; ++sh) acc += ys[(int64_t)(k + sh) * H + h];
            if (residual) acc += residual[(int64_t)t * H + h];
            o[h] = acc;
        }
    }
    free(J.ybuf);
    return 0;
}

/* Grouped evaluation over the batch-union lists (expert-major): each active
 * expert's FFN is applied to every token on its list and the weighted result
 * is added to that token's row; then the shared experts; then the residual.
 * Used only to check that grouping reproduces the per-token definition. */
int oracle_layer_grouped(int H, int I, int E, int k, int n_shared,
                         const oracle_expert *experts, int T, const uint16_t *x_bf16,
                         const double *w, const int32_t *offsets, const int32_t *pairs,
                         const int32_t *active, int n_active, const double *residual,
                         double *out) {
    double *x = (double *)malloc(sizeof(double) * (size_t)H);
    double *y = (double *)malloc(sizeof(double) * (size_t)H);
    double *tmp = (double *)malloc(sizeof(double) * (size_t)I);
    memset(out, 0, sizeof(double) * (size_t)T * H);
    for (int a = 0; a < n_active; ++a) {
        int e = active[a];
        for (int i = offsets[e]; i < offsets[e + 1]; ++i) {
            int p = pairs[i], t = p / k;
            for (int h = 0; h < H; ++h) x[h] = oracle_bf16_to_double(x_bf16[(int64_t)t * H + h]);
            expert_ffn(H, I, &experts[e], x, y, tmp);
            for (int h = 0; h < H; ++h) out[(int64_t)t * H + h] += w[p] * y[h];
        }
    }
    for (int s = 0; s < n_shared; ++s)
        for (int t = 0; t < T; ++t) {
            for (int h = 0; h < H; ++h) x[h] = oracle_bf16_to_double(x_bf16[(int64_t)t * H + h]);
            expert_ffn(H, I, &experts[E + s], x, y, tmp);
            for (int h = 0; h < H; ++h) out[(int64_t)t * H + h] += y[h];
        }
    if (residual)
        for (int64_t i = 0; i < (int64_t)T * H; ++i) out[i] += residual[i];
    free(x);
    free(y);
    free(tmp);
    return 0;
}
