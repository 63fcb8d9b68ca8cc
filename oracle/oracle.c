/*
 * oracle.c -- plain fp64 CPU oracle for grouped / latent-KV scaled-dot-product
 * attention.
 *
 * TEST INFRASTRUCTURE, NOT PRODUCT CODE.  Only the test-suite, the smoke check
 * and the benchmark's CPU-baseline leg may load this library.  It shares no
 * code, header, table or helper with the CUDA library in
 * latent_kv_attention_b200/: the two are independent implementations of the
 * same definitions, and the tests compare them.
 *
 * Every routine evaluates the textbook definition one output row at a time,
 * in double precision, with no blocking, fusion or reordering:
 *
 *   for a query q, a visible key set J, keys k_j and values v_j:
 *     s_j = scale * <q, k_j>
 *     p_j = exp(s_j - max s) / sum_j' exp(s_j' - max s)
 *     o   = sum_j p_j v_j
 *     lse = max s + ln sum_j exp(s_j - max s)          (natural log)
 *
 * Sources (web pages on the subject; cited by page title and section):
 *  - "Grouped Query Attention (GQA)" glossary page, section "How GQA works":
 *    per head, attention is plain scaled-dot-product attention; a group of
 *    h_q/h_kv consecutive query heads shares one key/value head (the page's
 *    PyTorch example copies each KV head to its group with repeat_interleave,
 *    so head i uses KV head floor(i / (h_q/h_kv))).  One group = MQA, as many
 *    groups as heads = MHA.
 *  - "GQLA: Group-Query Latent Attention ..." section 3.1, eq. (1): the latent
 *    c_t^KV (r_kv values) is expanded per group gamma by the rows of
 *    W^UK, W^UV in R^{g*d x r_kv}; the key of head i is
 *    [k^C_{t,gamma(i)} ; k^R_t] with one RoPE key k^R_t shared by all heads;
 *    the query is [q^C_{t,i} ; q^R_{t,i}].  Section 3.1 ("two equivalent
 *    decode paths") and Figure 2: the MQA-absorbed path folds W^UK into the
 *    query and W^UV into the output and attends to the cached latent; the GQA
 *    path attends to the per-group expanded cache (2*g*d_h + d_h^R values per
 *    token).  Both give the same output.
 *  - "GTA: Grouped-head latenT Attention" press article, section on the
 *    grouped shared attention matrix: heads are split into groups (e.g. 4
 *    heads) and one attention matrix per group is computed once and used by
 *    every head of the group with that head's own values.
 *
 * Readings where the pages are silent (the same list is kept with the design
 * notes of the repository):
 *  - cache_lens[b] counts the valid cache tokens of sequence b INCLUDING the
 *    s_q new query tokens, which sit at positions L_b - s_q .. L_b - 1.
 *  - causal masking is bottom-right aligned: query t (0 <= t < s_q) sees keys
 *    0 .. L_b - s_q + t.  Without causal masking every query sees 0 .. L_b-1.
 *  - the softmax scale is an explicit argument.
 *  - W^UK and W^UV are stored as [g][d_h][r_kv]: block gamma is the d_h x r_kv
 *    matrix that maps the latent to group gamma's key (value).
 *
 * Error behaviour: every routine returns 0 on success and 1 if an argument is
 * out of range (nothing is written in that case).
 */
#include <math.h>
#include <pthread.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

#define ORACLE_OK 0
#define ORACLE_BAD_ARG 1

/* ------------------------------------------------------------------------ */
/* A tiny thread pool: work items 0..n_items-1 are handed out round-robin.   */
/* ------------------------------------------------------------------------ */

typedef void (*item_fn)(void *ctx, long item, double *scratch);

typedef struct {
    item_fn fn;
    void *ctx;
    long n_items;
    int n_threads;
    int tid;
    size_t scratch_doubles;
} pool_arg;

static void *pool_worker(void *p) {
    pool_arg *a = (pool_arg *)p;
    double *scratch = NULL;
    if (a->scratch_doubles) scratch = (double *)malloc(a->scratch_doubles * sizeof(double));
    for (long it = a->tid; it < a->n_items; it += a->n_threads) a->fn(a->ctx, it, scratch);
    free(scratch);
    return NULL;
}

static int resolve_threads(int n_threads, long n_items) {
    if (n_threads <= 0) {
        long c = sysconf(_SC_NPROCESSORS_ONLN);
        n_threads = c > 0 ? (int)c : 1;
    }
    if (n_threads > n_items) n_threads = (int)(n_items > 0 ? n_items : 1);
    if (n_threads > 256) n_threads = 256;
    return n_threads;
}

static void run_pool(item_fn fn, void *ctx, long n_items, int n_threads, size_t scratch_doubles) {
    n_threads = resolve_threads(n_threads, n_items);
    pthread_t th[256];
    pool_arg args[256];
    for (int t = 0; t < n_threads; ++t) {
        args[t].fn = fn;
        args[t].ctx = ctx;
        args[t].n_items = n_items;
        args[t].n_threads = n_threads;
        args[t].tid = t;
        args[t].scratch_doubles = scratch_doubles;
    }
    if (n_threads == 1) {
        pool_worker(&args[0]);
        return;
    }
    for (int t = 0; t < n_threads; ++t) pthread_create(&th[t], NULL, pool_worker, &args[t]);
    for (int t = 0; t < n_threads; ++t) pthread_join(th[t], NULL);
}

/* Number of threads the pool would use for n_items (reported by the bench). */
int oracle_threads_used(int n_threads, long n_items) { return resolve_threads(n_threads, n_items); }

/* ------------------------------------------------------------------------ */
/* Softmax over n scores followed by the weighted sum of value rows.         */
/* value row j is vals[j * vstride .. j * vstride + dv - 1].                 */
/* ------------------------------------------------------------------------ */
static void softmax_combine(const double *s, int n, const double *vals, long vstride, int dv,
                            double *out, double *lse) {
    double m = -INFINITY;
    for (int j = 0; j < n; ++j)
        if (s[j] > m) m = s[j];
    double z = 0.0;
    for (int j = 0; j < n; ++j) z += exp(s[j] - m);
    for (int d = 0; d < dv; ++d) out[d] = 0.0;
    for (int j = 0; j < n; ++j) {
        double p = exp(s[j] - m) / z;
        const double *v = vals + (long)j * vstride;
        for (int d = 0; d < dv; ++d) out[d] += p * v[d];
    }
    if (lse) *lse = m + log(z);
}

/* Number of keys query t of a sequence with L valid tokens may see. */
static int visible_keys(int L, int s_q, int t, int causal) { return causal ? L - s_q + t + 1 : L; }

static int check_lens(const int *lens, int B, int Lmax, int s_q, int causal) {
    for (int b = 0; b < B; ++b) {
        if (lens[b] < 1 || lens[b] > Lmax) return 0;
        if (causal && lens[b] < s_q) return 0;
    }
    return 1;
}

/* Batch indices to evaluate: all of them, or the listed subset. */
static int batch_index(const int *rows_b, int n_rows_b, int B, long r) {
    (void)B;
    return rows_b ? rows_b[r] : (int)r;
}

static int check_rows(const int *rows_b, int n_rows_b, int B) {
    if (!rows_b) return 1;
    for (int r = 0; r < n_rows_b; ++r)
        if (rows_b[r] < 0 || rows_b[r] >= B) return 0;
    return 1;
}

/* ======================================================================== */
/* GQA: q [B,h_q,s_q,d], k,v [B,h_kv,Lmax,d], out [B,h_q,s_q,d], lse [B,h_q,s_q] */
/* ======================================================================== */
typedef struct {
    const double *q, *k, *v;
    const int *lens;
    int B, h_q, h_kv, s_q, d, Lmax, causal;
    double scale;
    double *out, *lse;
    const int *rows_b;
    int n_rows_b;
} gqa_ctx;

static void gqa_item(void *p, long item, double *s) {
    gqa_ctx *c = (gqa_ctx *)p;
    int i = (int)(item % c->h_q);
    int b = batch_index(c->rows_b, c->n_rows_b, c->B, item / c->h_q);
    int group = i / (c->h_q / c->h_kv); /* repeat_interleave grouping */
    int L = c->lens[b];
    const double *K = c->k + ((long)b * c->h_kv + group) * c->Lmax * c->d;
    const double *V = c->v + ((long)b * c->h_kv + group) * c->Lmax * c->d;
    for (int t = 0; t < c->s_q; ++t) {
        long row = ((long)b * c->h_q + i) * c->s_q + t;
        const double *q = c->q + row * c->d;
        int n = visible_keys(L, c->s_q, t, c->causal);
        for (int j = 0; j < n; ++j) {
            double acc = 0.0;
            for (int e = 0; e < c->d; ++e) acc += q[e] * K[(long)j * c->d + e];
            s[j] = c->scale * acc;
        }
        softmax_combine(s, n, V, c->d, c->d, c->out + row * c->d, c->lse ? c->lse + row : NULL);
    }
}

int oracle_gqa(const double *q, const double *k, const double *v, const int *lens, int B, int h_q,
               int h_kv, int s_q, int d, int Lmax, int causal, double scale, double *out, double *lse,
               const int *rows_b, int n_rows_b, int n_threads) {
    if (B < 1 || h_q < 1 || h_kv < 1 || s_q < 1 || d < 1 || Lmax < 1) return ORACLE_BAD_ARG;
    if (h_q % h_kv) return ORACLE_BAD_ARG;
    if (!check_lens(lens, B, Lmax, s_q, causal) || !check_rows(rows_b, n_rows_b, B)) return ORACLE_BAD_ARG;
    gqa_ctx c = {q, k, v, lens, B, h_q, h_kv, s_q, d, Lmax, causal, scale, out, lse, rows_b, n_rows_b};
    long nb = rows_b ? n_rows_b : B;
    run_pool(gqa_item, &c, nb * h_q, n_threads, (size_t)Lmax);
    return ORACLE_OK;
}

/* The attention probabilities p_j of one query row (b, head i, query t) of the
 * GQA definition; p must hold Lmax doubles.  Returns the number of visible
 * keys, or -1 on a bad argument. */
int oracle_gqa_probs(const double *q, const double *k, const int *lens, int B, int h_q, int h_kv,
                     int s_q, int d, int Lmax, int causal, double scale, int b, int i, int t,
                     double *p) {
    if (b < 0 || b >= B || i < 0 || i >= h_q || t < 0 || t >= s_q || h_q % h_kv) return -1;
    if (!check_lens(lens, B, Lmax, s_q, causal)) return -1;
    int group = i / (h_q / h_kv);
    int L = lens[b];
    int n = visible_keys(L, s_q, t, causal);
    const double *qr = q + (((long)b * h_q + i) * s_q + t) * d;
    const double *K = k + ((long)b * h_kv + group) * Lmax * d;
    double m = -INFINITY;
    for (int j = 0; j < n; ++j) {
        double acc = 0.0;
        for (int e = 0; e < d; ++e) acc += qr[e] * K[(long)j * d + e];
        p[j] = scale * acc;
        if (p[j] > m) m = p[j];
    }
    double z = 0.0;
    for (int j = 0; j < n; ++j) z += exp(p[j] - m);
    for (int j = 0; j < n; ++j) p[j] = exp(p[j] - m) / z;
    return n;
}

/* ======================================================================== */
/* GQLA latent attention.                                                   */
/* q_c [B,h_q,s_q,d_h], q_r [B,h_q,s_q,d_r], w_uk,w_uv [g,d_h,r_kv],         */
/* latent [B,Lmax,r_kv+d_r] holding c^KV (first r_kv) then k^R (last d_r).   */
/* ======================================================================== */
typedef struct {
    const double *q_c, *q_r, *w_uk, *w_uv, *latent;
    const int *lens;
    int B, h_q, g, s_q, d_h, r_kv, d_r, Lmax, causal;
    double scale;
    double *out, *lse;
    const int *rows_b;
    int n_rows_b;
} latent_ctx;

/* Expanded (per-group GQA) definition, eq. (1): one work item = (b, gamma).
 * scratch holds the expanded keys/values of this group: 2 * Lmax * d_h, then
 * Lmax scores. */
static void latent_expanded_item(void *p, long item, double *scratch) {
    latent_ctx *c = (latent_ctx *)p;
    int gamma = (int)(item % c->g);
    int b = batch_index(c->rows_b, c->n_rows_b, c->B, item / c->g);
    int L = c->lens[b];
    int W = c->r_kv + c->d_r;
    double *kc = scratch;                       /* [L][d_h] */
    double *vc = scratch + (long)c->Lmax * c->d_h; /* [L][d_h] */
    double *s = scratch + 2L * c->Lmax * c->d_h;
    const double *Wk = c->w_uk + (long)gamma * c->d_h * c->r_kv;
    const double *Wv = c->w_uv + (long)gamma * c->d_h * c->r_kv;
    for (int j = 0; j < L; ++j) {
        const double *cj = c->latent + ((long)b * c->Lmax + j) * W;
        for (int e = 0; e < c->d_h; ++e) {
            double ak = 0.0, av = 0.0;
            for (int r = 0; r < c->r_kv; ++r) {
                ak += Wk[(long)e * c->r_kv + r] * cj[r];
                av += Wv[(long)e * c->r_kv + r] * cj[r];
            }
            kc[(long)j * c->d_h + e] = ak;
            vc[(long)j * c->d_h + e] = av;
        }
    }
    int per_group = c->h_q / c->g;
    for (int i = gamma * per_group; i < (gamma + 1) * per_group; ++i) {
        for (int t = 0; t < c->s_q; ++t) {
            long row = ((long)b * c->h_q + i) * c->s_q + t;
            const double *qc = c->q_c + row * c->d_h;
            const double *qr = c->q_r + row * c->d_r;
            int n = visible_keys(L, c->s_q, t, c->causal);
            for (int j = 0; j < n; ++j) {
                const double *kr = c->latent + ((long)b * c->Lmax + j) * W + c->r_kv;
                double acc = 0.0;
                for (int e = 0; e < c->d_h; ++e) acc += qc[e] * kc[(long)j * c->d_h + e];
                for (int e = 0; e < c->d_r; ++e) acc += qr[e] * kr[e];
                s[j] = c->scale * acc;
            }
            softmax_combine(s, n, vc, c->d_h, c->d_h, c->out + row * c->d_h, c->lse ? c->lse + row : NULL);
        }
    }
}

/* Absorbed (MQA) form: q~ = W^UK_gamma^T q^C, scores against the latent
 * itself, o = W^UV_gamma (sum_j p_j c_j).  One work item = (b, head i).
 * scratch: Lmax scores, then q~ (r_kv), then the latent-space output (r_kv). */
static void latent_absorbed_item(void *p, long item, double *scratch) {
    latent_ctx *c = (latent_ctx *)p;
    int i = (int)(item % c->h_q);
    int b = batch_index(c->rows_b, c->n_rows_b, c->B, item / c->h_q);
    int gamma = i / (c->h_q / c->g);
    int L = c->lens[b];
    int W = c->r_kv + c->d_r;
    double *s = scratch;
    double *qt = scratch + c->Lmax;
    double *ot = qt + c->r_kv;
    const double *Wk = c->w_uk + (long)gamma * c->d_h * c->r_kv;
    const double *Wv = c->w_uv + (long)gamma * c->d_h * c->r_kv;
    const double *C = c->latent + (long)b * c->Lmax * W;
    for (int t = 0; t < c->s_q; ++t) {
        long row = ((long)b * c->h_q + i) * c->s_q + t;
        const double *qc = c->q_c + row * c->d_h;
        const double *qr = c->q_r + row * c->d_r;
        for (int r = 0; r < c->r_kv; ++r) {
            double a = 0.0;
            for (int e = 0; e < c->d_h; ++e) a += Wk[(long)e * c->r_kv + r] * qc[e];
            qt[r] = a;
        }
        int n = visible_keys(L, c->s_q, t, c->causal);
        for (int j = 0; j < n; ++j) {
            const double *cj = C + (long)j * W;
            double acc = 0.0;
            for (int r = 0; r < c->r_kv; ++r) acc += qt[r] * cj[r];
            for (int e = 0; e < c->d_r; ++e) acc += qr[e] * cj[c->r_kv + e];
            s[j] = c->scale * acc;
        }
        softmax_combine(s, n, C, W, c->r_kv, ot, c->lse ? c->lse + row : NULL);
        double *o = c->out + row * c->d_h;
        for (int e = 0; e < c->d_h; ++e) {
            double a = 0.0;
            for (int r = 0; r < c->r_kv; ++r) a += Wv[(long)e * c->r_kv + r] * ot[r];
            o[e] = a;
        }
    }
}

static int latent_args_ok(int B, int h_q, int g, int s_q, int d_h, int r_kv, int d_r, int Lmax) {
    if (B < 1 || h_q < 1 || g < 1 || s_q < 1 || d_h < 1 || r_kv < 1 || d_r < 0 || Lmax < 1) return 0;
    return h_q % g == 0;
}

int oracle_latent_expanded(const double *q_c, const double *q_r, const double *w_uk,
                           const double *w_uv, const double *latent, const int *lens, int B, int h_q,
                           int g, int s_q, int d_h, int r_kv, int d_r, int Lmax, int causal,
                           double scale, double *out, double *lse, const int *rows_b, int n_rows_b,
                           int n_threads) {
    if (!latent_args_ok(B, h_q, g, s_q, d_h, r_kv, d_r, Lmax)) return ORACLE_BAD_ARG;
    if (!check_lens(lens, B, Lmax, s_q, causal) || !check_rows(rows_b, n_rows_b, B)) return ORACLE_BAD_ARG;
    latent_ctx c = {q_c, q_r, w_uk, w_uv, latent, lens, B, h_q, g, s_q, d_h, r_kv, d_r, Lmax, causal,
                    scale, out, lse, rows_b, n_rows_b};
    long nb = rows_b ? n_rows_b : B;
    run_pool(latent_expanded_item, &c, nb * g, n_threads, (size_t)Lmax * (2 * d_h + 1));
    return ORACLE_OK;
}

int oracle_latent_absorbed(const double *q_c, const double *q_r, const double *w_uk,
                           const double *w_uv, const double *latent, const int *lens, int B, int h_q,
                           int g, int s_q, int d_h, int r_kv, int d_r, int Lmax, int causal,
                           double scale, double *out, double *lse, const int *rows_b, int n_rows_b,
                           int n_threads) {
    if (!latent_args_ok(B, h_q, g, s_q, d_h, r_kv, d_r, Lmax)) return ORACLE_BAD_ARG;
    if (!check_lens(lens, B, Lmax, s_q, causal) || !check_rows(rows_b, n_rows_b, B)) return ORACLE_BAD_ARG;
    latent_ctx c = {q_c, q_r, w_uk, w_uv, latent, lens, B, h_q, g, s_q, d_h, r_kv, d_r, Lmax, causal,
                    scale, out, lse, rows_b, n_rows_b};
    long nb = rows_b ? n_rows_b : B;
    run_pool(latent_absorbed_item, &c, nb * h_q, n_threads, (size_t)Lmax + 2 * (size_t)r_kv);
    return ORACLE_OK;
}

/* The one-time cache conversion of GQLA section 3.1 ("switching paths needs
 * only a one-time compression/expansion of the KV cache at deployment"):
 * kc[b,gamma,j,:] = W^UK_gamma c_j, vc[b,gamma,j,:] = W^UV_gamma c_j,
 * kr[b,j,:] = k^R_j, for every cache slot j < Lmax.
 * kc, vc [B,g,Lmax,d_h]; kr [B,Lmax,d_r]. */
typedef struct {
    const double *latent, *w_uk, *w_uv;
    int B, Lmax, g, d_h, r_kv, d_r;
    double *kc, *vc, *kr;
} expand_ctx;

static void expand_item(void *p, long item, double *unused) {
    (void)unused;
    expand_ctx *c = (expand_ctx *)p;
    int j = (int)(item % c->Lmax);
    int b = (int)(item / c->Lmax);
    int W = c->r_kv + c->d_r;
    const double *cj = c->latent + ((long)b * c->Lmax + j) * W;
    for (int gamma = 0; gamma < c->g; ++gamma) {
        const double *Wk = c->w_uk + (long)gamma * c->d_h * c->r_kv;
        const double *Wv = c->w_uv + (long)gamma * c->d_h * c->r_kv;
        double *ko = c->kc + (((long)b * c->g + gamma) * c->Lmax + j) * c->d_h;
        double *vo = c->vc + (((long)b * c->g + gamma) * c->Lmax + j) * c->d_h;
        for (int e = 0; e < c->d_h; ++e) {
            double ak = 0.0, av = 0.0;
            for (int r = 0; r < c->r_kv; ++r) {
                ak += Wk[(long)e * c->r_kv + r] * cj[r];
                av += Wv[(long)e * c->r_kv + r] * cj[r];
            }
            ko[e] = ak;
            vo[e] = av;
        }
    }
    for (int e = 0; e < c->d_r; ++e) c->kr[((long)b * c->Lmax + j) * c->d_r + e] = cj[c->r_kv + e];
}

int oracle_latent_expand_cache(const double *latent, const double *w_uk, const double *w_uv, int B,
                               int Lmax, int g, int d_h, int r_kv, int d_r, double *kc, double *vc,
                               double *kr, int n_threads) {
    if (B < 1 || Lmax < 1 || g < 1 || d_h < 1 || r_kv < 1 || d_r < 0) return ORACLE_BAD_ARG;
    expand_ctx c = {latent, w_uk, w_uv, B, Lmax, g, d_h, r_kv, d_r, kc, vc, kr};
    run_pool(expand_item, &c, (long)B * Lmax, n_threads, 0);
    return ORACLE_OK;
}

/* ======================================================================== */
/* GTA shared-score attention.                                              */
/* q_g [B,G,s_q,d_qk], k_g [B,G,Lmax,d_qk], v [B,H,Lmax,d_v],                */
/* out [B,H,s_q,d_v], lse [B,G,s_q].  Head h belongs to group               */
/* floor(h / (H/G)) and uses that group's score matrix with its own values.  */
/* ======================================================================== */
typedef struct {
    const double *q_g, *k_g, *v;
    const int *lens;
    int B, G, H, s_q, d_qk, d_v, Lmax, causal;
    double scale;
    double *out, *lse;
    const int *rows_b;
    int n_rows_b;
} gta_ctx;

static void gta_item(void *p, long item, double *s) {
    gta_ctx *c = (gta_ctx *)p;
    int h = (int)(item % c->H);
    int b = batch_index(c->rows_b, c->n_rows_b, c->B, item / c->H);
    int per_group = c->H / c->G;
    int gamma = h / per_group;
    int L = c->lens[b];
    const double *K = c->k_g + ((long)b * c->G + gamma) * c->Lmax * c->d_qk;
    const double *V = c->v + ((long)b * c->H + h) * c->Lmax * c->d_v;
    for (int t = 0; t < c->s_q; ++t) {
        const double *q = c->q_g + (((long)b * c->G + gamma) * c->s_q + t) * c->d_qk;
        int n = visible_keys(L, c->s_q, t, c->causal);
        for (int j = 0; j < n; ++j) {
            double acc = 0.0;
            for (int e = 0; e < c->d_qk; ++e) acc += q[e] * K[(long)j * c->d_qk + e];
            s[j] = c->scale * acc;
        }
        double lse_row;
        softmax_combine(s, n, V, c->d_v, c->d_v, c->out + (((long)b * c->H + h) * c->s_q + t) * c->d_v,
                        &lse_row);
        /* the score matrix is the group's: its first head records the lse */
        if (c->lse && h % per_group == 0) c->lse[((long)b * c->G + gamma) * c->s_q + t] = lse_row;
    }
}

int oracle_gta(const double *q_g, const double *k_g, const double *v, const int *lens, int B, int G,
               int H, int s_q, int d_qk, int d_v, int Lmax, int causal, double scale, double *out,
               double *lse, const int *rows_b, int n_rows_b, int n_threads) {
    if (B < 1 || G < 1 || H < 1 || s_q < 1 || d_qk < 1 || d_v < 1 || Lmax < 1) return ORACLE_BAD_ARG;
    if (H % G) return ORACLE_BAD_ARG;
    if (!check_lens(lens, B, Lmax, s_q, causal) || !check_rows(rows_b, n_rows_b, B)) return ORACLE_BAD_ARG;
    gta_ctx c = {q_g, k_g, v, lens, B, G, H, s_q, d_qk, d_v, Lmax, causal, scale, out, lse, rows_b, n_rows_b};
    long nb = rows_b ? n_rows_b : B;
    run_pool(gta_item, &c, nb * H, n_threads, (size_t)Lmax);
    return ORACLE_OK;
}

/* ======================================================================== */
/* Merge of partial attention results over disjoint key sets (the flash-    */
/* decoding combine), written from the definition: with weights             */
/* w_i = exp(lse_i - max lse), o = sum_i w_i o_i / sum_i w_i and            */
/* lse = max lse + ln sum_i w_i.  parts_o [n][dv], parts_lse [n].            */
/* ======================================================================== */
int oracle_merge_partials(const double *parts_o, const double *parts_lse, int n, int dv, double *out,
                          double *lse) {
    if (n < 1 || dv < 1) return ORACLE_BAD_ARG;
    double m = -INFINITY;
    for (int i = 0; i < n; ++i)
        if (parts_lse[i] > m) m = parts_lse[i];
    double z = 0.0;
    for (int i = 0; i < n; ++i) z += exp(parts_lse[i] - m);
    for (int d = 0; d < dv; ++d) {
        double a = 0.0;
        for (int i = 0; i < n; ++i) a += exp(parts_lse[i] - m) * parts_o[(long)i * dv + d];
        out[d] = a / z;
    }
    *lse = m + log(z);
    return ORACLE_OK;
}
