/*
 * fp64 CPU oracle for the LatentMoE layer forward pass.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product library links, includes
 * or calls this file; only the tests, the smoke check and the bench's CPU
 * baseline leg do.  It shares no header, helper, table or constant with the
 * CUDA path.
 *
 * What it computes, per token row x (applied to every row independently, as
 * the "Stable LatentMoE" problem statement requires), in double precision from
 * the already-rounded inputs:
 *
 *   a = W_r x                      router logits at model width
 *   r = sigmoid(a)                 "Stable LatentMoE", equation for r
 *   s = r + b                      biased scores, used for selection only
 *   T_k = TopK(s, k)               "Stable LatentMoE", equation for T_k(x);
 *                                  equal scores go to the lower expert index
 *                                  (cooking-agi LatentMoE page, section "Does
 *                                  the same latent vector imply the same
 *                                  output?", routed_example uses v0 >= v1)
 *   p_i = r_i / sum_{j in T_k} r_j "Stable LatentMoE", equation for p_i (raw r)
 *   z = W_down x                   shared down-projection to latent width l
 *   E_i(z) = D_i act(G_i z, U_i z) routed expert l -> f -> l
 *   u = sum_{i in T_k} p_i E_i(z)  "Stable LatentMoE", equation for u
 *   n = u / sqrt(mean(u^2) + eps)  RMSNorm, unit gain, eps inside the root
 *   y = S_1(x) + S_2(x) + W_up n   "Stable LatentMoE", equation for y;
 *                                  S_j(x) = Ds_j act(Gs_j x, Us_j x)
 *
 * act is one of
 *   SWIGLU : silu(g) * v                         (cooking-agi page: "SwiGLU
 *                                                 experts"; the workloads)
 *   SITU   : cg*tanh(g/cg)*sigmoid(g) * cu*tanh(v/cu)
 *            the SiTU-GLU gate named by "Stable LatentMoE"; the problem never
 *            writes the formula, this reading reproduces its worked example
 *            (gate_cap = 4, up_cap = 25) and tends to SWIGLU as the caps grow
 *   LINEAR : g (the up branch is ignored)         pin-only: lets the toy
 *            experts of the cooking-agi page (A(z) = 2z, B(z) = -z) be built
 * and the RMSNorm can be switched off (pin-only, same toy).
 *
 * Every function below is pinned by the -m "not gpu" tests: the worked example
 * and shape examples of "Stable LatentMoE", routed_example and the norm-order
 * example of the cooking-agi page, brute-force top-k, and invariants.
 *
 * Inputs are read through a dtype code (0 = fp32, 1 = bf16 stored as the
 * upper 16 bits of an fp32), so large bf16 weight stacks need no widened copy.
 * Threads run over token rows; the per-row arithmetic is a plain loop nest.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

enum { ORA_F32 = 0, ORA_BF16 = 1 };
enum { ORA_SWIGLU = 0, ORA_SITU = 1, ORA_LINEAR = 2 };

typedef struct {
    int64_t T;      /* rows in x */
    int d, l, f, E, k, fs, n_shared;
    double eps;
    int act;
    double gate_cap, up_cap;
    int use_norm;
    int n_threads;  /* 0: all online cores */
} ora_dims;

typedef struct {
    const void *x;  int x_dt;       /* [T, d] */
    const float *W_r;               /* [E, d] fp32 */
    const float *b;                 /* [E] fp32 */
    const void *W_down; const void *W_up;   /* [l, d], [d, l] */
    const void *G; const void *U;           /* [E, f, l] */
    const void *D;                          /* [E, l, f] */
    const void *Gs; const void *Us;         /* [n_shared, fs, d] */
    const void *Ds;                         /* [n_shared, d, fs] */
    int w_dt;                       /* dtype of every weight except W_r, b */
} ora_inputs;

typedef struct {
    double *y;      /* [n, d] */
    int32_t *sel;   /* [n, k] */
    double *p;      /* [n, k] */
    double *u;      /* [n, l] */
    double *r;      /* [n, E] or NULL: raw sigmoid scores */
    double *gap;    /* [n] or NULL: s_(k) - s_(k+1) (INFINITY when k == E) */
} ora_outputs;

static inline double ld(const void *p, int dt, int64_t i)
{
    if (dt == ORA_F32) return (double)((const float *)p)[i];
    uint32_t bits = (uint32_t)((const uint16_t *)p)[i] << 16;
    float v;
    memcpy(&v, &bits, sizeof v);
    return (double)v;
}

static inline double sigmoid(double a) { return 1.0 / (1.0 + exp(-a)); }

static double act_fn(const ora_dims *m, double g, double v)
{
    switch (m->act) {
    case ORA_SWIGLU:
        return g * sigmoid(g) * v;
    case ORA_SITU: {
        double cg = m->gate_cap, cu = m->up_cap;
        return cg * tanh(g / cg) * sigmoid(g) * cu * tanh(v / cu);
    }
    default:
        return g;
    }
}

/*
 * Top-k by repeated selection: k passes, each taking the largest remaining
 * score, scanning experts in ascending index so that on equal scores the
 * lower index is taken first.  Writes the chosen indices in the order chosen
 * (score descending, index ascending) and returns s_(k) - s_(k+1).
 */
static double topk_row(int E, int k, const double *s, int32_t *sel, char *taken)
{
    memset(taken, 0, (size_t)E);
    double kth = 0.0;
    for (int j = 0; j < k; ++j) {
        int best = -1;
        for (int e = 0; e < E; ++e) {
            if (taken[e]) continue;
            if (best < 0 || s[e] > s[best]) best = e;
        }
        taken[best] = 1;
        sel[j] = best;
        kth = s[best];
    }
    if (k == E) return INFINITY;
    double next = -INFINITY;
    for (int e = 0; e < E; ++e)
        if (!taken[e] && s[e] > next) next = s[e];
    return kth - next;
}

/* Exported for the brute-force pins: select the top k of n rows of E scores. */
void ora_topk(int64_t n, int E, int k, const double *s, int32_t *sel, double *gap)
{
    char *taken = (char *)malloc((size_t)E);
    for (int64_t i = 0; i < n; ++i) {
        double g = topk_row(E, k, s + i * E, sel + i * k, taken);
        if (gap) gap[i] = g;
    }
    free(taken);
}

typedef struct {
    const ora_dims *m;
    const ora_inputs *in;
    const ora_outputs *out;
    const int64_t *rows;        /* NULL: rows 0..n-1 */
    const int32_t *sel_in;      /* NULL: select; else [n, k] given selection */
    int64_t n;
    int64_t next;               /* work counter */
    pthread_mutex_t lock;
} job;

static void row_forward(const ora_dims *m, const ora_inputs *in, const ora_outputs *out,
                        int64_t t, int64_t o, const int32_t *sel_given, double *buf, char *taken)
{
    const int d = m->d, l = m->l, f = m->f, E = m->E, k = m->k, fs = m->fs;
    double *x = buf;            /* d */
    double *r = x + d;          /* E */
    double *s = r + E;          /* E */
    double *z = s + E;          /* l */
    double *h = z + l;          /* max(f, fs) */
    double *u = h + (f > fs ? f : fs);  /* l */
    double *y = u + l;          /* d */
    int32_t *sel = out->sel + o * k;
    double *p = out->p + o * k;

    for (int i = 0; i < d; ++i) x[i] = ld(in->x, in->x_dt, t * (int64_t)d + i);

    /* router at model width: r = sigmoid(W_r x), s = r + b */
    for (int e = 0; e < E; ++e) {
        double a = 0.0;
        for (int i = 0; i < d; ++i) a += (double)in->W_r[(int64_t)e * d + i] * x[i];
        r[e] = sigmoid(a);
        s[e] = r[e] + (double)in->b[e];
    }
    if (out->r) memcpy(out->r + o * E, r, sizeof(double) * (size_t)E);

    /* selection on biased scores */
    double gap;
    if (sel_given) {
        memcpy(sel, sel_given + o * k, sizeof(int32_t) * (size_t)k);
        gap = NAN;
    } else {
        gap = topk_row(E, k, s, sel, taken);
    }
    if (out->gap) out->gap[o] = gap;

    /* mixture weights from raw scores */
    double rsum = 0.0;
    for (int j = 0; j < k; ++j) rsum += r[sel[j]];
    for (int j = 0; j < k; ++j) p[j] = r[sel[j]] / rsum;

    /* z = W_down x */
    for (int c = 0; c < l; ++c) {
        double a = 0.0;
        for (int i = 0; i < d; ++i) a += ld(in->W_down, in->w_dt, (int64_t)c * d + i) * x[i];
        z[c] = a;
    }

    /* u = sum_j p_j E_{sel_j}(z) */
    for (int c = 0; c < l; ++c) u[c] = 0.0;
    for (int j = 0; j < k; ++j) {
        const int64_t e = sel[j];
        for (int q = 0; q < f; ++q) {
            double g = 0.0, v = 0.0;
            const int64_t row = (e * f + q) * (int64_t)l;
            for (int c = 0; c < l; ++c) {
                g += ld(in->G, in->w_dt, row + c) * z[c];
                v += ld(in->U, in->w_dt, row + c) * z[c];
            }
            h[q] = act_fn(m, g, v);
        }
        for (int c = 0; c < l; ++c) {
            double a = 0.0;
            const int64_t row = (e * l + c) * (int64_t)f;
            for (int q = 0; q < f; ++q) a += ld(in->D, in->w_dt, row + q) * h[q];
            u[c] += p[j] * a;
        }
    }
    memcpy(out->u + o * l, u, sizeof(double) * (size_t)l);

    /* RMSNorm(u), unit gain, eps inside the square root */
    if (m->use_norm) {
        double ss = 0.0;
        for (int c = 0; c < l; ++c) ss += u[c] * u[c];
        const double inv = 1.0 / sqrt(ss / (double)l + m->eps);
        for (int c = 0; c < l; ++c) u[c] *= inv;
    }

    /* y = W_up n */
    for (int i = 0; i < d; ++i) {
        double a = 0.0;
        for (int c = 0; c < l; ++c) a += ld(in->W_up, in->w_dt, (int64_t)i * l + c) * u[c];
        y[i] = a;
    }

    /* + shared experts at model width, each on the full-width x */
    for (int sh = 0; sh < m->n_shared; ++sh) {
        for (int q = 0; q < fs; ++q) {
            double g = 0.0, v = 0.0;
            const int64_t row = ((int64_t)sh * fs + q) * d;
            for (int i = 0; i < d; ++i) {
                g += ld(in->Gs, in->w_dt, row + i) * x[i];
                v += ld(in->Us, in->w_dt, row + i) * x[i];
            }
            h[q] = act_fn(m, g, v);
        }
        for (int i = 0; i < d; ++i) {
            double a = 0.0;
            const int64_t row = ((int64_t)sh * d + i) * fs;
            for (int q = 0; q < fs; ++q) a += ld(in->Ds, in->w_dt, row + q) * h[q];
            y[i] += a;
        }
    }
    memcpy(out->y + o * d, y, sizeof(double) * (size_t)d);
}

static void *worker(void *arg)
{
    job *J = (job *)arg;
    const ora_dims *m = J->m;
    const int hmax = m->f > m->fs ? m->f : m->fs;
    const size_t nbuf = (size_t)m->d * 2 + (size_t)m->E * 2 + (size_t)m->l * 2 + (size_t)hmax;
    double *buf = (double *)malloc(sizeof(double) * nbuf);
    char *taken = (char *)malloc((size_t)m->E);
    for (;;) {
        pthread_mutex_lock(&J->lock);
        int64_t o = J->next++;
        pthread_mutex_unlock(&J->lock);
        if (o >= J->n) break;
        int64_t t = J->rows ? J->rows[o] : o;
        row_forward(m, J->in, J->out, t, o, J->sel_in, buf, taken);
    }
    free(taken);
    free(buf);
    return NULL;
}

/*
 * Forward for n token rows.  rows == NULL means rows 0..n-1 of x; otherwise
 * output row o is token rows[o].  sel_in == NULL selects by top-k; otherwise
 * sel_in[o*k .. o*k+k) is used as the selection (for comparing against a
 * selection made elsewhere on near-tied rows).  Returns 0, or -1 on bad
 * arguments.
 */
int ora_forward(const ora_dims *m, const ora_inputs *in, const ora_outputs *out,
                const int64_t *rows, int64_t n, const int32_t *sel_in)
{
    if (!m || !in || !out || n < 0) return -1;
    if (m->d < 1 || m->l < 1 || m->f < 1 || m->E < 1 || m->k < 1 || m->k > m->E ||
        m->fs < 1 || m->n_shared < 0)
        return -1;
    if (n == 0) return 0;
    for (int64_t o = 0; rows && o < n; ++o)
        if (rows[o] < 0 || rows[o] >= m->T) return -1;
    if (!rows && n > m->T) return -1;

    job J;
    J.m = m; J.in = in; J.out = out; J.rows = rows; J.sel_in = sel_in; J.n = n; J.next = 0;
    pthread_mutex_init(&J.lock, NULL);
    int nt = m->n_threads > 0 ? m->n_threads : (int)sysconf(_SC_NPROCESSORS_ONLN);
    if (nt < 1) nt = 1;
    if (nt > n) nt = (int)n;
    pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)nt);
    for (int i = 0; i < nt; ++i) pthread_create(&th[i], NULL, worker, &J);
    for (int i = 0; i < nt; ++i) pthread_join(th[i], NULL);
    free(th);
    pthread_mutex_destroy(&J.lock);
    return 0;
}
