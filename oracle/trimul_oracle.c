/*
 * trimul_oracle.c - CPU float64 oracle for the triangle multiplicative update.
 *
 * TEST INFRASTRUCTURE ONLY. This file is the slow, plain definition that the
 * GPU kernels are checked against. It shares no code, header, table or helper
 * with the CUDA path; only the tests, the bench's CPU-baseline leg and the
 * smoke check may load it. Nothing in the product links against it.
 *
 * What it computes. The pages name the layer TriangleMultiplicationOutgoing
 * and call it as layer(x, mask) ("Scaling biomolecular modeling with context
 * parallelism in NVIDIA BioNeMo", section "Context-parallel implementation of
 * triangle multiplication"), but print no equations. The steps below are the
 * AlphaFold3 triangle multiplicative update (outgoing and incoming), read
 * plainly:
 *   1. zh_rs  = LayerNorm_in(z_rs) over the c_z channels
 *              (biased variance, eps inside the square root, affine gamma/beta).
 *   2. a_rs   = mask_rs * sigmoid(W_ag zh_rs + b_ag) (.) (W_a zh_rs + b_a)
 *      b_rs   = mask_rs * sigmoid(W_bg zh_rs + b_bg) (.) (W_b zh_rs + b_b)
 *   3. x_ij   = sum_k a_ik (.) b_jk          (outgoing)
 *      x_ij   = sum_k a_ki (.) b_kj          (incoming)
 *      summed over k in increasing order.
 *   4. xh_ij  = LayerNorm_out(x_ij) over the c_h channels.
 *   5. g_ij   = sigmoid(W_g zh_ij + b_g)
 *   6. out_ij = g_ij (.) (W_o xh_ij + b_o)
 * Weights are PyTorch Linear layout [out][in] (the pages load the layer from a
 * state dict), y = W x + b. NULL biases mean zero; NULL LayerNorm affines mean
 * gamma = 1, beta = 0.
 *
 * Inputs arrive as float32 arrays whose values the caller has already made
 * exact (bf16 workloads are rounded before they reach either side); every
 * operation here is carried out in double.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
    const float *w_a, *w_ag, *w_b, *w_bg; /* [c_h][c_z] */
    const float *w_g;                     /* [c_z][c_z] */
    const float *w_o;                     /* [c_z][c_h] */
    const float *b_a, *b_ag, *b_b, *b_bg; /* [c_h] or NULL */
    const float *b_g, *b_o;               /* [c_z] or NULL */
    const float *ln_in_w, *ln_in_b;       /* [c_z] or NULL */
    const float *ln_out_w, *ln_out_b;     /* [c_h] or NULL */
} oracle_weights;

/* ---- scalar building blocks ------------------------------------------- */

static double sigmoid(double t) { return 1.0 / (1.0 + exp(-t)); }

/* LayerNorm over c values: mean, biased variance, eps inside the root. */
static void layer_norm(const double *v, int c, const float *gamma, const float *beta,
                       double eps, double *out)
{
    double mean = 0.0;
    for (int k = 0; k < c; ++k) mean += v[k];
    mean /= c;
    double var = 0.0;
    for (int k = 0; k < c; ++k) var += (v[k] - mean) * (v[k] - mean);
    var /= c;
    double inv = 1.0 / sqrt(var + eps);
    for (int k = 0; k < c; ++k) {
        double g = gamma ? (double)gamma[k] : 1.0;
        double b = beta ? (double)beta[k] : 0.0;
        out[k] = g * (v[k] - mean) * inv + b;
    }
}

/* y = W x + bias, W row-major [n_out][n_in]. */
static void linear(const float *W, const float *bias, int n_out, int n_in,
                   const double *x, double *y)
{
    for (int o = 0; o < n_out; ++o) {
        double s = 0.0;
        const float *row = W + (size_t)o * n_in;
        for (int k = 0; k < n_in; ++k) s += (double)row[k] * x[k];
        y[o] = s + (bias ? (double)bias[o] : 0.0);
    }
}

typedef struct {
    int N, c_z, c_h;
    const float *z, *mask;
    const oracle_weights *w;
    double eps;
} layer_ctx;

/* Step 1: zh_rs = LayerNorm_in(z_rs). */
static void input_norm(const layer_ctx *L, int r, int s, double *zh /* c_z */, double *tmp)
{
    const float *zc = L->z + ((size_t)r * L->N + s) * L->c_z;
    for (int k = 0; k < L->c_z; ++k) tmp[k] = zc[k];
    layer_norm(tmp, L->c_z, L->w->ln_in_w, L->w->ln_in_b, L->eps, zh);
}

/* Steps 1-2 for one cell (r, s): the gated, masked projections a_rs and b_rs. */
static void project_cell(const layer_ctx *L, int r, int s, double *a, double *b, double *scratch)
{
    const int cz = L->c_z, ch = L->c_h;
    double *zh = scratch, *tmp = scratch + cz;
    double *pa = tmp + cz, *pag = pa + ch, *pb = pag + ch, *pbg = pb + ch;
    input_norm(L, r, s, zh, tmp);
    linear(L->w->w_a, L->w->b_a, ch, cz, zh, pa);
    linear(L->w->w_ag, L->w->b_ag, ch, cz, zh, pag);
    linear(L->w->w_b, L->w->b_b, ch, cz, zh, pb);
    linear(L->w->w_bg, L->w->b_bg, ch, cz, zh, pbg);
    double m = L->mask ? (double)L->mask[(size_t)r * L->N + s] : 1.0;
    for (int c = 0; c < ch; ++c) {
        a[c] = m * sigmoid(pag[c]) * pa[c];
        b[c] = m * sigmoid(pbg[c]) * pb[c];
    }
}
#define PROJECT_SCRATCH(cz, ch) (2 * (cz) + 4 * (ch))

/* Steps 4-6 for one cell (i, j), given x_ij. */
static void finish_cell(const layer_ctx *L, int i, int j, const double *x, double *out,
                        double *scratch)
{
    const int cz = L->c_z, ch = L->c_h;
    double *xh = scratch, *zh = xh + ch, *tmp = zh + cz, *g = tmp + cz, *o = g + cz;
    layer_norm(x, ch, L->w->ln_out_w, L->w->ln_out_b, L->eps, xh);
    input_norm(L, i, j, zh, tmp);
    linear(L->w->w_g, L->w->b_g, cz, cz, zh, g);
    linear(L->w->w_o, L->w->b_o, cz, ch, xh, o);
    for (int c = 0; c < cz; ++c) out[c] = sigmoid(g[c]) * o[c];
}
#define FINISH_SCRATCH(cz, ch) ((ch) + 4 * (cz))

/* ---- a tiny row-parallel driver ---------------------------------------- */

typedef struct {
    void (*fn)(void *arg, int row, double *scratch);
    void *arg;
    int rows;
    int scratch;
    int next;
    pthread_mutex_t lock;
} par_job;

static void *par_worker(void *p)
{
    par_job *J = (par_job *)p;
    double *scratch = (double *)malloc(sizeof(double) * (size_t)(J->scratch > 0 ? J->scratch : 1));
    for (;;) {
        pthread_mutex_lock(&J->lock);
        int r = J->next++;
        pthread_mutex_unlock(&J->lock);
        if (r >= J->rows) break;
        J->fn(J->arg, r, scratch);
    }
    free(scratch);
    return NULL;
}

static void par_rows(int rows, int scratch, int nthreads,
                     void (*fn)(void *, int, double *), void *arg)
{
    par_job J;
    J.fn = fn; J.arg = arg; J.rows = rows; J.scratch = scratch; J.next = 0;
    pthread_mutex_init(&J.lock, NULL);
    if (nthreads < 1) nthreads = 1;
    if (nthreads > 256) nthreads = 256;
    pthread_t th[256];
    int started = 0;
    for (int t = 1; t < nthreads; ++t)
        if (pthread_create(&th[started], NULL, par_worker, &J) == 0) ++started;
    par_worker(&J);
    for (int t = 0; t < started; ++t) pthread_join(th[t], NULL);
    pthread_mutex_destroy(&J.lock);
}

/* ---- stage 1-2: projections for every cell ------------------------------ */

typedef struct { const layer_ctx *L; double *a, *b; } project_arg;

static void project_row(void *p, int r, double *scratch)
{
    project_arg *A = (project_arg *)p;
    const layer_ctx *L = A->L;
    for (int s = 0; s < L->N; ++s) {
        size_t off = ((size_t)r * L->N + s) * L->c_h;
        project_cell(L, r, s, A->a + off, A->b + off, scratch);
    }
}

/* a, b: [N][N][c_h] cell-major doubles. */
int oracle_project(int N, int c_z, int c_h, const float *z, const float *mask,
                   const oracle_weights *w, double eps, double *a, double *b, int nthreads)
{
    if (N < 1 || c_z < 1 || c_h < 1 || !z || !w || !a || !b) return -1;
    layer_ctx L = {N, c_z, c_h, z, mask, w, eps};
    project_arg A = {&L, a, b};
    par_rows(N, PROJECT_SCRATCH(c_z, c_h), nthreads, project_row, &A);
    return 0;
}

/* ---- stage 3: the triangle contraction ---------------------------------- */

typedef struct { int N, c; const double *a, *b; int incoming; double *x; } contract_arg;

static void contract_row(void *p, int i, double *scratch)
{
    (void)scratch;
    contract_arg *C = (contract_arg *)p;
    const int N = C->N, c = C->c;
    for (int j = 0; j < N; ++j) {
        double *x = C->x + ((size_t)i * N + j) * c;
        for (int ch = 0; ch < c; ++ch) x[ch] = 0.0;
        for (int k = 0; k < N; ++k) {
            const double *ak, *bk;
            if (!C->incoming) { /* x_ij = sum_k a_ik * b_jk */
                ak = C->a + ((size_t)i * N + k) * c;
                bk = C->b + ((size_t)j * N + k) * c;
            } else {            /* x_ij = sum_k a_ki * b_kj */
                ak = C->a + ((size_t)k * N + i) * c;
                bk = C->b + ((size_t)k * N + j) * c;
            }
            for (int ch = 0; ch < c; ++ch) x[ch] += ak[ch] * bk[ch];
        }
    }
}

/* x: [N][N][c] cell-major doubles; direction 0 = outgoing, 1 = incoming. */
int oracle_contract(int N, int c, const double *a, const double *b, int direction,
                    double *x, int nthreads)
{
    if (N < 1 || c < 1 || !a || !b || !x || (direction != 0 && direction != 1)) return -1;
    contract_arg C = {N, c, a, b, direction, x};
    par_rows(N, 0, nthreads, contract_row, &C);
    return 0;
}

/* ---- stage 4-6: output normalisation, gate and projection --------------- */

typedef struct { const layer_ctx *L; const double *x; double *out; } finish_arg;

static void finish_row(void *p, int i, double *scratch)
{
    finish_arg *F = (finish_arg *)p;
    const layer_ctx *L = F->L;
    for (int j = 0; j < L->N; ++j) {
        size_t cell = (size_t)i * L->N + j;
        finish_cell(L, i, j, F->x + cell * L->c_h, F->out + cell * L->c_z, scratch);
    }
}

/* x: [N][N][c_h], out: [N][N][c_z], both cell-major doubles. */
int oracle_finish(int N, int c_z, int c_h, const float *z, const double *x,
                  const oracle_weights *w, double eps, double *out, int nthreads)
{
    if (N < 1 || c_z < 1 || c_h < 1 || !z || !x || !w || !out) return -1;
    layer_ctx L = {N, c_z, c_h, z, NULL, w, eps};
    finish_arg F = {&L, x, out};
    par_rows(N, FINISH_SCRATCH(c_z, c_h), nthreads, finish_row, &F);
    return 0;
}

/* ---- the whole layer ------------------------------------------------------ */

int oracle_trimul(int N, int c_z, int c_h, const float *z, const float *mask,
                  const oracle_weights *w, double eps, int direction, double *out, int nthreads)
{
    if (N < 1 || c_z < 1 || c_h < 1 || !z || !w || !out || (direction != 0 && direction != 1))
        return -1;
    size_t n = (size_t)N * N * c_h;
    double *a = (double *)malloc(n * sizeof(double));
    double *b = (double *)malloc(n * sizeof(double));
    double *x = (double *)malloc(n * sizeof(double));
    int rc = -2;
    if (a && b && x) {
        rc = oracle_project(N, c_z, c_h, z, mask, w, eps, a, b, nthreads);
        if (!rc) rc = oracle_contract(N, c_h, a, b, direction, x, nthreads);
        if (!rc) rc = oracle_finish(N, c_z, c_h, z, x, w, eps, out, nthreads);
    }
    free(a); free(b); free(x);
    return rc;
}

/* ---- sampled cells: the grid I x I --------------------------------------- *
 * Computes out_ij for i, j in the index list I without touching any other
 * output cell. Outgoing needs a_ik and b_jk for all k (rows i and j of a, b);
 * incoming needs a_ki and b_kj (columns i and j). Those lines are projected
 * with the same project_cell as above, then each output cell follows steps
 * 3-6 exactly as the full layer does.
 */
typedef struct {
    const layer_ctx *L;
    int incoming, nI;
    const int *I;
    double *aline, *bline; /* [nI][N][c_h]: the k-indexed line through each index */
    double *out;           /* [nI][nI][c_z] */
} grid_arg;

static void grid_project(void *p, int t, double *scratch)
{
    grid_arg *G = (grid_arg *)p;
    const layer_ctx *L = G->L;
    const int N = L->N, ch = L->c_h;
    const int idx = G->I[t];
    for (int k = 0; k < N; ++k) {
        double *a = G->aline + ((size_t)t * N + k) * ch;
        double *b = G->bline + ((size_t)t * N + k) * ch;
        if (!G->incoming) {
            /* a_{idx,k} and b_{idx,k}: both on row idx. */
            project_cell(L, idx, k, a, b, scratch);
        } else {
            /* a_{k,idx} and b_{k,idx}: both on column idx. */
            project_cell(L, k, idx, a, b, scratch);
        }
    }
}

static void grid_finish(void *p, int ti, double *scratch)
{
    grid_arg *G = (grid_arg *)p;
    const layer_ctx *L = G->L;
    const int N = L->N, ch = L->c_h, cz = L->c_z;
    double *x = scratch;
    double *fs = scratch + ch;
    for (int tj = 0; tj < G->nI; ++tj) {
        for (int c = 0; c < ch; ++c) x[c] = 0.0;
        for (int k = 0; k < N; ++k) {
            /* outgoing: a_ik (row i line) * b_jk (row j line)
               incoming: a_ki (column i line) * b_kj (column j line) */
            const double *ak = G->aline + ((size_t)ti * N + k) * ch;
            const double *bk = G->bline + ((size_t)tj * N + k) * ch;
            for (int c = 0; c < ch; ++c) x[c] += ak[c] * bk[c];
        }
        finish_cell(L, G->I[ti], G->I[tj], x,
                    G->out + ((size_t)ti * G->nI + tj) * cz, fs);
    }
}

int oracle_trimul_grid(int N, int c_z, int c_h, const float *z, const float *mask,
                       const oracle_weights *w, double eps, int direction,
                       int nI, const int *I, double *out, int nthreads)
{
    if (N < 1 || c_z < 1 || c_h < 1 || !z || !w || !out || !I || nI < 1 ||
        (direction != 0 && direction != 1))
        return -1;
    for (int t = 0; t < nI; ++t)
        if (I[t] < 0 || I[t] >= N) return -1;
    layer_ctx L = {N, c_z, c_h, z, mask, w, eps};
    size_t n = (size_t)nI * N * c_h;
    double *aline = (double *)malloc(n * sizeof(double));
    double *bline = (double *)malloc(n * sizeof(double));
    if (!aline || !bline) { free(aline); free(bline); return -2; }
    grid_arg G = {&L, direction, nI, I, aline, bline, out};
    int ps = PROJECT_SCRATCH(c_z, c_h);
    par_rows(nI, ps, nthreads, grid_project, &G);
    par_rows(nI, c_h + FINISH_SCRATCH(c_z, c_h), nthreads, grid_finish, &G);
    free(aline); free(bline);
    return 0;
}
