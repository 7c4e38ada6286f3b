/*
 * fp64 CPU oracle of the double-binary factorised layer forward.
 *
 * TEST INFRASTRUCTURE. Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg load this file's library. The CUDA product
 * path shares no code with it and never calls it.
 *
 * What it computes (the plain definition, factor by factor, in fp64):
 *
 *   LoRDBA page, section 2 "Arquitetura Central" (Delta-W equation):
 *     dW = sum_{i=1..ell} diag(alpha_i) B1 diag(beta_i) B2 diag(gamma_i),
 *     B1 in {+-1}^{N x R}, B2 in {+-1}^{R x M}; the same two sign matrices
 *     serve every envelope i, only the scales carry the superscript.
 *   LoRDBA page, section 2 "Kernel de Inferencia": the forward is two
 *     sign-accumulation products with per-channel scaling between them.
 *   LoRDBA page, sections 1 and 3 (unmerged adapter mode): the branch output
 *     is added to the base output when 'accumulate' is set.
 *   DBF page, section 2 (W ~ (a . A . m^T)(B . b^T)) is the same form with
 *     ell = 1 and a -> alpha, A -> B1, m -> beta, B -> B2, b -> gamma.
 *
 *   y[t,n] = [acc] y_in[t,n]
 *            + sum_i alpha_i[n] * sum_r B1[n,r] * beta_i[r]
 *                               * sum_m B2[r,m] * gamma_i[m] * x[t,m]
 *
 * Inputs are the unpacked +-1 int8 matrices and the bit patterns of the
 * fp16 scales and of the bf16 / fp32 activations; each is decoded to double
 * by exact bit arithmetic below. Rows (tokens) are independent; 'rows'
 * selects which ones are evaluated, so a subset of a large batch gives
 * exact per-row reference values.
 *
 * The packer below writes the packed sign layout of the library header from
 * its written definition (row-major, ceil(k/32) 32-bit words per row; in
 * word w, bit p (p < 16) holds k = 32w + 2p and bit 16 + p holds
 * k = 32w + 2p + 1; bit set means -1; padding bits zero).
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ---- exact decoders --------------------------------------------------- */

double dbf_oracle_f16_to_f64(uint16_t h)
{
    int s = (h >> 15) & 1;
    int e = (h >> 10) & 0x1f;
    int f = h & 0x3ff;
    double v;
    if (e == 0)
        v = ldexp((double)f, -24);                 /* subnormal: f * 2^-24 */
    else if (e == 31)
        v = f ? NAN : INFINITY;
    else
        v = ldexp((double)(f | 0x400), e - 25);    /* 1.f * 2^(e-15) */
    return s ? -v : v;
}

double dbf_oracle_bf16_to_f64(uint16_t b)
{
    int s = (b >> 15) & 1;
    int e = (b >> 7) & 0xff;
    int f = b & 0x7f;
    double v;
    if (e == 0)
        v = ldexp((double)f, -133);                /* subnormal: f * 2^-133 */
    else if (e == 255)
        v = f ? NAN : INFINITY;
    else
        v = ldexp((double)(f | 0x80), e - 134);    /* 1.f * 2^(e-127) */
    return s ? -v : v;
}

double dbf_oracle_f32_to_f64(uint32_t u)
{
    int s = (u >> 31) & 1;
    int e = (u >> 23) & 0xff;
    uint32_t f = u & 0x7fffff;
    double v;
    if (e == 0)
        v = ldexp((double)f, -149);
    else if (e == 255)
        v = f ? NAN : INFINITY;
    else
        v = ldexp((double)(f | 0x800000), e - 150);
    return s ? -v : v;
}

/* kind: 0 = fp32 bits (uint32), 1 = bf16 bits (uint16) */
static double load_act(const void *p, int kind, int64_t idx)
{
    if (kind == 0)
        return dbf_oracle_f32_to_f64(((const uint32_t *)p)[idx]);
    return dbf_oracle_bf16_to_f64(((const uint16_t *)p)[idx]);
}

/* ---- the forward ------------------------------------------------------ */

typedef struct {
    int64_t M, N, R, ell;
    const int8_t *b1, *b2;
    const uint16_t *alpha, *beta, *gamma;
    const void *x;
    int x_kind;
    const int64_t *rows;
    int64_t nrows;
    const void *y_in;
    int y_kind;
    int accumulate;
    double *y_out;
    int64_t row_begin, row_end;   /* slice of 'rows' for one worker */
} fwd_job;

static void forward_rows(const fwd_job *J)
{
    const int64_t M = J->M, N = J->N, R = J->R;
    double *u = (double *)malloc(sizeof(double) * (size_t)M);
    double *v = (double *)malloc(sizeof(double) * (size_t)R);
    for (int64_t q = J->row_begin; q < J->row_end; ++q) {
        const int64_t t = J->rows[q];
        double *y = J->y_out + q * N;
        for (int64_t n = 0; n < N; ++n)
            y[n] = J->accumulate ? load_act(J->y_in, J->y_kind, t * N + n) : 0.0;
        for (int64_t i = 0; i < J->ell; ++i) {
            /* gamma scaling of the input */
            for (int64_t m = 0; m < M; ++m)
                u[m] = dbf_oracle_f16_to_f64(J->gamma[i * M + m]) * load_act(J->x, J->x_kind, t * M + m);
            /* first sign accumulation (B2, R x M), then beta scaling */
            for (int64_t r = 0; r < R; ++r) {
                double h = 0.0;
                const int8_t *b2row = J->b2 + r * M;
                for (int64_t m = 0; m < M; ++m)
                    h += (double)b2row[m] * u[m];
                v[r] = dbf_oracle_f16_to_f64(J->beta[i * R + r]) * h;
            }
            /* second sign accumulation (B1, N x R), alpha scaling, envelope sum */
            for (int64_t n = 0; n < N; ++n) {
                double z = 0.0;
                const int8_t *b1row = J->b1 + n * R;
                for (int64_t r = 0; r < R; ++r)
                    z += (double)b1row[r] * v[r];
                y[n] += dbf_oracle_f16_to_f64(J->alpha[i * N + n]) * z;
            }
        }
    }
    free(u);
    free(v);
}

static void *forward_worker(void *arg)
{
    forward_rows((const fwd_job *)arg);
    return NULL;
}

/* Returns 0 on success, -1 on bad arguments. */
int dbf_oracle_forward(int64_t M, int64_t N, int64_t R, int64_t ell,
                       const int8_t *b1, const int8_t *b2,
                       const uint16_t *alpha, const uint16_t *beta, const uint16_t *gamma,
                       const void *x, int x_kind,
                       const int64_t *rows, int64_t nrows,
                       const void *y_in, int y_kind, int accumulate,
                       double *y_out, int nthreads)
{
    if (M <= 0 || N <= 0 || R <= 0 || ell <= 0 || nrows < 0 || !b1 || !b2 || !alpha || !beta ||
        !gamma || !x || !rows || !y_out || (accumulate && !y_in))
        return -1;
    if (nthreads < 1)
        nthreads = 1;
    if (nthreads > nrows)
        nthreads = nrows > 0 ? (int)nrows : 1;
    fwd_job *jobs = (fwd_job *)calloc((size_t)nthreads, sizeof(fwd_job));
    pthread_t *th = (pthread_t *)calloc((size_t)nthreads, sizeof(pthread_t));
    for (int k = 0; k < nthreads; ++k) {
        fwd_job *J = &jobs[k];
        J->M = M; J->N = N; J->R = R; J->ell = ell;
        J->b1 = b1; J->b2 = b2; J->alpha = alpha; J->beta = beta; J->gamma = gamma;
        J->x = x; J->x_kind = x_kind; J->rows = rows; J->nrows = nrows;
        J->y_in = y_in; J->y_kind = y_kind; J->accumulate = accumulate; J->y_out = y_out;
        J->row_begin = nrows * k / nthreads;
        J->row_end = nrows * (k + 1) / nthreads;
    }
    for (int k = 1; k < nthreads; ++k)
        pthread_create(&th[k], NULL, forward_worker, &jobs[k]);
    forward_rows(&jobs[0]);
    for (int k = 1; k < nthreads; ++k)
        pthread_join(th[k], NULL);
    free(jobs);
    free(th);
    return 0;
}

/* ---- packed sign layout ----------------------------------------------- */

/* Bit position inside a 32-bit word of in-word index j (k = 32w + j). */
static int bit_of(int j) { return (j & 1) ? 16 + (j >> 1) : (j >> 1); }

/* s: rows x k int8, any value < 0 is the sign -1, every other value +1. */
void dbf_oracle_pack(const int8_t *s, int64_t rows, int64_t k, uint32_t *out)
{
    const int64_t pitch = (k + 31) / 32;
    memset(out, 0, sizeof(uint32_t) * (size_t)(rows * pitch));
    for (int64_t i = 0; i < rows; ++i)
        for (int64_t c = 0; c < k; ++c)
            if (s[i * k + c] < 0)
                out[i * pitch + c / 32] |= 1u << bit_of((int)(c % 32));
}

void dbf_oracle_unpack(const uint32_t *w, int64_t rows, int64_t k, int8_t *s)
{
    const int64_t pitch = (k + 31) / 32;
    for (int64_t i = 0; i < rows; ++i)
        for (int64_t c = 0; c < k; ++c)
            s[i * k + c] = ((w[i * pitch + c / 32] >> bit_of((int)(c % 32))) & 1u) ? -1 : 1;
}

/* ---- the backward ----------------------------------------------------- */
/*
 * Gradients of a loss L through the forward above, given dL/dy = dy
 * (LoRDBA page, section 2, training pipeline: quantisation-aware training
 * of the factors with a straight-through estimator; the pages give the
 * forward only, so these are its derivatives, written out by the chain rule
 * in the forward's own order). Per token t and envelope i, in fp64:
 *
 *   u_i = gamma_i . x_t          h_i = B2 u_i        v_i = beta_i . h_i
 *   z_i = B1 v_i                 y_t = sum_i alpha_i . z_i
 *   a_i = alpha_i . dy_t         g_i = B1^T a_i      w_i = beta_i . g_i
 *   e_i = B2^T w_i
 *
 *   dalpha_i += dy_t . z_i       dbeta_i += g_i . h_i
 *   dgamma_i += x_t . e_i        dx_t = sum_i gamma_i . e_i
 *   dB1 += a_i v_i^T             dB2 += w_i u_i^T
 *
 * dB1 and dB2 are the gradients with respect to the sign matrices taken as
 * real variables: what a straight-through estimator hands to the latents.
 * Scale-gradient and dB outputs are sums over all tokens (rows); dx is per
 * row. Any output pointer may be NULL.
 */
typedef struct {
    int64_t M, N, R, ell;
    const int8_t *b1, *b2;
    const uint16_t *alpha, *beta, *gamma;
    const void *x;
    int x_kind;
    const void *dy;
    int dy_kind;
    int64_t row_begin, row_end;
    double *dx;                                  /* [T][M] */
    double *dalpha, *dbeta, *dgamma, *db1, *db2; /* private partial sums of this worker */
} bwd_job;

static void backward_rows(const bwd_job *J)
{
    const int64_t M = J->M, N = J->N, R = J->R;
    double *u = (double *)malloc(sizeof(double) * (size_t)M);
    double *h = (double *)malloc(sizeof(double) * (size_t)R);
    double *v = (double *)malloc(sizeof(double) * (size_t)R);
    double *z = (double *)malloc(sizeof(double) * (size_t)N);
    double *a = (double *)malloc(sizeof(double) * (size_t)N);
    double *g = (double *)malloc(sizeof(double) * (size_t)R);
    double *w = (double *)malloc(sizeof(double) * (size_t)R);
    double *e = (double *)malloc(sizeof(double) * (size_t)M);
    for (int64_t t = J->row_begin; t < J->row_end; ++t) {
        if (J->dx)
            for (int64_t m = 0; m < M; ++m) J->dx[t * M + m] = 0.0;
        for (int64_t i = 0; i < J->ell; ++i) {
            /* forward quantities of this token and envelope */
            for (int64_t m = 0; m < M; ++m)
                u[m] = dbf_oracle_f16_to_f64(J->gamma[i * M + m]) * load_act(J->x, J->x_kind, t * M + m);
            for (int64_t r = 0; r < R; ++r) {
                double s = 0.0;
                for (int64_t m = 0; m < M; ++m) s += (double)J->b2[r * M + m] * u[m];
                h[r] = s;
                v[r] = dbf_oracle_f16_to_f64(J->beta[i * R + r]) * s;
            }
            for (int64_t n = 0; n < N; ++n) {
                double s = 0.0;
                for (int64_t r = 0; r < R; ++r) s += (double)J->b1[n * R + r] * v[r];
                z[n] = s;
            }
            /* backward: alpha, then B1 transposed, beta, B2 transposed, gamma */
            for (int64_t n = 0; n < N; ++n) {
                const double d = load_act(J->dy, J->dy_kind, t * N + n);
                a[n] = dbf_oracle_f16_to_f64(J->alpha[i * N + n]) * d;
                if (J->dalpha) J->dalpha[i * N + n] += d * z[n];
            }
            for (int64_t r = 0; r < R; ++r) {
                double s = 0.0;
                for (int64_t n = 0; n < N; ++n) s += (double)J->b1[n * R + r] * a[n];
                g[r] = s;
                w[r] = dbf_oracle_f16_to_f64(J->beta[i * R + r]) * s;
                if (J->dbeta) J->dbeta[i * R + r] += s * h[r];
            }
            for (int64_t m = 0; m < M; ++m) {
                double s = 0.0;
                for (int64_t r = 0; r < R; ++r) s += (double)J->b2[r * M + m] * w[r];
                e[m] = s;
                if (J->dgamma) J->dgamma[i * M + m] += load_act(J->x, J->x_kind, t * M + m) * s;
                if (J->dx) J->dx[t * M + m] += dbf_oracle_f16_to_f64(J->gamma[i * M + m]) * s;
            }
            if (J->db1)
                for (int64_t n = 0; n < N; ++n)
                    for (int64_t r = 0; r < R; ++r) J->db1[n * R + r] += a[n] * v[r];
            if (J->db2)
                for (int64_t r = 0; r < R; ++r)
                    for (int64_t m = 0; m < M; ++m) J->db2[r * M + m] += w[r] * u[m];
        }
    }
    free(u); free(h); free(v); free(z); free(a); free(g); free(w); free(e);
}

static void *backward_worker(void *arg)
{
    backward_rows((const bwd_job *)arg);
    return NULL;
}

static double *zeros_or_null(int want, int64_t n)
{
    return want ? (double *)calloc((size_t)n, sizeof(double)) : NULL;
}

/* Returns 0 on success, -1 on bad arguments. Rows 0 .. T-1. */
int dbf_oracle_backward(int64_t M, int64_t N, int64_t R, int64_t ell,
                        const int8_t *b1, const int8_t *b2,
                        const uint16_t *alpha, const uint16_t *beta, const uint16_t *gamma,
                        const void *x, int x_kind, const void *dy, int dy_kind, int64_t T,
                        double *dx, double *dalpha, double *dbeta, double *dgamma,
                        double *db1, double *db2, int nthreads)
{
    if (M <= 0 || N <= 0 || R <= 0 || ell <= 0 || T < 0 || !b1 || !b2 || !alpha || !beta || !gamma ||
        !x || !dy)
        return -1;
    if (nthreads < 1)
        nthreads = 1;
    if (nthreads > T)
        nthreads = T > 0 ? (int)T : 1;
    bwd_job *jobs = (bwd_job *)calloc((size_t)nthreads, sizeof(bwd_job));
    pthread_t *th = (pthread_t *)calloc((size_t)nthreads, sizeof(pthread_t));
    for (int k = 0; k < nthreads; ++k) {
        bwd_job *J = &jobs[k];
        J->M = M; J->N = N; J->R = R; J->ell = ell;
        J->b1 = b1; J->b2 = b2; J->alpha = alpha; J->beta = beta; J->gamma = gamma;
        J->x = x; J->x_kind = x_kind; J->dy = dy; J->dy_kind = dy_kind;
        J->row_begin = T * k / nthreads;
        J->row_end = T * (k + 1) / nthreads;
        J->dx = dx;
        J->dalpha = zeros_or_null(dalpha != NULL, ell * N);
        J->dbeta = zeros_or_null(dbeta != NULL, ell * R);
        J->dgamma = zeros_or_null(dgamma != NULL, ell * M);
        J->db1 = zeros_or_null(db1 != NULL, N * R);
        J->db2 = zeros_or_null(db2 != NULL, R * M);
    }
    for (int k = 1; k < nthreads; ++k)
        pthread_create(&th[k], NULL, backward_worker, &jobs[k]);
    backward_rows(&jobs[0]);
    for (int k = 1; k < nthreads; ++k)
        pthread_join(th[k], NULL);
    /* sum the workers' partial sums in worker order */
    double *outs[5] = {dalpha, dbeta, dgamma, db1, db2};
    const int64_t lens[5] = {ell * N, ell * R, ell * M, N * R, R * M};
    for (int o = 0; o < 5; ++o) {
        if (!outs[o]) continue;
        for (int64_t q = 0; q < lens[o]; ++q) outs[o][q] = 0.0;
        for (int k = 0; k < nthreads; ++k) {
            double *part = o == 0 ? jobs[k].dalpha : o == 1 ? jobs[k].dbeta : o == 2 ? jobs[k].dgamma
                         : o == 3 ? jobs[k].db1 : jobs[k].db2;
            for (int64_t q = 0; q < lens[o]; ++q) outs[o][q] += part[q];
        }
    }
    for (int k = 0; k < nthreads; ++k) {
        free(jobs[k].dalpha); free(jobs[k].dbeta); free(jobs[k].dgamma); free(jobs[k].db1); free(jobs[k].db2);
    }
    free(jobs);
    free(th);
    return 0;
}

/* ---- multi-boolean-kernel layer (MBOK) --------------------------------- */
/*
 * Multi-Boolean Architectures page, section 2 ("Metodologia Proposta"):
 * a weight matrix is approximated by a sum of K boolean kernels, each with
 * an output and an input scale vector,
 *     W ~ sum_{k=1..K} W_bool^[k] . (s_out^[k] s_in^[k]^T),
 * so the layer's forward is
 *     y[t,n] = sum_k s_out^[k][n] * sum_m W^[k][n,m] * s_in^[k][m] * x[t,m].
 * w: int8 +-1 [K][N][M]; s_in: fp16 bits [K][M]; s_out: fp16 bits [K][N].
 * Rows 0 .. T-1. Returns 0, or -1 on bad arguments.
 */
int dbf_oracle_mbok_forward(int64_t M, int64_t N, int64_t K, const int8_t *w, const uint16_t *s_in,
                            const uint16_t *s_out, const void *x, int x_kind, int64_t T, double *y_out)
{
    if (M <= 0 || N <= 0 || K <= 0 || T < 0 || !w || !s_in || !s_out || !x || !y_out)
        return -1;
    double *u = (double *)malloc(sizeof(double) * (size_t)M);
    for (int64_t t = 0; t < T; ++t) {
        double *y = y_out + t * N;
        for (int64_t n = 0; n < N; ++n) y[n] = 0.0;
        for (int64_t k = 0; k < K; ++k) {
            for (int64_t m = 0; m < M; ++m)
                u[m] = dbf_oracle_f16_to_f64(s_in[k * M + m]) * load_act(x, x_kind, t * M + m);
            for (int64_t n = 0; n < N; ++n) {
                const int8_t *row = w + (k * N + n) * M;
                double s = 0.0;
                for (int64_t m = 0; m < M; ++m) s += (double)row[m] * u[m];
                y[n] += dbf_oracle_f16_to_f64(s_out[k * N + n]) * s;
            }
        }
    }
    free(u);
    return 0;
}
