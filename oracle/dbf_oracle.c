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
