/*
 * oracle.c -- float64 CPU oracle for the Hyena order-N forward and backward.
 *
 * TEST INFRASTRUCTURE ONLY. Only tests/, __graft_entry__.smoke() and the
 * CPU-baseline leg of bench.py may load this library. It shares no code,
 * header, table or constant with the CUDA library: it is the plain
 * definition of what that library computes, written so that it can be
 * checked against the pages by eye.
 *
 * Sources (page title, section):
 *  - Order-N recurrence z_1 = v, z_{n+1} = x_n * (h_n conv z_n), y = z_{N+1}:
 *    "Hyena Hierarchy - Towards Larger Convolutional Language Models" digest,
 *    section "방법 (Method) / 프레임워크 개요" (the framework graph); and the
 *    explainer "Hyena Hierarchy: Towards Larger Convolutional Language
 *    Models", section "Hyena 演算子の形".
 *  - Causal convolution (h conv z)_t = sum_{s=0..t} h_{t-s} z_s: "02. 3つの
 *    Hyena 演算子", section "4. FIR フィルタと効率的な生成" (the FIR sum).
 *  - FFT evaluation on a 2L zero-padded grid: glossary "Hyena（ハイエナ）",
 *    section "計算効率"; HyenaND summary, "境界の処理" (zero padding to twice
 *    the grid avoids wrap-around leakage).
 *  - Implicit filter h(t) = Window(t) * FFN(t/L, sin, cos): glossary
 *    "Hyena（ハイエナ）", section "暗黙的畳み込みフィルタ". The exact recipe
 *    (17-dim embedding, Linear-sin-Linear-sin-Linear, exp(-alpha_c t / L)
 *    window with alpha_c linearly spaced) is the workload specification.
 *
 * The backward (gradients w.r.t. v, x_n, h_n and the filter weights) is the
 * chain rule applied to these same definitions; the pages give no formulas
 * for it.
 *
 * Evaluation rules: direct O(L^2) causal sum for L <= 8192; above that a
 * naive recursive radix-2 FFT on the 2L zero-padded grid, keeping the first
 * L outputs. All arithmetic in double.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_DIRECT_MAX_L 8192

static const double ORACLE_PI = 3.14159265358979323846264338327950288;

/* ------------------------------------------------------------------------ */
/* Implicit filter                                                          */
/* ------------------------------------------------------------------------ */

/*
 * Positional embedding of tap t for a filter of length L:
 *   e = [ t/L, sin(2 pi k t / L) for k = 1..K, cos(2 pi k t / L) for k = 1..K ]
 * (1 + 2K values; block order: the linear term, then the K sines, then the
 * K cosines).
 */
void oracle_embedding(int t, int L, int n_bands, double *e)
{
    e[0] = (double)t / (double)L;
    for (int k = 1; k <= n_bands; ++k) {
        double a = 2.0 * ORACLE_PI * (double)k * (double)t / (double)L;
        e[k] = sin(a);
        e[n_bands + k] = cos(a);
    }
}

/* alpha_c linearly spaced over [lo, hi] with both ends included. */
double oracle_alpha(int c, int D, double lo, double hi)
{
    if (D <= 1) return lo;
    return lo + (hi - lo) * (double)c / (double)(D - 1);
}

typedef struct {
    const float *W1, *b1, *W2, *b2, *W3, *b3;
    int n_bands, width, N, D, L;
    double alpha_lo, alpha_hi;
    int n_rows;           /* number of (n, c) filter rows requested */
    const int *rows_n;    /* filter index n in [0, N) */
    const int *rows_c;    /* channel index c in [0, D) */
    double *h;            /* [n_rows][L] */
    int t_begin, t_end;
} filter_job;

static void *filter_worker(void *arg)
{
    filter_job *j = (filter_job *)arg;
    const int E = 1 + 2 * j->n_bands, H = j->width;
    double *e = (double *)malloc(sizeof(double) * E);
    double *s1 = (double *)malloc(sizeof(double) * H);
    double *s2 = (double *)malloc(sizeof(double) * H);
    for (int t = j->t_begin; t < j->t_end; ++t) {
        oracle_embedding(t, j->L, j->n_bands, e);
        /* layer 1: s1 = sin(W1 e + b1), W1 is [H][E] row-major */
        for (int o = 0; o < H; ++o) {
            double acc = (double)j->b1[o];
            for (int i = 0; i < E; ++i) acc += (double)j->W1[o * E + i] * e[i];
            s1[o] = sin(acc);
        }
        /* layer 2: s2 = sin(W2 s1 + b2), W2 is [H][H] */
        for (int o = 0; o < H; ++o) {
            double acc = (double)j->b2[o];
            for (int i = 0; i < H; ++i) acc += (double)j->W2[o * H + i] * s1[i];
            s2[o] = sin(acc);
        }
        /* layer 3 and window: output column (n * D + c) is filter n, channel c */
        for (int r = 0; r < j->n_rows; ++r) {
            int n = j->rows_n[r], c = j->rows_c[r];
            int o = n * j->D + c;
            double acc = (double)j->b3[o];
            for (int i = 0; i < H; ++i) acc += (double)j->W3[o * H + i] * s2[i];
            double alpha = oracle_alpha(c, j->D, j->alpha_lo, j->alpha_hi);
            double window = exp(-alpha * (double)t / (double)j->L);
            j->h[(size_t)r * j->L + t] = acc * window;
        }
    }
    free(e); free(s1); free(s2);
    return NULL;
}

/*
 * h[r][t] for the requested (n, c) rows, t in [0, L).
 * Weights are the float32 values the GPU receives, evaluated in double.
 */
void oracle_filter(const float *W1, const float *b1, const float *W2, const float *b2,
                   const float *W3, const float *b3, int n_bands, int width,
                   int N, int D, int L, double alpha_lo, double alpha_hi,
                   int n_rows, const int *rows_n, const int *rows_c,
                   double *h, int n_threads)
{
    if (n_threads < 1) n_threads = 1;
    if (n_threads > L) n_threads = L;
    pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * n_threads);
    filter_job *jobs = (filter_job *)malloc(sizeof(filter_job) * n_threads);
    for (int i = 0; i < n_threads; ++i) {
        filter_job j = {W1, b1, W2, b2, W3, b3, n_bands, width, N, D, L, alpha_lo, alpha_hi,
                        n_rows, rows_n, rows_c, h,
                        (int)((int64_t)L * i / n_threads), (int)((int64_t)L * (i + 1) / n_threads)};
        jobs[i] = j;
        pthread_create(&th[i], NULL, filter_worker, &jobs[i]);
    }
    for (int i = 0; i < n_threads; ++i) pthread_join(th[i], NULL);
    free(th); free(jobs);
}

/* ------------------------------------------------------------------------ */
/* Naive recursive radix-2 FFT                                              */
/* ------------------------------------------------------------------------ */

/*
 * In place, unnormalised: X[k] = sum_n x[n] exp(sign * 2 pi i n k / n_pts),
 * sign = -1 forward, +1 inverse. n_pts must be a power of two. Textbook
 * decimation in time: split even/odd samples, transform each half, combine
 * X[k] = E[k] + w^k O[k], X[k + n/2] = E[k] - w^k O[k].
 */
void oracle_fft(double *re, double *im, int64_t n, int sign)
{
    if (n <= 1) return;
    int64_t h = n / 2;
    double *er = (double *)malloc(sizeof(double) * h), *ei = (double *)malloc(sizeof(double) * h);
    double *or_ = (double *)malloc(sizeof(double) * h), *oi = (double *)malloc(sizeof(double) * h);
    for (int64_t i = 0; i < h; ++i) {
        er[i] = re[2 * i];     ei[i] = im[2 * i];
        or_[i] = re[2 * i + 1]; oi[i] = im[2 * i + 1];
    }
    oracle_fft(er, ei, h, sign);
    oracle_fft(or_, oi, h, sign);
    for (int64_t k = 0; k < h; ++k) {
        double ang = (double)sign * 2.0 * ORACLE_PI * (double)k / (double)n;
        double wr = cos(ang), wi = sin(ang);
        double tr = wr * or_[k] - wi * oi[k];
        double ti = wr * oi[k] + wi * or_[k];
        re[k] = er[k] + tr;      im[k] = ei[k] + ti;
        re[k + h] = er[k] - tr;  im[k + h] = ei[k] - ti;
    }
    free(er); free(ei); free(or_); free(oi);
}

/* ------------------------------------------------------------------------ */
/* Causal long convolution                                                  */
/* ------------------------------------------------------------------------ */

/* out[t] = sum_{s=0..t} h[t-s] z[s], t in [0, L): the plain definition. */
void oracle_causal_conv_direct(const double *h, const double *z, int64_t L, double *out)
{
    for (int64_t t = 0; t < L; ++t) {
        double acc = 0.0;
        for (int64_t s = 0; s <= t; ++s) acc += h[t - s] * z[s];
        out[t] = acc;
    }
}

/* Same result via FFT: zero-pad both to 2L, transform, multiply pointwise,
 * inverse transform, divide by 2L, keep the first L samples. */
void oracle_causal_conv_fft(const double *h, const double *z, int64_t L, double *out)
{
    int64_t n = 2 * L;
    double *hr = (double *)calloc(n, sizeof(double)), *hi = (double *)calloc(n, sizeof(double));
    double *zr = (double *)calloc(n, sizeof(double)), *zi = (double *)calloc(n, sizeof(double));
    memcpy(hr, h, sizeof(double) * L);
    memcpy(zr, z, sizeof(double) * L);
    oracle_fft(hr, hi, n, -1);
    oracle_fft(zr, zi, n, -1);
    for (int64_t k = 0; k < n; ++k) {
        double pr = hr[k] * zr[k] - hi[k] * zi[k];
        double pi = hr[k] * zi[k] + hi[k] * zr[k];
        zr[k] = pr; zi[k] = pi;
    }
    oracle_fft(zr, zi, n, +1);
    for (int64_t t = 0; t < L; ++t) out[t] = zr[t] / (double)n;
    free(hr); free(hi); free(zr); free(zi);
}

void oracle_causal_conv(const double *h, const double *z, int64_t L, double *out)
{
    if (L <= ORACLE_DIRECT_MAX_L) oracle_causal_conv_direct(h, z, L, out);
    else oracle_causal_conv_fft(h, z, L, out);
}

/* ------------------------------------------------------------------------ */
/* Filter spectrum                                                          */
/* ------------------------------------------------------------------------ */

/*
 * H[k] = sum_{t<L} h[t] exp(-2 pi i k t / (2L)), k = 0..L: the spectrum of
 * the filter on the 2L zero-padded grid (bins L+1..2L-1 are the conjugates).
 * Direct sum for L <= 8192, radix-2 FFT above.
 */
void oracle_filter_spectrum(const double *h, int64_t L, double *re, double *im)
{
    if (L <= ORACLE_DIRECT_MAX_L) {
        for (int64_t k = 0; k <= L; ++k) {
            double ar = 0.0, ai = 0.0;
            for (int64_t t = 0; t < L; ++t) {
                /* reduce k*t mod 2L exactly before forming the angle */
                int64_t e = (k * t) % (2 * L);
                double ang = -2.0 * ORACLE_PI * (double)e / (double)(2 * L);
                ar += h[t] * cos(ang);
                ai += h[t] * sin(ang);
            }
            re[k] = ar; im[k] = ai;
        }
        return;
    }
    int64_t n = 2 * L;
    double *xr = (double *)calloc(n, sizeof(double)), *xi = (double *)calloc(n, sizeof(double));
    memcpy(xr, h, sizeof(double) * L);
    oracle_fft(xr, xi, n, -1);
    for (int64_t k = 0; k <= L; ++k) { re[k] = xr[k]; im[k] = xi[k]; }
    free(xr); free(xi);
}

/* ------------------------------------------------------------------------ */
/* Order-N recurrence                                                       */
/* ------------------------------------------------------------------------ */

/*
 * One channel: z_1 = v; z_{n+1}[t] = x_n[t] * (h_n conv z_n)[t]; y = z_{N+1}.
 * x[n] and h[n] point at the length-L rows of gate n and filter n.
 */
void oracle_hyena_channel(const double *v, const double *const *x, const double *const *h,
                          int64_t L, int N, double *y)
{
    double *z = (double *)malloc(sizeof(double) * L);
    double *c = (double *)malloc(sizeof(double) * L);
    memcpy(z, v, sizeof(double) * L);
    for (int n = 0; n < N; ++n) {
        oracle_causal_conv(h[n], z, L, c);
        for (int64_t t = 0; t < L; ++t) z[t] = x[n][t] * c[t];
    }
    memcpy(y, z, sizeof(double) * L);
    free(z); free(c);
}

typedef struct {
    const double *v, *x, *h;
    const int *filter_row;   /* per channel: row of h (its channel c) */
    int64_t L, C;
    int N, n_filter_rows;
    double *y;
    int begin, end;
} fwd_job;

static void *fwd_worker(void *arg)
{
    fwd_job *j = (fwd_job *)arg;
    const double *xs[64];
    const double *hs[64];
    for (int r = j->begin; r < j->end; ++r) {
        for (int n = 0; n < j->N; ++n) {
            xs[n] = j->x + ((size_t)n * j->C + r) * j->L;
            hs[n] = j->h + ((size_t)n * j->n_filter_rows + j->filter_row[r]) * j->L;
        }
        oracle_hyena_channel(j->v + (size_t)r * j->L, xs, hs, j->L, j->N, j->y + (size_t)r * j->L);
    }
    return NULL;
}

/*
 * C independent channels.
 *   v [C][L], x [N][C][L], h [N][F][L], y [C][L];
 *   channel r uses filter row filter_row[r] of each h_n (its channel index c).
 * Work is split over n_threads POSIX threads by channel.
 */
int oracle_hyena_forward(const double *v, const double *x, const double *h,
                         const int *filter_row, int64_t C, int n_filter_rows,
                         int64_t L, int N, double *y, int n_threads)
{
    if (N < 1 || N > 64 || L < 1 || C < 0) return 1;
    if (C == 0) return 0;
    if (n_threads < 1) n_threads = 1;
    if (n_threads > C) n_threads = (int)C;
    pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * n_threads);
    fwd_job *jobs = (fwd_job *)malloc(sizeof(fwd_job) * n_threads);
    for (int i = 0; i < n_threads; ++i) {
        fwd_job j = {v, x, h, filter_row, L, C, N, n_filter_rows, y,
                     (int)(C * i / n_threads), (int)(C * (i + 1) / n_threads)};
        jobs[i] = j;
        pthread_create(&th[i], NULL, fwd_worker, &jobs[i]);
    }
    for (int i = 0; i < n_threads; ++i) pthread_join(th[i], NULL);
    free(th); free(jobs);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Backward (gradients of a scalar loss through the order-N recurrence)     */
/* ------------------------------------------------------------------------ */

/*
 * The pages print no backward formulas (they mention training at 1M tokens:
 * glossary "Hyena（ハイエナ）", section "超長系列タスクでの優位性"). What follows is the chain
 * rule applied to the forward definitions above, nothing more:
 *   u_n = h_n conv z_n,  z_{n+1} = x_n * u_n,  y = z_{N+1}.
 * With g_{N+1} = dL/dy and r_n = g_{n+1} * x_n:
 *   dL/dx_n[t]  = g_{n+1}[t] * u_n[t]
 *   dL/dz_n[s]  = sum_{t=s..L-1} h_n[t-s] r_n[t]         (adjoint of the causal sum)
 *   dL/dh_n[j]  = sum_{t=j..L-1} r_n[t] z_n[t-j]          (summed over the channels
 *                                                          that share filter n)
 *   dL/dv = g_1.
 */

/* out[s] = sum_{t=s..L-1} h[t-s] r[t]: the transpose of the causal sum. */
void oracle_causal_corr_direct(const double *h, const double *r, int64_t L, double *out)
{
    for (int64_t s = 0; s < L; ++s) {
        double acc = 0.0;
        for (int64_t t = s; t < L; ++t) acc += h[t - s] * r[t];
        out[s] = acc;
    }
}

/* out[j] = sum_{t=j..L-1} r[t] z[t-j]: the filter-gradient correlation. */
void oracle_causal_xcorr_direct(const double *r, const double *z, int64_t L, double *out)
{
    for (int64_t j = 0; j < L; ++j) {
        double acc = 0.0;
        for (int64_t t = j; t < L; ++t) acc += r[t] * z[t - j];
        out[j] = acc;
    }
}

/* Both correlations via the 2L zero-padded FFT: out[s] = IFFT(conj(A) B)[s]
 * for s < L, with A the transform of a (the lagged operand) and B of b.
 * corr:  a = h, b = r;  xcorr: a = z, b = r. */
static void corr_fft(const double *a, const double *b, int64_t L, double *out)
{
    int64_t n = 2 * L;
    double *ar = (double *)calloc(n, sizeof(double)), *ai = (double *)calloc(n, sizeof(double));
    double *br = (double *)calloc(n, sizeof(double)), *bi = (double *)calloc(n, sizeof(double));
    memcpy(ar, a, sizeof(double) * L);
    memcpy(br, b, sizeof(double) * L);
    oracle_fft(ar, ai, n, -1);
    oracle_fft(br, bi, n, -1);
    for (int64_t k = 0; k < n; ++k) {
        /* conj(A) * B */
        double pr = ar[k] * br[k] + ai[k] * bi[k];
        double pi = ar[k] * bi[k] - ai[k] * br[k];
        br[k] = pr; bi[k] = pi;
    }
    oracle_fft(br, bi, n, +1);
    for (int64_t s = 0; s < L; ++s) out[s] = br[s] / (double)n;
    free(ar); free(ai); free(br); free(bi);
}

void oracle_causal_corr_fft(const double *h, const double *r, int64_t L, double *out)
{
    corr_fft(h, r, L, out);
}

void oracle_causal_xcorr_fft(const double *r, const double *z, int64_t L, double *out)
{
    corr_fft(z, r, L, out);
}

void oracle_causal_corr(const double *h, const double *r, int64_t L, double *out)
{
    if (L <= ORACLE_DIRECT_MAX_L) oracle_causal_corr_direct(h, r, L, out);
    else oracle_causal_corr_fft(h, r, L, out);
}

void oracle_causal_xcorr(const double *r, const double *z, int64_t L, double *out)
{
    if (L <= ORACLE_DIRECT_MAX_L) oracle_causal_xcorr_direct(r, z, L, out);
    else oracle_causal_xcorr_fft(r, z, L, out);
}

/*
 * One channel. Forward again keeping every z_n and u_n, then the reverse
 * sweep above. dx[n] and dh[n] receive this channel's dL/dx_n and its
 * contribution to dL/dh_n (the caller sums contributions over channels that
 * share a filter row).
 */
void oracle_hyena_channel_backward(const double *v, const double *const *x, const double *const *h,
                                   const double *dy, int64_t L, int N,
                                   double *dv, double *const *dx, double *const *dh)
{
    double *z = (double *)malloc(sizeof(double) * (size_t)(N + 1) * L);   /* z_1..z_{N+1} */
    double *u = (double *)malloc(sizeof(double) * (size_t)N * L);         /* u_1..u_N */
    double *g = (double *)malloc(sizeof(double) * L);
    double *r = (double *)malloc(sizeof(double) * L);
    memcpy(z, v, sizeof(double) * L);
    for (int n = 0; n < N; ++n) {
        double *un = u + (size_t)n * L;
        oracle_causal_conv(h[n], z + (size_t)n * L, L, un);
        for (int64_t t = 0; t < L; ++t) z[(size_t)(n + 1) * L + t] = x[n][t] * un[t];
    }
    memcpy(g, dy, sizeof(double) * L);
    for (int n = N - 1; n >= 0; --n) {
        const double *un = u + (size_t)n * L;
        for (int64_t t = 0; t < L; ++t) {
            dx[n][t] = g[t] * un[t];
            r[t] = g[t] * x[n][t];
        }
        oracle_causal_xcorr(r, z + (size_t)n * L, L, dh[n]);
        oracle_causal_corr(h[n], r, L, g);
    }
    memcpy(dv, g, sizeof(double) * L);
    free(z); free(u); free(g); free(r);
}

typedef struct {
    const double *v, *x, *h, *dy;
    const int *filter_row;
    int64_t L, C;
    int N, n_filter_rows;
    double *dv, *dx, *dh;
    int begin, end;
} bwd_job;

static void *bwd_worker(void *arg)
{
    bwd_job *j = (bwd_job *)arg;
    const double *xs[64];
    const double *hs[64];
    double *dxs[64];
    double *dhs[64];
    for (int r = j->begin; r < j->end; ++r) {
        for (int n = 0; n < j->N; ++n) {
            xs[n] = j->x + ((size_t)n * j->C + r) * j->L;
            hs[n] = j->h + ((size_t)n * j->n_filter_rows + j->filter_row[r]) * j->L;
            dxs[n] = j->dx + ((size_t)n * j->C + r) * j->L;
            dhs[n] = j->dh + ((size_t)n * j->C + r) * j->L;
        }
        oracle_hyena_channel_backward(j->v + (size_t)r * j->L, xs, hs, j->dy + (size_t)r * j->L,
                                      j->L, j->N, j->dv + (size_t)r * j->L, dxs, dhs);
    }
    return NULL;
}

/*
 * C independent channels: v, dy, dv [C][L]; x, dx [N][C][L]; h [N][F][L];
 * dh [N][C][L] holds each channel's own contribution to dL/dh_n of its filter
 * row filter_row[r] (summed by the caller).
 */
int oracle_hyena_backward(const double *v, const double *x, const double *h, const double *dy,
                          const int *filter_row, int64_t C, int n_filter_rows, int64_t L, int N,
                          double *dv, double *dx, double *dh, int n_threads)
{
    if (N < 1 || N > 64 || L < 1 || C < 0) return 1;
    if (C == 0) return 0;
    if (n_threads < 1) n_threads = 1;
    if (n_threads > C) n_threads = (int)C;
    pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * n_threads);
    bwd_job *jobs = (bwd_job *)malloc(sizeof(bwd_job) * n_threads);
    for (int i = 0; i < n_threads; ++i) {
        bwd_job j = {v, x, h, dy, filter_row, L, C, N, n_filter_rows, dv, dx, dh,
                     (int)(C * i / n_threads), (int)(C * (i + 1) / n_threads)};
        jobs[i] = j;
        pthread_create(&th[i], NULL, bwd_worker, &jobs[i]);
    }
    for (int i = 0; i < n_threads; ++i) pthread_join(th[i], NULL);
    free(th); free(jobs);
    return 0;
}

/*
 * Gradients of the implicit-filter weights from dL/dh [N*D][L] (row n*D + c),
 * by the chain rule through h = window * (W3 s2 + b3), s2 = sin(W2 s1 + b2),
 * s1 = sin(W1 e + b1), e the positional embedding; all sums over t < L.
 *   dO_j(t) = dh_j(t) window_c(t)
 *   db3 = sum_t dO,  dW3 = sum_t dO s2^T,  ds2 = W3^T dO
 *   dp2 = ds2 cos(W2 s1 + b2),  db2 = sum_t dp2,  dW2 = sum_t dp2 s1^T,  ds1 = W2^T dp2
 *   dp1 = ds1 cos(W1 e + b1),   db1 = sum_t dp1,  dW1 = sum_t dp1 e^T
 * Outputs are float64 arrays shaped like the weights.
 */
typedef struct {
    const float *W1, *b1, *W2, *b2, *W3, *b3;
    int n_bands, width, N, D, L;
    double alpha_lo, alpha_hi;
    const double *dh;
    double *gW1, *gb1, *gW2, *gb2, *gW3, *gb3;   /* this worker's partial sums */
    int t_begin, t_end;
} fbwd_job;

static void *fbwd_worker(void *arg)
{
    fbwd_job *j = (fbwd_job *)arg;
    const int E = 1 + 2 * j->n_bands, H = j->width, O = j->N * j->D;
    double *e = (double *)malloc(sizeof(double) * E);
    double *p1 = (double *)malloc(sizeof(double) * H), *s1 = (double *)malloc(sizeof(double) * H);
    double *p2 = (double *)malloc(sizeof(double) * H), *s2 = (double *)malloc(sizeof(double) * H);
    double *ds2 = (double *)malloc(sizeof(double) * H), *dp2 = (double *)malloc(sizeof(double) * H);
    double *ds1 = (double *)malloc(sizeof(double) * H), *dp1 = (double *)malloc(sizeof(double) * H);
    for (int t = j->t_begin; t < j->t_end; ++t) {
        oracle_embedding(t, j->L, j->n_bands, e);
        for (int o = 0; o < H; ++o) {
            double acc = (double)j->b1[o];
            for (int i = 0; i < E; ++i) acc += (double)j->W1[o * E + i] * e[i];
            p1[o] = acc; s1[o] = sin(acc);
        }
        for (int o = 0; o < H; ++o) {
            double acc = (double)j->b2[o];
            for (int i = 0; i < H; ++i) acc += (double)j->W2[o * H + i] * s1[i];
            p2[o] = acc; s2[o] = sin(acc);
        }
        for (int i = 0; i < H; ++i) ds2[i] = 0.0;
        for (int o = 0; o < O; ++o) {
            int c = o % j->D;
            double alpha = oracle_alpha(c, j->D, j->alpha_lo, j->alpha_hi);
            double dO = j->dh[(size_t)o * j->L + t] * exp(-alpha * (double)t / (double)j->L);
            j->gb3[o] += dO;
            for (int i = 0; i < H; ++i) {
                j->gW3[(size_t)o * H + i] += dO * s2[i];
                ds2[i] += (double)j->W3[(size_t)o * H + i] * dO;
            }
        }
        for (int i = 0; i < H; ++i) dp2[i] = ds2[i] * cos(p2[i]);
        for (int i = 0; i < H; ++i) ds1[i] = 0.0;
        for (int o = 0; o < H; ++o) {
            j->gb2[o] += dp2[o];
            for (int i = 0; i < H; ++i) {
                j->gW2[o * H + i] += dp2[o] * s1[i];
                ds1[i] += (double)j->W2[o * H + i] * dp2[o];
            }
        }
        for (int i = 0; i < H; ++i) dp1[i] = ds1[i] * cos(p1[i]);
        for (int o = 0; o < H; ++o) {
            j->gb1[o] += dp1[o];
            for (int i = 0; i < E; ++i) j->gW1[o * E + i] += dp1[o] * e[i];
        }
    }
    free(e); free(p1); free(s1); free(p2); free(s2); free(ds2); free(dp2); free(ds1); free(dp1);
    return NULL;
}

void oracle_filter_backward(const float *W1, const float *b1, const float *W2, const float *b2,
                            const float *W3, const float *b3, int n_bands, int width,
                            int N, int D, int L, double alpha_lo, double alpha_hi, const double *dh,
                            double *gW1, double *gb1, double *gW2, double *gb2, double *gW3, double *gb3,
                            int n_threads)
{
    const int E = 1 + 2 * n_bands, H = width;
    const size_t O = (size_t)N * D;
    const size_t n1 = (size_t)H * E, n2 = (size_t)H * H, n3 = O * H;
    const size_t per = n1 + H + n2 + H + n3 + O;
    if (n_threads < 1) n_threads = 1;
    if (n_threads > L) n_threads = L;
    double *part = (double *)calloc(per * (size_t)n_threads, sizeof(double));
    pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * n_threads);
    fbwd_job *jobs = (fbwd_job *)malloc(sizeof(fbwd_job) * n_threads);
    for (int i = 0; i < n_threads; ++i) {
        double *q = part + per * (size_t)i;
        fbwd_job j = {W1, b1, W2, b2, W3, b3, n_bands, width, N, D, L, alpha_lo, alpha_hi, dh,
                      q, q + n1, q + n1 + H, q + n1 + H + n2, q + n1 + H + n2 + H, q + n1 + H + n2 + H + n3,
                      (int)((int64_t)L * i / n_threads), (int)((int64_t)L * (i + 1) / n_threads)};
        jobs[i] = j;
        pthread_create(&th[i], NULL, fbwd_worker, &jobs[i]);
    }
    for (int i = 0; i < n_threads; ++i) pthread_join(th[i], NULL);
    double *outs[6] = {gW1, gb1, gW2, gb2, gW3, gb3};
    size_t lens[6] = {n1, (size_t)H, n2, (size_t)H, n3, O};
    size_t off = 0;
    for (int k = 0; k < 6; ++k) {
        for (size_t m = 0; m < lens[k]; ++m) {
            double acc = 0.0;
            for (int i = 0; i < n_threads; ++i) acc += part[per * (size_t)i + off + m];
            outs[k][m] = acc;
        }
        off += lens[k];
    }
    free(part); free(th); free(jobs);
}

/* ------------------------------------------------------------------------ */
/* StripedHyena-form operator                                               */
/* ------------------------------------------------------------------------ */

/*
 * "02. 3つの Hyena 演算子", section 2 (the operator structure) and section 4
 * (the FIR sum y_t = sum_{k < l_h} h_k x_{t-k}):
 *   q = h_T * xq,  k = h_H * xk,  v = h_K * xv      (short explicit FIRs)
 *   y = q (.) (h_G * (k (.) v))
 * (the dense projections W, U, P, M of that section are outside this
 * operator: xq, xk, xv are their outputs). Every * is the causal FIR sum,
 * zero before t = 0. One channel, length L; filters of length lf (featurizers)
 * and lg (inner).
 */
static void fir_causal(const double *h, int lh, const double *x, int64_t L, double *out)
{
    for (int64_t t = 0; t < L; ++t) {
        double acc = 0.0;
        for (int j = 0; j < lh && j <= t; ++j) acc += h[j] * x[t - j];
        out[t] = acc;
    }
}

void oracle_striped_channel(const double *xq, const double *xk, const double *xv,
                            const double *hT, const double *hH, const double *hK, int lf,
                            const double *hG, int lg, int64_t L, double *y)
{
    double *q = (double *)malloc(sizeof(double) * L), *k = (double *)malloc(sizeof(double) * L);
    double *v = (double *)malloc(sizeof(double) * L), *w = (double *)malloc(sizeof(double) * L);
    fir_causal(hT, lf, xq, L, q);
    fir_causal(hH, lf, xk, L, k);
    fir_causal(hK, lf, xv, L, v);
    for (int64_t t = 0; t < L; ++t) k[t] *= v[t];
    fir_causal(hG, lg, k, L, w);
    for (int64_t t = 0; t < L; ++t) y[t] = q[t] * w[t];
    free(q); free(k); free(v); free(w);
}

typedef struct {
    const double *xq, *xk, *xv, *hT, *hH, *hK, *hG;
    const int *filter_row;
    int lf, lg;
    int64_t L;
    double *y;
    int begin, end;
} striped_job;

static void *striped_worker(void *arg)
{
    striped_job *j = (striped_job *)arg;
    for (int r = j->begin; r < j->end; ++r) {
        const int f = j->filter_row[r];
        const size_t o = (size_t)r * j->L;
        oracle_striped_channel(j->xq + o, j->xk + o, j->xv + o, j->hT + (size_t)f * j->lf,
                               j->hH + (size_t)f * j->lf, j->hK + (size_t)f * j->lf, j->lf,
                               j->hG + (size_t)f * j->lg, j->lg, j->L, j->y + o);
    }
    return NULL;
}

/* C channels [C][L]; filters [F][lf] / [F][lg], channel r uses row filter_row[r]. */
int oracle_striped_forward(const double *xq, const double *xk, const double *xv,
                           const double *hT, const double *hH, const double *hK, int lf,
                           const double *hG, int lg, const int *filter_row, int64_t C, int64_t L,
                           double *y, int n_threads)
{
    if (lf < 1 || lg < 1 || L < 1 || C < 0) return 1;
    if (C == 0) return 0;
    if (n_threads < 1) n_threads = 1;
    if (n_threads > C) n_threads = (int)C;
    pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * n_threads);
    striped_job *jobs = (striped_job *)malloc(sizeof(striped_job) * n_threads);
    for (int i = 0; i < n_threads; ++i) {
        striped_job j = {xq, xk, xv, hT, hH, hK, hG, filter_row, lf, lg, L, y,
                         (int)(C * i / n_threads), (int)(C * (i + 1) / n_threads)};
        jobs[i] = j;
        pthread_create(&th[i], NULL, striped_worker, &jobs[i]);
    }
    for (int i = 0; i < n_threads; ++i) pthread_join(th[i], NULL);
    free(th); free(jobs);
    return 0;
}
